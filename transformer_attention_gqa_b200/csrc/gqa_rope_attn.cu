// Host side of the C ABI (include/gqa_rope_attn.h): argument checks, TMA
// descriptor cache, the two launches of the fused forward (prologue, then
// the attention kernel, in stream order), the two of the masked forward (the
// same prologue, then the attention kernel in its masked form), the two of the decoding
// step (key-range kernel, then the merge), the three of the backward
// (prologue, attention backward, dq rotation) and the two of the QKV
// projection with its RoPE epilogue (cos/sin table, projection).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/gqa_rope_attn.h"
#include "attn_kernel.cuh"
#include "bwd_kernel.cuh"
#include "bwd_q_kernel.cuh"
#include "common.cuh"
#include "decode_kernel.cuh"
#include "prep_kernel.cuh"
#include "proj_kernel.cuh"

namespace gqa {

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool init = false;
  int sm_count = 0;
  bool attr_set[3][2] = {};
  bool bwd_attr_set[3] = {};
  bool proj_attr_set[3] = {};
  bool masked_attr_set[3] = {};
  bool dtc_attr_set[3] = {};
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
thread_local int t_last_launches = 0;
thread_local cudaEvent_t t_prof_ev[3] = {nullptr, nullptr, nullptr};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

struct TmapKey {
  int device;
  const void* ptr;
  uint64_t dims[3];
  uint64_t strides[2];
  uint32_t box[3];
  int swizzle;
  bool operator==(const TmapKey& o) const { return std::memcmp(this, &o, sizeof(TmapKey)) == 0; }
};

struct TmapEntry {
  TmapKey key;
  CUtensorMap map;
  uint64_t stamp;
  bool valid;
};

constexpr int kCacheSize = 64;
TmapEntry g_cache[kCacheSize];
uint64_t g_clock = 0;

// 3-D bf16 tensor map (innermost dimension first), cached by its arguments.
bool make_tmap(int device, const void* ptr, const uint64_t dims[3], const uint64_t strides[2],
               const uint32_t box[3], int swizzle_bytes, CUtensorMap* out) {
  TmapKey key;
  std::memset(&key, 0, sizeof(key));
  key.device = device;
  key.ptr = ptr;
  for (int i = 0; i < 3; ++i) key.dims[i] = dims[i], key.box[i] = box[i];
  key.strides[0] = strides[0];
  key.strides[1] = strides[1];
  key.swizzle = swizzle_bytes;
  int victim = 0;
  uint64_t oldest = ~0ull;
  for (int i = 0; i < kCacheSize; ++i) {
    if (g_cache[i].valid && g_cache[i].key == key) {
      g_cache[i].stamp = ++g_clock;
      *out = g_cache[i].map;
      return true;
    }
    const uint64_t st = g_cache[i].valid ? g_cache[i].stamp : 0;
    if (st < oldest) oldest = st, victim = i;
  }
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t gdim[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t gstr[2] = {strides[0], strides[1]};
  const cuuint32_t bdim[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap m;
  const CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), gdim, gstr, bdim, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  g_cache[victim].key = key;
  g_cache[victim].map = m;
  g_cache[victim].stamp = ++g_clock;
  g_cache[victim].valid = true;
  *out = m;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int dim_index(int d) { return d == 32 ? 0 : (d == 64 ? 1 : 2); }

// prerotated: q and k are already rotated (bf16 only); the prologue builds
// the schedule alone and K is read from the caller's token-major tensor.
// mask (bf16 only): the attention kernel's masked form adds mask[query,
// key] * sqrt(d) to every raw score.
template <int D, bool FP32>
int launch(const void* q, const void* k, const void* v, const int32_t* positions, double theta,
           const int32_t* cu, int num_seqs, int N, int nq, int nkv, int causal, void* out, float* lse,
           uint8_t* ws, const WsLayout& lay, cudaStream_t stream, int device, int sm_count,
           bool prerotated = false, const void* mask = nullptr, int mask_len = 0, int mask_ld = 0) {
  if (FP32 && (prerotated || mask)) return GQA_ERR_UNSUPPORTED;
  if (prerotated && mask) return GQA_ERR_UNSUPPORTED;
  using C = AttnCfg<D>;
  const int G = nq / nkv;
  const int tq = tokens_per_tile(G);

  {  // caller holds g_mu
    DeviceState& ds = g_dev[device];
    if (!ds.attr_set[dim_index(D)][FP32 ? 1 : 0]) {
      if (cudaFuncSetAttribute(gqa_attn_fwd_kernel<D, FP32, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES) != cudaSuccess)
        return GQA_ERR_CUDA;
      ds.attr_set[dim_index(D)][FP32 ? 1 : 0] = true;
    }
    if constexpr (!FP32) {
      if (mask && !ds.masked_attr_set[dim_index(D)]) {
        if (cudaFuncSetAttribute(gqa_attn_fwd_kernel<D, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES) != cudaSuccess)
          return GQA_ERR_CUDA;
        ds.masked_attr_set[dim_index(D)] = true;
      }
    }
  }

  PrepParams pp{};
  pp.q = q;
  pp.k = k;
  pp.v = v;
  pp.positions = positions;
  pp.cu = cu;
  pp.N = N;
  pp.num_seqs = num_seqs;
  pp.nq = nq;
  pp.nkv = nkv;
  pp.tq = tq;
  pp.causal = causal;
  pp.theta = theta;
  for (int i = 0; i < D / 2; ++i) pp.inv_freq[i] = std::pow(theta, -(2.0 * i) / D);
  pp.header = reinterpret_cast<int*>(ws + lay.header);
  pp.seq_pfx = reinterpret_cast<int*>(ws + lay.seq_pfx);
  pp.pairs = reinterpret_cast<int2*>(ws + lay.pairs);
  pp.table = reinterpret_cast<uint32_t*>(ws + lay.table);
  pp.kws = reinterpret_cast<__nv_bfloat16*>(ws + lay.kws);
  // the prologue rotates Q into the workspace when the layout has room for it
  // (fp32 inputs, or short work items), never for inputs already rotated
  const bool q_in_ws = !prerotated && lay.qws != 0;
  pp.qws = q_in_ws ? reinterpret_cast<__nv_bfloat16*>(ws + lay.qws) : nullptr;
  pp.vws = FP32 ? reinterpret_cast<__nv_bfloat16*>(ws + lay.vws) : nullptr;

  // Tensor maps. Q: [N][nq][d] (caller's, or the prologue's rotated Q');
  // K: RoPE'd, head-major [nkv][N][d] (or the caller's rotated K,
  // token-major); V: [N][nkv][d] (caller's, or its bf16 copy).
  CUtensorMap tmQ, tmK, tmV;
  const void* qsrc = q_in_ws ? (const void*)(ws + lay.qws) : q;
  const void* vsrc = FP32 ? (const void*)(ws + lay.vws) : v;
  const uint64_t es = 2;
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)nq, (uint64_t)N};
    const uint64_t str[2] = {(uint64_t)D * es, (uint64_t)nq * D * es};
    const uint32_t box[3] = {(uint32_t)C::BOXC, (uint32_t)G, (uint32_t)tq};
    if (!make_tmap(device, qsrc, dims, str, box, C::ROWB, &tmQ)) return GQA_ERR_CUDA;
  }
  if (prerotated) {  // the caller's K, token-major like V
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)nkv, (uint64_t)N};
    const uint64_t str[2] = {(uint64_t)D * es, (uint64_t)nkv * D * es};
    const uint32_t box[3] = {(uint32_t)C::BOXC, 1u, (uint32_t)BN};
    if (!make_tmap(device, k, dims, str, box, C::ROWB, &tmK)) return GQA_ERR_CUDA;
  } else {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)N, (uint64_t)nkv};
    const uint64_t str[2] = {(uint64_t)D * es, (uint64_t)N * D * es};
    const uint32_t box[3] = {(uint32_t)C::BOXC, (uint32_t)BN, 1u};
    if (!make_tmap(device, ws + lay.kws, dims, str, box, C::ROWB, &tmK)) return GQA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)nkv, (uint64_t)N};
    const uint64_t str[2] = {(uint64_t)D * es, (uint64_t)nkv * D * es};
    const uint32_t box[3] = {(uint32_t)C::BOXC, 1u, (uint32_t)BN};
    if (!make_tmap(device, vsrc, dims, str, box, C::ROWB, &tmV)) return GQA_ERR_CUDA;
  }


  const long long work = (long long)N * (D / 4);
  long long nb = (work + PREP_THREADS - 1) / PREP_THREADS;
  const long long cap = (long long)sm_count * 8;
  if (nb > cap) nb = cap;
  if (nb < 1) nb = 1;
  if (prerotated) nb = 0;  // block 0 alone: the schedule
  if (t_prof_ev[0] && cudaEventRecord(t_prof_ev[0], stream) != cudaSuccess) return GQA_ERR_CUDA;
  gqa_prep_kernel<D, FP32><<<(unsigned)(nb + 1), PREP_THREADS, 0, stream>>>(pp);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[1] && cudaEventRecord(t_prof_ev[1], stream) != cudaSuccess) return GQA_ERR_CUDA;


  AttnParams ap{};
  ap.cu = cu;
  ap.header = pp.header;
  ap.item_counter = pp.header + 8;
  ap.pairs = pp.pairs;
  ap.table = pp.table;
  ap.out = out;
  ap.lse = lse;
  ap.N = N;
  ap.nq = nq;
  ap.nkv = nkv;
  ap.G = G;
  ap.tq = tq;
  ap.causal = causal;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  ap.rescale_thr = (float)(8.0 / (1.4426950408889634 / std::sqrt((double)D)));
  ap.q_rotated = (prerotated || q_in_ws) ? 1 : 0;
  ap.k_token_major = prerotated ? 1 : 0;
  ap.mask = reinterpret_cast<const __nv_bfloat16*>(mask);
  ap.mask_len = mask_len;
  ap.mask_ld = mask_ld;
  ap.mask_scale = (float)std::sqrt((double)D);

  const long long max_items = lay.max_pairs * (long long)nkv;
  const unsigned grid = (unsigned)(max_items < sm_count ? max_items : sm_count);
  // Greedy claiming runs two items ahead of the work; with fewer than about
  // ten items per CTA that granularity balances worse than a static
  // alternating deal of the sorted list (measured on B200).
  ap.sched_dynamic = max_items >= 10LL * grid ? 1 : 0;

  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(ATTN_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  // Programmatic dependent launch: the attention grid may be scheduled as
  // soon as every prologue block has finished its stores (each block
  // triggers at its end), so its launch and setup overlap the prologue's
  // tail; it reads the prologue's results only after griddepcontrol.wait.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t le;
  if constexpr (!FP32) {
    le = mask ? cudaLaunchKernelEx(&cfg, gqa_attn_fwd_kernel<D, false, true>, tmQ, tmK, tmV, ap)
              : cudaLaunchKernelEx(&cfg, gqa_attn_fwd_kernel<D, false, false>, tmQ, tmK, tmV, ap);
  } else {
    le = cudaLaunchKernelEx(&cfg, gqa_attn_fwd_kernel<D, true, false>, tmQ, tmK, tmV, ap);
  }
  if (le != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[2] && cudaEventRecord(t_prof_ev[2], stream) != cudaSuccess) return GQA_ERR_CUDA;
  t_last_launches = 2;
  return GQA_OK;
}

// ---------------------------------------------------------------- decoding

struct DecLayout {
  size_t part_o, part_ml, total;
  int splits, kps;
};

// Key ranges: whole 64-key tiles, about DEC_TARGET_CTAS CTAs over the batch
// (a rule of the shape alone, so the workspace size needs no device query).
DecLayout dec_layout(int B, int Lmax, int nq, int nkv, int d) {
  DecLayout L{};
  const int G = nq / nkv;
  const long long tiles = (Lmax + DEC_KT - 1) / DEC_KT;
  long long want = (DEC_TARGET_CTAS + (long long)B * nkv - 1) / ((long long)B * nkv);
  if (want < 1) want = 1;
  if (want > tiles) want = tiles;
  const long long tps = (tiles + want - 1) / want;
  L.kps = (int)(tps * DEC_KT);
  L.splits = (int)((tiles + tps - 1) / tps);
  size_t off = 0;
  L.part_o = off;
  off = align_up(off + (size_t)B * nkv * L.splits * G * d * sizeof(float), 256);
  L.part_ml = off;
  off = align_up(off + (size_t)B * nkv * L.splits * G * sizeof(float2), 256);
  L.total = off;
  return L;
}

template <int D>
int launch_decode(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                  const int32_t* lens, double theta, int B, int Lmax, int nq, int nkv, void* out, float* lse,
                  uint8_t* ws, const DecLayout& lay, cudaStream_t stream, int device) {
  using C = DtcCfg<D>;
  // heads per softmax thread: G rounded up to 4, 8 or 16
  const int G = nq / nkv;
  void (*kern)(CUtensorMap, CUtensorMap, DecodeParams) =
      G <= 4 ? gqa_decode_tc_kernel<D, 4> : (G <= 8 ? gqa_decode_tc_kernel<D, 8> : gqa_decode_tc_kernel<D, 16>);
  {  // caller holds g_mu
    DeviceState& ds = g_dev[device];
    if (!ds.dtc_attr_set[dim_index(D)]) {
      if (cudaFuncSetAttribute(gqa_decode_tc_kernel<D, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(gqa_decode_tc_kernel<D, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(gqa_decode_tc_kernel<D, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES) != cudaSuccess)
        return GQA_ERR_CUDA;
      ds.dtc_attr_set[dim_index(D)] = true;
    }
  }
  // Cache maps: [B*Lmax rows][nkv][d], box (BOXC columns, 1 head, 64 rows).
  CUtensorMap tmK, tmV;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)nkv, (uint64_t)B * (uint64_t)Lmax};
  const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)nkv * D * 2};
  const uint32_t box[3] = {(uint32_t)C::A::BOXC, 1u, (uint32_t)DEC_KT};
  if (!make_tmap(device, k_cache, dims, str, box, C::A::ROWB, &tmK)) return GQA_ERR_CUDA;
  if (!make_tmap(device, v_cache, dims, str, box, C::A::ROWB, &tmV)) return GQA_ERR_CUDA;

  DecodeParams dp{};
  dp.q = reinterpret_cast<const __nv_bfloat16*>(q);
  dp.k_new = reinterpret_cast<const __nv_bfloat16*>(k_new);
  dp.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
  dp.k_cache = reinterpret_cast<__nv_bfloat16*>(k_cache);
  dp.v_cache = reinterpret_cast<__nv_bfloat16*>(v_cache);
  dp.cache_seqlens = lens;
  dp.part_o = reinterpret_cast<float*>(ws + lay.part_o);
  dp.part_ml = reinterpret_cast<float2*>(ws + lay.part_ml);
  dp.out = reinterpret_cast<__nv_bfloat16*>(out);
  dp.lse = lse;
  dp.theta = theta;
  for (int i = 0; i < D / 2; ++i) dp.inv_freq[i] = std::pow(theta, -(2.0 * i) / D);
  dp.B = B;
  dp.Lmax = Lmax;
  dp.nq = nq;
  dp.nkv = nkv;
  dp.G = G;
  dp.splits = lay.splits;
  dp.kps = lay.kps;
  dp.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  // Failure-detection test hook (off unless the variable is set to 1): the
  // first K/V tile of every key range is never loaded, so each CTA's bounded
  // wait runs out and the status word reads GQA_ERR_TIMEOUT.
  const char* drop = std::getenv("GQA_ROPE_ATTN_TEST_DROP_FIRST_LOAD");
  dp.test_drop_first_load = (drop && drop[0] == '1' && drop[1] == '\0') ? 1 : 0;

  if (t_prof_ev[0] && cudaEventRecord(t_prof_ev[0], stream) != cudaSuccess) return GQA_ERR_CUDA;
  kern<<<dim3(lay.splits, nkv, B), DTC_THREADS, C::SMEM_BYTES, stream>>>(tmK, tmV, dp);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[1] && cudaEventRecord(t_prof_ev[1], stream) != cudaSuccess) return GQA_ERR_CUDA;
  gqa_decode_combine_kernel<<<dim3(nkv, B), DEC_COMBINE_THREADS, 0, stream>>>(dp, D);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[2] && cudaEventRecord(t_prof_ev[2], stream) != cudaSuccess) return GQA_ERR_CUDA;
  t_last_launches = 2;
  return GQA_OK;
}

// ---------------------------------------------------------------- backward

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
               const int32_t* positions, double theta, const int32_t* cu, int num_seqs, int N, int nq, int nkv,
               int causal, void* dq, void* dk, void* dv, uint8_t* ws, const BwdWsLayout& lay, cudaStream_t stream,
               int device, int sm_count) {
  using C = BwdCfg<D>;
  const int G = nq / nkv;
  const int tq = tokens_per_tile(G);
  {  // caller holds g_mu
    DeviceState& ds = g_dev[device];
    if (!ds.bwd_attr_set[dim_index(D)]) {
      if (cudaFuncSetAttribute(gqa_attn_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(gqa_attn_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BwdQCfg<D>::SMEM_BYTES) != cudaSuccess)
        return GQA_ERR_CUDA;
      ds.bwd_attr_set[dim_index(D)] = true;
    }
  }
  BwdPrepParams pp{};
  pp.q = reinterpret_cast<const __nv_bfloat16*>(q);
  pp.k = reinterpret_cast<const __nv_bfloat16*>(k);
  pp.out = reinterpret_cast<const __nv_bfloat16*>(out);
  pp.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
  pp.lse = lse;
  pp.positions = positions;
  pp.cu = cu;
  pp.N = N;
  pp.num_seqs = num_seqs;
  pp.nq = nq;
  pp.nkv = nkv;
  pp.tq = tq;
  pp.causal = causal;
  for (int i = 0; i < D / 2; ++i) pp.inv_freq[i] = std::pow(theta, -(2.0 * i) / D);
  pp.header = reinterpret_cast<int*>(ws + lay.header);
  pp.seq_pfx = reinterpret_cast<int*>(ws + lay.seq_pfx);
  pp.pairs = reinterpret_cast<int2*>(ws + lay.pairs);
  pp.table = reinterpret_cast<float2*>(ws + lay.table);
  pp.kws = reinterpret_cast<__nv_bfloat16*>(ws + lay.kws);
  pp.qws = reinterpret_cast<__nv_bfloat16*>(ws + lay.qws);
  pp.lse2 = reinterpret_cast<float*>(ws + lay.lse2);
  pp.delta = reinterpret_cast<float*>(ws + lay.delta);
  pp.qheader = reinterpret_cast<int*>(ws + lay.qheader);
  pp.qseq_pfx = reinterpret_cast<int*>(ws + lay.qseq_pfx);
  pp.qpairs = reinterpret_cast<int2*>(ws + lay.qpairs);
  float* const dq_acc = reinterpret_cast<float*>(ws + lay.dq_acc);

  // Q' and dO: [N][nq][d], box (BOXC, G heads, tq tokens); K': [nkv][N][d],
  // box (BOXC, BN keys, 1); V: [N][nkv][d], box (BOXC, 1, BN keys).
  CUtensorMap tmQ, tmDO, tmK, tmV;
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)nq, (uint64_t)N};
    const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)nq * D * 2};
    const uint32_t box[3] = {(uint32_t)C::BOXC, (uint32_t)G, (uint32_t)tq};
    if (!make_tmap(device, ws + lay.qws, dims, str, box, C::ROWB, &tmQ)) return GQA_ERR_CUDA;
    if (!make_tmap(device, dout, dims, str, box, C::ROWB, &tmDO)) return GQA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)N, (uint64_t)nkv};
    const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)N * D * 2};
    const uint32_t box[3] = {(uint32_t)C::BOXC, (uint32_t)BN, 1u};
    if (!make_tmap(device, ws + lay.kws, dims, str, box, C::ROWB, &tmK)) return GQA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)nkv, (uint64_t)N};
    const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)nkv * D * 2};
    const uint32_t box[3] = {(uint32_t)C::BOXC, 1u, (uint32_t)BN};
    if (!make_tmap(device, v, dims, str, box, C::ROWB, &tmV)) return GQA_ERR_CUDA;
  }

  const long long work = (long long)N * (D / 4);
  long long nb = (work + PREP_THREADS - 1) / PREP_THREADS;
  const long long cap = (long long)sm_count * 8;
  if (nb > cap) nb = cap;
  if (nb < 1) nb = 1;
  if (t_prof_ev[0] && cudaEventRecord(t_prof_ev[0], stream) != cudaSuccess) return GQA_ERR_CUDA;
  gqa_bwd_prep_kernel<D><<<(unsigned)(nb + 2), PREP_THREADS, 0, stream>>>(pp);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[1] && cudaEventRecord(t_prof_ev[1], stream) != cudaSuccess) return GQA_ERR_CUDA;

  BwdParams bp{};
  bp.cu = cu;
  bp.header = pp.header;
  bp.pairs = pp.pairs;
  bp.table = pp.table;
  bp.lse2 = pp.lse2;
  bp.delta = pp.delta;
  bp.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  bp.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  bp.N = N;
  bp.nq = nq;
  bp.nkv = nkv;
  bp.G = G;
  bp.tq = tq;
  bp.causal = causal;
  bp.scale = (float)(1.0 / std::sqrt((double)D));
  bp.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  // one CTA per (sequence, key tile, KV head); CTAs past the prologue's
  // pair count exit at once
  const unsigned grid = (unsigned)(lay.max_pairs * (long long)nkv);
  gqa_attn_bwd_kernel<D><<<grid, BWD_THREADS, C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmDO, bp);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  // dQ' per (query tile, KV head); CTAs past the query-tile pair count exit at once
  BwdQParams qp{};
  qp.cu = cu;
  qp.header = pp.qheader;
  qp.pairs = pp.qpairs;
  qp.lse2 = pp.lse2;
  qp.delta = pp.delta;
  qp.dq_acc = dq_acc;
  qp.N = N;
  qp.nq = nq;
  qp.nkv = nkv;
  qp.G = G;
  qp.tq = tq;
  qp.causal = causal;
  qp.scale_log2 = bp.scale_log2;
  const unsigned qgrid = (unsigned)(lay.max_qpairs * (long long)nkv);
  gqa_attn_bwd_q_kernel<D><<<qgrid, BQ_THREADS, BwdQCfg<D>::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmDO, qp);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[2] && cudaEventRecord(t_prof_ev[2], stream) != cudaSuccess) return GQA_ERR_CUDA;

  const long long rows4 = (long long)N * nq * (D / 8);
  long long nbq = (rows4 + PREP_THREADS - 1) / PREP_THREADS;
  if (nbq > cap) nbq = cap;
  if (nbq < 1) nbq = 1;
  gqa_bwd_dq_kernel<D><<<(unsigned)nbq, PREP_THREADS, 0, stream>>>(dq_acc, pp.table,
                                                                 reinterpret_cast<__nv_bfloat16*>(dq), N, nq,
                                                                 bp.scale);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  t_last_launches = 4;
  return GQA_OK;
}

// ---------------------------------------------------------------- QKV projection

template <int D>
int launch_qkv_proj(const void* x, const void* w, const int32_t* positions, double theta, const int32_t* cu,
                    int num_seqs, int N, int C, int nq, int nkv, void* q, void* k, void* v, uint8_t* ws,
                    cudaStream_t stream, int device, int sm_count) {
  {  // caller holds g_mu
    DeviceState& ds = g_dev[device];
    if (!ds.proj_attr_set[dim_index(D)]) {
      if (cudaFuncSetAttribute(gqa_qkv_proj_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PJ_SMEM_BYTES) != cudaSuccess)
        return GQA_ERR_CUDA;
      ds.proj_attr_set[dim_index(D)] = true;
    }
  }
  const int F = (nq + 2 * nkv) * D;
  // x: [N][C], box (64 of C, 128 tokens); W: [F][C], box (64 of C, 256 features)
  CUtensorMap tmX, tmW;
  {
    const uint64_t dims[3] = {(uint64_t)C, (uint64_t)N, 1u};
    const uint64_t str[2] = {(uint64_t)C * 2, (uint64_t)C * N * 2};
    const uint32_t box[3] = {(uint32_t)PJ_BK, (uint32_t)PJ_BM, 1u};
    if (!make_tmap(device, x, dims, str, box, 128, &tmX)) return GQA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)C, (uint64_t)F, 1u};
    const uint64_t str[2] = {(uint64_t)C * 2, (uint64_t)C * F * 2};
    const uint32_t box[3] = {(uint32_t)PJ_BK, (uint32_t)PJ_BN, 1u};
    if (!make_tmap(device, w, dims, str, box, 128, &tmW)) return GQA_ERR_CUDA;
  }
  ProjTableParams tp{};
  tp.positions = positions;
  tp.cu = cu;
  tp.N = N;
  tp.num_seqs = num_seqs;
  tp.half = D / 2;
  for (int i = 0; i < D / 2; ++i) tp.inv_freq[i] = std::pow(theta, -(2.0 * i) / D);
  tp.table = reinterpret_cast<float2*>(ws);
  long long nb = ((long long)N * (D / 4) + PREP_THREADS - 1) / PREP_THREADS;
  if (nb > (long long)sm_count * 8) nb = (long long)sm_count * 8;
  if (nb < 1) nb = 1;
  if (t_prof_ev[0] && cudaEventRecord(t_prof_ev[0], stream) != cudaSuccess) return GQA_ERR_CUDA;
  gqa_qkv_table_kernel<<<(unsigned)nb, PREP_THREADS, 0, stream>>>(tp);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[1] && cudaEventRecord(t_prof_ev[1], stream) != cudaSuccess) return GQA_ERR_CUDA;
  ProjParams pp{};
  pp.table = tp.table;
  pp.q = reinterpret_cast<__nv_bfloat16*>(q);
  pp.k = reinterpret_cast<__nv_bfloat16*>(k);
  pp.v = reinterpret_cast<__nv_bfloat16*>(v);
  pp.N = N;
  pp.C = C;
  pp.nq = nq;
  pp.nkv = nkv;
  pp.n_tiles_n = (F + PJ_BN - 1) / PJ_BN;
  const long long n_tiles = (long long)pp.n_tiles_n * ((N + PJ_BM - 1) / PJ_BM);
  if (n_tiles > 0x7fffffffll) return GQA_ERR_UNSUPPORTED;
  pp.n_tiles = (int)n_tiles;
  // one persistent CTA per SM (each walks tiles b, b + grid, ...); with
  // fewer than two tiles per SM, one CTA per tile (measured faster there)
  const unsigned grid = (unsigned)(n_tiles <= 2LL * sm_count ? n_tiles : sm_count);
  gqa_qkv_proj_kernel<D><<<grid, PJ_THREADS, PJ_SMEM_BYTES, stream>>>(tmX, tmW, pp);
  if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
  if (t_prof_ev[2] && cudaEventRecord(t_prof_ev[2], stream) != cudaSuccess) return GQA_ERR_CUDA;
  t_last_launches = 2;
  return GQA_OK;
}

}  // namespace
}  // namespace gqa

using namespace gqa;

extern "C" size_t gqa_rope_attn_decode_workspace_size(int batch, int max_cache_len, int n_q_heads,
                                                      int n_kv_heads, int head_dim) {
  if (batch < 0 || max_cache_len < 1 || n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return 0;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return 0;
  if (n_q_heads / n_kv_heads > DEC_GMAX) return 0;
  if (batch == 0) return 256;
  return dec_layout(batch, max_cache_len, n_q_heads, n_kv_heads, head_dim).total;
}

extern "C" int gqa_rope_attn_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                    void* v_cache, const int32_t* cache_seqlens, double rope_theta, int batch,
                                    int max_cache_len, int n_q_heads, int n_kv_heads, int head_dim, void* out,
                                    float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  struct Disarm {
    ~Disarm() { t_prof_ev[0] = t_prof_ev[1] = t_prof_ev[2] = nullptr; }
  } disarm;
  if (batch < 0 || max_cache_len < 1) return GQA_ERR_INVALID_ARG;
  if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return GQA_ERR_INVALID_ARG;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return GQA_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED;
  if (n_q_heads / n_kv_heads > DEC_GMAX) return GQA_ERR_UNSUPPORTED;
  if (batch > 65535 || n_kv_heads > 65535) return GQA_ERR_UNSUPPORTED;
  if ((long long)batch * max_cache_len >= (1ll << 31)) return GQA_ERR_UNSUPPORTED;
  if (batch == 0) return GQA_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_seqlens || !out) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(out))
    return GQA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cache_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return GQA_ERR_INVALID_ARG;
  const DecLayout lay = dec_layout(batch, max_cache_len, n_q_heads, n_kv_heads, head_dim);
  if (!workspace || workspace_bytes < lay.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GQA_ERR_WORKSPACE;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return GQA_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& ds = g_dev[device];
    if (!ds.init) {
      int major = 0;
      if (cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
          cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
        return GQA_ERR_CUDA;
      if (major != 10) return GQA_ERR_UNSUPPORTED;
      ds.init = true;
    }
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  std::lock_guard<std::mutex> lk(g_mu);  // descriptor cache
#define GQA_DEC_CASE(DD)                                                                                      \
  if (head_dim == DD)                                                                                         \
    return launch_decode<DD>(q, k_new, v_new, k_cache, v_cache, cache_seqlens, rope_theta, batch, max_cache_len, \
                             n_q_heads, n_kv_heads, out, lse, ws, lay, st, device);
  GQA_DEC_CASE(32) GQA_DEC_CASE(64) GQA_DEC_CASE(128)
#undef GQA_DEC_CASE
  return GQA_ERR_UNSUPPORTED;
}

extern "C" size_t gqa_rope_attn_workspace_size(int num_seqs, int total_tokens, int n_q_heads, int n_kv_heads,
                                               int head_dim, int dtype) {
  if (num_seqs < 0 || total_tokens < 0 || n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return 0;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return 0;
  if (n_q_heads / n_kv_heads > BM) return 0;
  if (dtype != GQA_DTYPE_BF16 && dtype != GQA_DTYPE_FP32) return 0;
  return ws_layout(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim, dtype == GQA_DTYPE_FP32).total;
}

// Current device and its SM count; the first call per device checks that it
// is a compute capability 10.x part.
static int device_init(int* device_out, int* sm_count_out) {
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return GQA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& ds = g_dev[device];
  if (!ds.init) {
    int major = 0;
    if (cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
      return GQA_ERR_CUDA;
    if (major != 10) return GQA_ERR_UNSUPPORTED;
    ds.init = true;
  }
  *device_out = device;
  *sm_count_out = ds.sm_count;
  return GQA_OK;
}

// The forward's argument checks that need no CUDA call (shared by the
// forward and its no-allocation variant). GQA_OK with *empty set means there
// is nothing to compute (no tokens).
static int fwd_check_args(const void* q, const void* k, const void* v, const int32_t* positions, double rope_theta,
                          const int32_t* cu_seqlens, int num_seqs, int total_tokens, int n_q_heads, int n_kv_heads,
                          int head_dim, int causal, int dtype, const void* out, const float* lse, bool* empty) {
  *empty = false;
  if (total_tokens < 0 || num_seqs < 0) return GQA_ERR_INVALID_ARG;
  if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return GQA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return GQA_ERR_INVALID_ARG;
  if (dtype != GQA_DTYPE_BF16 && dtype != GQA_DTYPE_FP32) return GQA_ERR_INVALID_ARG;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return GQA_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED;
  if (n_q_heads / n_kv_heads > BM) return GQA_ERR_UNSUPPORTED;
  if ((long long)total_tokens * n_q_heads * head_dim > (1ll << 40)) return GQA_ERR_UNSUPPORTED;
  if (total_tokens == 0) {
    *empty = true;
    return GQA_OK;
  }
  if (num_seqs < 1) return GQA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !cu_seqlens) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GQA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(positions) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return GQA_ERR_INVALID_ARG;
  return GQA_OK;
}

extern "C" int gqa_rope_attn_fwd(const void* q, const void* k, const void* v, const int32_t* positions,
                                 double rope_theta, const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                                 int n_q_heads, int n_kv_heads, int head_dim, int causal, int dtype, void* out,
                                 float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  struct Disarm {
    ~Disarm() { t_prof_ev[0] = t_prof_ev[1] = t_prof_ev[2] = nullptr; }
  } disarm;
  // ---- checks that need no CUDA call
  bool empty = false;
  const int arg_rc = fwd_check_args(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,
                                    n_kv_heads, head_dim, causal, dtype, out, lse, &empty);
  if (arg_rc != GQA_OK || empty) return arg_rc;
  const bool fp32 = dtype == GQA_DTYPE_FP32;
  const WsLayout lay = ws_layout(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim, fp32);
  if (!workspace || workspace_bytes < lay.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GQA_ERR_WORKSPACE;

  // ---- device state
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return GQA_ERR_CUDA;
  int sm_count = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& ds = g_dev[device];
    if (!ds.init) {
      int major = 0;
      if (cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
          cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
        return GQA_ERR_CUDA;
      if (major != 10) return GQA_ERR_UNSUPPORTED;
      ds.init = true;
    }
    sm_count = ds.sm_count;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int rc;
  std::lock_guard<std::mutex> lk(g_mu);  // descriptor cache
#define GQA_FWD_CASE(KEY, DD, FP)                                                                           \
  case KEY:                                                                                                 \
    rc = launch<DD, FP>(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,     \
                        n_kv_heads, causal, out, lse, ws, lay, st, device, sm_count);                       \
    break;
  switch (head_dim * 2 + (fp32 ? 1 : 0)) {
    GQA_FWD_CASE(64, 32, false)
    GQA_FWD_CASE(65, 32, true)
    GQA_FWD_CASE(128, 64, false)
    GQA_FWD_CASE(129, 64, true)
    GQA_FWD_CASE(256, 128, false)
    GQA_FWD_CASE(257, 128, true)
    default: rc = GQA_ERR_UNSUPPORTED; break;
  }
#undef GQA_FWD_CASE
  return rc;
}

extern "C" int gqa_rope_attn_fwd_rotated(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                                         int num_seqs, int total_tokens, int n_q_heads, int n_kv_heads,
                                         int head_dim, int causal, void* out, float* lse, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  struct Disarm {
    ~Disarm() { t_prof_ev[0] = t_prof_ev[1] = t_prof_ev[2] = nullptr; }
  } disarm;
  bool empty = false;
  const int arg_rc = fwd_check_args(q, k, v, nullptr, 1.0, cu_seqlens, num_seqs, total_tokens, n_q_heads,
                                    n_kv_heads, head_dim, causal, GQA_DTYPE_BF16, out, lse, &empty);
  if (arg_rc != GQA_OK || empty) return arg_rc;
  const WsLayout lay = ws_layout(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim, false);
  if (!workspace || workspace_bytes < lay.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GQA_ERR_WORKSPACE;
  int device = 0, sm_count = 0;
  const int init_rc = device_init(&device, &sm_count);
  if (init_rc != GQA_OK) return init_rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  std::lock_guard<std::mutex> lk(g_mu);  // descriptor cache
#define GQA_ROT_CASE(DD)                                                                                    \
  if (head_dim == DD)                                                                                       \
    return launch<DD, false>(q, k, v, nullptr, 1.0, cu_seqlens, num_seqs, total_tokens, n_q_heads,          \
                             n_kv_heads, causal, out, lse, ws, lay, st, device, sm_count, true);
  GQA_ROT_CASE(32) GQA_ROT_CASE(64) GQA_ROT_CASE(128)
#undef GQA_ROT_CASE
  return GQA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// No-allocation variant: the workspace is a static device array of the
// library (one per device that loads it).

static __device__ __align__(256) uint8_t g_noalloc_scratch[GQA_ROPE_ATTN_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

extern "C" int gqa_rope_attn_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* positions,
                                         double rope_theta, const int32_t* cu_seqlens, int num_seqs,
                                         int total_tokens, int n_q_heads, int n_kv_heads, int head_dim,
                                         int causal, int dtype, void* out, float* lse, void* stream) {
  // the same argument checks as the forward, before any CUDA call
  bool empty = false;
  const int arg_rc = fwd_check_args(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,
                                    n_kv_heads, head_dim, causal, dtype, out, lse, &empty);
  if (arg_rc != GQA_OK || empty) return arg_rc;
  const size_t need =
      gqa_rope_attn_workspace_size(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim, dtype);
  if (need > (size_t)GQA_ROPE_ATTN_NOALLOC_SCRATCH_BYTES) return GQA_ERR_NOALLOC_LIMIT;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return GQA_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[device]) {
      // The array's name is only a host-side handle; its device address is
      // looked up once per device, with that device current.
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return GQA_ERR_CUDA;
      g_noalloc_ptr[device] = ptr;
    }
    scratch = g_noalloc_ptr[device];
  }
  return gqa_rope_attn_fwd(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,
                           n_kv_heads, head_dim, causal, dtype, out, lse, scratch,
                           (size_t)GQA_ROPE_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int gqa_rope_attn_get_device_status(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GQA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return GQA_ERR_CUDA;
  }
  return v;
}

extern "C" const char* gqa_rope_attn_strerror(int status) {
  switch (status) {
    case GQA_OK: return "ok";
    case GQA_ERR_INVALID_ARG: return "invalid argument";
    case GQA_ERR_UNSUPPORTED: return "unsupported shape or device";
    case GQA_ERR_CUDA: return "CUDA error";
    case GQA_ERR_BAD_SEQLENS:
      return "cu_seqlens is not a valid prefix sum of total_tokens, or a decode cache_seqlens entry is "
             "outside [0, max_cache_len)";
    case GQA_ERR_TIMEOUT: return "a bounded wait inside the kernel ran out";
    case GQA_ERR_WORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case GQA_ERR_NOALLOC_LIMIT:
      return "shape needs more scratch than the no-allocation entry point's built-in buffer "
             "(GQA_ROPE_ATTN_NOALLOC_SCRATCH_BYTES)";
    default: return "unknown status";
  }
}

extern "C" int gqa_rope_attn_abi_version(void) { return GQA_ROPE_ATTN_ABI_VERSION; }

extern "C" int gqa_rope_attn_last_launch_count(void) { return t_last_launches; }

extern "C" void gqa_rope_attn_set_profile_events(void* ev_start, void* ev_mid, void* ev_end) {
  t_prof_ev[0] = reinterpret_cast<cudaEvent_t>(ev_start);
  t_prof_ev[1] = reinterpret_cast<cudaEvent_t>(ev_mid);
  t_prof_ev[2] = reinterpret_cast<cudaEvent_t>(ev_end);
}

// ---------------------------------------------------------------------------
// Backward

extern "C" size_t gqa_rope_attn_bwd_workspace_size(int num_seqs, int total_tokens, int n_q_heads, int n_kv_heads,
                                                   int head_dim) {
  if (num_seqs < 0 || total_tokens < 0 || n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return 0;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return 0;
  if (n_q_heads / n_kv_heads > BM) return 0;
  return bwd_ws_layout(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim).total;
}

extern "C" int gqa_rope_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                                 const void* dout, const int32_t* positions, double rope_theta,
                                 const int32_t* cu_seqlens, int num_seqs, int total_tokens, int n_q_heads,
                                 int n_kv_heads, int head_dim, int causal, void* dq, void* dk, void* dv,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  struct Disarm {
    ~Disarm() { t_prof_ev[0] = t_prof_ev[1] = t_prof_ev[2] = nullptr; }
  } disarm;
  if (total_tokens < 0 || num_seqs < 0) return GQA_ERR_INVALID_ARG;
  if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return GQA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return GQA_ERR_INVALID_ARG;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return GQA_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED;
  if (n_q_heads / n_kv_heads > BM) return GQA_ERR_UNSUPPORTED;
  if ((long long)total_tokens * n_q_heads * head_dim > (1ll << 40)) return GQA_ERR_UNSUPPORTED;
  if (total_tokens == 0) return GQA_OK;
  if (num_seqs < 1) return GQA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !lse || !dout || !cu_seqlens || !dq || !dk || !dv) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return GQA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(positions) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return GQA_ERR_INVALID_ARG;
  const BwdWsLayout lay = bwd_ws_layout(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim);
  if (lay.max_pairs * (long long)n_kv_heads > 0x7fffffffll) return GQA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < lay.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GQA_ERR_WORKSPACE;

  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return GQA_ERR_CUDA;
  int sm_count = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& ds = g_dev[device];
    if (!ds.init) {
      int major = 0;
      if (cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
          cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
        return GQA_ERR_CUDA;
      if (major != 10) return GQA_ERR_UNSUPPORTED;
      ds.init = true;
    }
    sm_count = ds.sm_count;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  std::lock_guard<std::mutex> lk(g_mu);  // descriptor cache
#define GQA_BWD_CASE(DD)                                                                                        \
  if (head_dim == DD)                                                                                           \
    return launch_bwd<DD>(q, k, v, out, lse, dout, positions, rope_theta, cu_seqlens, num_seqs, total_tokens,  \
                          n_q_heads, n_kv_heads, causal, dq, dk, dv, ws, lay, st, device, sm_count);
  GQA_BWD_CASE(32) GQA_BWD_CASE(64) GQA_BWD_CASE(128)
#undef GQA_BWD_CASE
  return GQA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// QKV projection with the RoPE epilogue

extern "C" size_t gqa_rope_attn_qkv_proj_workspace_size(int total_tokens, int head_dim) {
  if (total_tokens < 0 || (head_dim != 32 && head_dim != 64 && head_dim != 128)) return 0;
  return align_up((size_t)total_tokens * (head_dim / 2) * sizeof(float2), 256) + 256;
}

extern "C" int gqa_rope_attn_qkv_proj(const void* x, const void* w_qkv, const int32_t* positions, double rope_theta,
                                      const int32_t* cu_seqlens, int num_seqs, int total_tokens, int hidden,
                                      int n_q_heads, int n_kv_heads, int head_dim, void* q, void* k, void* v,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  struct Disarm {
    ~Disarm() { t_prof_ev[0] = t_prof_ev[1] = t_prof_ev[2] = nullptr; }
  } disarm;
  if (total_tokens < 0 || num_seqs < 0 || hidden < 1) return GQA_ERR_INVALID_ARG;
  if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return GQA_ERR_INVALID_ARG;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return GQA_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED;
  if (hidden % 8) return GQA_ERR_UNSUPPORTED;  // rows of x and W start on 16-byte boundaries
  if ((long long)(n_q_heads + 2 * n_kv_heads) * head_dim > (1ll << 24)) return GQA_ERR_UNSUPPORTED;
  if ((long long)total_tokens > 65535ll * PJ_BM) return GQA_ERR_UNSUPPORTED;
  if (total_tokens == 0) return GQA_OK;
  if (!x || !w_qkv || !q || !k || !v) return GQA_ERR_INVALID_ARG;
  if (!positions && (!cu_seqlens || num_seqs < 1)) return GQA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v)) return GQA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(positions) & 3u))
    return GQA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < gqa_rope_attn_qkv_proj_workspace_size(total_tokens, head_dim) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GQA_ERR_WORKSPACE;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return GQA_ERR_CUDA;
  int sm_count = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& ds = g_dev[device];
    if (!ds.init) {
      int major = 0;
      if (cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
          cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
        return GQA_ERR_CUDA;
      if (major != 10) return GQA_ERR_UNSUPPORTED;
      ds.init = true;
    }
    sm_count = ds.sm_count;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  std::lock_guard<std::mutex> lk(g_mu);  // descriptor cache
#define GQA_PROJ_CASE(DD)                                                                                   \
  if (head_dim == DD)                                                                                       \
    return launch_qkv_proj<DD>(x, w_qkv, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, hidden, \
                               n_q_heads, n_kv_heads, q, k, v, ws, st, device, sm_count);
  GQA_PROJ_CASE(32) GQA_PROJ_CASE(64) GQA_PROJ_CASE(128)
#undef GQA_PROJ_CASE
  return GQA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------
// Forward with an additive mask

extern "C" int gqa_rope_attn_fwd_masked(const void* q, const void* k, const void* v, const int32_t* positions,
                                        double rope_theta, const int32_t* cu_seqlens, int num_seqs,
                                        int total_tokens, int n_q_heads, int n_kv_heads, int head_dim, int causal,
                                        const void* mask, int mask_len, int mask_ld, void* out, float* lse,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  t_last_launches = 0;
  struct Disarm {
    ~Disarm() { t_prof_ev[0] = t_prof_ev[1] = t_prof_ev[2] = nullptr; }
  } disarm;
  if (total_tokens < 0 || num_seqs < 0) return GQA_ERR_INVALID_ARG;
  if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return GQA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return GQA_ERR_INVALID_ARG;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return GQA_ERR_INVALID_ARG;
  if (mask_len < 1 || mask_ld < mask_len || mask_ld % 8) return GQA_ERR_INVALID_ARG;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return GQA_ERR_UNSUPPORTED;
  if (n_q_heads / n_kv_heads > BM) return GQA_ERR_UNSUPPORTED;
  if ((long long)total_tokens * n_q_heads * head_dim > (1ll << 40)) return GQA_ERR_UNSUPPORTED;
  if (total_tokens == 0) return GQA_OK;
  if (num_seqs < 1) return GQA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !cu_seqlens || !mask) return GQA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(mask))
    return GQA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(positions) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return GQA_ERR_INVALID_ARG;
  const WsLayout lay = ws_layout(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim, false);
  if (lay.max_pairs * (long long)n_kv_heads > 0x7fffffffll) return GQA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < lay.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return GQA_ERR_WORKSPACE;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return GQA_ERR_CUDA;
  int sm_count = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState& ds = g_dev[device];
    if (!ds.init) {
      int major = 0;
      if (cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, device) != cudaSuccess ||
          cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
        return GQA_ERR_CUDA;
      if (major != 10) return GQA_ERR_UNSUPPORTED;
      ds.init = true;
    }
    sm_count = ds.sm_count;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  std::lock_guard<std::mutex> lk(g_mu);  // descriptor cache
#define GQA_MASKED_CASE(DD)                                                                                   \
  if (head_dim == DD)                                                                                         \
    return launch<DD, false>(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,  \
                             n_kv_heads, causal, out, lse, ws, lay, st, device, sm_count, false, mask,        \
                             mask_len, mask_ld);
  GQA_MASKED_CASE(32) GQA_MASKED_CASE(64) GQA_MASKED_CASE(128)
#undef GQA_MASKED_CASE
  return GQA_ERR_UNSUPPORTED;
}
