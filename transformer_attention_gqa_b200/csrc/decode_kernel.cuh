// Decoding step of causal GQA + RoPE attention for sm_100a: one new token per
// sequence against a KV cache.
//
// What it computes ("Attention from Scratch", section "Attention, the math:
// Grouped-Query Attention with RoPE'd Q/K", and its paragraph on the KV
// cache GQA shrinks: one K and one V vector per token and KV head is kept
// for every token so far): the new token of sequence b sits at position
// p = cache_seqlens[b]; its key is rotated at p and appended, with its
// value, as cache row p; its rotated queries attend to cache rows 0..p. It
// is the causal mask's last row of the prefill computation.
//
// The step reads every cached K and V row once, so it is bound by HBM
// bandwidth; the G heads that share a KV head make G multiply-adds per
// cached value, which the tensor cores take (see gqa_decode_tc_kernel).
//
// Kernel 1 (key ranges): one CTA per (key range, KV head, sequence). It
// rotates the G queries of the KV head at p (and the new key, in the CTA
// whose range holds p), then walks its key range in tiles of 128 keys through
// a TMA ring: scores of the tile for the G heads, an online softmax, and the
// weighted sum of V. It leaves (running max, sum, un-normalised output) per
// head in the workspace.
// Kernel 2 (combine): per (sequence, KV head) merges the ranges: out =
// sum_s o_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), lse = (M + log2 L) ln 2.
#pragma once

#include "attn_kernel.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "rope_round.cuh"

namespace gqa {

constexpr int DEC_COMBINE_THREADS = 256;
constexpr int DEC_KT = 128;     // keys per tile (the cache maps' box height)
constexpr int DEC_GMAX = 16;    // query heads per KV head
// The split count aims at about this many CTAs over the batch (measured:
// fewer, longer CTAs amortise the per-CTA RoPE setup).
constexpr int DEC_TARGET_CTAS = 256;

struct DecodeParams {
  const __nv_bfloat16* q;        // [B, nq, d]
  const __nv_bfloat16* k_new;    // [B, nkv, d], not rotated
  const __nv_bfloat16* v_new;    // [B, nkv, d]
  __nv_bfloat16* k_cache;        // [B, Lmax, nkv, d], rotated keys
  __nv_bfloat16* v_cache;        // [B, Lmax, nkv, d]
  const int* cache_seqlens;      // [B]
  float* part_o;                 // [B, nkv, splits, G, d]
  float2* part_ml;               // [B, nkv, splits, G]: (max, sum), scores in log2 units
  __nv_bfloat16* out;            // [B, nq, d]
  float* lse;                    // [nq, B] or null
  double theta;
  double inv_freq[64];           // theta^(-2i/d), i < d/2, evaluated once on the host
  int B, Lmax, nq, nkv, G, splits, kps;  // kps: keys per split, a multiple of DEC_KT
  int test_drop_first_load;      // failure-detection test: never issue the first tile's load (0 normally)
  float scale_log2;              // log2(e) / sqrt(d)
};

// ---------------------------------------------------------------- key ranges on the tensor cores
//
// Keys in the rows of the products. Per 128-key tile of one (sequence, KV
// head) key range:
//   S^T = K Q^T    one M = 128 (keys) x N = 16 (heads) x K = d MMA,
//                  A = the K tile as loaded (K-major), B = the G rotated
//                  query heads in rows 0..G-1 of a 16-row tile (rows past
//                  G zero), scores into tensor memory (lane = key);
//   O^T += V^T P^T one M = 128 (features) x N = 16 x K = 128 (keys) MMA,
//                  A = the V tile read feature-major (MN-major), B = the
//                  bf16 weights P^T (row = head) that the softmax threads
//                  write to shared memory; O^T in tensor memory
//                  (lane = feature; for d < 128 the upper lanes repeat the
//                  lower ones and are not read).
// The G heads of a KV head are the N dimension, so no tensor-core row or
// softmax thread is spent on padding: per tile the tensor core does
// 2 * 128 * 16 * 128 multiply-adds and each softmax thread (one key) G
// exponentials. (The previous form, heads in the rows of an M = 128 tile
// and 64 keys in N, did 32 times the tensor work at G = 4 and ran the
// exponentials of 128 rows, G of them real: 4.2 TB/s at G = 4.)
//
// Online softmax per head over the range's tiles: the tile's max over its
// keys (warp shuffles, then the four warps through shared memory); the
// running max moves only when a score exceeds it by more than 2^8 in p
// (then O^T's column and the thread's partial sum are rescaled); the row
// sum is kept per thread and summed over the keys at the end.
//
// Warps 0-3: RoPE of the queries and the new key, the softmax (one key of
// the tile per thread), the partial results. Warp 4: TMA of the K/V tiles
// through a ring of 192 KB, the fix-up of the range's last tile (the new
// token's row from this CTA, rows past the range zeroed in V so that their
// zero weights meet finite values) and the appended cache row. Warp 5:
// tensor memory and the S^T MMAs; warp 6: the O^T MMAs. (A tcgen05.mma
// issue or a wait blocks its thread: with one issuing thread, O^T(j) and
// the release of tile j's stage waited for tile j + 1 to land, which cost
// the ring a stage.)
constexpr int DTC_KT = DEC_KT;   // keys per tile
constexpr int DTC_N = DEC_GMAX;  // heads per MMA
constexpr int DTC_THREADS = 224;

template <int D_>
struct DtcCfg {
  using A = AttnCfg<D_>;
  static constexpr int D = D_;
  static constexpr int KV_BOX_BYTES = DTC_KT * A::ROWB;      // one box (BOXC features) of a tile
  static constexpr int TILE_BYTES = A::NBOX * KV_BOX_BYTES;  // one K or V tile
  static constexpr int STAGES = 2 * 3 * 32768 / (2 * TILE_BYTES) < 8 ? 2 * 3 * 32768 / (2 * TILE_BYTES) : 8;
  static constexpr int Q_BOX_BYTES = DTC_N * A::ROWB;        // query tile: 16 rows per box
  static constexpr int Q_BYTES = A::NBOX * Q_BOX_BYTES;
  static constexpr int P_BOX_BYTES = DTC_N * 128;            // P^T: 16 rows x 64 keys (128-byte swizzle)
  static constexpr int P_BYTES = 2 * P_BOX_BYTES;            // 128 keys
  static constexpr int OFF_K = 0;                            // [stage] K tiles
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;  // [stage] V tiles
  static constexpr int OFF_Q = OFF_V + STAGES * TILE_BYTES;
  static constexpr int OFF_P = OFF_Q + Q_BYTES;              // [2] P^T buffers
  static constexpr int OFF_CS = OFF_P + 2 * P_BYTES;         // uint2 [D/4]: bf16x2 (cos, sin) at pos
  static constexpr int OFF_NEW = OFF_CS + D * 2;             // bf16 [2][D]: rotated new key, value
  static constexpr int OFF_RED = OFF_NEW + 2 * D * 2;        // float [3][4 warps][16]: maxima x2, sums
  static constexpr int OFF_BAR = OFF_RED + 3 * 4 * DTC_N * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;    // + barriers + alignment slack
  static constexpr uint32_t S_COL = 0;                       // two 16-column S^T buffers
  static constexpr uint32_t O_COL = 2 * DTC_N;               // O^T
  static constexpr uint32_t TMEM_COLS = 64;
  // bf16 x bf16 -> fp32, M = 128, N = 16; S^T: A and B K-major; O^T: A MN-major
  static constexpr uint32_t IDESC_S =
      (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(DTC_N >> 3) << 17) | ((uint32_t)(DTC_KT >> 4) << 24);
  static constexpr uint32_t IDESC_O = IDESC_S | (1u << 15);
  // V^T's M = 128 features span 128 / BOXC swizzle atoms; for d < 128 they
  // all start at the same box (stride 0), so the upper lanes repeat d.
  static constexpr uint32_t V_LBO = D == 128 ? (uint32_t)KV_BOX_BYTES : 0u;
  static_assert(DTC_KT == 128 && DTC_N == 16, "MMA shape M = 128, N = 16");
  static_assert(OFF_V % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_P % 1024 == 0 && TILE_BYTES % 1024 == 0,
                "swizzle atoms 1024-aligned");
  static_assert(O_COL + DTC_N <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct DtcBarriers {
  uint64_t full[8], empty[8];
  uint64_t fixed;     // the range's last tile patched in shared memory
  uint64_t q_ready;   // query tile, new key and value written (128 arrivals)
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_full, drain;
  uint64_t xchg[2];   // per-head tile maxima of the four softmax warps published (by tile parity)
  uint64_t lsum;      // per-head partial sums of the four softmax warps published
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(DtcBarriers) <= 256, "barrier area");

__device__ __forceinline__ void dtc_softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int D, int NH>
__global__ void __launch_bounds__(DTC_THREADS, 1)
    gqa_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const DecodeParams p) {
  using C = DtcCfg<D>;
  using A = AttnCfg<D>;
  constexpr int HALF = D / 2;
  constexpr int ST = C::STAGES;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = p.G;  // <= NH
  static_assert(NH % 4 == 0 && NH <= DTC_N, "heads per thread");
  const int pos = __ldg(p.cache_seqlens + b);
  if (pos < 0 || pos >= p.Lmax) {  // the combine kernel skips this sequence too
    if (threadIdx.x == 0 && split == 0 && h == 0) atomicCAS(&g_status, 0, kStatusBadSeqlens);
    return;
  }
  const int k0 = split * p.kps;
  const int k1 = min(k0 + p.kps, pos + 1);
  const size_t part = ((size_t)b * p.nkv + h) * p.splits + split;
  if (k0 >= k1) {  // no visible key in this range (the whole CTA, before any barrier or TMEM use)
    for (int i = threadIdx.x; i < G; i += DTC_THREADS) p.part_ml[part * G + i] = make_float2(-INFINITY, 0.f);
    return;
  }
  const int ntiles = (k1 - k0 + DTC_KT - 1) / DTC_KT;
  const bool has_new = pos >= k0 && pos < k1;
  const int last_start = k0 + (ntiles - 1) * DTC_KT;
  const int last_valid = k1 - last_start;  // keys of the last tile inside the range, 1..128
  const bool fix_last = has_new || last_valid < DTC_KT;

  extern __shared__ uint8_t dtc_smem_raw[];
  uint8_t* smem = dtc_smem_raw + ((1024u - (ptx::smem_u32(dtc_smem_raw) & 1023u)) & 1023u);
  DtcBarriers* bars = reinterpret_cast<DtcBarriers*>(smem + C::OFF_BAR);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  auto B = [&](uint64_t& x) { return ptx::smem_u32(&x); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      ptx::mbar_init(B(bars->full[s]), 1);
      ptx::mbar_init(B(bars->empty[s]), 1);
    }
    ptx::mbar_init(B(bars->fixed), 1);
    ptx::mbar_init(B(bars->q_ready), 128);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(B(bars->s_full[s]), 1);
      ptx::mbar_init(B(bars->p_full[s]), 128);
      ptx::mbar_init(B(bars->pv_done[s]), 1);
    }
    ptx::mbar_init(B(bars->o_full), 1);
    ptx::mbar_init(B(bars->drain), 2);  // one commit per MMA-issuing thread
    for (int s = 0; s < 2; ++s) ptx::mbar_init(B(bars->xchg[s]), 4);
    ptx::mbar_init(B(bars->lsum), 4);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
  }
  if (warp == 5) {
    ptx::tmem_alloc(ptx::smem_u32(&bars->tmem_base), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int row0 = b * p.Lmax + k0;  // key coordinate of the range's first row in the maps

  if (warp == 4) {
    // ------------------------------------------------------------ TMA, last-tile fix-up, appended row
    int issued = 0;
    bool ok = true;
    if (lane == 0) {
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % ST;
        // (a spinning wait: the ring is three tiles deep, so a sleeping
        // producer's late refill would stall the stream)
        if (!(ok = bwait(B(bars->empty[st]), ((t / ST) & 1) ^ 1, abort_flag))) break;
        ptx::mbar_arrive_expect_tx(B(bars->full[st]), 2u * C::TILE_BYTES);
        if (!(p.test_drop_first_load && t == 0)) {
          for (int bx = 0; bx < A::NBOX; ++bx) {
            ptx::tma_load_3d(sbase + C::OFF_K + st * C::TILE_BYTES + bx * C::KV_BOX_BYTES, &tmK, B(bars->full[st]),
                             bx * A::BOXC, h, row0 + t * DTC_KT);
            ptx::tma_load_3d(sbase + C::OFF_V + st * C::TILE_BYTES + bx * C::KV_BOX_BYTES, &tmV, B(bars->full[st]),
                             bx * A::BOXC, h, row0 + t * DTC_KT);
          }
          ++issued;
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    const int tl = ntiles - 1, stl = tl % ST;
    if (ok && fix_last) {
      // the last tile: the new token's rotated key and value in row pos, and
      // V rows past the range zero (their weights are zero; the cache rows
      // there may hold anything)
      ok = __all_sync(0xffffffffu, bwait(B(bars->full[stl]), (tl / ST) & 1, abort_flag) &&
                                       bwait(B(bars->q_ready), 0, abort_flag));
      if (ok) {
        uint8_t* kt = smem + C::OFF_K + stl * C::TILE_BYTES;
        uint8_t* vt = smem + C::OFF_V + stl * C::TILE_BYTES;
        const __nv_bfloat16* knew = reinterpret_cast<const __nv_bfloat16*>(smem + C::OFF_NEW);
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        if (has_new) {
          const int r = pos - last_start;
          for (int c = lane; c < CPR; c += 32) {
            const int bx = c / (A::BOXC / 8), ch = c % (A::BOXC / 8);
            const uint32_t off = bx * C::KV_BOX_BYTES + swz(r * A::ROWB + ch * 16, A::SWZ_MASK);
            *reinterpret_cast<uint4*>(kt + off) = *reinterpret_cast<const uint4*>(knew + c * 8);
            *reinterpret_cast<uint4*>(vt + off) = *reinterpret_cast<const uint4*>(knew + D + c * 8);
          }
        }
        for (int i = lane; i < (DTC_KT - last_valid) * CPR; i += 32) {
          const int r = last_valid + i / CPR, c = i % CPR;
          const int bx = c / (A::BOXC / 8), ch = c % (A::BOXC / 8);
          *reinterpret_cast<uint4*>(vt + bx * C::KV_BOX_BYTES + swz(r * A::ROWB + ch * 16, A::SWZ_MASK)) =
              make_uint4(0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(B(bars->fixed));
      }
    }
    if (ok) {
      // all MMAs done: every load of this CTA has landed; append the new row
      ok = __all_sync(0xffffffffu, bwait_lazy(B(bars->o_full), 0, abort_flag));
      if (ok && has_new) {
        const size_t row = (((size_t)b * p.Lmax + pos) * p.nkv + h) * D;
        const uint4* kv4 = reinterpret_cast<const uint4*>(smem + C::OFF_NEW);
        for (int i = lane; i < D / 8; i += 32) {
          reinterpret_cast<uint4*>(p.k_cache + row)[i] = kv4[i];
          reinterpret_cast<uint4*>(p.v_cache + row)[i] = kv4[D / 8 + i];
        }
      }
    }
    if (!ok && lane == 0) {  // every copy issued lands before the CTA exits
      const int first = p.test_drop_first_load ? 1 : 0;
      for (int t = first; t < first + issued; ++t) drain_wait(B(bars->full[t % ST]), (t / ST) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ S^T issuer
    if (lane == 0) {
      const uint64_t dq = umma_desc(sbase + C::OFF_Q, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t dk0 = umma_desc(sbase + C::OFF_K, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t stage = (uint64_t)(C::TILE_BYTES >> 4);
      bool ok = bwait(B(bars->q_ready), 0, abort_flag);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int sb = j & 1, st = j % ST;
        // S buffer sb held S^T(j - 2): the softmax read it before releasing P^T(j - 2)
        if (j >= 2 && !(ok = bwait(B(bars->p_full[sb]), ((j - 2) >> 1) & 1, abort_flag))) break;
        if (!(ok = (j == ntiles - 1 && fix_last) ? bwait(B(bars->fixed), 0, abort_flag)
                                                 : bwait(B(bars->full[st]), (j / ST) & 1, abort_flag)))
          break;
        ptx::tc_fence_after();
        const uint64_t dk = dk0 + st * stage;
#pragma unroll
        for (int kk = 0; kk < A::KSTEPS_S; ++kk) {
          const uint32_t off_k = (kk / A::STEPS_PER_BOX) * C::KV_BOX_BYTES + (kk % A::STEPS_PER_BOX) * 32;
          const uint32_t off_q = (kk / A::STEPS_PER_BOX) * C::Q_BOX_BYTES + (kk % A::STEPS_PER_BOX) * 32;
          ptx::mma_ss(tmem + C::S_COL + sb * DTC_N, dk + (uint64_t)(off_k >> 4), dq + (uint64_t)(off_q >> 4),
                      C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(B(bars->s_full[sb]));
      }
      // all tensor-core work issued here has finished before TMEM is freed
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ O^T issuer
    if (lane == 0) {
      const uint64_t dv0 = umma_desc(sbase + C::OFF_V, C::V_LBO, A::SBO, A::UMMA_LAYOUT);
      const uint64_t dp0 = umma_desc(sbase + C::OFF_P, 16, 1024, 2);  // P^T: 128-byte swizzle
      const uint64_t stage = (uint64_t)(C::TILE_BYTES >> 4);
      bool ok = true;
      for (int j = 0; ok && j < ntiles; ++j) {
        const int sb = j & 1, st = j % ST;
        if (!(ok = bwait(B(bars->p_full[sb]), (j >> 1) & 1, abort_flag))) break;
        ptx::tc_fence_after();
        // O^T (+)= V^T P^T: 128 keys in 8 K-steps of 16
#pragma unroll
        for (int kk = 0; kk < DTC_KT / 16; ++kk) {
          const uint32_t off_p = sb * C::P_BYTES + (kk / 4) * C::P_BOX_BYTES + (kk % 4) * 32;
          ptx::mma_ss(tmem + C::O_COL, dv0 + st * stage + (uint64_t)((kk * 16 * A::ROWB) >> 4),
                      dp0 + (uint64_t)(off_p >> 4), C::IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(B(bars->pv_done[sb]));
        // the stage's K was read by S^T(j), issued and finished before P^T(j) existed
        ptx::mma_commit(B(bars->empty[st]));
      }
      if (ok) ptx::mma_commit(B(bars->o_full));
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
  } else {
    // ------------------------------------------------------------ RoPE, softmax, partial results
    const int tid = threadIdx.x;  // 0..127 == tile row (key, then feature) == TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    uint2* cs = reinterpret_cast<uint2*>(smem + C::OFF_CS);
    __nv_bfloat16* knew = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_NEW);
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [3][4][16], 16-byte aligned
    // zero query tile and both P^T buffers (rows past G stay zero); bf16x2
    // (cos, sin) words of frequencies (2j, 2j + 1) at pos (float64 angle,
    // rounded to fp32, then to bf16 as in the prefill)
    for (int i = tid; i < (C::Q_BYTES + 2 * C::P_BYTES) / 16; i += 128)
      reinterpret_cast<uint4*>(smem + C::OFF_Q)[i] = make_uint4(0, 0, 0, 0);
    for (int j = tid; j < HALF / 2; j += 128) {
      float c[2], sn[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        double sd, cd;
        sincos((double)pos * p.inv_freq[2 * j + e], &sd, &cd);
        c[e] = (float)cd;
        sn[e] = (float)sd;
      }
      cs[j] = make_uint2(bf16x2_rn(c[0], c[1]), bf16x2_rn(sn[0], sn[1]));
    }
    dtc_softmax_sync();
    // rotated queries into rows 0..G-1 of the query tile, and the new key (if
    // this range holds pos), two frequencies per item, in the prefill's bf16
    // rotation
    constexpr int NPAIR = HALF / 2;
    const int nrot = (G + (has_new ? 1 : 0)) * NPAIR;
    for (int it = tid; it < nrot; it += 128) {
      const int hg = it / NPAIR, i = 2 * (it - hg * NPAIR);
      const uint2 c = cs[i / 2];
      const __nv_bfloat16* src =
          hg < G ? p.q + ((size_t)b * p.nq + h * G + hg) * D : p.k_new + ((size_t)b * p.nkv + h) * D;
      uint32_t lo, hi;
      rope_bf16x2(*reinterpret_cast<const uint32_t*>(src + i), *reinterpret_cast<const uint32_t*>(src + i + HALF),
                  c.x, c.y, lo, hi);
      if (hg < G) {
        const int cl = i, chh = i + HALF;
        *reinterpret_cast<uint32_t*>(smem + C::OFF_Q + (cl / A::BOXC) * C::Q_BOX_BYTES +
                                     swz(hg * A::ROWB + (cl % A::BOXC) * 2, A::SWZ_MASK)) = lo;
        *reinterpret_cast<uint32_t*>(smem + C::OFF_Q + (chh / A::BOXC) * C::Q_BOX_BYTES +
                                     swz(hg * A::ROWB + (chh % A::BOXC) * 2, A::SWZ_MASK)) = hi;
      } else {
        *reinterpret_cast<uint32_t*>(knew + i) = lo;
        *reinterpret_cast<uint32_t*>(knew + i + HALF) = hi;
      }
    }
    if (has_new)
      for (int i = tid; i < D; i += 128) knew[D + i] = p.v_new[((size_t)b * p.nkv + h) * D + i];
    ptx::fence_proxy_async_smem();
    ptx::mbar_arrive(B(bars->q_ready));

    const float sl2 = p.scale_log2;
    const float thr = 8.f / sl2;  // raw-score growth that forces an O rescale (2^8 in p)
    // NH >= G heads per thread, without branches on G: the query rows past G
    // are zero, so those heads' scores are 0, their weights land in P^T rows
    // and O^T columns that nothing reads, and their max never moves
    float m[NH], l[NH];
#pragma unroll
    for (int g = 0; g < NH; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
    }
    // this thread's key in the P^T tile: box, and byte offset in row 0
    uint8_t* const p_base = smem + C::OFF_P + (tid / 64) * C::P_BOX_BYTES;
    const uint32_t p_col = (uint32_t)(tid % 64) * 2;
    bool ok = true;
    uint32_t sv[DTC_N];
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, bwait(B(bars->s_full[sb]), (j >> 1) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      ptx::tmem_ld16(trow + C::S_COL + sb * DTC_N, sv);
      ptx::tmem_wait_ld();
      float s[NH], mx[NH];
#pragma unroll
      for (int g = 0; g < NH; ++g) s[g] = __uint_as_float(sv[g]);
      if (j == ntiles - 1 && k0 + j * DTC_KT + tid >= k1) {  // keys past the range (last tile only)
#pragma unroll
        for (int g = 0; g < NH; ++g) s[g] = -INFINITY;
      }
      // the tile's max per head over its 128 keys: shuffles interleaved over
      // the heads, then each warp publishes its maxima and waits (bounded)
      // for the other three
#pragma unroll
      for (int g = 0; g < NH; ++g) mx[g] = s[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int g = 0; g < NH; ++g) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
      }
      float4* rx = reinterpret_cast<float4*>(red + sb * 4 * DTC_N);
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < NH; g += 4) rx[(warp * DTC_N + g) / 4] = make_float4(mx[g], mx[g + 1], mx[g + 2], mx[g + 3]);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(B(bars->xchg[sb]));
      ok = __all_sync(0xffffffffu, bwait(B(bars->xchg[sb]), (j >> 1) & 1, abort_flag));
      if (!ok) break;
#pragma unroll
      for (int g = 0; g < NH; g += 4) {
        const float4 a = rx[g / 4], b2 = rx[(DTC_N + g) / 4], c = rx[(2 * DTC_N + g) / 4], d4 = rx[(3 * DTC_N + g) / 4];
        mx[g] = fmaxf(fmaxf(a.x, b2.x), fmaxf(c.x, d4.x));
        mx[g + 1] = fmaxf(fmaxf(a.y, b2.y), fmaxf(c.y, d4.y));
        mx[g + 2] = fmaxf(fmaxf(a.z, b2.z), fmaxf(c.z, d4.z));
        mx[g + 3] = fmaxf(fmaxf(a.w, b2.w), fmaxf(c.w, d4.w));
      }
      // the running max moves when a head's tile max exceeds it by more than
      // the threshold (every thread sees the same maxima: uniform branches)
      bool need_any = false;
      float alpha[NH];
#pragma unroll
      for (int g = 0; g < NH; ++g) {
        alpha[g] = 1.f;
        if (mx[g] > m[g] + thr) {
          if (j > 0) {
            alpha[g] = ptx::ex2((m[g] - mx[g]) * sl2);
            need_any = true;
          }
          m[g] = mx[g];
        }
      }
      if (need_any) {
        // O^T holds the sum up to the previous tile: wait for PV(j - 1), then
        // scale the heads' columns of this thread's feature row
        const int jp = j - 1;
        ok = __all_sync(0xffffffffu, bwait(B(bars->pv_done[jp & 1]), (jp >> 1) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        uint32_t ov[DTC_N];
        ptx::tmem_ld16(trow + C::O_COL, ov);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < NH; ++g) ov[g] = __float_as_uint(__uint_as_float(ov[g]) * alpha[g]);
        ptx::tmem_st16(trow + C::O_COL, ov);
        ptx::tmem_wait_st();
#pragma unroll
        for (int g = 0; g < NH; ++g) l[g] *= alpha[g];
      }
      // P^T buffer sb was read by PV(j - 2)
      if (j >= 2) {
        const int jq = j - 2;
        ok = __all_sync(0xffffffffu, bwait(B(bars->pv_done[sb]), (jq >> 1) & 1, abort_flag));
        if (!ok) break;
      }
      uint8_t* pt = p_base + sb * C::P_BYTES;
#pragma unroll
      for (int g = 0; g < NH; ++g) {
        const float pg = ptx::ex2((s[g] - m[g]) * sl2);
        l[g] += pg;
        *reinterpret_cast<__nv_bfloat16*>(pt + swz(g * 128 + p_col, 7)) = __float2bfloat16_rn(pg);
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(B(bars->p_full[sb]));
    }
    if (ok) ok = __all_sync(0xffffffffu, bwait(B(bars->o_full), 0, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
      // partial sums per head over this range's keys
      float* rl = red + 2 * 4 * DTC_N;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int g = 0; g < NH; ++g) l[g] += __shfl_xor_sync(0xffffffffu, l[g], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < NH; ++g) rl[warp * DTC_N + g] = l[g];
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(B(bars->lsum));
      uint32_t ov[DTC_N];
      ptx::tmem_ld16(trow + C::O_COL, ov);
      ptx::tmem_wait_ld();
      if (tid < D) {
        float* po = p.part_o + part * G * D + tid;
#pragma unroll
        for (int g = 0; g < NH; ++g)
          if (g < G) po[(size_t)g * D] = __uint_as_float(ov[g]);
      }
      ok = __all_sync(0xffffffffu, bwait(B(bars->lsum), 0, abort_flag));
      if (ok && tid < G) {
        float mg = 0.f;
#pragma unroll
        for (int g = 0; g < NH; ++g)
          if (g == tid) mg = m[g];
        const float lg = rl[tid] + rl[DTC_N + tid] + rl[2 * DTC_N + tid] + rl[3 * DTC_N + tid];
        p.part_ml[part * G + tid] = make_float2(mg * sl2, lg);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Merge of the key ranges of one (sequence, KV head); threads over
// (head, column).
__global__ void __launch_bounds__(DEC_COMBINE_THREADS) gqa_decode_combine_kernel(const DecodeParams p, int D) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = p.G;
  const int pos = __ldg(p.cache_seqlens + b);
  if (pos < 0 || pos >= p.Lmax) return;
  const int used = min(p.splits, pos / p.kps + 1);  // ranges holding a visible key
  const size_t part0 = ((size_t)b * p.nkv + h) * p.splits;
  for (int u = threadIdx.x; u < G * D; u += DEC_COMBINE_THREADS) {
    const int g = u / D, d = u - g * D;
    float M = -INFINITY;
    for (int s = 0; s < used; ++s) M = fmaxf(M, p.part_ml[(part0 + s) * G + g].x);
    float L = 0.f, acc = 0.f;
    for (int s = 0; s < used; ++s) {
      const float2 ml = p.part_ml[(part0 + s) * G + g];
      if (ml.x == -INFINITY) continue;
      const float w = ptx::ex2(ml.x - M);
      L = fmaf(ml.y, w, L);
      acc = fmaf(p.part_o[((part0 + s) * G + g) * D + d], w, acc);
    }
    const int hq = h * G + g;
    p.out[((size_t)b * p.nq + hq) * D + d] = __float2bfloat16_rn(acc / L);
    if (d == 0 && p.lse) p.lse[(size_t)hq * p.B + b] = (M + __log2f(L)) * 0.69314718055994531f;
  }
}

}  // namespace gqa
