// Backward of the fused causal GQA + RoPE attention (sm_100a).
//
// Gradients of sum(dout * out) with respect to q, k and v, for the forward of
// attn_kernel.cuh ("Attention from Scratch", section "Attention, the math";
// the chain rule through its steps, using the forward's fp32 log-sum-exp):
//   P   = exp(S - lse),  S = rope(q) rope(k)^T / sqrt(d)  (causal mask)
//   dV  = P^T dO                      (summed over the G heads of a group)
//   dP  = dO V^T
//   dS  = P * (dP - Delta),           Delta_i = sum_c dO_ic O_ic
//   dQ' = dS K' / sqrt(d),  dK' = dS^T Q' / sqrt(d)   (summed over the group)
//   dq  = rope^T(dQ'),      dk  = rope^T(dK')  (rotation by the negative angle)
// The rotated operands Q', K' are the forward's, rounded to bf16 exactly as
// the forward rounds them; the rounding passes gradients straight through.
//
// Four launches:
//  * gqa_bwd_prep_kernel: the (sequence, key-tile) schedule and the
//    (sequence, query-tile) schedule, longest first; each token's (cos, sin)
//    row; K' head-major and Q' [N, n_q, d] in the workspace; Delta and
//    lse * log2(e) per (head, token).
//  * gqa_attn_bwd_kernel: dK' and dV, one CTA per (KV head, 128-key tile).
//    It loops over the packed query tiles (tq tokens x G heads = 128 rows,
//    the forward's packing) that the causal mask lets see its keys. Per
//    query tile, four tensor-core products:
//        S^T  = K' Q'^T   (M = keys, N = packed q rows, K = d)  SS
//        dP^T = V dO^T    (M = keys, N = packed q rows, K = d)  SS
//        dV  += P^T dO    (A = P^T from TMEM, bf16)             TS
//        dK' += dS^T Q'   (A = dS^T from shared memory)         SS
//    P^T and dS^T are formed by one thread per key row (a TMEM lane); dV
//    and dK' stay in TMEM over the whole loop and are written once.
//  * gqa_attn_bwd_q_kernel (bwd_q_kernel.cuh): dQ' = dS K', one CTA per
//    (query tile, KV head), summed over its key tiles in TMEM and written
//    once (P and dP recomputed there).
//  * gqa_bwd_dq_kernel: dq = rope^T(dQ' / sqrt(d)) -> bf16.
//
// Warp roles of the key-tile kernel (512 threads):
//   warp 0      TMA: K', V once; Q', dO per query tile (two stages each);
//               lse * log2(e) and Delta of the tile's 128 rows into shared
//               memory (all 32 lanes)
//   warp 1      TMEM allocator; one thread issues every MMA
//   warps 4-11  P^T and dS^T, one key row per thread: warps 4-7 the packed
//               query columns [0, 64), warps 8-11 [64, 128)
//   warps 12-15 at the end dV and dK' -> bf16
// Tensor memory (512 columns): [0,128) S^T, then P^T (bf16 pairs: packed
// columns [0, 64) over S columns [0, 32), [64, 128) over [64, 96), so each
// warpgroup overwrites only S columns it has read); [128,256) dP^T;
// [256, 256+d) dV; [256+d, 256+2d) dK'.
#pragma once

#include "attn_kernel.cuh"
#include "common.cuh"
#include "prep_kernel.cuh"
#include "ptx.cuh"
#include "rope_round.cuh"

namespace gqa {

constexpr int BWD_THREADS = 512;
// Register split (launch: 512 threads x 128, the most __launch_bounds__(512, 1)
// allows): loaders and MMA issuer 104, the two P^T/dS^T warpgroups (half of
// the packed query columns each) 136, dQ'/dK'/dV epilogue 136.
constexpr int BWD_LAUNCH_REGS = 128;
constexpr int BWD_REG_PRODUCER = 104;
constexpr int BWD_REG_SOFTMAX = 136;
constexpr int BWD_REG_READOUT = 136;
static_assert(BWD_REG_PRODUCER * 128 + 2 * BWD_REG_SOFTMAX * 128 + BWD_REG_READOUT * 128 <= BWD_LAUNCH_REGS * BWD_THREADS,
              "register split exceeds the launch's registers");

// Workspace regions of the backward (byte offsets from the 256-byte aligned base).
struct BwdWsLayout {
  size_t header;   // int[16]: [0] number of (sequence, key-tile) pairs
  size_t seq_pfx;  // int[num_seqs + 1]
  size_t pairs;    // int2[max_pairs]: (sequence, key tile), decreasing cost
  size_t table;    // float2[N * d/2]: (cos, sin)
  size_t kws;      // bf16[n_kv][N][d]: K'
  size_t qws;      // bf16[N][n_q][d]: Q'
  size_t lse2;     // float[n_q][N]: lse * log2(e)
  size_t delta;    // float[n_q][N]: Delta
  size_t dq_acc;   // float[N][n_q][d]: dQ' (written once per row by the query-tile kernel)
  size_t qheader;  // int[16]: [0] number of (sequence, query tile) pairs
  size_t qseq_pfx; // int[num_seqs + 1]
  size_t qpairs;   // int2[max_qpairs]: (sequence, query tile), decreasing cost
  size_t total;
  long long max_pairs, max_qpairs;
};

__host__ inline BwdWsLayout bwd_ws_layout(int num_seqs, int N, int nq, int nkv, int d) {
  BwdWsLayout w{};
  w.max_pairs = (long long)(N + BN - 1) / BN + num_seqs;
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  w.header = take(16 * sizeof(int));
  w.seq_pfx = take((size_t)(num_seqs + 1) * sizeof(int));
  w.pairs = take((size_t)w.max_pairs * 8);
  w.table = take((size_t)N * (d / 2) * 8);
  w.kws = take((size_t)nkv * N * d * 2);
  w.qws = take((size_t)N * nq * d * 2);
  w.lse2 = take((size_t)nq * N * 4);
  w.delta = take((size_t)nq * N * 4);
  w.dq_acc = take((size_t)N * nq * d * 4);
  const int tq = tokens_per_tile(nq / nkv);
  w.max_qpairs = (long long)(N + tq - 1) / tq + num_seqs;
  w.qheader = take(16 * sizeof(int));
  w.qseq_pfx = take((size_t)(num_seqs + 1) * sizeof(int));
  w.qpairs = take((size_t)w.max_qpairs * 8);
  w.total = off;
  return w;
}

struct BwdPrepParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* out;
  const __nv_bfloat16* dout;
  const float* lse;
  const int* positions;
  const int* cu;
  int N, num_seqs, nq, nkv, tq, causal;
  double inv_freq[64];  // theta^(-2i/d), i < d/2
  int* header;
  int* seq_pfx;
  int2* pairs;
  float2* table;
  __nv_bfloat16* kws;
  __nv_bfloat16* qws;
  float* lse2;
  float* delta;
  int* qheader;
  int* qseq_pfx;
  int2* qpairs;
};

struct BwdParams {
  const int* cu;
  const int* header;
  const int2* pairs;
  const float2* table;
  const float* lse2;
  const float* delta;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int N, nq, nkv, G, tq, causal;
  float scale;       // 1 / sqrt(d)
  float scale_log2;  // log2(e) / sqrt(d)
};

// ------------------------------------------------------------------ prologue

// Query tiles that see key tile l of a sequence of length L: with the causal
// mask, those whose last token is at or after the tile's first key.
__device__ __forceinline__ int kv_tile_cost(int L, int l, int tq, int causal) {
  const int qt = (L + tq - 1) / tq;
  return causal ? qt - (l * BN) / tq : qt;
}

// Block 0: checks cu_seqlens and lists every (sequence, key tile) pair in
// decreasing cost order (counting sort over cost bins).
__device__ void build_kv_schedule(const BwdPrepParams& p) {
  __shared__ int s_scan[PREP_THREADS];
  __shared__ int s_bins[SCHED_BINS];
  const int tid = threadIdx.x;
  const int ns = p.num_seqs;
  const int* cu = p.cu;
  int* pfx = p.seq_pfx;

  int bad = 0;
  for (int s = tid; s < ns; s += PREP_THREADS)
    if (__ldg(cu + s + 1) < __ldg(cu + s)) bad = 1;
  if (tid == 0 && (__ldg(cu) != 0 || __ldg(cu + ns) != p.N)) bad = 1;
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      set_status(kStatusBadSeqlens);
      p.header[0] = 0;
    }
    return;
  }

  int running = 0;
  for (int base = 0; base < ns; base += PREP_THREADS) {
    const int s = base + tid;
    int nt = 0;
    if (s < ns) nt = (__ldg(cu + s + 1) - __ldg(cu + s) + BN - 1) / BN;
    int tot;
    const int ex = block_exclusive_scan(nt, s_scan, tot);
    if (s < ns) pfx[s] = running + ex;
    running += tot;
  }
  if (tid == 0) pfx[ns] = running;
  const int P = running;

  for (int i = tid; i < SCHED_BINS; i += PREP_THREADS) s_bins[i] = 0;
  __syncthreads();  // pfx and s_bins visible to the whole block

  for (int q = tid; q < P; q += PREP_THREADS) {
    const int s = upper_index_plain(pfx, ns, q);
    const int L = __ldg(cu + s + 1) - __ldg(cu + s);
    const int c = min(kv_tile_cost(L, q - pfx[s], p.tq, p.causal), SCHED_BINS - 1);
    atomicAdd(&s_bins[c], 1);
  }
  __syncthreads();

  constexpr int PER = SCHED_BINS / PREP_THREADS;
  int local[PER];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    local[i] = s_bins[SCHED_BINS - 1 - (tid * PER + i)];
    sum += local[i];
  }
  int tot;
  int off = block_exclusive_scan(sum, s_scan, tot);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    s_bins[SCHED_BINS - 1 - (tid * PER + i)] = off;
    off += local[i];
  }
  __syncthreads();

  for (int q = tid; q < P; q += PREP_THREADS) {
    const int s = upper_index_plain(pfx, ns, q);
    const int l = q - pfx[s];
    const int L = __ldg(cu + s + 1) - __ldg(cu + s);
    const int c = min(kv_tile_cost(L, l, p.tq, p.causal), SCHED_BINS - 1);
    const int slot = atomicAdd(&s_bins[c], 1);
    p.pairs[slot] = make_int2(s, l);
  }
  if (tid == 0) p.header[0] = P;
}

// (cos, sin) row of every token (fp32, for the transposed rotations of dq
// and dk), K' head-major and Q' token-major in the forward's bf16 rotation
// (rope_bf16x2 in rope_round.cuh), so that the recomputed scores are the
// forward's. One thread per (token, pair of frequencies).
template <int D>
__device__ void bwd_rope_rows(const BwdPrepParams& p, int block, int nblocks) {
  constexpr int HALF = D / 2;
  constexpr int PAIRS = HALF / 2;
  const long long total = (long long)p.N * PAIRS;
  for (long long idx = (long long)block * PREP_THREADS + threadIdx.x; idx < total;
       idx += (long long)nblocks * PREP_THREADS) {
    const int t = (int)(idx / PAIRS);
    const int i = (int)(idx % PAIRS) * 2;
    int pos;
    if (p.positions) {
      pos = __ldg(p.positions + t);
    } else {
      const int s = upper_index(p.cu, p.num_seqs, t);
      pos = t - __ldg(p.cu + s);
    }
    float c[2], sn[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      double sd, cd;
      sincos((double)pos * p.inv_freq[i + e], &sd, &cd);
      c[e] = (float)cd;
      sn[e] = (float)sd;
    }
    *reinterpret_cast<float4*>(p.table + (size_t)t * HALF + i) = make_float4(c[0], sn[0], c[1], sn[1]);
    const uint32_t c2 = bf16x2_rn(c[0], c[1]), s2 = bf16x2_rn(sn[0], sn[1]);
    // heads in groups of HB: the group's words are all loaded before any is
    // stored, so one memory latency covers the group
    constexpr int HB = 8;
    auto rotate_heads = [&](const __nv_bfloat16* src, int src_stride, __nv_bfloat16* dst, size_t dst_stride,
                            int nh) {
      for (int h0 = 0; h0 < nh; h0 += HB) {
        uint32_t wl[HB], wh[HB];
#pragma unroll
        for (int u = 0; u < HB; ++u) {
          if (h0 + u < nh) {
            const __nv_bfloat16* r = src + (size_t)(h0 + u) * src_stride;
            wl[u] = __ldg(reinterpret_cast<const unsigned int*>(r + i));
            wh[u] = __ldg(reinterpret_cast<const unsigned int*>(r + i + HALF));
          }
        }
#pragma unroll
        for (int u = 0; u < HB; ++u) {
          if (h0 + u < nh) {
            uint32_t ol, oh;
            rope_bf16x2(wl[u], wh[u], c2, s2, ol, oh);
            __nv_bfloat16* w = dst + (size_t)(h0 + u) * dst_stride;
            *reinterpret_cast<uint32_t*>(w + i) = ol;
            *reinterpret_cast<uint32_t*>(w + i + HALF) = oh;
          }
        }
      }
    };
    rotate_heads(p.k + (size_t)t * p.nkv * D, D, p.kws + (size_t)t * D, (size_t)p.N * D, p.nkv);
    rotate_heads(p.q + (size_t)t * p.nq * D, D, p.qws + (size_t)t * p.nq * D, (size_t)D, p.nq);
  }
}

// Delta = rowsum(dout * out) and lse * log2(e) per (token, head) row: d/8
// lanes per row, 16-byte loads, shuffle reduction.
template <int D>
__device__ void bwd_delta_rows(const BwdPrepParams& p, int block, int nblocks) {
  constexpr int LPR = D / 8;
  constexpr int RPW = 32 / LPR;
  constexpr int WPB = PREP_THREADS / 32;
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)p.N * p.nq;
  const long long stride = (long long)nblocks * WPB * RPW;
  for (long long base = ((long long)block * WPB + (threadIdx.x >> 5)) * RPW; base < rows; base += stride) {
    const long long row = base + lane / LPR;
    const int ch = lane % LPR;
    float acc = 0.f;
    if (row < rows) {
      const uint4 a = *reinterpret_cast<const uint4*>(p.out + row * D + ch * 8);
      const uint4 b = *reinterpret_cast<const uint4*>(p.dout + row * D + ch * 8);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(a2[e]);
        const float2 fb = __bfloat1622float2(b2[e]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (row < rows && ch == 0) {
      const int t = (int)(row / p.nq);
      const int h = (int)(row - (long long)t * p.nq);
      const size_t at = (size_t)h * p.N + t;
      p.delta[at] = acc;
      p.lse2[at] = p.lse[at] * 1.4426950408889634f;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(PREP_THREADS) gqa_bwd_prep_kernel(const BwdPrepParams p) {
  if (blockIdx.x == 0) {
    build_kv_schedule(p);
    return;
  }
  if (blockIdx.x == 1) {
    // the query-tile schedule of gqa_attn_bwd_q_kernel: the forward's (sequence,
    // q-tile) pairs, longest first
    PrepParams q{};
    q.cu = p.cu;
    q.N = p.N;
    q.num_seqs = p.num_seqs;
    q.tq = p.tq;
    q.causal = p.causal;
    q.header = p.qheader;
    q.seq_pfx = p.qseq_pfx;
    q.pairs = p.qpairs;
    build_schedule(q);
    return;
  }
  const int b = blockIdx.x - 2, nb = gridDim.x - 2;
  bwd_rope_rows<D>(p, b, nb);
  bwd_delta_rows<D>(p, b, nb);
}

// ------------------------------------------------------------------ main kernel

template <int D_>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr int BOXC = D >= 64 ? 64 : 32;  // columns per TMA box
  static constexpr int NBOX = D / BOXC;
  static constexpr int ROWB = BOXC * 2;
  static constexpr int SWZ_MASK = ROWB == 128 ? 7 : 3;
  static constexpr uint64_t UMMA_LAYOUT = ROWB == 128 ? 2 : 4;  // SWIZZLE_128B / SWIZZLE_64B
  static constexpr int SBO = 8 * ROWB;
  static constexpr int TILE_BOX_BYTES = 128 * ROWB;  // 128 rows (keys or packed q rows)
  static constexpr int TILE_BYTES = NBOX * TILE_BOX_BYTES;
  // dS^T: 128 key rows x 128 packed-q-row columns, two 64-column SW128 boxes
  static constexpr int DS_BOX_BYTES = 128 * 128;
  static constexpr int DS_BYTES = 2 * DS_BOX_BYTES;
  // d = 128: dS of query tile i overwrites dO of tile i (dP and dV have read it)
  static constexpr bool DS_IN_DO = TILE_BYTES == DS_BYTES;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE_BYTES;
  static constexpr int OFF_Q = OFF_V + TILE_BYTES;   // two stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE_BYTES;  // two stages
  static constexpr int OFF_DS = DS_IN_DO ? OFF_DO : OFF_DO + 2 * TILE_BYTES;
  // float [2 stages][lse2, Delta][128], after the dO stages and the dS buffer
  static constexpr int OFF_ST = DS_IN_DO ? OFF_DO + 2 * TILE_BYTES : OFF_DS + DS_BYTES;
  static constexpr int OFF_BAR = OFF_ST + 2 * 2 * BM * 4;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_USED = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
  // at least 120 KB, so that one CTA (which takes all 512 TMEM columns) runs per SM
  static constexpr int SMEM_BYTES = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0, DP_COL = 128, DV_COL = 256, DK_COL = 256 + D;
  static constexpr int STEPS_PER_BOX = BOXC / 16;
  // bf16 x bf16 -> fp32, M = 128
  static constexpr uint32_t IDESC_RR = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BM >> 3) << 17) |
                                       ((uint32_t)(BM >> 4) << 24);  // N = 128, A and B K-major
  static constexpr uint32_t IDESC_D = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(D >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);  // N = d, B MN-major
  __host__ __device__ static constexpr int ds_off(int stage) {
    return DS_IN_DO ? OFF_DO + stage * TILE_BYTES : OFF_DS;
  }
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(DK_COL + D <= TMEM_COLS, "tensor memory budget");
  static_assert(OFF_DS % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_DO % 1024 == 0, "swizzle atoms 1024-aligned");
  // regions in order, none overlapping the next
  static_assert(OFF_V >= OFF_K + TILE_BYTES && OFF_Q >= OFF_V + TILE_BYTES && OFF_DO >= OFF_Q + 2 * TILE_BYTES,
                "K', V, Q' regions overlap");
  static_assert(DS_IN_DO ? (OFF_DS == OFF_DO && DS_BYTES <= TILE_BYTES) : OFF_DS >= OFF_DO + 2 * TILE_BYTES,
                "dS region");
  static_assert(OFF_ST >= OFF_DO + 2 * TILE_BYTES && OFF_ST >= OFF_DS + DS_BYTES, "statistics overlap dO or dS");
  static_assert(OFF_BAR >= OFF_ST + 2 * 2 * BM * 4, "barriers overlap the statistics");
};

struct BwdBarriers {
  uint64_t kv_full;
  uint64_t q_full[2], do_full[2], st_full[2];
  uint64_t q_empty[2], do_empty[2], st_empty[2];
  uint64_t s_full, dp_full, p_full, dv_done, ds_full, acc_done, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(BwdBarriers) <= BwdCfg<128>::BAR_BYTES, "barrier area");

struct BwdItem {
  int seq_start, L, k0, kvh, qi0, nt;  // k0: first key of the tile; qi0, nt: query tiles visited
};

__device__ __forceinline__ BwdItem bwd_decode_item(const BwdParams& p, int w) {
  BwdItem it;
  const int pair = w / p.nkv;
  it.kvh = w - pair * p.nkv;
  const int2 sl = ptx::ld_cg_v2s32(p.pairs + pair);  // written by the prologue grid
  it.seq_start = __ldg(p.cu + sl.x);
  it.L = __ldg(p.cu + sl.x + 1) - it.seq_start;
  it.k0 = sl.y * BN;
  const int qt = (it.L + p.tq - 1) / p.tq;
  it.qi0 = p.causal ? it.k0 / p.tq : 0;
  it.nt = qt - it.qi0;
  return it;
}

// D = A B^T over d for two 128-row K-major tiles (S^T = K' Q'^T, dP^T = V dO^T).
template <class C>
__device__ __forceinline__ void bwd_mma_rows(uint32_t d_tmem, uint64_t da, uint64_t db) {
#pragma unroll
  for (int kk = 0; kk < C::D / 16; ++kk) {
    const uint32_t off = (kk / C::STEPS_PER_BOX) * C::TILE_BOX_BYTES + (kk % C::STEPS_PER_BOX) * 32;
    ptx::mma_ss(d_tmem, da + (uint64_t)(off >> 4), db + (uint64_t)(off >> 4), C::IDESC_RR, kk > 0 ? 1u : 0u);
  }
}

// dV (+)= P^T dO: A = P^T in TMEM (bf16 pairs, 16 packed q rows per 8
// columns), B = dO (MN-major, 16 rows per step).
template <class C>
__device__ __forceinline__ void bwd_mma_dv(uint32_t d_tmem, uint32_t p_tmem, uint64_t db, bool acc) {
#pragma unroll
  for (int kk = 0; kk < BM / 16; ++kk)  // packed columns [0, 64) at p_tmem, [64, 128) at p_tmem + 64
    ptx::mma_ts(d_tmem, p_tmem + (kk >> 2) * 64 + (kk & 3) * 8, db + (uint64_t)((kk * 16 * C::ROWB) >> 4),
                C::IDESC_D, (acc || kk > 0) ? 1u : 0u);
}

// dK' (+)= dS^T Q': A = dS^T (K-major SW128, 64 columns per box), B = Q' (MN-major).
template <class C>
__device__ __forceinline__ void bwd_mma_dk(uint32_t d_tmem, uint64_t da, uint64_t db, bool acc) {
#pragma unroll
  for (int kk = 0; kk < BM / 16; ++kk) {
    const uint32_t off_a = (kk / 4) * C::DS_BOX_BYTES + (kk % 4) * 32;
    ptx::mma_ss(d_tmem, da + (uint64_t)(off_a >> 4), db + (uint64_t)((kk * 16 * C::ROWB) >> 4), C::IDESC_D,
                (acc || kk > 0) ? 1u : 0u);
  }
}

template <int D>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    gqa_attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                        const BwdParams p) {
  using C = BwdCfg<D>;
  // one work item per CTA: (pair, KV head) in the longest-first list
  const int n_items = ptx::ld_cg_s32(p.header) * p.nkv;
  if ((int)blockIdx.x >= n_items) return;  // the whole CTA, before any barrier or TMEM use

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base derived by pointer arithmetic (accesses through it
  // stay shared-memory accesses)
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + C::OFF_BAR);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  auto B = [&](uint64_t& b) { return ptx::smem_u32(&b); };

  const BwdItem it = bwd_decode_item(p, blockIdx.x);
  const int G = p.G, tq = p.tq, rows = tq * G;

  if (threadIdx.x == 0) {
    ptx::mbar_init(B(bars->kv_full), 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(B(bars->q_full[s]), 1);
      ptx::mbar_init(B(bars->do_full[s]), 1);
      ptx::mbar_init(B(bars->st_full[s]), 32);
      ptx::mbar_init(B(bars->q_empty[s]), 1);
      ptx::mbar_init(B(bars->do_empty[s]), 1);
      ptx::mbar_init(B(bars->st_empty[s]), 8);
    }
    ptx::mbar_init(B(bars->s_full), 1);
    ptx::mbar_init(B(bars->dp_full), 1);
    ptx::mbar_init(B(bars->p_full), 256);
    ptx::mbar_init(B(bars->dv_done), 1);
    ptx::mbar_init(B(bars->ds_full), 256);
    ptx::mbar_init(B(bars->acc_done), 1);
    ptx::mbar_init(B(bars->drain), 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    ptx::prefetch_tmap(&tmDO);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&bars->tmem_base), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  // Padding rows (packed q rows >= tq * G, never written by TMA) of the Q'
  // and dO stage buffers are zero, so their scores are finite.
  if (rows < BM) {
    constexpr int CPR = C::ROWB / 16;  // 16-byte chunks per box row
    const int per_box = (BM - rows) * CPR;
    const int per_buf = C::NBOX * per_box;
    for (int i = threadIdx.x; i < 4 * per_buf; i += BWD_THREADS) {
      const int buf = i / per_buf;  // 0, 1: Q' stages; 2, 3: dO stages
      int rem = i - buf * per_buf;
      const int bx = rem / per_box;
      rem -= bx * per_box;
      const int row = rows + rem / CPR;
      const int ch = rem % CPR;
      const int base = buf < 2 ? C::OFF_Q + buf * C::TILE_BYTES : C::OFF_DO + (buf - 2) * C::TILE_BYTES;
      *reinterpret_cast<uint4*>(smem + base + bx * C::TILE_BOX_BYTES + swz(row * C::ROWB + ch * 16, C::SWZ_MASK)) =
          make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_smem();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 4) {
   ptx::setmaxnreg_dec<BWD_REG_PRODUCER>();
   if (warp == 0) {
    // ------------------------------------------------------------ loads
    bool ok = true;
    int n_q = 0, n_do = 0;
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(B(bars->kv_full), 2u * C::TILE_BYTES);
      for (int b = 0; b < C::NBOX; ++b) {
        ptx::tma_load_3d(sbase + C::OFF_K + b * C::TILE_BOX_BYTES, &tmK, B(bars->kv_full), b * C::BOXC,
                         it.seq_start + it.k0, it.kvh);
        ptx::tma_load_3d(sbase + C::OFF_V + b * C::TILE_BOX_BYTES, &tmV, B(bars->kv_full), b * C::BOXC, it.kvh,
                         it.seq_start + it.k0);
      }
    }
    for (int i = 0; i < it.nt; ++i) {
      const int s = i & 1;
      const uint32_t par = ((i >> 1) & 1) ^ 1;  // previous use of stage s released
      const int t0 = (it.qi0 + i) * tq;
      int lok = 1;
      if (lane == 0) {
        lok = bwait_lazy(B(bars->q_empty[s]), par, abort_flag);
        if (lok) {
          ptx::mbar_arrive_expect_tx(B(bars->q_full[s]), (uint32_t)(D * 2 * rows));
          for (int b = 0; b < C::NBOX; ++b)
            ptx::tma_load_3d(sbase + C::OFF_Q + s * C::TILE_BYTES + b * C::TILE_BOX_BYTES, &tmQ,
                             B(bars->q_full[s]), b * C::BOXC, it.kvh * G, it.seq_start + t0);
          ++n_q;
          lok = bwait_lazy(B(bars->do_empty[s]), par, abort_flag);
        }
        if (lok) {
          ptx::mbar_arrive_expect_tx(B(bars->do_full[s]), (uint32_t)(D * 2 * rows));
          for (int b = 0; b < C::NBOX; ++b)
            ptx::tma_load_3d(sbase + C::OFF_DO + s * C::TILE_BYTES + b * C::TILE_BOX_BYTES, &tmDO,
                             B(bars->do_full[s]), b * C::BOXC, it.kvh * G, it.seq_start + t0);
          ++n_do;
        }
      }
      ok = __shfl_sync(0xffffffffu, lok, 0) != 0;
      if (!ok) break;
      ok = __all_sync(0xffffffffu, bwait_lazy(B(bars->st_empty[s]), par, abort_flag));
      if (!ok) break;
      // lse * log2(e) and Delta of the tile's rows; rows past the sequence
      // (or padding) get +inf and 0, so that their P and dS are 0.
      float* st = reinterpret_cast<float*>(smem + C::OFF_ST) + s * 2 * BM;
#pragma unroll
      for (int u = 0; u < BM / 32; ++u) {
        const int r = lane + 32 * u;
        const int tt = r / G;
        const int tok = t0 + tt;
        float l2 = INFINITY, dl = 0.f;
        if (r < rows && tok < it.L) {
          const size_t at = (size_t)(it.kvh * G + (r - tt * G)) * p.N + it.seq_start + tok;
          l2 = __ldg(p.lse2 + at);
          dl = __ldg(p.delta + at);
        }
        st[r] = l2;
        st[BM + r] = dl;
      }
      ptx::mbar_arrive(B(bars->st_full[s]));
    }
    if (!ok && lane == 0) {  // every copy issued lands before the CTA exits
      drain_wait(B(bars->kv_full), 0);
      for (int s = 0; s < 2; ++s) {
        const int uq = (n_q - s + 1) / 2, ud = (n_do - s + 1) / 2;
        if (uq > 0) drain_wait(B(bars->q_full[s]), (uq - 1) & 1);
        if (ud > 0) drain_wait(B(bars->do_full[s]), (ud - 1) & 1);
      }
    }
   } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Per query tile i (stage s = i & 1), in issue order:
    //   dV(i) after P(i); S(i+1) once dV(i) has read P(i); dK(i), dQ'(i)
    //   after dS(i); dP(i+1) once dQ'(i) has been read out of TMEM.
    if (lane == 0) {
      const uint64_t dK_a = umma_desc(sbase + C::OFF_K, 16, C::SBO, C::UMMA_LAYOUT);
      const uint64_t dV_a = umma_desc(sbase + C::OFF_V, 16, C::SBO, C::UMMA_LAYOUT);
      const uint64_t dQ_k0 = umma_desc(sbase + C::OFF_Q, 16, C::SBO, C::UMMA_LAYOUT);
      const uint64_t dQ_mn0 = umma_desc(sbase + C::OFF_Q, C::TILE_BOX_BYTES, C::SBO, C::UMMA_LAYOUT);
      const uint64_t dO_k0 = umma_desc(sbase + C::OFF_DO, 16, C::SBO, C::UMMA_LAYOUT);
      const uint64_t dO_mn0 = umma_desc(sbase + C::OFF_DO, C::TILE_BOX_BYTES, C::SBO, C::UMMA_LAYOUT);
      const uint64_t stage_step = (uint64_t)(C::TILE_BYTES >> 4);
      auto dS_k = [&](int s) { return umma_desc(sbase + C::ds_off(s), 16, 1024, 2); };
      bool ok = bwait(B(bars->kv_full), 0, abort_flag);
      if (ok && (ok = bwait(B(bars->q_full[0]), 0, abort_flag))) {
        ptx::tc_fence_after();
        bwd_mma_rows<C>(tmem + C::S_COL, dK_a, dQ_k0);
        ptx::mma_commit(B(bars->s_full));
      }
      if (ok && (ok = bwait(B(bars->do_full[0]), 0, abort_flag))) {
        ptx::tc_fence_after();
        bwd_mma_rows<C>(tmem + C::DP_COL, dV_a, dO_k0);
        ptx::mma_commit(B(bars->dp_full));
      }
      for (int i = 0; ok && i < it.nt; ++i) {
        const int s = i & 1;
        const uint32_t ph = i & 1;
        const bool more = i + 1 < it.nt;
        const uint32_t nph = ((i + 1) >> 1) & 1;
        if (!(ok = bwait(B(bars->p_full), ph, abort_flag))) break;
        ptx::tc_fence_after();
        bwd_mma_dv<C>(tmem + C::DV_COL, tmem + C::S_COL, dO_mn0 + s * stage_step, i > 0);
        ptx::mma_commit(B(bars->dv_done));
        if (more) {
          if (!(ok = bwait(B(bars->q_full[s ^ 1]), nph, abort_flag))) break;
          if (!(ok = bwait(B(bars->dv_done), ph, abort_flag))) break;
          ptx::tc_fence_after();
          bwd_mma_rows<C>(tmem + C::S_COL, dK_a, dQ_k0 + (s ^ 1) * stage_step);
          ptx::mma_commit(B(bars->s_full));
        }
        if (!(ok = bwait(B(bars->ds_full), ph, abort_flag))) break;
        ptx::tc_fence_after();
        bwd_mma_dk<C>(tmem + C::DK_COL, dS_k(s), dQ_mn0 + s * stage_step, i > 0);
        ptx::mma_commit(B(bars->q_empty[s]));
        ptx::mma_commit(B(bars->do_empty[s]));
        if (more) {
          // dS(i) is formed: the softmax threads have read dP(i), its columns are free
          if (!(ok = bwait(B(bars->do_full[s ^ 1]), nph, abort_flag))) break;
          ptx::tc_fence_after();
          bwd_mma_rows<C>(tmem + C::DP_COL, dV_a, dO_k0 + (s ^ 1) * stage_step);
          ptx::mma_commit(B(bars->dp_full));
        }
      }
      if (ok) ptx::mma_commit(B(bars->acc_done));
      // all tensor-core work issued here has finished before TMEM is freed
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
   }
  } else if (warp < 12) {
    ptx::setmaxnreg_inc<BWD_REG_SOFTMAX>();
    // ------------------------------------------------------------ P^T, dS^T
    // Two warpgroups: warps 4-7 the packed query columns [0, 64), warps 8-11
    // [64, 128), of the same key rows (one per thread, TMEM lane quadrant
    // warp % 4).
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;
    constexpr int HC = BM / 2;        // columns per warpgroup
    const int c_lo = half * (HC / 32);  // first 32-column chunk of this half
    const int j = quad * 32 + lane;  // key row of the tile == TMEM lane
    const int key = it.k0 + j;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = true;
    uint32_t pw[HC / 2];  // this half of the P^T row, bf16 pairs
    uint32_t v[32];
    for (int i = 0; i < it.nt; ++i) {
      const int s = i & 1;
      const uint32_t ph = i & 1;
      const int t0 = (it.qi0 + i) * tq;
      // packed column r is query token t0 + r / G; with the causal mask it
      // sees this key iff r >= (key - t0) * G. Keys past the sequence see nothing.
      int r_lo = 0;
      if (key >= it.L) r_lo = BM;
      else if (p.causal && key > t0) r_lo = min(BM, (key - t0) * G);
      const float* st = reinterpret_cast<const float*>(smem + C::OFF_ST) + s * 2 * BM;
      ok = __all_sync(0xffffffffu, bwait(B(bars->st_full[s]), (i >> 1) & 1, abort_flag));
      if (!ok) break;
      ok = __all_sync(0xffffffffu, bwait(B(bars->s_full), ph, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < HC / 32; ++cc) {
        const int c = c_lo + cc;
        ptx::tmem_ld32(trow + C::S_COL + c * 32, v);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(v);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int col = c * 32 + e;
          const float x0 = fmaf(__uint_as_float(v[e]), sl2, -st[col]);
          const float x1 = fmaf(__uint_as_float(v[e + 1]), sl2, -st[col + 1]);
          const float p0 = col >= r_lo ? ptx::ex2(x0) : 0.f;
          const float p1 = col + 1 >= r_lo ? ptx::ex2(x1) : 0.f;
          pw[(cc * 32 + e) >> 1] = pack_bf16x2(p0, p1);
        }
      }
      // P^T of packed columns [64 half, 64 half + 64) as bf16 pairs over the
      // first 32 of the S columns this warpgroup has just read
      ptx::tmem_st32(trow + C::S_COL + half * 64, pw);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(B(bars->p_full));

      ok = __all_sync(0xffffffffu, bwait(B(bars->dp_full), ph, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      // dS^T of this half row into registers first (bf16 pairs), then, once
      // its shared-memory destination is free, stored
      uint32_t dw[HC / 2];
#pragma unroll
      for (int cc = 0; cc < HC / 32; ++cc) {
        const int c = c_lo + cc;
        ptx::tmem_ld32(trow + C::DP_COL + c * 32, v);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(v);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int col = c * 32 + e;
          const uint32_t pp = pw[(cc * 32 + e) >> 1];
          const float d0 = __uint_as_float(pp << 16) * (__uint_as_float(v[e]) - st[BM + col]);
          const float d1 = __uint_as_float(pp & 0xFFFF0000u) * (__uint_as_float(v[e + 1]) - st[BM + col + 1]);
          dw[(cc * 32 + e) >> 1] = pack_bf16x2(d0, d1);
        }
      }
      if (C::DS_IN_DO) {  // dS(i) overwrites dO(i): dV(i) must have read it
        ok = __all_sync(0xffffffffu, bwait(B(bars->dv_done), ph, abort_flag));
        if (!ok) break;
      }
      uint8_t* ds = smem + C::ds_off(s);
#pragma unroll
      for (int cc = 0; cc < HC / 32; ++cc) {
        const int c = c_lo + cc;
        // columns [32c, 32c + 32) of row j: box c / 2, 16-byte chunks 4 (c & 1) .. + 3
        uint8_t* box = ds + (c >> 1) * C::DS_BOX_BYTES;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int w0 = (cc * 32 + q4 * 8) >> 1;
          const int ch = (c & 1) * 4 + q4;
          *reinterpret_cast<uint4*>(box + swz(j * 128 + ch * 16, 7)) =
              make_uint4(dw[w0], dw[w0 + 1], dw[w0 + 2], dw[w0 + 3]);
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(B(bars->ds_full));
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(B(bars->st_empty[s]));
    }
  } else {
    ptx::setmaxnreg_inc<BWD_REG_READOUT>();
    // ------------------------------------------------------------ dV, dK' at the end
    const int quad = warp - 12;
    const int r = quad * 32 + lane;  // key row (dV, dK') == TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = true;
    uint32_t v[32];
    // (a sleeping wait: these warps idle for the whole loop and share their
    // schedulers with the P^T/dS^T warps)
    if (ok) ok = __all_sync(0xffffffffu, bwait_lazy(B(bars->acc_done), 0, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
      const int key = it.k0 + r;
      const bool kvalid = key < it.L;
      const size_t orow = ((size_t)(it.seq_start + (kvalid ? key : 0)) * p.nkv + it.kvh) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        ptx::tmem_ld32(trow + C::DV_COL + c * 32, v);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(v);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        if (kvalid) {
          uint4* o = reinterpret_cast<uint4*>(p.dv + orow + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) o[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
      }
      // dk = rope^T(dK') / sqrt(d): pairs (i, i + d/2) rotated by the negative angle
      constexpr int HALF = D / 2;
      const float sc = p.scale;
#pragma unroll
      for (int i0 = 0; i0 < HALF; i0 += 16) {
        uint32_t lo[16], hi[16];
        ptx::tmem_ld16(trow + C::DK_COL + i0, lo);
        ptx::tmem_ld16(trow + C::DK_COL + HALF + i0, hi);
        ptx::tmem_wait_ld();
        ptx::reg_fence16(lo);
        ptx::reg_fence16(hi);
        if (kvalid) {
          const float4* tab = reinterpret_cast<const float4*>(p.table + (size_t)(it.seq_start + key) * HALF + i0);
          uint32_t ol[8], oh[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float4 cs = __ldg(tab + e / 2);  // cos_e, sin_e, cos_e+1, sin_e+1
            const float g0 = __uint_as_float(lo[e]), g1 = __uint_as_float(lo[e + 1]);
            const float h0 = __uint_as_float(hi[e]), h1 = __uint_as_float(hi[e + 1]);
            ol[e / 2] = pack_bf16x2((g0 * cs.x + h0 * cs.y) * sc, (g1 * cs.z + h1 * cs.w) * sc);
            oh[e / 2] = pack_bf16x2((h0 * cs.x - g0 * cs.y) * sc, (h1 * cs.z - g1 * cs.w) * sc);
          }
          uint4* olo = reinterpret_cast<uint4*>(p.dk + orow + i0);
          uint4* ohi = reinterpret_cast<uint4*>(p.dk + orow + HALF + i0);
          olo[0] = make_uint4(ol[0], ol[1], ol[2], ol[3]);
          olo[1] = make_uint4(ol[4], ol[5], ol[6], ol[7]);
          ohi[0] = make_uint4(oh[0], oh[1], oh[2], oh[3]);
          ohi[1] = make_uint4(oh[4], oh[5], oh[6], oh[7]);
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ dq

// dq = rope^T(dQ' / sqrt(d)) in bf16: dx_i = g_i cos + g_{i+d/2} sin,
// dx_{i+d/2} = g_{i+d/2} cos - g_i sin. Four frequencies per thread.
template <int D>
__global__ void __launch_bounds__(PREP_THREADS)
    gqa_bwd_dq_kernel(const float* __restrict__ dq_acc, const float2* __restrict__ table,
                      __nv_bfloat16* __restrict__ dq, int N, int nq, float scale) {
  constexpr int HALF = D / 2;
  constexpr int QPR = HALF / 4;
  const long long total = (long long)N * nq * QPR;
  for (long long idx = (long long)blockIdx.x * PREP_THREADS + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * PREP_THREADS) {
    const long long row = idx / QPR;
    const int i0 = (int)(idx - row * QPR) * 4;
    const int t = (int)(row / nq);
    const float4 g = *reinterpret_cast<const float4*>(dq_acc + row * D + i0);
    const float4 h = *reinterpret_cast<const float4*>(dq_acc + row * D + HALF + i0);
    const float4 a = *reinterpret_cast<const float4*>(table + (size_t)t * HALF + i0);      // c0 s0 c1 s1
    const float4 b = *reinterpret_cast<const float4*>(table + (size_t)t * HALF + i0 + 2);  // c2 s2 c3 s3
    const uint32_t l01 = pack_bf16x2((g.x * a.x + h.x * a.y) * scale, (g.y * a.z + h.y * a.w) * scale);
    const uint32_t l23 = pack_bf16x2((g.z * b.x + h.z * b.y) * scale, (g.w * b.z + h.w * b.w) * scale);
    const uint32_t h01 = pack_bf16x2((h.x * a.x - g.x * a.y) * scale, (h.y * a.z - g.y * a.w) * scale);
    const uint32_t h23 = pack_bf16x2((h.z * b.x - g.z * b.y) * scale, (h.w * b.z - g.w * b.w) * scale);
    *reinterpret_cast<uint2*>(dq + row * D + i0) = make_uint2(l01, l23);
    *reinterpret_cast<uint2*>(dq + row * D + HALF + i0) = make_uint2(h01, h23);
  }
}

}  // namespace gqa
