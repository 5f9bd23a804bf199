// dQ' of the backward, per query tile (sm_100a).
//
// Of the backward's products ("Attention from Scratch", section "Attention,
// the math", through the chain rule; see bwd_kernel.cuh), this kernel
// computes
//   dQ' = dS K',   dS = P * (dP - Delta),   P = exp(S - lse),
//   S = Q' K'^T,   dP = dO V^T
// with the query tile as the owner: one CTA per (sequence, packed query
// tile, KV head), the forward's packing of tq tokens x G heads into 128 rows,
// looping over the key tiles that the causal mask lets the tile see. Each
// dQ' row is summed over all its keys in tensor memory and written once, in
// fp32, to the accumulator that gqa_bwd_dq_kernel rotates back; no atomics.
// (The key-tile kernel of bwd_kernel.cuh computes dK' and dV; P and dP are
// recomputed here, three products per key tile instead of the single dQ'
// product that a shared kernel would add, which measured slower there: its
// dQ' atomics and the tensor-memory hand-offs they needed serialised every
// query tile.)
//
// Per key tile j (stage s = j & 1 of the K'/V ring):
//   S(j)  = Q' K'_j^T   M = 128 rows, N = 128 keys, K = d   SS (the forward's S form)
//   dP(j) = dO V_j^T    the same form with dO and V
//   dS(j) = bf16(P) * (dP - Delta), bf16, written over S(j) in tensor memory
//   dQ'  += dS(j) K'_j  A = dS from tensor memory, B = K'_j read key-major (the forward's P V form)
// P uses the forward's lse (lse * log2(e) per row, from the prologue), so
// there is no running max. Rows past the sequence or padding rows take
// lse = +inf and Delta = 0: their P and dS are 0.
//
// Warp roles (384 threads): warp 0 TMA (Q' and dO once, K' through three
// stages, V through two) and the rows' statistics; warp 1 tensor memory and every MMA;
// warps 4-11 dS, one row per thread and half of the tile's keys per
// warpgroup (warps 4-7 keys [0, 64), 8-11 [64, 128)), then dQ' out.
// Tensor memory: S/dS buffers at columns 0 and 128, dP at 256, dQ' at 384.
#pragma once

#include "attn_kernel.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace gqa {

constexpr int BQ_THREADS = 384;

struct BwdQParams {
  const int* cu;
  const int* header;   // [0]: number of (sequence, query tile) pairs
  const int2* pairs;   // (sequence, query tile), decreasing cost
  const float* lse2;   // [n_q][N]: lse * log2(e)
  const float* delta;  // [n_q][N]
  float* dq_acc;       // [N][n_q][d]: dQ' (fp32, unscaled)
  int N, nq, nkv, G, tq, causal;
  float scale_log2;    // log2(e) / sqrt(d)
};

template <int D>
struct BwdQCfg {
  using A = AttnCfg<D>;
  static constexpr int OFF_Q = 0;                          // Q' tile
  static constexpr int OFF_DO = A::Q_BYTES;                // dO tile (same layout)
  // K'_j is read by S(j) and dQ'(j), V_j by dP(j) only: K' has a deeper ring,
  // so that K'_{j+3} loads once dQ'(j) is done and V_{j+2} once dP(j) is
  static constexpr int KST = 3;
  static constexpr int VST = 2;
  static constexpr int OFF_K = OFF_DO + A::Q_BYTES;        // KST stages
  static constexpr int OFF_V = OFF_K + KST * A::KV_BYTES;  // VST stages
  static constexpr int OFF_ST = OFF_V + VST * A::KV_BYTES;  // float [lse2, Delta][BM]
  static constexpr int OFF_BAR = OFF_ST + 2 * BM * 4;
  static constexpr int SMEM_USED = OFF_BAR + 256 + 1024;  // + barriers + alignment slack
  // at least 120 KB, so that one CTA (which takes all 512 TMEM columns) runs per SM
  static constexpr int SMEM_BYTES = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t DP_COL = 256, DQ_COL = 384;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(OFF_DO % 1024 == 0 && OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "swizzle atoms 1024-aligned");
  static_assert(DQ_COL + D <= TMEM_COLS, "tensor memory budget");
};

struct BwdQBarriers {
  uint64_t q_full, st_full;
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], dp_full, ds_full[2], dq_done[2];
  uint64_t o_full, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(BwdQBarriers) <= 256, "barrier area");

template <int D>
__global__ void __launch_bounds__(BQ_THREADS, 1)
    gqa_attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                          const BwdQParams p) {
  using A = AttnCfg<D>;
  using C = BwdQCfg<D>;
  const int n_items = ptx::ld_cg_s32(p.header) * p.nkv;
  if ((int)blockIdx.x >= n_items) return;  // the whole CTA, before any barrier or TMEM use
  // the work item: (sequence, query tile) pair and KV head
  const int pair = (int)blockIdx.x / p.nkv;
  const int kvh = (int)blockIdx.x - pair * p.nkv;
  const int2 sl = ptx::ld_cg_v2s32(p.pairs + pair);  // written by the prologue grid
  const int seq_start = __ldg(p.cu + sl.x);
  const int L = __ldg(p.cu + sl.x + 1) - seq_start;
  const int t0 = sl.y * p.tq;
  const int t_end = p.causal ? min(t0 + p.tq, L) : L;
  const int nkt = (t_end + BN - 1) / BN;  // key tiles this query tile sees
  const int G = p.G, rows = p.tq * G;

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base derived by pointer arithmetic (accesses through it
  // stay shared-memory accesses)
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  BwdQBarriers* bars = reinterpret_cast<BwdQBarriers*>(smem + C::OFF_BAR);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  auto B = [&](uint64_t& b) { return ptx::smem_u32(&b); };

  if (threadIdx.x == 0) {
    ptx::mbar_init(B(bars->q_full), 1);
    ptx::mbar_init(B(bars->st_full), 1);
    for (int s = 0; s < C::KST; ++s) {
      ptx::mbar_init(B(bars->k_full[s]), 1);
      ptx::mbar_init(B(bars->k_empty[s]), 1);
    }
    for (int s = 0; s < C::VST; ++s) {
      ptx::mbar_init(B(bars->v_full[s]), 1);
      ptx::mbar_init(B(bars->v_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(B(bars->s_full[s]), 1);
      ptx::mbar_init(B(bars->ds_full[s]), 256);
      ptx::mbar_init(B(bars->dq_done[s]), 1);
    }
    ptx::mbar_init(B(bars->dp_full), 1);
    ptx::mbar_init(B(bars->o_full), 1);
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
  // padding rows of the Q' and dO tiles (never written by TMA) are zero
  if (rows < BM) {
    constexpr int CPR = A::ROWB / 16;
    const int per_box = (BM - rows) * CPR;
    for (int i = threadIdx.x; i < 2 * A::NBOX * per_box; i += BQ_THREADS) {
      const int t = i / (A::NBOX * per_box);  // 0: Q', 1: dO
      int rem = i - t * A::NBOX * per_box;
      const int bx = rem / per_box;
      rem -= bx * per_box;
      *reinterpret_cast<uint4*>(smem + (t ? C::OFF_DO : C::OFF_Q) + bx * A::Q_BOX_BYTES +
                                swz((rows + rem / CPR) * A::ROWB + (rem % CPR) * 16, A::SWZ_MASK)) =
          make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_smem();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer, statistics
    int nk = 0, nv = 0;
    bool ok = true;
    if (lane == 0) {
      ptx::mbar_arrive_expect_tx(B(bars->q_full), (uint32_t)(2 * D * 2 * rows));
      for (int b = 0; b < A::NBOX; ++b) {
        ptx::tma_load_3d(sbase + C::OFF_Q + b * A::Q_BOX_BYTES, &tmQ, B(bars->q_full), b * A::BOXC, kvh * G,
                         seq_start + t0);
        ptx::tma_load_3d(sbase + C::OFF_DO + b * A::Q_BOX_BYTES, &tmDO, B(bars->q_full), b * A::BOXC, kvh * G,
                         seq_start + t0);
      }
    }
    // lse * log2(e) and Delta of the tile's rows; rows past the sequence
    // (or padding) get +inf and 0, so that their P and dS are 0
    float* st = reinterpret_cast<float*>(smem + C::OFF_ST);
#pragma unroll
    for (int u = 0; u < BM / 32; ++u) {
      const int r = lane + 32 * u;
      const int tt = r / G;
      const int tok = t0 + tt;
      float l2 = INFINITY, dl = 0.f;
      if (r < rows && tok < L) {
        const size_t at = (size_t)(kvh * G + (r - tt * G)) * p.N + seq_start + tok;
        l2 = __ldg(p.lse2 + at);
        dl = __ldg(p.delta + at);
      }
      st[r] = l2;
      st[BM + r] = dl;
    }
    __syncwarp();
    if (lane == 0) {
      ptx::mbar_arrive(B(bars->st_full));
      for (int j = 0; j < nkt; ++j) {
        const int ks = j % C::KST, vs = j % C::VST;
        // previous use of each stage released
        if (!(ok = bwait_lazy(B(bars->k_empty[ks]), ((j / C::KST) & 1) ^ 1, abort_flag))) break;
        ptx::mbar_arrive_expect_tx(B(bars->k_full[ks]), (uint32_t)A::KV_BYTES);
        for (int b = 0; b < A::NBOX; ++b)
          ptx::tma_load_3d(sbase + C::OFF_K + ks * A::KV_BYTES + b * A::KV_BOX_BYTES, &tmK, B(bars->k_full[ks]),
                           b * A::BOXC, seq_start + j * BN, kvh);
        ++nk;
        if (!(ok = bwait_lazy(B(bars->v_empty[vs]), ((j / C::VST) & 1) ^ 1, abort_flag))) break;
        ptx::mbar_arrive_expect_tx(B(bars->v_full[vs]), (uint32_t)A::KV_BYTES);
        for (int b = 0; b < A::NBOX; ++b)
          ptx::tma_load_3d(sbase + C::OFF_V + vs * A::KV_BYTES + b * A::KV_BOX_BYTES, &tmV, B(bars->v_full[vs]),
                           b * A::BOXC, kvh, seq_start + j * BN);
        ++nv;
      }
      if (!ok) {  // every copy issued lands before the CTA exits
        drain_wait(B(bars->q_full), 0);
        for (int s = 0; s < C::KST; ++s) {
          const int uk = (nk - s + C::KST - 1) / C::KST;  // loads issued into stage s
          if (uk > 0) drain_wait(B(bars->k_full[s]), (uk - 1) & 1);
        }
        for (int s = 0; s < C::VST; ++s) {
          const int uv = (nv - s + C::VST - 1) / C::VST;
          if (uv > 0) drain_wait(B(bars->v_full[s]), (uv - 1) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // In issue order per key tile j: S(j + 1) once dQ'(j - 1) has read dS(j - 1)
    // from that buffer; dQ'(j) after dS(j); dP(j + 1) after dS(j) (which read dP(j)).
    if (lane == 0) {
      const uint64_t dq = umma_desc(sbase + C::OFF_Q, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t ddo = umma_desc(sbase + C::OFF_DO, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t dk0 = umma_desc(sbase + C::OFF_K, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t dv0 = umma_desc(sbase + C::OFF_V, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t dkmn0 = umma_desc(sbase + C::OFF_K, A::KV_BOX_BYTES, A::SBO, A::UMMA_LAYOUT);
      const uint64_t stage = (uint64_t)(A::KV_BYTES >> 4);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1, ks = j % C::KST;
        if (j >= 2 && !bwait(B(bars->dq_done[s]), ((j - 2) >> 1) & 1, abort_flag)) return false;
        if (!bwait(B(bars->k_full[ks]), (j / C::KST) & 1, abort_flag)) return false;
        ptx::tc_fence_after();
        issue_s_mmas<A>(tmem + s * 128, dq, dk0 + ks * stage);
        ptx::mma_commit(B(bars->s_full[s]));
        return true;
      };
      auto issue_dp = [&](int j) -> bool {
        const int vs = j % C::VST;
        if (!bwait(B(bars->v_full[vs]), (j / C::VST) & 1, abort_flag)) return false;
        ptx::tc_fence_after();
        issue_s_mmas<A>(tmem + C::DP_COL, ddo, dv0 + vs * stage);
        ptx::mma_commit(B(bars->dp_full));
        ptx::mma_commit(B(bars->v_empty[vs]));  // dP(j) is V_j's only reader
        return true;
      };
      bool ok = bwait(B(bars->q_full), 0, abort_flag) && issue_s(0) && issue_dp(0);
      for (int j = 0; ok && j < nkt; ++j) {
        const int s = j & 1;
        if (j + 1 < nkt && !(ok = issue_s(j + 1))) break;
        if (!(ok = bwait(B(bars->ds_full[s]), (j >> 1) & 1, abort_flag))) break;
        ptx::tc_fence_after();
        issue_pv_mmas<A>(tmem + C::DQ_COL, tmem + s * 128, dkmn0 + (j % C::KST) * stage, j > 0);
        ptx::mma_commit(B(bars->dq_done[s]));
        ptx::mma_commit(B(bars->k_empty[j % C::KST]));  // S(j) and dQ'(j) have read K'_j
        if (j + 1 < nkt && !(ok = issue_dp(j + 1))) break;
      }
      if (ok) ptx::mma_commit(B(bars->o_full));
      // all tensor-core work issued here has finished before TMEM is freed
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dS, then dQ' out
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;      // keys [64 * half, 64 * half + 64) of each tile
    const int r = quad * 32 + lane;        // row of the tile == TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const int tt = r / G;
    const int tok = t0 + tt;
    const bool row_valid = r < rows && tok < L;
    const int last_key = p.causal ? tok : L - 1;  // keys past it are hidden (in-sequence index)
    const float sl2 = p.scale_log2;
    bool ok = __all_sync(0xffffffffu, bwait(B(bars->st_full), 0, abort_flag));
    const float* st = reinterpret_cast<const float*>(smem + C::OFF_ST);
    const float lse2 = ok ? st[r] : INFINITY, dl = ok ? st[BM + r] : 0.f;
    // Per key tile: P from S first (its exponentials overlap dP's MMA), rounded
    // to bf16 as it enters dV's product; then dS = P (dP - Delta) once dP is in.
    uint32_t v[32], pw[32], pk[16];
    for (int j = 0; ok && j < nkt; ++j) {
      const int s = j & 1;
      ok = __all_sync(0xffffffffu, bwait(B(bars->s_full[s]), (j >> 1) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = half * 64 + cc * 32;      // first key (column) of this chunk
        const int lim = last_key - j * BN - c0;  // columns > lim are hidden
        ptx::tmem_ld32(trow + s * 128 + c0, v);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(v);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = e <= lim ? ptx::ex2(fmaf(__uint_as_float(v[e]), sl2, -lse2)) : 0.f;
          const float p1 = e + 1 <= lim ? ptx::ex2(fmaf(__uint_as_float(v[e + 1]), sl2, -lse2)) : 0.f;
          pw[(cc * 32 + e) >> 1] = pack_bf16x2(p0, p1);
        }
      }
      ok = __all_sync(0xffffffffu, bwait(B(bars->dp_full), j & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = half * 64 + cc * 32;
        ptx::tmem_ld32(trow + C::DP_COL + c0, v);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(v);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t pp = pw[(cc * 32 + e) >> 1];
          const float d0 = __uint_as_float(pp << 16) * (__uint_as_float(v[e]) - dl);
          const float d1 = __uint_as_float(pp & 0xFFFF0000u) * (__uint_as_float(v[e + 1]) - dl);
          pk[e >> 1] = pack_bf16x2(d0, d1);
        }
        // dS (bf16 pairs) over this row's S columns, all read above: keys
        // [0, 64) at columns 0..31, keys [64, 128) at columns 64..95
        ptx::tmem_st16(trow + s * 128 + half * 64 + cc * 16, pk);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(B(bars->ds_full[s]));
    }
    if (ok) ok = __all_sync(0xffffffffu, bwait(B(bars->o_full), 0, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
      // this half of the dQ' row (D / 2 fp32 columns) into the accumulator
      float* dst = row_valid ? p.dq_acc + ((size_t)(seq_start + tok) * p.nq + kvh * G + (r - tt * G)) * D : nullptr;
#pragma unroll
      for (int c = 0; c < D / 2; c += 16) {
        uint32_t o[16];
        ptx::tmem_ld16(trow + C::DQ_COL + half * (D / 2) + c, o);
        ptx::tmem_wait_ld();
        ptx::reg_fence16(o);
        if (row_valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + half * (D / 2) + c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            d4[q4] = make_float4(__uint_as_float(o[4 * q4]), __uint_as_float(o[4 * q4 + 1]),
                                 __uint_as_float(o[4 * q4 + 2]), __uint_as_float(o[4 * q4 + 3]));
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

}  // namespace gqa
