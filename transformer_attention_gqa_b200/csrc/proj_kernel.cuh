// Q, K, V projection with the RoPE epilogue (sm_100a).
//
// Steps 1 and 2 of the attention module's walk-through ("Attention from
// Scratch", section "Attention, the math": Project, then Rotate), for the
// tokens x [N, C] of the residual stream:
//   [q | k | v] = x W^T,  W = [W_q; W_k; W_v]  ([(n_q + 2 n_kv) d, C], the
//   three linear layers' weights stacked, no bias)
//   q, k: each head's feature i rotated with feature i + d/2 by the token's
//   angle ("Embeddings & the Residual Stream", section "Positional
//   information: RoPE, not a learned table"); v: not rotated.
// The rotation is applied to the fp32 accumulator and rounded once to bf16
// (rope_round.cuh): no bf16 rounding between the product and the rotation.
//
// One persistent CTA per SM (one CTA per tile when there are at most two
// tiles per SM) walks the tiles of 128 tokens x 256 output features (256 is a multiple of d in {32, 64, 128}, so a tile holds whole
// heads), CTA b taking tiles b, b + grid, ... (feature tiles of the same
// tokens next to each other, so x stays in L2): a TMA ring of PJ_STAGES
// (x, W) blocks of 64 along C, continuous across tiles, feeds one thread
// issuing tcgen05.mma (kind::f16, M = 128, N = 256, K = 16, both operands
// K-major SW128) into one of two 256-column fp32 accumulators in tensor
// memory, alternating by tile; four epilogue warps read a finished
// accumulator (32 rows each) and write q, k (rotated) and v while the next
// tile's products fill the other one.
//
// Warp roles (192 threads): warp 0 TMA producer; warp 1 TMEM allocation and
// the MMA issuer; warps 2-5 epilogue (TMEM lane quadrant = warp % 4).
//
// A small kernel ahead of it writes each token's (cos, sin) row, as the
// attention prologue does.
#pragma once

#include "attn_kernel.cuh"
#include "common.cuh"
#include "prep_kernel.cuh"
#include "ptx.cuh"
#include "rope_round.cuh"

namespace gqa {

constexpr int PJ_BM = 128;  // tokens per tile
constexpr int PJ_BN = 256;  // output features per tile
constexpr int PJ_BK = 64;   // C per stage (one 128-byte swizzle row)
constexpr int PJ_STAGES = 4;
constexpr int PJ_THREADS = 192;
constexpr int PJ_A_BYTES = PJ_BM * PJ_BK * 2;  // 16 KB
constexpr int PJ_B_BYTES = PJ_BN * PJ_BK * 2;  // 32 KB
constexpr int PJ_STAGE_BYTES = PJ_A_BYTES + PJ_B_BYTES;
constexpr int PJ_OFF_BAR = PJ_STAGES * PJ_STAGE_BYTES;
constexpr int PJ_SMEM_BYTES = PJ_OFF_BAR + 256 + 1024;  // + barriers + alignment slack
constexpr uint32_t PJ_TMEM_COLS = 512;  // two accumulators of PJ_BN columns
// bf16 x bf16 -> fp32, A and B K-major, M = 128, N = 256
constexpr uint32_t PJ_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(PJ_BN >> 3) << 17) |
                              ((uint32_t)(PJ_BM >> 4) << 24);
static_assert(PJ_SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(PJ_A_BYTES % 1024 == 0 && PJ_STAGE_BYTES % 1024 == 0, "swizzle atoms 1024-aligned");

struct ProjBarriers {
  uint64_t full[PJ_STAGES], empty[PJ_STAGES];
  uint64_t acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(ProjBarriers) <= 256, "barrier area");

struct ProjTableParams {
  const int* positions;
  const int* cu;
  int N, num_seqs, half;
  double inv_freq[64];
  float2* table;
};

struct ProjParams {
  const float2* table;  // [N][d/2] (cos, sin)
  __nv_bfloat16* q;     // [N][n_q][d]
  __nv_bfloat16* k;     // [N][n_kv][d]
  __nv_bfloat16* v;     // [N][n_kv][d]
  int N, C, nq, nkv;
  int n_tiles_n;        // feature tiles of PJ_BN per token tile
  int n_tiles;          // token tiles x feature tiles
};

// (cos, sin) of every token's angles: fp64 angle and sincos, stored as fp32.
// One thread per (token, pair of frequencies).
__global__ void __launch_bounds__(PREP_THREADS) gqa_qkv_table_kernel(const ProjTableParams p) {
  const int pairs = p.half / 2;
  const long long total = (long long)p.N * pairs;
  for (long long idx = (long long)blockIdx.x * PREP_THREADS + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * PREP_THREADS) {
    const int t = (int)(idx / pairs);
    const int i = (int)(idx % pairs) * 2;
    int pos;
    if (p.positions) {
      pos = __ldg(p.positions + t);
    } else {
      const int s = upper_index(p.cu, p.num_seqs, t);
      pos = t - __ldg(p.cu + s);
    }
    double s0, c0, s1, c1;
    sincos((double)pos * p.inv_freq[i], &s0, &c0);
    sincos((double)pos * p.inv_freq[i + 1], &s1, &c1);
    *reinterpret_cast<float4*>(p.table + (size_t)t * p.half + i) =
        make_float4((float)c0, (float)s0, (float)c1, (float)s1);
  }
}

template <int D>
__global__ void __launch_bounds__(PJ_THREADS, 1)
    gqa_qkv_proj_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                        const ProjParams p) {
  constexpr int HALF = D / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  ProjBarriers* bars = reinterpret_cast<ProjBarriers*>(smem + PJ_OFF_BAR);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  auto B = [&](uint64_t& b) { return ptx::smem_u32(&b); };

  const int nk = (p.C + PJ_BK - 1) / PJ_BK;
  const int G = (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PJ_STAGES; ++s) {
      ptx::mbar_init(B(bars->full[s]), 1);
      ptx::mbar_init(B(bars->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(B(bars->acc_full[a]), 1);
      ptx::mbar_init(B(bars->acc_empty[a]), 128);
    }
    ptx::mbar_init(B(bars->drain), 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&bars->tmem_base), PJ_TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.n_tiles; t += G) {
        const int n0 = (t % p.n_tiles_n) * PJ_BN, m0 = (t / p.n_tiles_n) * PJ_BM;
        for (int kb = 0; kb < nk; ++kb, ++issued) {
          const int s = issued % PJ_STAGES;
          if (!(ok = bwait_lazy(B(bars->empty[s]), ((issued / PJ_STAGES) & 1) ^ 1, abort_flag))) break;
          const uint32_t a = sbase + s * PJ_STAGE_BYTES;
          ptx::mbar_arrive_expect_tx(B(bars->full[s]), (uint32_t)PJ_STAGE_BYTES);
          ptx::tma_load_3d(a, &tmX, B(bars->full[s]), kb * PJ_BK, m0, 0);
          ptx::tma_load_3d(a + PJ_A_BYTES, &tmW, B(bars->full[s]), kb * PJ_BK, n0, 0);
        }
      }
      if (!ok) {  // every copy issued lands before the CTA exits
        for (int s = 0; s < PJ_STAGES; ++s) {
          const int uses = (issued - s + PJ_STAGES - 1) / PJ_STAGES;
          if (uses > 0) drain_wait(B(bars->full[s]), (uses - 1) & 1);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint64_t da0 = umma_desc(sbase, 16, 1024, 2);
      const uint64_t db0 = umma_desc(sbase + PJ_A_BYTES, 16, 1024, 2);
      int used = 0;
      bool ok = true;
      for (int t = blockIdx.x, i = 0; ok && t < p.n_tiles; t += G, ++i) {
        const int acc = i & 1;
        // the epilogue has read this accumulator's previous tile (i - 2)
        if (!(ok = bwait(B(bars->acc_empty[acc]), ((i >> 1) & 1) ^ 1, abort_flag))) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++used) {
          const int s = used % PJ_STAGES;
          if (!(ok = bwait(B(bars->full[s]), (used / PJ_STAGES) & 1, abort_flag))) break;
          ptx::tc_fence_after();
          const uint64_t st = (uint64_t)((s * PJ_STAGE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < PJ_BK / 16; ++kk)
            ptx::mma_ss(tmem + acc * PJ_BN, da0 + st + (uint64_t)kk * 2, db0 + st + (uint64_t)kk * 2, PJ_IDESC,
                        (kb > 0 || kk > 0) ? 1u : 0u);
          ptx::mma_commit(B(bars->empty[s]));
        }
        if (ok) ptx::mma_commit(B(bars->acc_full[acc]));
      }
      // all tensor-core work issued here has finished before TMEM is freed
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int quad = warp & 3;         // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;  // == TMEM lane
    const uint32_t trow0 = tmem + ((uint32_t)(quad * 32) << 16);
    const int heads = p.nq + 2 * p.nkv;
    bool ok = true;
    for (int t = blockIdx.x, i = 0; ok && t < p.n_tiles; t += G, ++i) {
      const int acc = i & 1;
      const int n0 = (t % p.n_tiles_n) * PJ_BN, m0 = (t / p.n_tiles_n) * PJ_BM;
      ok = __all_sync(0xffffffffu, bwait(B(bars->acc_full[acc]), (i >> 1) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      const int tok = m0 + row;
      const bool valid = tok < p.N;
      const uint32_t trow = trow0 + (uint32_t)(acc * PJ_BN);
#pragma unroll 1
      for (int hd = 0; hd < PJ_BN / D; ++hd) {
        const int head = n0 / D + hd;  // head index in [q | k | v]
        if (head >= heads) break;      // the same for every thread of the CTA
        const uint32_t tc = trow + (uint32_t)(hd * D);
        if (head < p.nq + p.nkv) {
          // q or k: rotate, round once to bf16
          __nv_bfloat16* dst = head < p.nq ? p.q + ((size_t)tok * p.nq + head) * D
                                           : p.k + ((size_t)tok * p.nkv + (head - p.nq)) * D;
#pragma unroll 1
          for (int i0 = 0; i0 < HALF; i0 += 16) {
            uint32_t lo[16], hi[16];
            ptx::tmem_ld16(tc + i0, lo);
            ptx::tmem_ld16(tc + HALF + i0, hi);
            ptx::tmem_wait_ld();
            ptx::reg_fence16(lo);
            ptx::reg_fence16(hi);
            if (valid) {
              const float4* tab = reinterpret_cast<const float4*>(p.table + (size_t)tok * HALF + i0);
              uint32_t ol[8], oh[8];
#pragma unroll
              for (int e = 0; e < 16; e += 2) {
                const float4 cs = __ldg(tab + e / 2);  // cos_e, sin_e, cos_e+1, sin_e+1
                const float x0 = __uint_as_float(lo[e]), x1 = __uint_as_float(lo[e + 1]);
                const float y0 = __uint_as_float(hi[e]), y1 = __uint_as_float(hi[e + 1]);
                ol[e / 2] = (uint32_t)rope_round_bf16(x0, cs.x, y0, -cs.y) |
                            ((uint32_t)rope_round_bf16(x1, cs.z, y1, -cs.w) << 16);
                oh[e / 2] = (uint32_t)rope_round_bf16(y0, cs.x, x0, cs.y) |
                            ((uint32_t)rope_round_bf16(y1, cs.z, x1, cs.w) << 16);
              }
              uint4* plo = reinterpret_cast<uint4*>(dst + i0);
              uint4* phi = reinterpret_cast<uint4*>(dst + HALF + i0);
              plo[0] = make_uint4(ol[0], ol[1], ol[2], ol[3]);
              plo[1] = make_uint4(ol[4], ol[5], ol[6], ol[7]);
              phi[0] = make_uint4(oh[0], oh[1], oh[2], oh[3]);
              phi[1] = make_uint4(oh[4], oh[5], oh[6], oh[7]);
            }
          }
        } else {
          // v: round to bf16
          __nv_bfloat16* dst = p.v + ((size_t)tok * p.nkv + (head - p.nq - p.nkv)) * D;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t x[16];
            ptx::tmem_ld16(tc + c0, x);
            ptx::tmem_wait_ld();
            ptx::reg_fence16(x);
            if (valid) {
              uint32_t o[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = pack_bf16x2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]));
              uint4* pv = reinterpret_cast<uint4*>(dst + c0);
              pv[0] = make_uint4(o[0], o[1], o[2], o[3]);
              pv[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
          }
        }
      }
      // this accumulator is read: the tile after next may overwrite it
      ptx::tc_fence_before();
      ptx::mbar_arrive(B(bars->acc_empty[acc]));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, PJ_TMEM_COLS);
  }
}

}  // namespace gqa
