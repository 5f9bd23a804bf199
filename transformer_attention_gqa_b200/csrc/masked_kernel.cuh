// Attention forward with an additive mask (sm_100a).
//
// The attention kernel of "Attention from Scratch" (section "The compute
// thread") adds a mask tile to the scaled scores before the softmax:
// score(i, j) = q_i' . k_j' / sqrt(d) + mask(i, j), with -inf hiding a key;
// the "Kohaku-TT" page lists masks among its flash-attention features. Here
// the mask is one bf16 [mask_len, mask_ld] array over in-sequence (query,
// key) indices, shared by every sequence and head, optionally combined with
// the causal mask. A row that sees no key gets out = 0 and lse = -inf.
//
// It runs after the forward's own prologue (schedule, cos/sin table, K'
// head-major) and reuses the forward's operand layouts and MMA issue
// helpers, but with a plain structure: one CTA per work item (sequence,
// packed q-tile, KV head) and an exact online softmax (O rescaled whenever
// the row maximum grows), one row per thread. The mask is added to the raw
// scores as mask * sqrt(d), so the forward's log2(e)/sqrt(d) scaling of the
// exponent applies unchanged.
//
// Warp roles (256 threads): warp 0 TMA (Q once, then K/V tiles through two
// stages); warp 1 TMEM allocation and the S = Q K^T / O += P V issuer (S of
// tile j+1 issued before P V of tile j, two S buffers); warps 4-7 the Q
// rotation, the softmax (mask row of the next tile loaded before its scores
// are ready) and the epilogue. Tensor memory: S buffers at columns 0 and
// 128 (P overwrites the first half of each 64-key half, as in the forward),
// O at column 256.
#pragma once

#include "attn_kernel.cuh"
#include "common.cuh"
#include "prep_kernel.cuh"
#include "ptx.cuh"
#include "rope_round.cuh"

namespace gqa {

constexpr int MK_THREADS = 256;

struct MaskedParams {
  AttnParams base;            // the forward's schedule, table, outputs and shapes
  const __nv_bfloat16* mask;  // [mask_len][mask_ld], additive, in scaled-score units
  int mask_len;               // every sequence must be at most this long
  int mask_ld;                // elements between mask rows (a multiple of 8)
  float sqrt_d;               // raw score += mask * sqrt(d)
};

template <int D>
struct MaskedCfg {
  using A = AttnCfg<D>;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = A::Q_BYTES;             // two stages
  static constexpr int OFF_V = OFF_K + 2 * A::KV_BYTES;  // two stages
  static constexpr int OFF_BAR = OFF_V + 2 * A::KV_BYTES;
  static constexpr int SMEM_USED = OFF_BAR + 256 + 1024;
  // at least 120 KB, so that one CTA (which takes all 512 TMEM columns) runs per SM
  static constexpr int SMEM_BYTES = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t O_COL = 256;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0, "swizzle atoms 1024-aligned");
};

struct MaskedBarriers {
  uint64_t q_loaded, q_ready;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_full, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(MaskedBarriers) <= 256, "barrier area");

// The 128 mask values of query row `mrow` for keys [key0, key0 + 128) as
// bf16 pairs (key0 + 2e in the low half of m[e]); keys at or past L read 0
// (the length mask hides them).
__device__ __forceinline__ void load_mask_row(const __nv_bfloat16* mrow, int key0, int L, uint32_t* m) {
#pragma unroll
  for (int q4 = 0; q4 < 16; ++q4) {
    const int key = key0 + 8 * q4;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (mrow) {
      if (key + 8 <= L) {
        w = __ldg(reinterpret_cast<const uint4*>(mrow + key));
      } else if (key < L) {
        uint32_t h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = key + e < L ? (uint32_t)__bfloat16_as_ushort(mrow[key + e]) : 0u;
        w = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
      }
    }
    m[4 * q4] = w.x;
    m[4 * q4 + 1] = w.y;
    m[4 * q4 + 2] = w.z;
    m[4 * q4 + 3] = w.w;
  }
}

template <int D>
__global__ void __launch_bounds__(MK_THREADS, 1)
    gqa_attn_fwd_masked_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const MaskedParams mp) {
  using A = AttnCfg<D>;
  using C = MaskedCfg<D>;
  const AttnParams& p = mp.base;
  const int n_items = ptx::ld_cg_s32(p.header) * p.nkv;
  if ((int)blockIdx.x >= n_items) return;  // the whole CTA, before any barrier or TMEM use
  const WorkItem wi = decode_item(p, blockIdx.x);
  if (wi.L > mp.mask_len) {  // the mask does not cover this sequence
    if (threadIdx.x == 0) atomicCAS(&g_status, 0, kStatusBadSeqlens);
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  MaskedBarriers* bars = reinterpret_cast<MaskedBarriers*>(smem + C::OFF_BAR);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  auto B = [&](uint64_t& b) { return ptx::smem_u32(&b); };
  const int G = p.G, rows = p.tq * G;

  if (threadIdx.x == 0) {
    ptx::mbar_init(B(bars->q_loaded), 1);
    ptx::mbar_init(B(bars->q_ready), 128);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(B(bars->k_full[s]), 1);
      ptx::mbar_init(B(bars->k_empty[s]), 1);
      ptx::mbar_init(B(bars->v_full[s]), 1);
      ptx::mbar_init(B(bars->v_empty[s]), 1);
      ptx::mbar_init(B(bars->s_full[s]), 1);
      ptx::mbar_init(B(bars->p_full[s]), 128);
      ptx::mbar_init(B(bars->pv_done[s]), 1);
    }
    ptx::mbar_init(B(bars->o_full), 1);
    ptx::mbar_init(B(bars->drain), 1);
    bars->abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(&bars->tmem_base), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  // padding rows of the Q tile (never written by TMA) are zero
  if (rows < BM) {
    constexpr int CPR = A::ROWB / 16;
    const int per_box = (BM - rows) * CPR;
    for (int i = threadIdx.x; i < A::NBOX * per_box; i += MK_THREADS) {
      const int bx = i / per_box;
      const int rem = i - bx * per_box;
      const int row = rows + rem / CPR;
      *reinterpret_cast<uint4*>(smem + C::OFF_Q + bx * A::Q_BOX_BYTES +
                                swz(row * A::ROWB + (rem % CPR) * 16, A::SWZ_MASK)) = make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_smem();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    ptx::mbar_arrive_expect_tx(B(bars->q_loaded), (uint32_t)(D * 2 * rows));
    for (int b = 0; b < A::NBOX; ++b)
      ptx::tma_load_3d(sbase + C::OFF_Q + b * A::Q_BOX_BYTES, &tmQ, B(bars->q_loaded), b * A::BOXC, wi.kvh * G,
                       wi.seq_start + wi.t0);
    int nk = 0, nv = 0;
    bool ok = true;
    for (int j = 0; j < wi.nkv; ++j) {
      const int s = j & 1;
      const uint32_t par = ((j >> 1) & 1) ^ 1;
      if (!(ok = bwait_lazy(B(bars->k_empty[s]), par, abort_flag))) break;
      ptx::mbar_arrive_expect_tx(B(bars->k_full[s]), (uint32_t)A::KV_BYTES);
      for (int b = 0; b < A::NBOX; ++b)
        ptx::tma_load_3d(sbase + C::OFF_K + s * A::KV_BYTES + b * A::KV_BOX_BYTES, &tmK, B(bars->k_full[s]),
                         b * A::BOXC, wi.seq_start + j * BN, wi.kvh);
      ++nk;
      if (!(ok = bwait_lazy(B(bars->v_empty[s]), par, abort_flag))) break;
      ptx::mbar_arrive_expect_tx(B(bars->v_full[s]), (uint32_t)A::KV_BYTES);
      for (int b = 0; b < A::NBOX; ++b)
        ptx::tma_load_3d(sbase + C::OFF_V + s * A::KV_BYTES + b * A::KV_BOX_BYTES, &tmV, B(bars->v_full[s]),
                         b * A::BOXC, wi.kvh, wi.seq_start + j * BN);
      ++nv;
    }
    if (!ok) {  // every copy issued lands before the CTA exits
      drain_wait(B(bars->q_loaded), 0);
      for (int s = 0; s < 2; ++s) {
        const int uk = (nk - s + 1) / 2, uv = (nv - s + 1) / 2;
        if (uk > 0) drain_wait(B(bars->k_full[s]), (uk - 1) & 1);
        if (uv > 0) drain_wait(B(bars->v_full[s]), (uv - 1) & 1);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dq = umma_desc(sbase + C::OFF_Q, 16, A::SBO, A::UMMA_LAYOUT);
    const uint64_t dk0 = umma_desc(sbase + C::OFF_K, 16, A::SBO, A::UMMA_LAYOUT);
    const uint64_t dv0 = umma_desc(sbase + C::OFF_V, A::KV_BOX_BYTES, A::SBO, A::UMMA_LAYOUT);
    const uint64_t stage = (uint64_t)(A::KV_BYTES >> 4);
    // S(j) into buffer j & 1 once P V(j - 2), which read P from it, is done
    auto issue_s = [&](int j) -> bool {
      const int s = j & 1;
      if (j >= 2 && !bwait(B(bars->pv_done[s]), ((j - 2) >> 1) & 1, abort_flag)) return false;
      if (!bwait(B(bars->k_full[s]), (j >> 1) & 1, abort_flag)) return false;
      ptx::tc_fence_after();
      issue_s_mmas<A>(tmem + s * 128, dq, dk0 + s * stage);
      ptx::mma_commit(B(bars->s_full[s]));
      ptx::mma_commit(B(bars->k_empty[s]));
      return true;
    };
    bool ok = bwait(B(bars->q_ready), 0, abort_flag) && issue_s(0);
    for (int j = 0; ok && j < wi.nkv; ++j) {
      const int s = j & 1;
      if (j + 1 < wi.nkv && !(ok = issue_s(j + 1))) break;
      if (!(ok = bwait(B(bars->v_full[s]), (j >> 1) & 1, abort_flag))) break;
      if (!(ok = bwait(B(bars->p_full[s]), (j >> 1) & 1, abort_flag))) break;
      ptx::tc_fence_after();
      issue_pv_mmas<A>(tmem + C::O_COL, tmem + s * 128, dv0 + s * stage, j > 0);
      ptx::mma_commit(B(bars->pv_done[s]));
      ptx::mma_commit(B(bars->v_empty[s]));
    }
    if (ok) ptx::mma_commit(B(bars->o_full));
    // all tensor-core work issued here has finished before TMEM is freed
    ptx::mma_commit(B(bars->drain));
    drain_wait(B(bars->drain), 0);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ Q rotation, softmax, epilogue
    constexpr int HALF = D / 2;
    constexpr int NCH = D / 16;  // 16-byte chunks in the first half of a row
    const int tid = threadIdx.x - 128;
    const int quad = warp - 4;
    const int r = quad * 32 + lane;  // row of the tile == TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const int tt = r / G;
    const int tok = wi.t0 + tt;
    const bool row_valid = r < rows && tok < wi.L;
    bool ok = __all_sync(0xffffffffu, bwait(B(bars->q_loaded), 0, abort_flag));
    if (ok) {
      // rotate the Q tile in shared memory (the forward's bf16 rotation)
      uint8_t* qbuf = smem + C::OFF_Q;
      for (int item = tid; item < p.tq * NCH; item += 128) {
        const int it_t = item / NCH;
        const int ch = item - it_t * NCH;
        const int qt = wi.t0 + it_t;
        if (qt >= wi.L) continue;
        const float4* tab = reinterpret_cast<const float4*>(p.table + table_word(wi.seq_start + qt, HALF, ch * 8));
        const float4 cf = ptx::ld_cg_v4f32(tab), sf = ptx::ld_cg_v4f32(tab + 1);
        const uint32_t cw[4] = {__float_as_uint(cf.x), __float_as_uint(cf.y), __float_as_uint(cf.z),
                                __float_as_uint(cf.w)};
        const uint32_t sw[4] = {__float_as_uint(sf.x), __float_as_uint(sf.y), __float_as_uint(sf.z),
                                __float_as_uint(sf.w)};
        const int col_lo = ch * 8, col_hi = ch * 8 + HALF;
        for (int hh = 0; hh < G; ++hh) {
          const int row = it_t * G + hh;
          uint4* plo = reinterpret_cast<uint4*>(qbuf + (col_lo / A::BOXC) * A::Q_BOX_BYTES +
                                                swz(row * A::ROWB + (col_lo % A::BOXC) * 2, A::SWZ_MASK));
          uint4* phi = reinterpret_cast<uint4*>(qbuf + (col_hi / A::BOXC) * A::Q_BOX_BYTES +
                                                swz(row * A::ROWB + (col_hi % A::BOXC) * 2, A::SWZ_MASK));
          uint4 vlo = *plo, vhi = *phi;
          rope_bf16x2(vlo.x, vhi.x, cw[0], sw[0], vlo.x, vhi.x);
          rope_bf16x2(vlo.y, vhi.y, cw[1], sw[1], vlo.y, vhi.y);
          rope_bf16x2(vlo.z, vhi.z, cw[2], sw[2], vlo.z, vhi.z);
          rope_bf16x2(vlo.w, vhi.w, cw[3], sw[3], vlo.w, vhi.w);
          *plo = vlo;
          *phi = vhi;
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(B(bars->q_ready));
    }

    const float sl2 = p.scale_log2;
    const float sqd = mp.sqrt_d;
    const int last_key = p.causal ? tok : wi.L - 1;
    const __nv_bfloat16* mrow = row_valid ? mp.mask + (size_t)tok * mp.mask_ld : nullptr;
    float m = -INFINITY, l = 0.f;
    uint32_t sr[BN];
    uint32_t mk[BN / 2];
    for (int j = 0; ok && j < wi.nkv; ++j) {
      const int s = j & 1;
      load_mask_row(mrow, j * BN, wi.L, mk);  // before the scores are ready
      ok = __all_sync(0xffffffffu, bwait(B(bars->s_full[s]), (j >> 1) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      load_s_cols<BN>(trow + s * 128, sr);
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const uint32_t w = mk[c >> 1];
        sr[c] = __float_as_uint(fmaf(__uint_as_float(w << 16), sqd, __uint_as_float(sr[c])));
        sr[c + 1] = __float_as_uint(fmaf(__uint_as_float(w & 0xFFFF0000u), sqd, __uint_as_float(sr[c + 1])));
      }
      const int lim = last_key - j * BN;  // causal or length mask: columns > lim hidden
      if (lim < BN - 1) mask_cols<BN>(sr, lim);
      const float mx = cols_max<BN>(sr);
      const float m_new = fmaxf(m, mx);
      // The rescale is decided per row, but its wait and the tensor-memory
      // accesses are warp-collective (.sync.aligned): the whole warp enters
      // the branch when any of its rows needs it, the others scale by 1.
      const bool need = j > 0 && m != -INFINITY && m_new > m;
      if (__any_sync(0xffffffffu, need)) {
        // O holds the sum up to tile j - 1: wait for P V(j - 1), then rescale
        const float alpha = need ? ptx::ex2((m - m_new) * sl2) : 1.f;
        const uint32_t jp = j - 1;
        ok = __all_sync(0xffffffffu, bwait(B(bars->pv_done[jp & 1]), (jp >> 1) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        scale_o_cols<D>(trow + C::O_COL, alpha, mk);  // (the mask words are no longer needed)
        l *= alpha;
      }
      m = m_new;
      // a row that has seen no visible key yet keeps p = 0 (bias 0, scores -inf)
      const float bias = m == -INFINITY ? 0.f : -m * sl2;
      l += exp_pack<BN, emu_period(D)>(sr, bias, sl2, nullptr);
      ptx::tmem_st32(trow + s * 128, sr);            // keys [0, 64): columns 0..31
      ptx::tmem_st32(trow + s * 128 + 64, sr + 32);  // keys [64, 128): columns 64..95
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(B(bars->p_full[s]));
    }
    if (ok) ok = __all_sync(0xffffffffu, bwait(B(bars->o_full), 0, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
      // a row with no visible key: out = 0, lse = -inf
      const bool seen = m != -INFINITY && l > 0.f;
      const float inv_l = seen ? 1.f / l : 0.f;
      const int h = wi.kvh * G + (r - tt * G);
      const size_t orow = (size_t)(wi.seq_start + (row_valid ? tok : 0)) * p.nq + h;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        ptx::tmem_ld32(trow + C::O_COL + c * 32, sr);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(sr);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + orow * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o[e] = pack_bf16x2(__uint_as_float(sr[8 * q4 + 2 * e]) * inv_l,
                                 __uint_as_float(sr[8 * q4 + 2 * e + 1]) * inv_l);
            dst[q4] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
      if (row_valid && p.lse)
        p.lse[(size_t)h * p.N + wi.seq_start + tok] =
            seen ? (m * sl2 + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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
