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
// whose range holds p), then walks its key range in tiles of 64 keys through
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
constexpr int DEC_KT = 64;      // keys per tile (the cache maps' box height)
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
// Both products on the tensor cores (tcgen05): the G rotated query heads of KV head
// h fill G rows of a 128-row operand tile (the other rows are zero), so
// S = Q K^T over a 64-key tile is one M = 128, N = 64 MMA into tensor memory
// and O += P V one M = 128, N = d MMA with P read from tensor memory, the
// operand forms of the prefill kernel. Head g sits at tile row
// 32 (g % 4) + g / 4, so each of the four softmax warps (one TMEM lane
// quadrant each) holds a share of the heads. Per CTA: one key range of one
// (sequence, KV head), its partial (max, sum, un-normalised output) per head
// for the combine kernel. (A CUDA-core version of this kernel, scores and
// weighted sum on the FP32 pipes, reached 3.5 TB/s at G = 4 and 2.1 TB/s at
// G = 8 on B200; this one 4.2 and 4.0.)
//
// Warps 0-3: RoPE of the queries and the new key, then the online softmax
// (one row per thread; rows that hold no head compute zeros) and the partial
// results. Warp 4: TMA of the K/V tiles through a two-stage ring, the
// fix-up of the range's last tile (the new token's row from this CTA, rows
// past the range zeroed in V so that their zero weights meet finite values)
// and the appended cache row. Warp 5: tensor memory and the MMAs.
// One CTA per SM with a four-stage ring (measured: two stages with two CTAs
// per SM reached 2.7 TB/s, three 3.7, four to six 4.1-4.2).
constexpr int DTC_KT = DEC_KT;   // keys per tile
constexpr int DTC_STAGES = 4;
constexpr int DTC_THREADS = 192;

template <int D_>
struct DtcCfg {
  using A = AttnCfg<D_>;
  static constexpr int D = D_;
  static constexpr int KV_BOX_BYTES = DTC_KT * A::ROWB;      // one box of a 64-key tile
  static constexpr int TILE_BYTES = A::NBOX * KV_BOX_BYTES;  // one K or V tile
  static constexpr int OFF_Q = 0;                            // 128-row query tile
  static constexpr int OFF_K = A::Q_BYTES;                   // [stage] K tiles
  static constexpr int OFF_V = OFF_K + DTC_STAGES * TILE_BYTES;  // [stage] V tiles
  static constexpr int OFF_CS = OFF_V + DTC_STAGES * TILE_BYTES;  // uint2 [D/4]: bf16x2 (cos, sin) at pos
  static constexpr int OFF_NEW = OFF_CS + (D / 2) * 8;           // bf16 [2][D]: rotated new key, value
  static constexpr int OFF_BAR = OFF_NEW + 2 * D * 2;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;       // + barriers + alignment slack
  static constexpr uint32_t S_COL = 0;                          // two 64-column S/P buffers
  static constexpr uint32_t O_COL = 2 * DTC_KT;
  static constexpr uint32_t TMEM_COLS = 256;
  // bf16 x bf16 -> fp32, both K-major, M = 128, N = 64 keys
  static constexpr uint32_t IDESC_S =
      (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(DTC_KT >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
  static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && TILE_BYTES % 1024 == 0, "swizzle atoms 1024-aligned");
  static_assert(O_COL + D <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct DtcBarriers {
  uint64_t full[DTC_STAGES], empty[DTC_STAGES];
  uint64_t fixed;     // the range's last tile patched in shared memory
  uint64_t q_ready;   // query tile, new key and value written (128 arrivals)
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_full, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(DtcBarriers) <= 256, "barrier area");

__device__ __forceinline__ void dtc_softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(DTC_THREADS, 1)
    gqa_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const DecodeParams p) {
  using C = DtcCfg<D>;
  using A = AttnCfg<D>;
  constexpr int HALF = D / 2;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = p.G;
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
  const int last_valid = k1 - last_start;  // keys of the last tile inside the range, 1..64
  const bool fix_last = has_new || last_valid < DTC_KT;

  extern __shared__ uint8_t dtc_smem_raw[];
  uint8_t* smem = dtc_smem_raw + ((1024u - (ptx::smem_u32(dtc_smem_raw) & 1023u)) & 1023u);
  DtcBarriers* bars = reinterpret_cast<DtcBarriers*>(smem + C::OFF_BAR);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;
  auto B = [&](uint64_t& x) { return ptx::smem_u32(&x); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < DTC_STAGES; ++s) {
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
    ptx::mbar_init(B(bars->drain), 1);
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
        const int st = t % DTC_STAGES;
        if (!(ok = bwait_lazy(B(bars->empty[st]), ((t / DTC_STAGES) & 1) ^ 1, abort_flag))) break;
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
    const int tl = ntiles - 1, stl = tl % DTC_STAGES;
    if (ok && fix_last) {
      // the last tile: the new token's rotated key and value in row pos, and
      // V rows past the range zero (their weights are zero; the cache rows
      // there may hold anything)
      ok = __all_sync(0xffffffffu, bwait(B(bars->full[stl]), (tl / DTC_STAGES) & 1, abort_flag) &&
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
      for (int t = first; t < first + issued; ++t)
        drain_wait(B(bars->full[t % DTC_STAGES]), (t / DTC_STAGES) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dq = umma_desc(sbase + C::OFF_Q, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t dk0 = umma_desc(sbase + C::OFF_K, 16, A::SBO, A::UMMA_LAYOUT);
      const uint64_t dv0 = umma_desc(sbase + C::OFF_V, C::KV_BOX_BYTES, A::SBO, A::UMMA_LAYOUT);
      const uint64_t stage = (uint64_t)(C::TILE_BYTES >> 4);
      // S(j) into S buffer j & 1 once K(j) is in place and P V(j - 2), which
      // read P from that buffer, is done
      auto issue_s = [&](int j) -> bool {
        const int sb = j & 1, st = j % DTC_STAGES;
        if (j >= 2 && !bwait(B(bars->pv_done[sb]), ((j - 2) >> 1) & 1, abort_flag)) return false;
        const bool w = (j == ntiles - 1 && fix_last) ? bwait(B(bars->fixed), 0, abort_flag)
                                                     : bwait(B(bars->full[st]), (j / DTC_STAGES) & 1, abort_flag);
        if (!w) return false;
        ptx::tc_fence_after();
        const uint64_t dk = dk0 + st * stage;
#pragma unroll
        for (int kk = 0; kk < A::KSTEPS_S; ++kk) {
          const uint32_t off_q = (kk / A::STEPS_PER_BOX) * A::Q_BOX_BYTES + (kk % A::STEPS_PER_BOX) * 32;
          const uint32_t off_k = (kk / A::STEPS_PER_BOX) * C::KV_BOX_BYTES + (kk % A::STEPS_PER_BOX) * 32;
          ptx::mma_ss(tmem + C::S_COL + sb * DTC_KT, dq + (uint64_t)(off_q >> 4), dk + (uint64_t)(off_k >> 4),
                      C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(B(bars->s_full[sb]));
        return true;
      };
      bool ok = bwait(B(bars->q_ready), 0, abort_flag) && issue_s(0);
      for (int j = 0; ok && j < ntiles; ++j) {
        const int sb = j & 1, st = j % DTC_STAGES;
        if (j + 1 < ntiles && !(ok = issue_s(j + 1))) break;
        if (!(ok = bwait(B(bars->p_full[sb]), (j >> 1) & 1, abort_flag))) break;
        ptx::tc_fence_after();
        // O (+)= P V: 64 keys in 4 K-steps of 16, P from the S buffer's first 32 columns
#pragma unroll
        for (int kk = 0; kk < DTC_KT / 16; ++kk)
          ptx::mma_ts(tmem + C::O_COL, tmem + C::S_COL + sb * DTC_KT + kk * 8,
                      dv0 + st * stage + (uint64_t)((kk * 16 * A::ROWB) >> 4), A::IDESC_O,
                      (j > 0 || kk > 0) ? 1u : 0u);
        ptx::mma_commit(B(bars->pv_done[sb]));
        ptx::mma_commit(B(bars->empty[st]));
      }
      if (ok) ptx::mma_commit(B(bars->o_full));
      // all tensor-core work issued here has finished before TMEM is freed
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
  } else {
    // ------------------------------------------------------------ RoPE, softmax, partial results
    const int tid = threadIdx.x;  // 0..127 == tile row == TMEM lane
    const int g = 4 * lane + warp;  // the head of this row (a row past G holds none)
    const bool active = g < G;
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    uint2* cs = reinterpret_cast<uint2*>(smem + C::OFF_CS);
    __nv_bfloat16* knew = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_NEW);
    // zero query tile; bf16x2 (cos, sin) words of frequencies (2j, 2j + 1) at
    // pos (float64 angle, rounded to fp32, then to bf16 as in the prefill)
    for (int i = tid; i < A::Q_BYTES / 16; i += 128)
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
    // rotated queries into their tile rows, and the new key (if this range
    // holds pos), two frequencies per item, in the prefill's bf16 rotation
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
        const int row = 32 * (hg % 4) + hg / 4;
        const int cl = i, chh = i + HALF;
        *reinterpret_cast<uint32_t*>(smem + C::OFF_Q + (cl / A::BOXC) * A::Q_BOX_BYTES +
                                     swz(row * A::ROWB + (cl % A::BOXC) * 2, A::SWZ_MASK)) = lo;
        *reinterpret_cast<uint32_t*>(smem + C::OFF_Q + (chh / A::BOXC) * A::Q_BOX_BYTES +
                                     swz(row * A::ROWB + (chh % A::BOXC) * 2, A::SWZ_MASK)) = hi;
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
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t sr[DTC_KT];
    uint32_t ob[32];  // scratch of the O rescale
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, bwait(B(bars->s_full[sb]), (j >> 1) & 1, abort_flag));
      if (!ok) break;
      ptx::tc_fence_after();
      load_s_cols<DTC_KT>(trow + C::S_COL + sb * DTC_KT, sr);
      const int nvalid = min(DTC_KT, k1 - (k0 + j * DTC_KT));
      if (nvalid < DTC_KT) mask_cols<DTC_KT>(sr, nvalid - 1);
      const float mx = cols_max<DTC_KT>(sr);
      // exponentials against the running max; it moves only when a score
      // exceeds it by more than the threshold (the first tile sets it)
      const bool need = mx > m + thr;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? mx : m;
        if (j > 0) {
          const float alpha = need ? ptx::ex2((m - m_new) * sl2) : 1.f;
          const int jp = j - 1;
          ok = __all_sync(0xffffffffu, bwait(B(bars->pv_done[jp & 1]), (jp >> 1) & 1, abort_flag));
          if (!ok) break;
          ptx::tc_fence_after();
          scale_o_cols<D>(trow + C::O_COL, alpha, ob);
          l *= alpha;
        }
        m = m_new;
      }
      l += exp_pack<DTC_KT, emu_period(D)>(sr, -m * sl2, sl2, nullptr);
      ptx::tmem_st32(trow + C::S_COL + sb * DTC_KT, sr);  // P (bf16 pairs) in the buffer's first 32 columns
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(B(bars->p_full[sb]));
    }
    if (ok) ok = __all_sync(0xffffffffu, bwait(B(bars->o_full), 0, abort_flag));
    if (ok) {
      ptx::tc_fence_after();
      float* po = p.part_o + (part * G + (active ? g : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        ptx::tmem_ld32(trow + C::O_COL + c * 32, sr);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(sr);
        if (active) {
          float4* dst = reinterpret_cast<float4*>(po + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(sr[4 * e]), __uint_as_float(sr[4 * e + 1]),
                                 __uint_as_float(sr[4 * e + 2]), __uint_as_float(sr[4 * e + 3]));
        }
      }
      if (active) p.part_ml[part * G + g] = make_float2(m * sl2, l);
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
