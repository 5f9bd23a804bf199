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
// bandwidth, not by arithmetic: the scores and the weighted sum run on the
// FP32 pipes, and the cache streams through shared memory in TMA tiles.
//
// Kernel 1 (split): one CTA per (key range, KV head, sequence). It rotates
// the G queries of the KV head at p (and the new key, in the CTA whose range
// holds p), then walks its key range in tiles of 64 keys (2-stage TMA ring
// for K and V): scores of the tile for the G heads, an online softmax, and
// the weighted sum of V. It leaves (running max, sum, un-normalised output)
// per head in the workspace.
// Kernel 2 (combine): per (sequence, KV head) merges the ranges: out =
// sum_s o_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), lse = (M + log2 L) ln 2.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "rope_round.cuh"

namespace gqa {

constexpr int DEC_THREADS = 256;
constexpr int DEC_KT = 64;      // keys per tile
constexpr int DEC_STAGES = 2;
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

template <int D_, int GM_>
struct DecCfg {
  static constexpr int D = D_;
  static constexpr int GM = GM_;                   // query heads per KV head, at most
  static constexpr int BOXC = D >= 64 ? 64 : 32;   // columns per TMA box
  static constexpr int NBOX = D / BOXC;
  static constexpr int ROWB = BOXC * 2;            // bytes per box row (swizzle span)
  static constexpr int SWZ_MASK = ROWB == 128 ? 7 : 3;
  static constexpr int BOX_BYTES = DEC_KT * ROWB;
  static constexpr int TILE_BYTES = NBOX * BOX_BYTES;  // one K or V tile
  // Score phase: 4 lanes per key (a quarter of d each: CPQ 16-byte chunks),
  // 8 keys per warp. Weighted-sum phase: thread = (4 output columns, key
  // group of KPG keys), all heads.
  static constexpr int CPQ = D / 32;
  // Query chunk c (8 features) is stored at slot (c % CPQ) * 4 + c / CPQ, so
  // the four lanes of a key, reading chunk i of their quarters at once, hit
  // four different bank groups.
  static __device__ __forceinline__ int qslot(int c) { return (c % CPQ) * 4 + c / CPQ; }
  static constexpr int KGROUPS = DEC_THREADS / (D / 4);
  static constexpr int KPG = DEC_KT / KGROUPS;
  static constexpr int OFF_KV = 0;                                 // [stage][K tile, V tile]
  static constexpr int OFF_Q = OFF_KV + DEC_STAGES * 2 * TILE_BYTES;  // float [GM][D]
  static constexpr int OFF_S = OFF_Q + GM * D * 4;                    // float [KT][GM]
  static constexpr int OFF_CS = OFF_S + GM * DEC_KT * 4;              // float2 [D/2] (cos, sin)
  static constexpr int OFF_ML = OFF_CS + (D / 2) * 8;                 // float2 [GM] running (max, sum)
  static constexpr int OFF_A = OFF_ML + GM * 8;                       // float [GM] rescale of the tile
  static constexpr int OFF_NEW = OFF_A + GM * 4;                      // bf16 [2][D]: rotated new key, value
  static constexpr int OFF_BAR = OFF_NEW + 2 * D * 2;                 // mbarriers [STAGES]
  static constexpr int SMEM_BYTES = ((OFF_BAR + DEC_STAGES * 8 + 15) / 16) * 16 + 1024;  // + alignment slack
  static_assert(DEC_THREADS == 4 * DEC_KT, "score phase: four lanes per key");
  static_assert(KPG * KGROUPS == DEC_KT, "weighted-sum key groups");
  static_assert(GM * D * 4 <= DEC_STAGES * 2 * TILE_BYTES, "final reduction buffer in the stage area");
  static_assert(SMEM_BYTES <= 113 * 1024, "two CTAs per SM");
};

__device__ __forceinline__ uint32_t dswz(uint32_t lin, int mask) { return lin ^ (((lin >> 7) & mask) << 4); }

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Bounded wait (2 s) for one mbarrier phase; false (and the device status
// word set) when it runs out.
__device__ __forceinline__ bool dec_wait(uint32_t bar, uint32_t parity) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer() - t0 > WAIT_TIMEOUT_NS) {
      atomicCAS(&g_status, 0, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// d = a * b + c on pairs of fp32 (one packed .f32x2 instruction).
__device__ __forceinline__ float2 dec_ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

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

template <int D, int GM>
__global__ void __launch_bounds__(DEC_THREADS, 2)
    gqa_decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const DecodeParams p) {
  using C = DecCfg<D, GM>;
  extern __shared__ uint8_t dec_smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer
  // arithmetic so that accesses through it stay shared-memory accesses
  uint8_t* sm = dec_smem_raw + ((1024u - (ptx::smem_u32(dec_smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = p.G;
  const int pos = __ldg(p.cache_seqlens + b);
  if (pos < 0 || pos >= p.Lmax) {  // the combine kernel skips this sequence too
    if (tid == 0 && split == 0 && h == 0) atomicCAS(&g_status, 0, kStatusBadSeqlens);
    return;
  }
  const int k0 = split * p.kps;
  const int k1 = min(k0 + p.kps, pos + 1);
  const size_t part = ((size_t)b * p.nkv + h) * p.splits + split;
  float2* pml = p.part_ml + part * G;
  float* po = p.part_o + part * G * D;
  if (k0 >= k1) {  // no visible key in this range
    for (int i = tid; i < G; i += DEC_THREADS) pml[i] = make_float2(-INFINITY, 0.f);
    return;
  }
  const int ntiles = (k1 - k0 + DEC_KT - 1) / DEC_KT;
  const bool has_new = pos >= k0 && pos < k1;

  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  if (tid == 0) {
    for (int i = 0; i < DEC_STAGES; ++i) ptx::mbar_init(ptx::smem_u32(&full[i]), 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();

  const int row0 = b * p.Lmax + k0;  // key coordinate of the range's first row in the maps
  auto issue = [&](int t) {
    const int st = t % DEC_STAGES;
    const uint32_t bar = ptx::smem_u32(&full[st]);
    const uint32_t dk = ptx::smem_u32(sm + C::OFF_KV + st * 2 * C::TILE_BYTES);
    ptx::mbar_arrive_expect_tx(bar, 2u * C::TILE_BYTES);
#pragma unroll
    for (int bx = 0; bx < C::NBOX; ++bx) {
      ptx::tma_load_3d(dk + bx * C::BOX_BYTES, &tmK, bar, bx * C::BOXC, h, row0 + t * DEC_KT);
      ptx::tma_load_3d(dk + C::TILE_BYTES + bx * C::BOX_BYTES, &tmV, bar, bx * C::BOXC, h, row0 + t * DEC_KT);
    }
  };
  if (tid == 0)
    for (int t = 0; t < min(DEC_STAGES, ntiles); ++t)
      if (!(p.test_drop_first_load && t == 0)) issue(t);

  // ---- RoPE at position pos: cos/sin (float64 angle, fp32 values, as in the
  // prefill), the G queries of KV head h, and the new key if this range
  // holds pos. The rotated values are rounded once to bf16.
  float* qs = reinterpret_cast<float*>(sm + C::OFF_Q);
  float2* cs = reinterpret_cast<float2*>(sm + C::OFF_CS);
  __nv_bfloat16* knew = reinterpret_cast<__nv_bfloat16*>(sm + C::OFF_NEW);
  __nv_bfloat16* vnew = knew + D;
  for (int i = tid; i < D / 2; i += DEC_THREADS) {
    double sd, cd;
    sincos((double)pos * p.inv_freq[i], &sd, &cd);
    cs[i] = make_float2((float)cd, (float)sd);
  }
  __syncthreads();
  const int nrot = (G + (has_new ? 1 : 0)) * (D / 2);
  for (int it = tid; it < nrot; it += DEC_THREADS) {
    const int row = it / (D / 2), i = it - row * (D / 2);
    const float2 c = cs[i];
    const __nv_bfloat16* src =
        row < G ? p.q + ((size_t)b * p.nq + h * G + row) * D : p.k_new + ((size_t)b * p.nkv + h) * D;
    const float xl = __bfloat162float(src[i]), xh = __bfloat162float(src[i + D / 2]);
    const uint16_t lo = rope_round_bf16(xl, c.x, xh, -c.y), hi = rope_round_bf16(xh, c.x, xl, c.y);
    if (row < G) {
      qs[row * D + C::qslot(i / 8) * 8 + i % 8] = __uint_as_float((uint32_t)lo << 16);
      qs[row * D + C::qslot((i + D / 2) / 8) * 8 + i % 8] = __uint_as_float((uint32_t)hi << 16);
    } else {
      knew[i] = __ushort_as_bfloat16(lo);
      knew[i + D / 2] = __ushort_as_bfloat16(hi);
    }
  }
  if (has_new)
    for (int i = tid; i < D; i += DEC_THREADS) vnew[i] = p.v_new[((size_t)b * p.nkv + h) * D + i];
  float* sp = reinterpret_cast<float*>(sm + C::OFF_S);
  float2* mls = reinterpret_cast<float2*>(sm + C::OFF_ML);
  float* alpha_s = reinterpret_cast<float*>(sm + C::OFF_A);
  if (tid < GM) mls[tid] = make_float2(-INFINITY, 0.f);
  __syncthreads();

  // weighted-sum phase: this thread's columns and key group
  const int cq = tid % (D / 4);
  const int kg = tid / (D / 4);
  const int col = cq * 4;
  const uint32_t vcol_off = (col / C::BOXC) * C::BOX_BYTES;
  const uint32_t vcol_in = (col % C::BOXC) * 2;
  float2 o[GM][2];  // columns (col, col + 1), (col + 2, col + 3) per head
#pragma unroll
  for (int g = 0; g < GM; ++g) o[g][0] = o[g][1] = make_float2(0.f, 0.f);

  int t_fail = -1;
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % DEC_STAGES;
    uint8_t* kt = sm + C::OFF_KV + st * 2 * C::TILE_BYTES;
    uint8_t* vt = kt + C::TILE_BYTES;
    const bool landed = dec_wait(ptx::smem_u32(&full[st]), (t / DEC_STAGES) & 1);
    if (__syncthreads_or(!landed)) {
      t_fail = t;
      break;
    }
    const int tstart = k0 + t * DEC_KT;
    const int nvalid = min(DEC_KT, k1 - tstart);
    if (has_new && pos >= tstart && pos < tstart + DEC_KT) {
      // the new token's row comes from this CTA, not from the cache
      const int r = pos - tstart;
      for (int c = tid; c < D / 8; c += DEC_THREADS) {
        const int bx = c / (C::BOXC / 8), ch = c % (C::BOXC / 8);
        const uint32_t off = bx * C::BOX_BYTES + dswz(r * C::ROWB + ch * 16, C::SWZ_MASK);
        *reinterpret_cast<uint4*>(kt + off) = *reinterpret_cast<const uint4*>(knew + c * 8);
        *reinterpret_cast<uint4*>(vt + off) = *reinterpret_cast<const uint4*>(vnew + c * 8);
      }
      ptx::fence_proxy_async_smem();
      __syncthreads();
    }

    // ---- scores, log2 units: lanes (key, d quarter), all heads
    {
      const int key = warp * 8 + (lane & 7);
      const int dq = lane >> 3;
      float2 acc2[GM];  // two partial sums per head (even / odd features)
#pragma unroll
      for (int g = 0; g < GM; ++g) acc2[g] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < C::CPQ; ++i) {
        const int c = dq * C::CPQ + i;
        const int bx = c / (C::BOXC / 8), ch = c % (C::BOXC / 8);
        const uint4 kw = *reinterpret_cast<const uint4*>(kt + bx * C::BOX_BYTES +
                                                         dswz(key * C::ROWB + ch * 16, C::SWZ_MASK));
        const float2 k01 = make_float2(bf_lo(kw.x), bf_hi(kw.x)), k23 = make_float2(bf_lo(kw.y), bf_hi(kw.y));
        const float2 k45 = make_float2(bf_lo(kw.z), bf_hi(kw.z)), k67 = make_float2(bf_lo(kw.w), bf_hi(kw.w));
#pragma unroll
        for (int g = 0; g < GM; ++g) {
          if (g < G) {
            const float4 qa = *reinterpret_cast<const float4*>(qs + g * D + (i * 4 + dq) * 8);
            const float4 qb = *reinterpret_cast<const float4*>(qs + g * D + (i * 4 + dq) * 8 + 4);
            float2 a = acc2[g];
            a = dec_ffma2(make_float2(qa.x, qa.y), k01, a);
            a = dec_ffma2(make_float2(qa.z, qa.w), k23, a);
            a = dec_ffma2(make_float2(qb.x, qb.y), k45, a);
            a = dec_ffma2(make_float2(qb.z, qb.w), k67, a);
            acc2[g] = a;
          }
        }
      }
      float acc[GM];
#pragma unroll
      for (int g = 0; g < GM; ++g) acc[g] = acc2[g].x + acc2[g].y;
#pragma unroll
      for (int g = 0; g < GM; ++g) {
        acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 8);
        acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 16);
        if (g < G && (g & 3) == dq) sp[key * GM + g] = key < nvalid ? acc[g] * p.scale_log2 : -INFINITY;
      }
    }
    __syncthreads();

    // ---- online softmax: warp w takes heads w, w + 8
    for (int g = warp; g < G; g += DEC_THREADS / 32) {
      const float s0 = sp[lane * GM + g], s1 = sp[(lane + 32) * GM + g];
      const float2 ml = mls[g];
      const float mnew = fmaxf(ml.x, warp_max(fmaxf(s0, s1)));  // finite: key tstart is visible
      const float p0 = ptx::ex2(s0 - mnew), p1 = ptx::ex2(s1 - mnew);
      const float sum = warp_sum(p0 + p1);
      const float a = ptx::ex2(ml.x - mnew);
      sp[lane * GM + g] = p0;
      sp[(lane + 32) * GM + g] = p1;
      __syncwarp();
      if (lane == 0) {
        mls[g] = make_float2(mnew, ml.y * a + sum);
        alpha_s[g] = a;
      }
    }
    __syncthreads();

    // ---- O = O * a + P V: this thread's 4 columns, its key group, all heads
    {
#pragma unroll
      for (int g = 0; g < GM; ++g) {
        if (g < G) {
          const float a = alpha_s[g];
          o[g][0].x *= a; o[g][0].y *= a; o[g][1].x *= a; o[g][1].y *= a;
        }
      }
#pragma unroll 2
      for (int j = 0; j < C::KPG; ++j) {
        const int k = kg * C::KPG + j;
        if (k < nvalid) {  // uniform across the warp
          const uint2 vw = *reinterpret_cast<const uint2*>(vt + vcol_off + dswz(k * C::ROWB + vcol_in, C::SWZ_MASK));
          const float2 v01 = make_float2(bf_lo(vw.x), bf_hi(vw.x)), v23 = make_float2(bf_lo(vw.y), bf_hi(vw.y));
#pragma unroll
          for (int g4 = 0; g4 < GM / 4; ++g4) {
            if (4 * g4 < G) {
              const float4 pk = *reinterpret_cast<const float4*>(sp + k * GM + 4 * g4);
              const float pv[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int g = 4 * g4 + e;
                if (g < G) {
                  const float2 pp = make_float2(pv[e], pv[e]);
                  o[g][0] = dec_ffma2(pp, v01, o[g][0]);
                  o[g][1] = dec_ffma2(pp, v23, o[g][1]);
                }
              }
            }
          }
        }
      }
    }
    __syncthreads();  // stage and scores free
    if (tid == 0 && t + DEC_STAGES < ntiles) issue(t + DEC_STAGES);
  }

  if (t_fail >= 0) {
    // tiles t_fail .. t_fail + STAGES - 1 may still be in flight: let them
    // land (bounded waits) before the CTA exits
    if (tid == 0)
      for (int t = t_fail; t < min(ntiles, t_fail + DEC_STAGES); ++t)
        dec_wait(ptx::smem_u32(&full[t % DEC_STAGES]), (t / DEC_STAGES) & 1);
    __syncthreads();
    return;
  }

  // ---- this range's partial results: the key groups' sums, added in a
  // fixed order (group 0 first) in shared memory (the stage area is free)
  float* red = reinterpret_cast<float*>(sm + C::OFF_KV);  // [G][D]
  for (int i = tid; i < G * D; i += DEC_THREADS) red[i] = 0.f;
  __syncthreads();
  for (int r = 0; r < C::KGROUPS; ++r) {
    if (kg == r) {
#pragma unroll
      for (int g = 0; g < GM; ++g) {
        if (g < G) {
          float4* dst = reinterpret_cast<float4*>(red + g * D + col);
          const float4 cur = *dst;
          *dst = make_float4(cur.x + o[g][0].x, cur.y + o[g][0].y, cur.z + o[g][1].x, cur.w + o[g][1].y);
        }
      }
    }
    __syncthreads();
  }
  for (int i = tid; i < G * D / 4; i += DEC_THREADS)
    reinterpret_cast<float4*>(po)[i] = reinterpret_cast<const float4*>(red)[i];
  for (int i = tid; i < G; i += DEC_THREADS) pml[i] = mls[i];
  // the appended cache row (after every load of this CTA has landed)
  if (has_new) {
    const size_t row = (((size_t)b * p.Lmax + pos) * p.nkv + h) * D;
    for (int i = tid; i < D / 8; i += DEC_THREADS) {
      reinterpret_cast<uint4*>(p.k_cache + row)[i] = reinterpret_cast<const uint4*>(knew)[i];
      reinterpret_cast<uint4*>(p.v_cache + row)[i] = reinterpret_cast<const uint4*>(vnew)[i];
    }
  }
}

// Merge of the key ranges of one (sequence, KV head); threads over
// (head, column).
__global__ void __launch_bounds__(DEC_THREADS) gqa_decode_combine_kernel(const DecodeParams p, int D) {
  const int h = blockIdx.x, b = blockIdx.y;
  const int G = p.G;
  const int pos = __ldg(p.cache_seqlens + b);
  if (pos < 0 || pos >= p.Lmax) return;
  const int used = min(p.splits, pos / p.kps + 1);  // ranges holding a visible key
  const size_t part0 = ((size_t)b * p.nkv + h) * p.splits;
  for (int u = threadIdx.x; u < G * D; u += DEC_THREADS) {
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
