// Fused causal GQA + RoPE attention forward for sm_100a.
//
// What it computes ("Attention from Scratch", section "Attention, the math:
// Grouped-Query Attention with RoPE'd Q/K"): for every query head h of KV
// group kv = h / G, softmax(rope(q) . rope(k)^T / sqrt(d) + causal mask) . v,
// plus the natural-log log-sum-exp of every row. The score matrix never
// leaves the SM ("Coming from CUDA: FlashAttention"): each KV tile's scores
// are produced in tensor memory, turned into probabilities by an online
// (running max / running sum) softmax and consumed by the P.V product.
//
// Masked form (MASK): the additive mask of the same page's section "The
// compute thread" (and the masks of the "Kohaku-TT" page): each softmax
// thread adds mask[token, key] * sqrt(d) to its raw scores, the values of
// the next KV tile loaded from global memory while the current one runs; a
// row that sees no key gets out = 0 and lse = -inf.
//
// One persistent CTA per SM takes work items (sequence, q-tile, KV head)
// from a longest-first list: its first item statically, every further one
// from a global counter (greedy list scheduling, so that faster CTAs take
// more items), or, for short lists, from a static alternating deal. A q-tile
// packs tq = 128 / G tokens times the G query heads of one KV head into 128
// MMA rows, so every K/V tile loaded by TMA is used by all G heads at once.
//
// Warp roles (512 threads):
//   warp 0      TMA producer: K tiles (K is RoPE'd already); work items
//   warp 1      TMEM allocator; one thread issues the S = Q K^T MMAs
//   warp 2      TMA producer: V tiles
//   warp 3      one thread issues the O += P V MMAs
//   warps 4-11  softmax: a row (TMEM lane) is shared by two threads, warps
//               4-7 take its columns [0, 64) and warps 8-11 columns
//               [64, 128); S -> P, running max and partial sums, O
//               rescale. At d <= 64 each half keeps its own running max
//               and sum and accumulates into its own partial output (O_a
//               or O_b), so the two never wait for each other; at d = 128
//               they share one O and exchange their tile maxima once per
//               tile (two outputs would not leave room for three S buffers)
//   warps 12-15 Q tiles: TMA load, RoPE applied in shared memory before the
//               first S MMA reads it; epilogue: O / l from TMEM, LSE
// Two softmax warps per SM sub-partition keep the special-function unit
// busy while either one waits on its in-order instruction stream.
//
// Tensor memory (512 columns x 128 lanes of 32 bit):
//   [0,128) [128,256) [256,384): three S buffers; the bf16 P of each column
//   half overwrites the first 32 columns of that half's S columns (keys
//   [0, 64) at +0, keys [64, 128) at +64); from 384: O (d = 128), or O_a and
//   O_b (d <= 64, d columns each), which the epilogue combines as the two
//   partial sums of a split softmax: O = (a_a O_a + a_b O_b) / (a_a l_a +
//   a_b l_b) with a_h = 2^(m_h - max(m_a, m_b)).
// MMAs: S = Q K^T     kind::f16, A = Q (smem, K-major), B = K (smem,
//                     K-major), M = 128, N = 128, fp32 accumulate, d/16 steps;
//       O += P V        A = P (tmem), B = V (smem, MN-major), M = 128,
//                     N = d, 8 steps of 16 keys; at d <= 64 as
//                     O_h += P_h V_h, 4 steps over the keys of half h.
#pragma once

#include "common.cuh"
#include "exp2_poly.cuh"
#include "ptx.cuh"
#include "rope_round.cuh"

namespace gqa {


// Work-item hand-off ring: the K producer takes item indices and publishes
// them, decoded; every other role (V producer, S issuer, PV issuer: one
// thread each; softmax and Q warps: one arrival per warp) reads each slot
// once.
constexpr int ITEM_SLOTS = 8;
constexpr int ITEM_READERS = 3 + 8 + 4;
constexpr int KSTEPS_PV_HALF = BN / 2 / 16;  // P V K-steps of one column half

// Register split (launch: 512 threads x 128): producers/MMA 56, softmax 160
// (8 warps), Q rotation/epilogue 128 (the launch value).
constexpr int REG_PRODUCER = 56;
constexpr int REG_SOFTMAX = 160;
constexpr int REG_ROPE = 128;
static_assert(REG_PRODUCER * 128 + REG_SOFTMAX * 256 + REG_ROPE * 128 <= 65536 / ATTN_THREADS * ATTN_THREADS,
              "register split exceeds the launch's register file share");
// masked form: 8 more per softmax thread for the mask words, from the Q
// warpgroup (56 x 128 + 168 x 256 + 112 x 128 = 64512)
constexpr int REG_SOFTMAX_MASKED = 168;
constexpr int REG_ROPE_MASKED = 112;
static_assert(REG_PRODUCER * 128 + REG_SOFTMAX_MASKED * 256 + REG_ROPE_MASKED * 128 <= 65536,
              "register split exceeds the launch's register file share");

struct WorkItem {
  int seq_start, L, t0, nkv, kvh;
};

struct Barriers {
  uint64_t q_loaded[2], q_ready[2], q_empty[2];
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[NUM_S_BUF], p_full[NUM_S_BUF][2], pv_done[NUM_S_BUF];  // p_full: [buffer][column half]
  uint64_t o_free, drain;
  uint64_t stats_full, stats_empty;
  uint64_t xchg[2][4];  // (d = 128) row-max exchange of the two softmax halves: [tile parity][lane quadrant]
  uint64_t item_full[ITEM_SLOTS], item_empty[ITEM_SLOTS];
  int item[ITEM_SLOTS];  // work-item index, -1 = no more items
  WorkItem witem[ITEM_SLOTS];  // the item decoded (sequence, tile, KV head), by the publisher
  uint32_t tmem_base;
  int abort_flag;
};

template <int D_>
struct AttnCfg {
  static constexpr int D = D_;
  static constexpr int BOXC = D >= 64 ? 64 : 32;   // columns per TMA box
  static constexpr int NBOX = D / BOXC;            // boxes per row of a tile
  static constexpr int ROWB = BOXC * 2;            // bytes per box row (swizzle span)
  static constexpr int SWZ_MASK = ROWB == 128 ? 7 : 3;
  static constexpr uint64_t UMMA_LAYOUT = ROWB == 128 ? 2 : 4;  // SWIZZLE_128B / SWIZZLE_64B
  static constexpr int SBO = 8 * ROWB;             // bytes between 8-row core-matrix groups
  static constexpr int Q_BOX_BYTES = BM * ROWB;
  static constexpr int KV_BOX_BYTES = BN * ROWB;
  static constexpr int Q_BYTES = NBOX * Q_BOX_BYTES;
  static constexpr int KV_BYTES = NBOX * KV_BOX_BYTES;
  static constexpr int KST = D == 128 ? 2 : (D == 64 ? 3 : 4);
  static constexpr int VST = KST;
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_STATS = OFF_V + VST * KV_BYTES;  // float2 (m, l_half) [2][BM], softmax -> epilogue
  static constexpr int OFF_XMAX = OFF_STATS + 2 * BM * 8;   // float [2 parities][2 halves][BM]: row max exchange
  static constexpr int OFF_BAR = OFF_XMAX + 4 * BM * 4;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  // d <= 64 (SPLIT): the two softmax column halves keep their own running
  // max and sum and their own partial output, O_a (keys [0, 64) of every
  // tile) at O_COL and O_b (keys [64, 128)) at O_COL + D, and never wait
  // for each other. d = 128: one O and a running max that the halves
  // exchange once per tile (two outputs would cost the third S buffer, and
  // measured slower there).
  static constexpr bool SPLIT = D <= 64;
  static constexpr int NSB = NUM_S_BUF;
  static constexpr uint32_t O_COL = NSB * 128;
  static constexpr int KSTEPS_S = D / 16;
  static constexpr int KSTEPS_PV = BN / 16;
  static constexpr int STEPS_PER_BOX = BOXC / 16;
  // instruction descriptors: bf16 x bf16 -> fp32, M = 128
  static constexpr uint32_t IDESC_S =
      (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
  static constexpr uint32_t IDESC_O = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(D >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(sizeof(Barriers) <= BAR_BYTES, "barrier area");
  static_assert(O_COL + (SPLIT ? 2 : 1) * D <= TMEM_COLS, "tensor memory budget");
};

// Shared-memory matrix descriptor (tcgen05): start, leading/stride byte
// offsets (in 16-byte units), fixed version field 1, swizzle layout type.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint64_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (layout << 61);
}

__device__ __forceinline__ WorkItem decode_item(const AttnParams& p, int w) {
  WorkItem it;
  const int pair = w / p.nkv;
  it.kvh = w - pair * p.nkv;
  const int2 sl = ptx::ld_cg_v2s32(p.pairs + pair);  // written by the prologue grid
  it.seq_start = __ldg(p.cu + sl.x);
  it.L = __ldg(p.cu + sl.x + 1) - it.seq_start;
  it.t0 = sl.y * p.tq;
  const int t_end = p.causal ? min(it.t0 + p.tq, it.L) : it.L;
  it.nkv = (t_end + BN - 1) / BN;
  return it;
}

// Bounded wait on an mbarrier phase. Returns false if the CTA is aborting or
// the wait exceeded WAIT_TIMEOUT_NS (then the abort flag and the device
// status word are set). The abort flag and the clock are checked only every
// 8 polls.
__device__ __forceinline__ bool bwait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer() - t0 > WAIT_TIMEOUT_NS) {
      *abort_flag = 1;
      atomicCAS(&g_status, 0, kStatusTimeout);
      return false;
    }
  }
}

// Bounded wait for waiters off the critical path (TMA producers, the Q
// rotation warps): between polls the warp sleeps with exponential backoff
// (32 ns .. 1 us), so that it takes no issue slots from the softmax warps
// that share its scheduler.
__device__ __forceinline__ bool bwait_lazy(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  uint32_t ns = 32;
  while (true) {
    __nanosleep(ns);
    if (ns < 1024) ns <<= 1;
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer() - t0 > WAIT_TIMEOUT_NS) {
      *abort_flag = 1;
      atomicCAS(&g_status, 0, kStatusTimeout);
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if (ptx::globaltimer() - t0 > WAIT_TIMEOUT_NS) {
      atomicCAS(&g_status, 0, kStatusTimeout);
      return;
    }
  }
}

__device__ __forceinline__ WorkItem load_witem(const WorkItem* src) {
  const volatile int* v = reinterpret_cast<const volatile int*>(src);
  WorkItem wi;
  wi.seq_start = v[0];
  wi.L = v[1];
  wi.t0 = v[2];
  wi.nkv = v[3];
  wi.kvh = v[4];
  return wi;
}

__device__ __forceinline__ void store_witem(WorkItem* dst, const WorkItem& wi) {
  volatile int* v = reinterpret_cast<volatile int*>(dst);
  v[0] = wi.seq_start;
  v[1] = wi.L;
  v[2] = wi.t0;
  v[3] = wi.nkv;
  v[4] = wi.kvh;
}

// Work item k of this CTA from the hand-off ring (-1: none left) with its
// decoded fields, read by one thread (take_item) or by a whole warp
// (take_item_warp, one arrival).
__device__ __forceinline__ bool take_item(Barriers* bars, int k, int& w, WorkItem& wi, volatile int* abort_flag) {
  const int slot = k & (ITEM_SLOTS - 1);
  if (!bwait(ptx::smem_u32(&bars->item_full[slot]), (k / ITEM_SLOTS) & 1, abort_flag)) return false;
  w = *reinterpret_cast<volatile int*>(&bars->item[slot]);
  wi = load_witem(&bars->witem[slot]);
  ptx::mbar_arrive(ptx::smem_u32(&bars->item_empty[slot]));
  return true;
}
// Index of the CTA's k-th work item (k >= 1) in the longest-first list.
// Dynamic: the next unclaimed item (greedy list scheduling; it adapts to
// the actual duration of every item). Static, for lists of only a few items
// per CTA, where a claim made two items ahead is too coarse: rounds of
// gridDim.x items dealt in alternating direction (CTA b takes item b of even
// rounds and gridDim.x - 1 - b of odd ones).
__device__ __forceinline__ int next_item_index(const AttnParams& p, int k) {
  const int G = (int)gridDim.x, b = (int)blockIdx.x;
  if (p.sched_dynamic) return atomicAdd(p.item_counter, 1) + G;
  return k * G + ((k & 1) ? G - 1 - b : b);
}

// Publishes work item k (index w, -1 = none left), decoded (its global
// loads are paid here, by the producer that runs ahead, not by the roles
// that start the item), once every reader has taken item k - ITEM_SLOTS
// from the same slot.
__device__ __forceinline__ bool publish_item(const AttnParams& p, Barriers* bars, int k, int w,
                                             volatile int* abort_flag) {
  const int slot = k & (ITEM_SLOTS - 1);
  WorkItem wi{};
  if (w >= 0) wi = decode_item(p, w);
  if (k >= ITEM_SLOTS &&
      !bwait_lazy(ptx::smem_u32(&bars->item_empty[slot]), ((k / ITEM_SLOTS) - 1) & 1, abort_flag))
    return false;
  *reinterpret_cast<volatile int*>(&bars->item[slot]) = w;
  store_witem(&bars->witem[slot], wi);
  ptx::mbar_arrive(ptx::smem_u32(&bars->item_full[slot]));
  return true;
}
__device__ __forceinline__ bool take_item_warp(Barriers* bars, int k, int& w, WorkItem& wi, volatile int* abort_flag) {
  const int slot = k & (ITEM_SLOTS - 1);
  if (!__all_sync(0xffffffffu, bwait(ptx::smem_u32(&bars->item_full[slot]), (k / ITEM_SLOTS) & 1, abort_flag)))
    return false;
  w = *reinterpret_cast<volatile int*>(&bars->item[slot]);
  wi = load_witem(&bars->witem[slot]);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(ptx::smem_u32(&bars->item_empty[slot]));
  return true;
}

// 2^x on the FMA pipe, for x <= 8: x = n + f with n = rint(x) (the 1.5*2^23
// addition leaves n in the low mantissa bits), 2^f from the degree-4
// minimax polynomial of exp2_poly.cuh, n added to the exponent as an
// integer. x is clamped to -125 so the result stays a normal number
// (2^-125 is negligible next to the row maximum's 1).
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  float p = fmaf(kExp2C4, f, kExp2C3);
  p = fmaf(p, f, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, kExp2C0);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// Two fp32 -> one bf16x2 word (lo in the low half), rounded to nearest even:
// one cvt.rn.bf16x2.f32 (measured faster than packing with integer ops).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Of every emu_period(d) groups of 4 exponentials of a row, one is evaluated
// on the FMA pipe, the rest on the special-function unit (0: all on the
// SFU). Measured: at d = 128, 1 in 16 (1 in 8 while the Q rotation's fp64
// conversions also used the special-function unit); 1 in 4 and more run out
// of issue slots; at d = 64, 1 in 8.
__host__ __device__ constexpr int emu_period(int d) { return d == 128 ? 16 : 8; }

__device__ __forceinline__ uint32_t swz(uint32_t lin, int mask) { return lin ^ (((lin >> 7) & mask) << 4); }

// The packed P row (BN/2 words) into its TMEM columns.
__device__ __forceinline__ void store_p_row(uint32_t taddr, const uint32_t* r) {
#pragma unroll
  for (int c = 0; c < BN / 64; ++c) ptx::tmem_st32(taddr + c * 32, r + c * 32);
}

// D = A * B + C and A + B on pairs of fp32 (packed .f32x2 instructions).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// ---- softmax helpers (one thread = NC columns of one row of the S tile) ----

// NC columns of the row from TMEM into r[] (fp32 bit patterns).
template <int NC>
__device__ __forceinline__ void load_s_cols(uint32_t taddr, uint32_t* r) {
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) ptx::tmem_ld32(taddr + c * 32, r + c * 32);
  ptx::tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) ptx::reg_fence32(r + c * 32);
}

// Columns > lim get -inf (causal diagonal tile, or keys past the sequence).
template <int NC>
__device__ __forceinline__ void mask_cols(uint32_t* r, int lim) {
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if (c > lim) r[c] = __float_as_uint(-INFINITY);
}

// Max of the NC values: 8 independent chains of 3-input max, then a tree.
template <int NC>
__device__ __forceinline__ float cols_max(const uint32_t* r) {
  float mx8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(__uint_as_float(r[e]), __uint_as_float(r[e + 8]));
#pragma unroll
  for (int c = 16; c < NC; c += 16)
#pragma unroll
    for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], __uint_as_float(r[c + e]), __uint_as_float(r[c + 8 + e]));
  return fmaxf(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
}

// p = 2^(s * scale + bias) for the NC values, packed in place to bf16 pairs
// (r[c/2], c = 0..NC-1). Returns the fp32 sum of p; if mx_out is given, also
// the max of s.
template <int NC, int EMU_PERIOD>
__device__ __forceinline__ float exp_pack(uint32_t* r, float bias, float scale, float* mx_out) {
  float2 ls[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) ls[e] = make_float2(0.f, 0.f);
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  const float2 sc2 = make_float2(scale, scale), bi2 = make_float2(bias, bias);
#pragma unroll
  for (int c = 0; c < NC; c += 4) {
    const float2 s01 = make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1]));
    const float2 s23 = make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
    if (mx_out) mx4[(c >> 2) & 3] = fmax3(mx4[(c >> 2) & 3], fmaxf(s01.x, s01.y), fmaxf(s23.x, s23.y));
    const float2 x01 = ffma2(s01, sc2, bi2);
    const float2 x23 = ffma2(s23, sc2, bi2);
    float2 p01, p23;
    if (EMU_PERIOD > 0 && ((c >> 2) % (EMU_PERIOD > 0 ? EMU_PERIOD : 1)) == EMU_PERIOD - 1) {
      p01 = make_float2(exp2_fma(x01.x), exp2_fma(x01.y));
      p23 = make_float2(exp2_fma(x23.x), exp2_fma(x23.y));
    } else {
      p01 = make_float2(ptx::ex2(x01.x), ptx::ex2(x01.y));
      p23 = make_float2(ptx::ex2(x23.x), ptx::ex2(x23.y));
    }
    ls[(c >> 2) & 3] = fadd2(ls[(c >> 2) & 3], fadd2(p01, p23));
    r[c >> 1] = pack_bf16x2(p01.x, p01.y);
    r[(c >> 1) + 1] = pack_bf16x2(p23.x, p23.y);
  }
  if (mx_out) *mx_out = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
  const float2 t = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
  return t.x + t.y;
}

// The NC/2 packed P words into TMEM.
template <int NC>
__device__ __forceinline__ void store_p(uint32_t taddr, const uint32_t* r) {
  static_assert(NC == 64, "one 32-column store per half row");
  ptx::tmem_st32(taddr, r);
}

// Multiplies NCOL columns of O (this thread's row) by alpha.
template <int NCOL>
__device__ __forceinline__ void scale_o_cols(uint32_t taddr, float alpha, uint32_t* o) {
  if constexpr (NCOL >= 32) {
#pragma unroll
    for (int c = 0; c < NCOL / 32; ++c) {
      ptx::tmem_ld32(taddr + c * 32, o);
      ptx::tmem_wait_ld();
      ptx::reg_fence32(o);
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
      ptx::tmem_st32(taddr + c * 32, o);
    }
  } else {
    static_assert(NCOL == 16, "O half widths are 64, 32 or 16 columns");
    ptx::tmem_ld16(taddr, o);
    ptx::tmem_wait_ld();
    ptx::reg_fence16(o);
#pragma unroll
    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
    ptx::tmem_st16(taddr, o);
  }
}

// One Q tile (tokens [t_first, t_first + tq) of item wi, the G heads of its
// KV head) into the shared-memory buffer qbuf, rotated there by the Q
// warpgroup (128 threads): thread 0 loads the tile once the buffer's
// previous tile has finished its S MMAs (bar_empty, phase ph ^ 1); each
// thread's first cos/sin words are loaded before the tile lands and the next
// ones while it rotates the current ones; then bar_ready. With have = false
// nothing is loaded but every barrier still completes its phase. Returns
// false on abort.
template <class C>
__device__ __forceinline__ bool load_rope_q(const AttnParams& p, uint8_t* qbuf, uint32_t bar_empty,
                                            uint32_t bar_loaded, uint32_t bar_ready, uint32_t ph, bool have,
                                            const WorkItem& wi, int t_first, const CUtensorMap* tmQ, int tid,
                                            volatile int* abort_flag) {
  constexpr int D = C::D;
  constexpr int NCH = D / 16;  // 16-byte chunks in the first half of a row
  constexpr int HALF = D / 2;
  const int G = p.G;
  bool issued = false;
  if (tid == 0 && bwait(bar_empty, ph ^ 1, abort_flag)) {
    if (have) {
      issued = true;
      ptx::mbar_arrive_expect_tx(bar_loaded, (uint32_t)(D * 2 * G * p.tq));
#pragma unroll
      for (int b = 0; b < C::NBOX; ++b)
        ptx::tma_load_3d(ptx::smem_u32(qbuf + b * C::Q_BOX_BYTES), tmQ, bar_loaded, b * C::BOXC, wi.kvh * G,
                         wi.seq_start + t_first);
    } else {
      ptx::mbar_arrive(bar_loaded);
    }
  }
  // this thread's work: (token, 8-column chunk) pairs item = tid, tid + 128, ...
  const int items = (!have || p.q_rotated) ? 0 : p.tq * NCH;  // rotated Q tiles are used as loaded
  auto load_tab = [&](int item, float4& cf, float4& sf) {
    const int tt = item / NCH;
    const int ch = item - tt * NCH;
    if (t_first + tt < wi.L) {
      // bf16 cos and sin of frequencies ch*8 .. ch*8+7 (table_word layout)
      const float4* tab = reinterpret_cast<const float4*>(p.table + table_word(wi.seq_start + t_first + tt, HALF, ch * 8));
      cf = ptx::ld_cg_v4f32(tab);
      sf = ptx::ld_cg_v4f32(tab + 1);
    }
  };
  float4 cf = make_float4(0.f, 0.f, 0.f, 0.f), sf = cf;
  if (tid < items) load_tab(tid, cf, sf);
  const bool ok = __all_sync(0xffffffffu, bwait_lazy(bar_loaded, ph, abort_flag));
  if (!ok) {  // a load issued above lands before the CTA may exit
    if (issued) drain_wait(bar_loaded, ph);
    return false;
  }
  if (!have) return true;
  for (int item = tid; item < items; item += 128) {
    float4 cfn = cf, sfn = sf;
    if (item + 128 < items) load_tab(item + 128, cfn, sfn);
    const int tt = item / NCH;
    const int ch = item - tt * NCH;
    if (t_first + tt < wi.L) {
      const uint32_t cw[4] = {__float_as_uint(cf.x), __float_as_uint(cf.y), __float_as_uint(cf.z),
                              __float_as_uint(cf.w)};
      const uint32_t sw[4] = {__float_as_uint(sf.x), __float_as_uint(sf.y), __float_as_uint(sf.z),
                              __float_as_uint(sf.w)};
      const int col_lo = ch * 8, col_hi = ch * 8 + HALF;
      const int bx_lo = col_lo / C::BOXC, bx_hi = col_hi / C::BOXC;
      for (int hh = 0; hh < G; ++hh) {
        const int row = tt * G + hh;
        uint4* plo = reinterpret_cast<uint4*>(qbuf + bx_lo * C::Q_BOX_BYTES +
                                              swz(row * C::ROWB + (col_lo % C::BOXC) * 2, C::SWZ_MASK));
        uint4* phi = reinterpret_cast<uint4*>(qbuf + bx_hi * C::Q_BOX_BYTES +
                                              swz(row * C::ROWB + (col_hi % C::BOXC) * 2, C::SWZ_MASK));
        uint4 vlo = *plo, vhi = *phi;
        rope_bf16x2(vlo.x, vhi.x, cw[0], sw[0], vlo.x, vhi.x);
        rope_bf16x2(vlo.y, vhi.y, cw[1], sw[1], vlo.y, vhi.y);
        rope_bf16x2(vlo.z, vhi.z, cw[2], sw[2], vlo.z, vhi.z);
        rope_bf16x2(vlo.w, vhi.w, cw[3], sw[3], vlo.w, vhi.w);
        *plo = vlo;
        *phi = vhi;
      }
    }
    cf = cfn;
    sf = sfn;
  }
  ptx::fence_proxy_async_smem();
  ptx::mbar_arrive(bar_ready);
  return true;
}

// Q tile of the CTA's work item `it` into Q buffer it & 1: every warp of the
// Q warpgroup takes the item from the hand-off ring (w_out = its index, -1
// when no items are left), then load_rope_q. Returns false on abort.
template <class C>
__device__ __forceinline__ bool rope_q_tile(const AttnParams& p, uint8_t* smem, Barriers* bars,
                                            const CUtensorMap* tmQ, int it, int tid, volatile int* abort_flag,
                                            int& w_out, WorkItem& wi_out) {
  const int qb = it & 1;
  int w;
  WorkItem wi;
  if (!take_item_warp(bars, it, w, wi, abort_flag)) return false;
  w_out = w;
  wi_out = wi;
  return load_rope_q<C>(p, smem + qb * C::Q_BYTES, ptx::smem_u32(&bars->q_empty[qb]),
                        ptx::smem_u32(&bars->q_loaded[qb]), ptx::smem_u32(&bars->q_ready[qb]), (it >> 1) & 1,
                        w >= 0, wi, wi.t0, tmQ, tid, abort_flag);
}

template <class C, bool OUT_FP32, bool MASK>
__device__ __forceinline__ bool epilogue_tile(const AttnParams& p, const WorkItem& wi, uint8_t* smem, Barriers* bars,
                                              uint32_t tmem, int it, uint32_t g, int tid,
                                              volatile int* abort_flag) {
  constexpr int D = C::D;
  const int warp = tid >> 5;  // 0..3 inside the warpgroup == TMEM lane quadrant
  const int r = tid;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
  const int G = p.G;
  const int tok_off = r / G;
  const int hin = r - tok_off * G;
  const int tok = wi.t0 + tok_off;
  const bool row_valid = r < p.tq * G && tok < wi.L;
  bool ok = __all_sync(0xffffffffu, bwait(ptx::smem_u32(&bars->stats_full), it & 1, abort_flag));
  if (!ok) return false;
  // (running max, sum) of the two column halves, each against its own max
  const float2 ml0 = reinterpret_cast<const float2*>(smem + C::OFF_STATS)[r];
  const float2 ml1 = reinterpret_cast<const float2*>(smem + C::OFF_STATS)[BM + r];
  ptx::mbar_arrive(ptx::smem_u32(&bars->stats_empty));
  const uint32_t gl = g + wi.nkv - 1;
  ok = __all_sync(0xffffffffu,
                  bwait(ptx::smem_u32(&bars->pv_done[gl % C::NSB]), (gl / C::NSB) & 1, abort_flag));
  if (!ok) return false;
  ptx::tc_fence_after();

  float mrow, lrow, w0, w1;
  bool dead = false;  // masked form: the row saw no visible key (its running max stayed -inf): out 0, lse -inf
  if constexpr (C::SPLIT) {
    // O = (a0 O_a + a1 O_b) / (a0 l_a + a1 l_b), a_h = 2^((m_h - m) scale) for
    // the row max m; a half that saw no unmasked key (m_h = -inf) weighs 0
    mrow = fmaxf(ml0.x, ml1.x);
    const float a0 = ml0.x == -INFINITY ? 0.f : ptx::ex2((ml0.x - mrow) * p.scale_log2);
    const float a1 = ml1.x == -INFINITY ? 0.f : ptx::ex2((ml1.x - mrow) * p.scale_log2);
    lrow = a0 * ml0.y + a1 * ml1.y;
    dead = MASK && mrow == -INFINITY;
    const float inv_l = dead ? 0.f : 1.f / lrow;
    w0 = a0 * inv_l;
    w1 = a1 * inv_l;
  } else {
    mrow = ml0.x;  // both halves hold the same running max
    lrow = ml0.y + ml1.y;
    dead = MASK && mrow == -INFINITY;
    w0 = dead ? 0.f : 1.f / lrow;
    w1 = 0.f;
  }
  const int h = wi.kvh * G + hin;
  const size_t orow = (size_t)(wi.seq_start + tok) * p.nq + h;
  // 16 columns of O (of O_a and O_b) at a time
  uint32_t oa[16], ob[16];
#pragma unroll
  for (int c = 0; c < D / 16; ++c) {
    ptx::tmem_ld16(trow + C::O_COL + c * 16, oa);
    if constexpr (C::SPLIT) ptx::tmem_ld16(trow + C::O_COL + D + c * 16, ob);
    ptx::tmem_wait_ld();
    ptx::reg_fence16(oa);
    if constexpr (C::SPLIT) ptx::reg_fence16(ob);
    if (c == D / 16 - 1) {  // O fully read: the next tile's first P.V may overwrite it
      ptx::tc_fence_before();
      ptx::mbar_arrive(ptx::smem_u32(&bars->o_free));
    }
    auto o = [&](int e) {
      if constexpr (C::SPLIT) return fmaf(__uint_as_float(oa[e]), w0, __uint_as_float(ob[e]) * w1);
      else return __uint_as_float(oa[e]) * w0;
    };
    if constexpr (OUT_FP32) {
      if (row_valid) {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + orow * D + c * 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_float4(o(4 * e), o(4 * e + 1), o(4 * e + 2), o(4 * e + 3));
      }
    } else {
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(o(2 * e), o(2 * e + 1));
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + orow * D + c * 16);
        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
  }
  if (row_valid && p.lse)
    p.lse[(size_t)h * p.N + wi.seq_start + tok] =
        dead ? -INFINITY : (mrow * p.scale_log2 + __log2f(lrow)) * 0.69314718055994531f;
  return true;
}

// The 64 mask values of query row mrow for keys [key0, key0 + 64) as bf16
// pairs (key0 + 2e in the low half of m[e]); keys at or past L, and every
// key of a null row, read 0 (the length mask hides them).
__device__ __forceinline__ void load_mask_half(const __nv_bfloat16* mrow, int key0, int L, uint32_t* m) {
#pragma unroll
  for (int q4 = 0; q4 < 8; ++q4) {
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

// s += mask * scale on 64 raw scores (the bf16 pairs of load_mask_half).
__device__ __forceinline__ void add_mask_half(uint32_t* sr, const uint32_t* m, float scale) {
  const float2 sc2 = make_float2(scale, scale);
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const uint32_t w = m[c >> 1];
    const float2 mv = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    const float2 r = ffma2(mv, sc2, make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])));
    sr[c] = __float_as_uint(r.x);
    sr[c + 1] = __float_as_uint(r.y);
  }
}

// S = Q K^T for one KV tile: D/16 K-steps, K-major A and B (SW128/SW64).
template <class C>
__device__ __forceinline__ void issue_s_mmas(uint32_t d_tmem, uint64_t dq, uint64_t dk) {
#pragma unroll
  for (int kk = 0; kk < C::KSTEPS_S; ++kk) {
    const uint32_t off_q = (kk / C::STEPS_PER_BOX) * C::Q_BOX_BYTES + (kk % C::STEPS_PER_BOX) * 32;
    const uint32_t off_k = (kk / C::STEPS_PER_BOX) * C::KV_BOX_BYTES + (kk % C::STEPS_PER_BOX) * 32;
    ptx::mma_ss(d_tmem, dq + (uint64_t)(off_q >> 4), dk + (uint64_t)(off_k >> 4), C::IDESC_S, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V for one KV tile: 8 K-steps of 16 keys, P from TMEM (keys
// [0, 64) at S buffer column 0, keys [64, 128) at column 64), V MN-major.
template <class C>
__device__ __forceinline__ void issue_pv_mmas(uint32_t o_tmem, uint32_t p_tmem, uint64_t dv, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < C::KSTEPS_PV; ++kk)
    ptx::mma_ts(o_tmem, p_tmem + (kk >> 2) * 64 + (kk & 3) * 8, dv + (uint64_t)((kk * 16 * C::ROWB) >> 4),
                C::IDESC_O, (accumulate || kk > 0) ? 1u : 0u);
}

// O_h (+)= P_h V_h for one column half h of a KV tile: 4 K-steps of 16 keys;
// p_tmem = the half's packed P columns, dv = V's descriptor at the half's
// first key.
template <class C>
__device__ __forceinline__ void issue_pv_half(uint32_t o_tmem, uint32_t p_tmem, uint64_t dv, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < KSTEPS_PV_HALF; ++kk)
    ptx::mma_ts(o_tmem, p_tmem + kk * 8, dv + (uint64_t)((kk * 16 * C::ROWB) >> 4), C::IDESC_O,
                (accumulate || kk > 0) ? 1u : 0u);
}

template <int D, bool OUT_FP32, bool MASK>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
    gqa_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array by pointer
  // arithmetic so that accesses through it stay shared-memory accesses
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::OFF_BAR);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;

  auto B = [&](uint64_t& b) { return ptx::smem_u32(&b); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(B(bars->q_loaded[i]), 1);
      ptx::mbar_init(B(bars->q_ready[i]), 128);
      ptx::mbar_init(B(bars->q_empty[i]), 1);
    }
    for (int i = 0; i < C::KST; ++i) {
      ptx::mbar_init(B(bars->k_full[i]), 1);
      ptx::mbar_init(B(bars->k_empty[i]), 1);
    }
    for (int i = 0; i < C::VST; ++i) {
      ptx::mbar_init(B(bars->v_full[i]), 1);
      ptx::mbar_init(B(bars->v_empty[i]), 1);
    }
    for (int i = 0; i < NUM_S_BUF; ++i) {
      ptx::mbar_init(B(bars->s_full[i]), 1);
      ptx::mbar_init(B(bars->p_full[i][0]), C::SPLIT ? 128 : 256);
      ptx::mbar_init(B(bars->p_full[i][1]), 128);  // (SPLIT only)
      ptx::mbar_init(B(bars->pv_done[i]), 1);
    }
    ptx::mbar_init(B(bars->o_free), 128);
    ptx::mbar_init(B(bars->stats_full), 256);
    ptx::mbar_init(B(bars->stats_empty), 128);
    for (int i = 0; i < 2; ++i)
      for (int qd = 0; qd < 4; ++qd) ptx::mbar_init(B(bars->xchg[i][qd]), 64);
    ptx::mbar_init(B(bars->drain), 2);  // one commit per MMA-issuing thread
    for (int i = 0; i < ITEM_SLOTS; ++i) {
      ptx::mbar_init(B(bars->item_full[i]), 1);
      ptx::mbar_init(B(bars->item_empty[i]), ITEM_READERS);
    }
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
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  // Everything below reads what the prologue kernel wrote. The forward
  // launches this kernel as a programmatic dependent of the prologue, so the
  // setup above overlaps the prologue's tail; this wait returns once the
  // prologue grid has completed and its stores are visible (at once for a
  // launch in plain stream order).
  ptx::griddep_wait();
  const int n_items = ptx::ld_cg_s32(p.header) * p.nkv;

  // Register split (launch: 512 threads x 128): producers/MMA 56, softmax
  // 160, Q rotation 128 -> 56 x 128 + 160 x 256 + 128 x 128 = 64512 <= 65536.
  if (warp < 4) {
   ptx::setmaxnreg_dec<REG_PRODUCER>();
   if (warp == 0) {
    // ------------------------------------------------------------ K producer
    // Also the scheduler: when it starts the K loads of item k it publishes
    // item k + 1 in ring slot (k + 1) % ITEM_SLOTS (so the Q warps can rotate
    // that tile early) and asks the global counter for item k + 2, whose
    // index is needed only one item later.
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      int w = (int)blockIdx.x < n_items ? (int)blockIdx.x : -1;  // first item of CTA b: item b
      int nxt = w >= 0 ? next_item_index(p, 1) : n_items;
      ok = publish_item(p, bars, 0, w, abort_flag);
      for (int k = 0; ok && w >= 0; ++k) {
        const int wn = nxt < n_items ? nxt : -1;
        if (!(ok = publish_item(p, bars, k + 1, wn, abort_flag))) break;
        if (wn >= 0) nxt = next_item_index(p, k + 2);
        const WorkItem wi = decode_item(p, w);
        for (int j = 0; j < wi.nkv; ++j, ++g) {
          const int ks = g % C::KST;
          if (!(ok = bwait_lazy(B(bars->k_empty[ks]), ((g / C::KST) & 1) ^ 1, abort_flag))) break;
          ptx::mbar_arrive_expect_tx(B(bars->k_full[ks]), (uint32_t)C::KV_BYTES);
          // K' head-major (token, head) or, for rotated inputs, the caller's
          // token-major K (head, token): the same 128-byte rows in shared memory
          const int c1 = p.k_token_major ? wi.kvh : wi.seq_start + j * BN;
          const int c2 = p.k_token_major ? wi.seq_start + j * BN : wi.kvh;
          for (int b = 0; b < C::NBOX; ++b)
            ptx::tma_load_3d(sbase + C::OFF_K + ks * C::KV_BYTES + b * C::KV_BOX_BYTES, &tmK,
                             B(bars->k_full[ks]), b * C::BOXC, c1, c2);
        }
        w = wn;
      }
      if (!ok) {  // let every copy already issued land before the CTA exits
        // loads issued: K tiles 0..g-1 (stage x % KST)
        for (int i = 0; i < C::KST; ++i) {
          const int uses = ((int)g - i + C::KST - 1) / C::KST;
          if (uses > 0) drain_wait(B(bars->k_full[i]), (uses - 1) & 1);
        }
      }
    }
   } else if (warp == 2) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        int w;
        WorkItem wi;
        if (!(ok = take_item(bars, k, w, wi, abort_flag)) || w < 0) break;
        for (int j = 0; j < wi.nkv; ++j, ++g) {
          const int vs = g % C::VST;
          if (!(ok = bwait_lazy(B(bars->v_empty[vs]), ((g / C::VST) & 1) ^ 1, abort_flag))) break;
          ptx::mbar_arrive_expect_tx(B(bars->v_full[vs]), (uint32_t)C::KV_BYTES);
          for (int b = 0; b < C::NBOX; ++b)
            ptx::tma_load_3d(sbase + C::OFF_V + vs * C::KV_BYTES + b * C::KV_BOX_BYTES, &tmV,
                             B(bars->v_full[vs]), b * C::BOXC, wi.kvh, wi.seq_start + j * BN);
        }
      }
      if (!ok) {
        for (int i = 0; i < C::VST; ++i) {
          const int uses = ((int)g - i + C::VST - 1) / C::VST;
          if (uses > 0) drain_wait(B(bars->v_full[i]), (uses - 1) & 1);
        }
      }
    }
   } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    // S(x) = Q K(x)^T into S buffer x % 3; it needs PV(x - 3) done (that PV
    // read P from the same columns). Runs ahead of the softmax by up to three
    // KV tiles; a tcgen05.mma blocks its issuing thread while the tensor core
    // works, so S and PV have separate issuing threads.
    if (lane == 0) {
      const uint64_t dq_base = umma_desc(sbase, 16, C::SBO, C::UMMA_LAYOUT);
      const uint64_t dk_base = umma_desc(sbase + C::OFF_K, 16, C::SBO, C::UMMA_LAYOUT);
      const uint32_t bar_pv0 = B(bars->pv_done[0]), bar_s0 = B(bars->s_full[0]);
      const uint32_t bar_kf0 = B(bars->k_full[0]), bar_ke0 = B(bars->k_empty[0]);
      const uint32_t bar_qr0 = B(bars->q_ready[0]), bar_qe0 = B(bars->q_empty[0]);
      uint32_t gs = 0;
      int it = 0;
      bool ok = true;
      for (; ok; ++it) {
        int w;
        WorkItem wi;
        if (!(ok = take_item(bars, it, w, wi, abort_flag)) || w < 0) break;
        const int qb = it & 1;
        if (!(ok = bwait(bar_qr0 + 8 * qb, (it >> 1) & 1, abort_flag))) break;
        const uint64_t dq = dq_base + (uint64_t)((qb * C::Q_BYTES) >> 4);
        for (int j = 0; j < wi.nkv; ++j, ++gs) {
          const int bs = gs % C::NSB, ks = gs % C::KST;
          if (gs >= C::NSB && !(ok = bwait(bar_pv0 + 8 * bs, ((gs / C::NSB) - 1) & 1, abort_flag))) break;
          if (!(ok = bwait(bar_kf0 + 8 * ks, (gs / C::KST) & 1, abort_flag))) break;
          ptx::tc_fence_after();
          issue_s_mmas<C>(tmem + bs * 128, dq, dk_base + (uint64_t)((ks * C::KV_BYTES) >> 4));
          ptx::mma_commit(bar_s0 + 8 * bs);
          ptx::mma_commit(bar_ke0 + 8 * ks);
        }
        if (ok) ptx::mma_commit(bar_qe0 + 8 * qb);  // every S of this tile read Q
      }
      // all tensor-core work issued here has finished before TMEM is freed
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
   } else if (warp == 3) {
    // ------------------------------------------------------------ PV issuer
    // O += P(x) V(x) once the softmax has written P(x) into S buffer x % 3.
    if (lane == 0) {
      const uint64_t dv_base = umma_desc(sbase + C::OFF_V, C::KV_BOX_BYTES, C::SBO, C::UMMA_LAYOUT);
      const uint32_t bar_pv0 = B(bars->pv_done[0]), bar_p0 = B(bars->p_full[0][0]);
      const uint32_t bar_vf0 = B(bars->v_full[0]), bar_ve0 = B(bars->v_empty[0]), bar_of = B(bars->o_free);
      uint32_t g = 0;
      int it = 0;
      bool ok = true;
      for (; ok; ++it) {
        int w;
        WorkItem wi;
        if (!(ok = take_item(bars, it, w, wi, abort_flag)) || w < 0) break;
        for (int j = 0; j < wi.nkv; ++j, ++g) {
          const int b = g % C::NSB, vs = g % C::VST;
          if (!(ok = bwait(bar_vf0 + 8 * vs, (g / C::VST) & 1, abort_flag))) break;
          if (j == 0 && !(ok = bwait(bar_of, (it & 1) ^ 1, abort_flag))) break;
          const uint64_t dv = dv_base + (uint64_t)((vs * C::KV_BYTES) >> 4);
          if constexpr (C::SPLIT) {
            // each column half's P V as soon as that half has written its P
            for (int h = 0; h < 2; ++h) {
              if (!(ok = bwait(bar_p0 + 16 * b + 8 * h, (g / C::NSB) & 1, abort_flag))) break;
              ptx::tc_fence_after();
              issue_pv_half<C>(tmem + C::O_COL + h * D, tmem + b * 128 + h * (BN / 2),
                               dv + (uint64_t)((h * (BN / 2) * C::ROWB) >> 4), j > 0);
            }
          } else {
            if ((ok = bwait(bar_p0 + 16 * b, (g / C::NSB) & 1, abort_flag))) {
              ptx::tc_fence_after();
              issue_pv_mmas<C>(tmem + C::O_COL, tmem + b * 128, dv, j > 0);
            }
          }
          if (!ok) break;
          ptx::mma_commit(bar_pv0 + 8 * b);
          ptx::mma_commit(bar_ve0 + 8 * vs);
        }
      }
      ptx::mma_commit(B(bars->drain));
      drain_wait(B(bars->drain), 0);
    }
   }
  } else if (warp < 12) {
    ptx::setmaxnreg_inc<MASK ? REG_SOFTMAX_MASKED : REG_SOFTMAX>();
    // ------------------------------------------------------------ softmax
    constexpr int NC = BN / 2;           // columns per thread
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;    // 0: columns [0, 64), 1: [64, 128)
    const int r = quad * 32 + lane;      // row of the tile == TMEM lane
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16) + half * NC;
    const int G = p.G;
    const int tok_off = r / G;
    const float sl2 = p.scale_log2;
    float2* stats = reinterpret_cast<float2*>(smem + C::OFF_STATS) + half * BM;
    float* xmax = reinterpret_cast<float*>(smem + C::OFF_XMAX);  // [parity][half][BM] (d = 128)
    uint32_t g = 0;
    int it = 0;
    bool ok = true;
    uint32_t sr[NC];
    for (; ok; ++it) {
      int w;
      WorkItem wi;
      if (!(ok = take_item_warp(bars, it, w, wi, abort_flag)) || w < 0) break;
      const int tok = wi.t0 + tok_off;  // index inside the sequence
      const int last_key = p.causal ? tok : wi.L - 1;
      // masked form: the row's mask values, a tile ahead (null row past the
      // sequence; a sequence longer than the mask is reported and unmasked)
      const __nv_bfloat16* mrow = nullptr;
      uint32_t mk[MASK ? NC / 2 : 1];
      if constexpr (MASK) {
        if (wi.L > p.mask_len) {
          if (warp == 4 && lane == 0) atomicCAS(&g_status, 0, kStatusBadSeqlens);
        } else if (tok < wi.L) {
          mrow = p.mask + (size_t)tok * p.mask_ld;
        }
        load_mask_half(mrow, half * NC, wi.L, mk);
      }
      float m = -INFINITY;
      float l = 0.f;
      for (int j = 0; j < wi.nkv; ++j) {
        const uint32_t gg = g + j;
        const int b = gg % C::NSB;
        const uint32_t tS = trow + b * 128;
        ok = __all_sync(0xffffffffu, bwait(B(bars->s_full[b]), (gg / C::NSB) & 1, abort_flag));
        if (!ok) break;
        ptx::tc_fence_after();
        load_s_cols<NC>(tS, sr);
        if constexpr (MASK) add_mask_half(sr, mk, p.mask_scale);
        const int lim = last_key - j * BN - half * NC;  // this half's columns > lim are masked
        if (lim < NC - 1) mask_cols<NC>(sr, lim);
        float alpha = 1.f;
        float lsum;
        if constexpr (C::SPLIT) {
          // The halves keep their own running max and sum (and their own O),
          // so neither waits for the other. A half whose keys were all masked
          // so far keeps m = -inf; its p are 0 (bias 0 on -inf scores).
          if (j == 0) {
            m = cols_max<NC>(sr);
            lsum = exp_pack<NC, emu_period(D)>(sr, m == -INFINITY ? 0.f : -m * sl2, sl2, nullptr);
          } else {
            // Exponentials with the running max m, the tile's max alongside;
            // if the tile's max exceeds m by more than the threshold (2^8 in
            // p) the tile is redone below with the new max.
            float mh;
            lsum = exp_pack<NC, emu_period(D)>(sr, m == -INFINITY ? 0.f : -m * sl2, sl2, &mh);
            const bool need = mh > m + p.rescale_thr;
            if (__any_sync(0xffffffffu, need)) {
              if (need) {
                alpha = ptx::ex2((m - mh) * sl2);
                m = mh;
              }
              load_s_cols<NC>(tS, sr);  // S is intact: P has not been stored yet
              if constexpr (MASK) {
                load_mask_half(mrow, j * BN + half * NC, wi.L, mk);
                add_mask_half(sr, mk, p.mask_scale);
              }
              if (lim < NC - 1) mask_cols<NC>(sr, lim);
              lsum = exp_pack<NC, emu_period(D)>(sr, m == -INFINITY ? 0.f : -m * sl2, sl2, nullptr);
              // O_h holds this half's sum up to the previous tile: wait for
              // PV(gg-1), then scale it (alpha = 1 on rows that kept their max)
              const uint32_t gp = gg - 1;
              ok = __all_sync(0xffffffffu, bwait(B(bars->pv_done[gp % C::NSB]), (gp / C::NSB) & 1, abort_flag));
              if (!ok) break;
              ptx::tc_fence_after();
              // (sr[0, NC/2) holds the packed P; the upper half is free scratch)
              scale_o_cols<D>(tmem + ((uint32_t)(quad * 32) << 16) + C::O_COL + half * D, alpha, sr + NC / 2);
            }
          }
        } else {
          // Both halves publish their max, then read the other's (mbarrier of
          // 64 arrivals per lane quadrant, alternating by tile parity).
          const int xp = gg & 1;
          float* xm_mine = xmax + (xp * 2 + half) * BM + r;
          const float* xm_other = xmax + (xp * 2 + (half ^ 1)) * BM + r;
          const uint32_t xbar = B(bars->xchg[xp][quad]);
          const uint32_t xpar = (gg >> 1) & 1;
          if (j == 0) {
            const float mh = cols_max<NC>(sr);
            *xm_mine = mh;
            ptx::mbar_arrive(xbar);
            ok = __all_sync(0xffffffffu, bwait(xbar, xpar, abort_flag));
            if (!ok) break;
            m = fmaxf(mh, *xm_other);
            lsum = exp_pack<NC, emu_period(D)>(sr, (MASK && m == -INFINITY) ? 0.f : -m * sl2, sl2, nullptr);
          } else {
            // Exponentials with the running max m, the tile's max alongside;
            // if the row's max exceeds m by more than the threshold (2^8 in p)
            // the tile is redone below with the new max.
            float mh;
            lsum = exp_pack<NC, emu_period(D)>(sr, (MASK && m == -INFINITY) ? 0.f : -m * sl2, sl2, &mh);
            *xm_mine = mh;
            ptx::mbar_arrive(xbar);
            ok = __all_sync(0xffffffffu, bwait(xbar, xpar, abort_flag));
            if (!ok) break;
            const float mx = fmaxf(mh, *xm_other);
            bool need = false;
            if (mx > m + p.rescale_thr) {
              alpha = ptx::ex2((m - mx) * sl2);
              m = mx;
              need = true;
            }
            // Both halves see the same maxima, so they take this branch together.
            if (__any_sync(0xffffffffu, need)) {
              load_s_cols<NC>(tS, sr);  // S is intact: P has not been stored yet
              if constexpr (MASK) {
                load_mask_half(mrow, j * BN + half * NC, wi.L, mk);
                add_mask_half(sr, mk, p.mask_scale);
              }
              if (lim < NC - 1) mask_cols<NC>(sr, lim);
              lsum = exp_pack<NC, emu_period(D)>(sr, (MASK && m == -INFINITY) ? 0.f : -m * sl2, sl2, nullptr);
              // O holds the sum up to the previous tile: wait for PV(gg-1), then
              // scale this half's share of O's columns.
              const uint32_t gp = gg - 1;
              ok = __all_sync(0xffffffffu, bwait(B(bars->pv_done[gp % C::NSB]), (gp / C::NSB) & 1, abort_flag));
              if (!ok) break;
              ptx::tc_fence_after();
              // (sr[0, NC/2) holds the packed P; the upper half is free scratch)
              scale_o_cols<D / 2>(tmem + ((uint32_t)(quad * 32) << 16) + C::O_COL + half * (D / 2), alpha,
                                  sr + NC / 2);
            }
          }
        }
        l = l * alpha + lsum;
        store_p<NC>(tS, sr);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(B(bars->p_full[b][C::SPLIT ? half : 0]));
        if constexpr (MASK)
          if (j + 1 < wi.nkv) load_mask_half(mrow, (j + 1) * BN + half * NC, wi.L, mk);
      }
      if (!ok) break;
      // ---- hand (m, this half's l) of every row to the epilogue warps
      ok = __all_sync(0xffffffffu, bwait(B(bars->stats_empty), (it & 1) ^ 1, abort_flag));
      if (!ok) break;
      stats[r] = make_float2(m, l);
      ptx::mbar_arrive(B(bars->stats_full));
      g += wi.nkv;
    }
  } else {
    // (runs with the launch's REG_ROPE registers; REG_ROPE_MASKED in the masked form)
    if constexpr (MASK) ptx::setmaxnreg_dec<REG_ROPE_MASKED>();
    // ------------------------------------------------------------ Q rotation + epilogue
    const int tid = threadIdx.x - 384;
    const int rows = p.tq * p.G;
    // padding rows (never written by TMA) are zero in both Q buffers
    for (int i = tid; i < 2 * C::NBOX * (BM - rows) * (C::ROWB / 16); i += 128) {
      const int per_buf = C::NBOX * (BM - rows) * (C::ROWB / 16);
      const int qb = i / per_buf;
      int rem = i - qb * per_buf;
      const int bx = rem / ((BM - rows) * (C::ROWB / 16));
      rem -= bx * (BM - rows) * (C::ROWB / 16);
      const int row = rows + rem / (C::ROWB / 16);
      const int ch = rem % (C::ROWB / 16);
      uint4* dst = reinterpret_cast<uint4*>(smem + qb * C::Q_BYTES + bx * C::Q_BOX_BYTES +
                                            swz(row * C::ROWB + ch * 16, C::SWZ_MASK));
      *dst = make_uint4(0, 0, 0, 0);
    }
    // Order: rope(0); then for every tile t: rope(t + 1), epilogue(t). The
    // next tile's Q is rotated while tile t still runs; the epilogue of t
    // runs once its last P.V is done.
    int w;
    WorkItem wi{};
    bool ok = rope_q_tile<C>(p, smem, bars, &tmQ, 0, tid, abort_flag, w, wi);
    int it = 0;
    uint32_t g = 0;
    while (ok && w >= 0) {
      int wn;
      WorkItem win{};
      if (!(ok = rope_q_tile<C>(p, smem, bars, &tmQ, it + 1, tid, abort_flag, wn, win))) break;
      ok = epilogue_tile<C, OUT_FP32, MASK>(p, wi, smem, bars, tmem, it, g, tid, abort_flag);
      g += wi.nkv;
      w = wn;
      wi = win;
      ++it;
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
