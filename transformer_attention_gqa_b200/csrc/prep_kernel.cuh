// Prologue kernel of the fused forward. Runs once per call, ahead of the
// attention kernel:
//
//  * block 0 checks cu_seqlens and builds the tile schedule: every
//    (sequence, q-tile) pair, sorted by decreasing cost (number of KV tiles
//    the causal q-tile visits), so that persistent CTAs take the longest
//    tiles first;
//  * the other blocks compute each token's RoPE (cos, sin) table row and
//    write the RoPE'd K once, head-major, into the workspace. K is shared by
//    every query tile that attends to it, so it is rotated once per
//    (token, KV head) instead of once per visiting tile. When asked (short
//    work items, or fp32 inputs) they also write the rotated Q.
//
// RoPE ("Embeddings & the Residual Stream", section "Positional information:
// RoPE, not a learned table"): inv_freq[i] = theta^(-2i/d); angle =
// position * inv_freq[i]; feature i is rotated with feature i + d/2:
//   out[i]       = x[i]       * cos - x[i + d/2] * sin
//   out[i + d/2] = x[i + d/2] * cos + x[i]       * sin
// The angle and cos/sin are evaluated in float64 and rounded to fp32 (the
// page's table is fp32), then cast to bf16 as the page's apply_rope casts
// them to the bf16 inputs' dtype; the rotation is evaluated in bf16
// arithmetic (rope_bf16x2 in rope_round.cuh).
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "rope_round.cuh"

namespace gqa {


__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

// largest s in [0, n) with a[s] <= x (a nondecreasing, a[0] <= x)
__device__ __forceinline__ int upper_index(const int* a, int n, int x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a + mid) <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int tile_cost(int L, int l, int tq, int causal) {
  const int t_end = causal ? min((l + 1) * tq, L) : L;
  return (t_end + BN - 1) / BN;
}

// Block-wide exclusive scan of one int per thread (PREP_THREADS threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_buf, int& total) {
  const int tid = threadIdx.x;
  s_buf[tid] = v;
  __syncthreads();
  for (int off = 1; off < PREP_THREADS; off <<= 1) {
    const int add = tid >= off ? s_buf[tid - off] : 0;
    __syncthreads();
    s_buf[tid] += add;
    __syncthreads();
  }
  total = s_buf[PREP_THREADS - 1];
  const int excl = s_buf[tid] - v;
  __syncthreads();
  return excl;
}

// largest s in [0, n) with a[s] <= x (a nondecreasing, a[0] <= x); plain
// loads, for arrays this block has written (shared or global memory).
__device__ __forceinline__ int upper_index_plain(const int* a, int n, int x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Up to this many sequences, cu_seqlens and the per-sequence pair offsets are
// kept in shared memory while the schedule is built (beyond: global memory).
constexpr int SCHED_SMEM_SEQS = 2048;

__device__ void build_schedule(const PrepParams& p) {
  __shared__ int s_scan[PREP_THREADS];
  __shared__ int s_bins[SCHED_BINS];
  __shared__ int s_cu[SCHED_SMEM_SEQS + 1];
  __shared__ int s_pfx[SCHED_SMEM_SEQS + 1];
  const int tid = threadIdx.x;
  const int ns = p.num_seqs;

  const int* cu = p.cu;
  int* pfx = p.seq_pfx;
  if (ns <= SCHED_SMEM_SEQS) {
    for (int i = tid; i <= ns; i += PREP_THREADS) s_cu[i] = __ldg(p.cu + i);
    cu = s_cu;
    pfx = s_pfx;
  }
  if (tid == 0) p.header[8] = 0;  // work-item counter of the attention kernel
  __syncthreads();

  int bad = 0;
  for (int s = tid; s < ns; s += PREP_THREADS)
    if (cu[s + 1] < cu[s]) bad = 1;
  if (tid == 0 && (cu[0] != 0 || cu[ns] != p.N)) bad = 1;
  if (__syncthreads_or(bad)) {
    if (tid == 0) {
      set_status(kStatusBadSeqlens);
      p.header[0] = 0;
    }
    return;
  }

  // First pair index of every sequence.
  int running = 0;
  for (int base = 0; base < ns; base += PREP_THREADS) {
    const int s = base + tid;
    int nt = 0;
    if (s < ns) nt = (cu[s + 1] - cu[s] + p.tq - 1) / p.tq;
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
    const int l = q - pfx[s];
    const int L = cu[s + 1] - cu[s];
    const int c = min(tile_cost(L, l, p.tq, p.causal), SCHED_BINS - 1);
    atomicAdd(&s_bins[c], 1);
  }
  __syncthreads();

  // Offsets in decreasing-cost order: thread t owns reversed bins [8t, 8t+8).
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
    s_bins[SCHED_BINS - 1 - (tid * PER + i)] = off;  // each bin written by its owner only
    off += local[i];
  }
  __syncthreads();

  for (int q = tid; q < P; q += PREP_THREADS) {
    const int s = upper_index_plain(pfx, ns, q);
    const int l = q - pfx[s];
    const int L = cu[s + 1] - cu[s];
    const int c = min(tile_cost(L, l, p.tq, p.causal), SCHED_BINS - 1);
    const int slot = atomicAdd(&s_bins[c], 1);
    p.pairs[slot] = make_int2(s, l);
  }
  if (tid == 0) p.header[0] = P;
}

template <int D, bool FP32_IN>
__device__ void rope_k_and_table(const PrepParams& p, int block, int nblocks) {
  constexpr int HALF = D / 2;
  constexpr int PAIRS = HALF / 2;  // each thread handles frequencies i, i+1

  const long long total = (long long)p.N * PAIRS;
  for (long long idx = (long long)block * PREP_THREADS + threadIdx.x; idx < total;
       idx += (long long)nblocks * PREP_THREADS) {
    const int t = (int)(idx / PAIRS);
    const int i = (int)(idx % PAIRS) * 2;
    // K words of up to HB heads are loaded before the sincos, so that one
    // memory latency covers them all.
    constexpr int HB = 8;
    uint32_t wl[HB], wh[HB];  // bf16 pairs (i, i + 1) and (i + d/2, i + d/2 + 1)
    auto load_heads = [&](int h0) {
#pragma unroll
      for (int u = 0; u < HB; ++u) {
        if (h0 + u >= p.nkv) break;
        const size_t src = ((size_t)t * p.nkv + h0 + u) * D;
        if constexpr (FP32_IN) {
          // inputs are rounded to bf16 before anything else
          const float2 a = *reinterpret_cast<const float2*>((const float*)p.k + src + i);
          const float2 b = *reinterpret_cast<const float2*>((const float*)p.k + src + i + HALF);
          wl[u] = bf16x2_rn(a.x, a.y);
          wh[u] = bf16x2_rn(b.x, b.y);
        } else {
          wl[u] = *reinterpret_cast<const uint32_t*>((const __nv_bfloat16*)p.k + src + i);
          wh[u] = *reinterpret_cast<const uint32_t*>((const __nv_bfloat16*)p.k + src + i + HALF);
        }
      }
    };
    load_heads(0);

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
    const uint32_t c2 = bf16x2_rn(c[0], c[1]), s2 = bf16x2_rn(sn[0], sn[1]);
    const size_t tw = table_word(t, HALF, i);
    p.table[tw] = c2;
    p.table[tw + 4] = s2;

    for (int h0 = 0; h0 < p.nkv; h0 += HB) {
      if (h0 > 0) load_heads(h0);
#pragma unroll
      for (int u = 0; u < HB; ++u) {
        if (h0 + u >= p.nkv) break;
        uint32_t ol, oh;
        rope_bf16x2(wl[u], wh[u], c2, s2, ol, oh);
        const size_t dst = ((size_t)(h0 + u) * p.N + t) * D;
        *reinterpret_cast<uint32_t*>(p.kws + dst + i) = ol;
        *reinterpret_cast<uint32_t*>(p.kws + dst + i + HALF) = oh;
      }
    }

    if (p.qws) {
      // rotated queries Q' (inputs rounded to bf16 first, as for K)
      for (int h = 0; h < p.nq; ++h) {
        const size_t o = ((size_t)t * p.nq + h) * D;
        uint32_t wa, wb;
        if constexpr (FP32_IN) {
          const float2 a = *reinterpret_cast<const float2*>((const float*)p.q + o + i);
          const float2 b = *reinterpret_cast<const float2*>((const float*)p.q + o + i + HALF);
          wa = bf16x2_rn(a.x, a.y);
          wb = bf16x2_rn(b.x, b.y);
        } else {
          wa = *reinterpret_cast<const uint32_t*>((const __nv_bfloat16*)p.q + o + i);
          wb = *reinterpret_cast<const uint32_t*>((const __nv_bfloat16*)p.q + o + i + HALF);
        }
        uint32_t ol, oh;
        rope_bf16x2(wa, wb, c2, s2, ol, oh);
        *reinterpret_cast<uint32_t*>(p.qws + o + i) = ol;
        *reinterpret_cast<uint32_t*>(p.qws + o + i + HALF) = oh;
      }
    }
    if constexpr (FP32_IN) {
      // bf16 copy of v
      for (int h = 0; h < p.nkv; ++h) {
        const size_t o = ((size_t)t * p.nkv + h) * D;
        const float2 a = *reinterpret_cast<const float2*>((const float*)p.v + o + i);
        const float2 b = *reinterpret_cast<const float2*>((const float*)p.v + o + i + HALF);
        *reinterpret_cast<__nv_bfloat162*>(p.vws + o + i) = __floats2bfloat162_rn(a.x, a.y);
        *reinterpret_cast<__nv_bfloat162*>(p.vws + o + i + HALF) = __floats2bfloat162_rn(b.x, b.y);
      }
    }
  }
}

template <int D, bool FP32_IN>
__global__ void __launch_bounds__(PREP_THREADS) gqa_prep_kernel(const PrepParams p) {
  if (blockIdx.x == 0) {
    build_schedule(p);
  } else {
    rope_k_and_table<D, FP32_IN>(p, blockIdx.x - 1, gridDim.x - 1);
  }
  // This block's stores are issued: the attention grid (a programmatic
  // dependent launch) may be scheduled once every block got here; it reads
  // nothing written here before its griddepcontrol.wait, which returns once
  // this grid has completed and its stores are visible.
  ptx::griddep_launch_dependents();
}

}  // namespace gqa
