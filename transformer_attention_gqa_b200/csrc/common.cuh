// Shared constants, parameter blocks and workspace layout of the fused
// causal GQA + RoPE attention forward (sm_100a).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace gqa {

// A query tile packs BM rows = (tq tokens) x (G query heads of one KV group),
// row r <-> (token t0 + r / G, head kv*G + r % G). One K/V tile of BN keys
// feeds every head of the group in a single MMA.
constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NUM_S_BUF = 3;        // S/P buffers in tensor memory
constexpr int ATTN_THREADS = 512;   // 16 warps (roles: attention kernel)
constexpr int PREP_THREADS = 256;
constexpr int SCHED_BINS = 2048;    // cost histogram bins of the tile scheduler
constexpr unsigned long long WAIT_TIMEOUT_NS = 2000000000ull;  // bounded waits: 2 s
// bf16 inputs with at most this many tokens per sequence on average have Q
// rotated by the prologue instead of the attention kernel (0: never).
constexpr int kQPrologueMaxTokensPerSeq = 0;

// Device status word: first device-detected error since the host last read
// it. The library is a single translation unit, so it is defined here.
__device__ int g_status = 0;

// Status codes (same values as the C ABI).
constexpr int kStatusBadSeqlens = 4;
constexpr int kStatusTimeout = 5;

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// tokens per packed query tile for a group of G heads
__host__ __device__ constexpr int tokens_per_tile(int G) { return BM / G; }

// Workspace regions (byte offsets from the 256-byte aligned base).
struct WsLayout {
  size_t header;   // int[16]: [0] number of (sequence, q-tile) pairs, [8] work-item counter
  size_t seq_pfx;  // int[num_seqs + 1]: first pair index of each sequence
  size_t pairs;    // int2[max_pairs]: (sequence, q-tile) in decreasing cost order
  size_t table;    // uint32[N * d/2]: bf16 (cos, sin) of each token's angles (table_word)
  size_t kws;      // bf16[n_kv][N][d]: RoPE'd K, head-major
  size_t qws;      // bf16[N][n_q][d]: rotated q (when the prologue rotates it)
  size_t vws;      // bf16[N][n_kv][d]: v rounded to bf16 (fp32 inputs only)
  size_t total;
  long long max_pairs;
};

// Whether the prologue writes the rotated queries Q' (bf16, [N][n_q][d]) into
// the workspace, so that the attention kernel uses the Q tiles as loaded:
// always for fp32 inputs (the prologue writes a bf16 copy of q anyway), and
// for bf16 inputs when the work items are short (see the forward's launch).
__host__ inline bool q_rotated_in_prologue(int num_seqs, int N, bool fp32_in) {
  return fp32_in || (kQPrologueMaxTokensPerSeq > 0 && num_seqs > 0 &&
                     (long long)N <= (long long)kQPrologueMaxTokensPerSeq * num_seqs);
}

__host__ inline WsLayout ws_layout(int num_seqs, int N, int nq, int nkv, int d, bool fp32_in) {
  WsLayout w{};
  const int G = nq / nkv;
  const int tq = tokens_per_tile(G);
  w.max_pairs = (long long)(N + tq - 1) / tq + num_seqs;
  size_t off = 0;
  w.header = off;
  off = align_up(off + 16 * sizeof(int), 256);
  w.seq_pfx = off;
  off = align_up(off + (size_t)(num_seqs + 1) * sizeof(int), 256);
  w.pairs = off;
  off = align_up(off + (size_t)w.max_pairs * 8, 256);
  w.table = off;
  off = align_up(off + (size_t)N * (d / 2) * 4, 256);
  w.kws = off;
  off = align_up(off + (size_t)nkv * N * d * 2, 256);
  w.qws = w.vws = 0;
  if (q_rotated_in_prologue(num_seqs, N, fp32_in)) {
    w.qws = off;
    off = align_up(off + (size_t)N * nq * d * 2, 256);
  }
  if (fp32_in) {
    w.vws = off;
    off = align_up(off + (size_t)N * nkv * d * 2, 256);
  }
  w.total = off;
  return w;
}

// The forward's RoPE table holds, for each token, d/16 chunks of 8
// frequencies: the chunk's bf16 cos values as 4 bf16x2 words, then its bf16
// sin values as 4 words (d/2 words per token). Word of the cos of the even
// frequency i and i + 1 (the sin word follows 4 words later):
__host__ __device__ constexpr size_t table_word(int t, int half, int i) {
  return (size_t)t * half + (size_t)(i / 8) * 8 + (i % 8) / 2;
}

struct PrepParams {
  const void* q;  // read when the prologue rotates q
  const void* k;
  const void* v;  // fp32 inputs only
  const int* positions;
  const int* cu;
  int N, num_seqs, nq, nkv, tq, causal;
  double theta;
  double inv_freq[64];  // theta^(-2i/d), i < d/2, evaluated once on the host
  int* header;
  int* seq_pfx;
  int2* pairs;
  uint32_t* table;  // table_word layout
  __nv_bfloat16* kws;
  __nv_bfloat16* qws;
  __nv_bfloat16* vws;
};

struct AttnParams {
  const int* cu;
  const int* header;
  int* item_counter;    // work items taken so far beyond the first of each CTA (zeroed by the prologue)
  const int2* pairs;
  const uint32_t* table;  // table_word layout
  void* out;
  float* lse;
  int N, nq, nkv, G, tq, causal;
  int sched_dynamic;    // 1: items beyond the first from item_counter; 0: static alternating deal
  float scale_log2;     // log2(e) / sqrt(d)
  float rescale_thr;    // raw-score growth that triggers an O rescale
  int q_rotated;        // 1: the Q tiles arrive rotated (the caller's, or the prologue's Q'); 0: rotate them
  int k_token_major;    // 1: K is the caller's rotated token-major [N][n_kv][d] tensor; 0: K' head-major
                        // from the prologue
  // additive mask (masked form of the kernel only): bf16 [mask_len][mask_ld]
  // over in-sequence (query, key) indices, raw score += mask * mask_scale
  const __nv_bfloat16* mask;
  int mask_len, mask_ld;
  float mask_scale;
};

}  // namespace gqa
