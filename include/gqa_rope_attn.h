/*
 * gqa_rope_attn.h -- C ABI of the B200 (sm_100a) fused causal grouped-query
 * attention with rotary position embeddings.
 *
 * The operation (per sequence s of a packed batch, per query head h, with
 * G = n_q_heads / n_kv_heads and kv = h / G):
 *
 *   out[t, h, :] = softmax_j( rope(q[t, h]) . rope(k[j, kv]) / sqrt(d) ) v[j, kv]
 *   lse[h, t]    = ln sum_j exp( rope(q[t, h]) . rope(k[j, kv]) / sqrt(d) )
 *
 * over keys j of the same sequence with j <= t (causal) or all j of the
 * sequence (causal = 0). Sources:
 *   - "Attention from Scratch", section "Attention, the math: Grouped-Query
 *     Attention with RoPE'd Q/K": rotate Q and K (never V), share each KV
 *     head over a group of consecutive query heads (repeat_interleave),
 *     score q.k^T / sqrt(head_dim), fill the future with -inf, softmax,
 *     weights @ v.
 *   - "Embeddings & the Residual Stream", section "Positional information:
 *     RoPE, not a learned table": inv_freq[i] = theta^(-2i/d), angle =
 *     position * inv_freq[i], x*cos + rotate_half(x)*sin, i.e. feature i is
 *     rotated together with feature i + d/2.
 *   - "Kohaku-TT", Highlights: flash attention over packed variable-length
 *     batches (cu_seqlens prefix sums).
 *   The log-sum-exp output is not on the pages; it is the natural-log
 *   normaliser of each row's scaled, masked scores.
 * A forward on already rotated q and k (gqa_rope_attn_fwd_rotated), a
 * forward with an additive mask (gqa_rope_attn_fwd_masked), a decoding
 * step against a KV cache (gqa_rope_attn_decode), the backward
 * (gqa_rope_attn_bwd) and the QKV projection with its RoPE epilogue
 * (gqa_rope_attn_qkv_proj) are declared further down.
 *
 * Precision: q, k, v, out are bf16 (or fp32 with dtype GQA_DTYPE_FP32; then
 * q, k, v are rounded to bf16 on load and out is written as fp32). RoPE is
 * evaluated in bf16, as the RoPE page's apply_rope evaluates it on bf16
 * tensors: cos/sin are the fp32 values of the float64 angle's cos/sin cast to
 * bf16, and x*cos and rotate_half(x)*sin are each rounded to bf16, then their
 * sum (round to nearest even throughout); the rotated q and k are the
 * tensor-core operands. Scores and the output accumulate in fp32; the softmax
 * weights enter P.V as bf16. lse is fp32.
 *
 * Memory layout ("THD", all row-major, contiguous, device memory):
 *   q          [total_tokens, n_q_heads,  head_dim]
 *   k, v       [total_tokens, n_kv_heads, head_dim]
 *   out        [total_tokens, n_q_heads,  head_dim]
 *   lse        [n_q_heads, total_tokens]  fp32
 *   positions  [total_tokens] int32
 *   cu_seqlens [num_seqs + 1] int32, cu[0] = 0, nondecreasing,
 *              cu[num_seqs] = total_tokens
 * A fixed batch [B, T, ...] is the same memory with cu = {0, T, 2T, ..., BT}.
 *
 * Ownership: the caller allocates and owns every buffer, the workspace
 * included. The library keeps only a cache of TMA descriptors (per device)
 * and a device status word. It allocates nothing per call and never
 * synchronises inside gqa_rope_attn_fwd.
 */
#ifndef GQA_ROPE_ATTN_H_
#define GQA_ROPE_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GQA_ROPE_ATTN_ABI_VERSION 1

/* Element type of q, k, v and out. */
typedef enum gqa_dtype_e {
  GQA_DTYPE_BF16 = 0,
  GQA_DTYPE_FP32 = 1
} gqa_dtype_t;

/* Status codes. Host-detected errors are returned by the call itself before
 * any CUDA work is queued; device-detected ones are read later with
 * gqa_rope_attn_get_device_status. */
enum {
  GQA_OK = 0,
  GQA_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or flag   */
  GQA_ERR_UNSUPPORTED = 2, /* head_dim not in {32,64,128}, group > 128, ... */
  GQA_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed          */
  GQA_ERR_BAD_SEQLENS = 4, /* device: cu_seqlens not a valid prefix sum     */
  GQA_ERR_TIMEOUT = 5,     /* device: a bounded wait in the kernel ran out  */
  GQA_ERR_WORKSPACE = 6,   /* workspace missing, too small or misaligned    */
  GQA_ERR_NOALLOC_LIMIT = 7 /* shape needs more scratch than the built-in
                               buffer of gqa_rope_attn_fwd_noalloc holds    */
};

/* Bytes of scratch the caller must pass to gqa_rope_attn_fwd for this shape
 * (the RoPE'd K in head-major layout, the cos/sin table, the tile schedule
 * and, for fp32 inputs, bf16 copies of q and v). Returns 0 for invalid
 * arguments. Pure host arithmetic: no CUDA call. */
size_t gqa_rope_attn_workspace_size(int num_seqs, int total_tokens, int n_q_heads,
                                    int n_kv_heads, int head_dim, int dtype);

/* The fused forward.
 *
 * q, k, v      device pointers, layout above, 16-byte aligned.
 * positions    device int32 [total_tokens] giving each token's RoPE
 *              position, or NULL for the index inside its sequence. The
 *              causal mask always uses the index inside the sequence.
 * rope_theta   RoPE base, finite and > 0.
 * cu_seqlens   device int32 [num_seqs + 1]. Checked on the device: a bad
 *              array makes the call write nothing and sets
 *              GQA_ERR_BAD_SEQLENS in the device status word.
 * num_seqs     >= 1 (or 0 with total_tokens == 0).
 * total_tokens >= 0; 0 is a no-op returning GQA_OK.
 * n_q_heads, n_kv_heads  >= 1, n_q_heads % n_kv_heads == 0,
 *              n_q_heads / n_kv_heads <= 128.
 * head_dim     32, 64 or 128.
 * causal       1: key j visible to query t iff j <= t inside the sequence;
 *              0: every key of the sequence is visible.
 * dtype        GQA_DTYPE_BF16 or GQA_DTYPE_FP32 (for q, k, v and out).
 * out          device pointer, written for every token of every sequence.
 * lse          device fp32 [n_q_heads, total_tokens] or NULL.
 * workspace    device scratch of at least gqa_rope_attn_workspace_size()
 *              bytes, 256-byte aligned; contents need not be initialised;
 *              it must not be shared by calls that may overlap on the GPU.
 * stream       a cudaStream_t (passed as void*), NULL for the default
 *              stream. Work is queued on it; the call does not wait.
 *
 * Returns GQA_OK or an error code; on an error nothing has been queued.
 */
int gqa_rope_attn_fwd(const void* q, const void* k, const void* v, const int32_t* positions,
                      double rope_theta, const int32_t* cu_seqlens, int num_seqs,
                      int total_tokens, int n_q_heads, int n_kv_heads, int head_dim,
                      int causal, int dtype, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream);

/* The forward on q and k that are already rotated, e.g. the outputs of
 * gqa_rope_attn_qkv_proj. "Attention from Scratch", section "Attention, the
 * math": the module rotates Q and K once (step 2) and then scores, masks and
 * normalises them (steps 4-6); this call is steps 4-6 alone:
 *
 *   out[t, h, :] = softmax_j( q[t, h] . k[j, kv] / sqrt(d) ) v[j, kv]
 *
 * with lse, masks, GQA sharing and packed sequences as in gqa_rope_attn_fwd.
 * bf16 only; no positions or rope_theta (nothing is rotated); K is read in
 * place from the caller's [total_tokens, n_kv_heads, head_dim] tensor, so
 * the call skips the forward's K pass (its prologue only builds the tile
 * schedule). Arguments, alignment, workspace (gqa_rope_attn_workspace_size()
 * with GQA_DTYPE_BF16 is enough), status codes and stream behaviour as for
 * gqa_rope_attn_fwd. */
int gqa_rope_attn_fwd_rotated(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                              int num_seqs, int total_tokens, int n_q_heads, int n_kv_heads,
                              int head_dim, int causal, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Waits for `stream` (a cudaStream_t as void*, NULL for the default stream),
 * then returns and clears the current device's status word: GQA_OK, or the
 * first device-detected error (GQA_ERR_BAD_SEQLENS, GQA_ERR_TIMEOUT) since
 * the last read. Returns GQA_ERR_CUDA if the synchronisation fails. */
int gqa_rope_attn_get_device_status(void* stream);

/* Static, NUL-terminated description of a status code. */
const char* gqa_rope_attn_strerror(int status);

/* GQA_ROPE_ATTN_ABI_VERSION of the loaded library. */
int gqa_rope_attn_abi_version(void);

/* Number of kernel launches the last successful gqa_rope_attn_fwd queued on
 * the calling thread (0 for a no-op). */
int gqa_rope_attn_last_launch_count(void);

/* Size of the scratch buffer built into the library for
 * gqa_rope_attn_fwd_noalloc: 32 MiB of device memory on every GPU where the
 * library's device code is loaded, held until the process exits. */
#define GQA_ROPE_ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)

/* The fused forward for callers that cannot allocate device memory: for
 * instance code running inside a host application that owns every device
 * allocation and forbids its plug-ins from making their own, or callers that
 * cannot afford the device-wide synchronisation cudaMalloc/cudaFree imply.
 * (The pages have no counterpart; this is a deployment convenience.)
 *
 * Same arguments and results as gqa_rope_attn_fwd, minus the workspace: the
 * scratch lives in a static device array of GQA_ROPE_ATTN_NOALLOC_SCRATCH_BYTES
 * inside the library. The caller still provides q, k, v, positions,
 * cu_seqlens, out and lse. The call makes no cudaMalloc or cudaFree, and
 * neither does anything it calls.
 *   - Invalid arguments get the same codes as from gqa_rope_attn_fwd, before
 *     any CUDA call. Shapes whose gqa_rope_attn_workspace_size() exceeds the
 *     buffer are then rejected with GQA_ERR_NOALLOC_LIMIT, also before any
 *     CUDA call.
 *   - The first call on a device (per process) looks the buffer's device
 *     address up with cudaGetSymbolAddress, with that device current; make
 *     that first call before any stream capture on the device. CUDA loads a
 *     library's device code lazily by default, so this first call may be
 *     the one that loads it onto the device: that reserves the buffer there
 *     and may synchronise the device.
 *   - The buffer is reserved on every device where the library's device
 *     code is loaded (by any of its entry points), whether or not this entry
 *     point is ever called, and held until the process exits.
 *   - All calls on a device share the one buffer: calls that may overlap on
 *     the GPU (different streams without ordering, several host threads)
 *     race on it and must be serialised by the caller. The buffer keeps the
 *     last call's contents; nothing in it needs to start at zero, since each
 *     call writes every byte it later reads.
 */
int gqa_rope_attn_fwd_noalloc(const void* q, const void* k, const void* v, const int32_t* positions,
                              double rope_theta, const int32_t* cu_seqlens, int num_seqs,
                              int total_tokens, int n_q_heads, int n_kv_heads, int head_dim,
                              int causal, int dtype, void* out, float* lse, void* stream);

/* ---- Forward with an additive mask -----------------------------------------
 *
 * The attention kernel of "Attention from Scratch" (section "The compute
 * thread") adds a mask tile to the scaled scores: here
 *
 *   score(t, j) = rope(q[t, h]) . rope(k[j, kv]) / sqrt(d) + mask[t', j']
 *
 * with t', j' the indices of query t and key j inside their sequence; -inf
 * hides a key. The mask is shared by every sequence and head and is combined
 * with the causal mask when causal = 1. A row that sees no key gets out = 0
 * and lse = -inf. Arguments as for gqa_rope_attn_fwd (bf16 only), plus:
 *   mask      bf16 [mask_len, mask_ld] device array, 16-byte aligned
 *   mask_len  >= the longest sequence (checked on the device: a longer one
 *             is attended without the mask, so its output has no meaning,
 *             and sets GQA_ERR_BAD_SEQLENS; no mask element past mask_len
 *             is read)
 *   mask_ld   elements between mask rows, >= mask_len, a multiple of 8
 * workspace: gqa_rope_attn_workspace_size(..., GQA_DTYPE_BF16) bytes. Two
 * kernels are queued (the forward's prologue, then the attention kernel in
 * its masked form: each softmax thread adds its mask values, loaded from
 * global memory a tile ahead, to the raw scores); the call does not wait.
 */
int gqa_rope_attn_fwd_masked(const void* q, const void* k, const void* v, const int32_t* positions,
                             double rope_theta, const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                             int n_q_heads, int n_kv_heads, int head_dim, int causal, const void* mask,
                             int mask_len, int mask_ld, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ---- Decoding step (one new token per sequence against a KV cache) ------
 *
 * "Attention from Scratch", section "Attention, the math: Grouped-Query
 * Attention with RoPE'd Q/K", the paragraph on the KV cache GQA shrinks: one
 * K and one V vector per token and KV head is kept for every token so far.
 * For sequence b the new token sits at position p = cache_seqlens[b]:
 *
 *   k_cache[b, p, kv, :] = rope(k_new[b, kv], p)   (bf16, the prefill's rotation)
 *   v_cache[b, p, kv, :] = v_new[b, kv]
 *   out[b, h, :] = softmax_j( rope(q[b, h], p) . k_cache[b, j, kv] / sqrt(d) ) v_cache[b, j, kv],
 *                  j = 0 .. p, kv = h / G
 *   lse[h, b]    = ln sum_j exp( rope(q[b, h], p) . k_cache[b, j, kv] / sqrt(d) )
 *
 * i.e. the causal mask's last row of the prefill above, with the earlier
 * keys read from the cache (which holds keys after rotation). RoPE and the
 * rounding of the rotated operands are those of gqa_rope_attn_fwd.
 *
 * All tensors bf16 (lse fp32), contiguous, device memory, 16-byte aligned:
 *   q          [batch, n_q_heads, head_dim]
 *   k_new      [batch, n_kv_heads, head_dim]   (not rotated)
 *   v_new      [batch, n_kv_heads, head_dim]
 *   k_cache    [batch, max_cache_len, n_kv_heads, head_dim]  rotated keys;
 *              rows 0 .. p-1 are read, row p is written
 *   v_cache    same layout; rows 0 .. p-1 read, row p written
 *   cache_seqlens  int32 [batch]: tokens already cached, 0 <= p < max_cache_len.
 *              Checked on the device: a sequence outside the range gets no
 *              output and sets GQA_ERR_BAD_SEQLENS in the status word.
 *   out        [batch, n_q_heads, head_dim]
 *   lse        [n_q_heads, batch] fp32, or NULL
 * head_dim 32, 64 or 128; n_q_heads / n_kv_heads <= 16; batch <= 65535.
 * workspace: at least gqa_rope_attn_decode_workspace_size() bytes, 256-byte
 * aligned, contents need not be initialised, not shared by calls that may
 * overlap. Two kernels are queued on `stream`; the call does not wait.
 * Returns GQA_OK or an error code; on an error nothing has been queued.
 */
size_t gqa_rope_attn_decode_workspace_size(int batch, int max_cache_len, int n_q_heads, int n_kv_heads,
                                           int head_dim);

int gqa_rope_attn_decode(const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                         const int32_t* cache_seqlens, double rope_theta, int batch, int max_cache_len,
                         int n_q_heads, int n_kv_heads, int head_dim, void* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream);

/* ---- Backward (gradients of the prefill) --------------------------------
 *
 * The chain rule through the forward's steps ("Attention from Scratch",
 * section "Attention, the math"), for a loss with gradient dout = dL/dout:
 *
 *   P  = exp(S - lse),  S = rope(q) rope(k)^T / sqrt(d) + mask (per head)
 *   dv = sum over the G heads of a group of P^T dout
 *   dS = P * (dout v^T - Delta),  Delta[t, h] = sum_c dout[t, h, c] out[t, h, c]
 *   dq = rope^T(dS rope(k) / sqrt(d)),  dk = rope^T(sum over the group of dS^T rope(q) / sqrt(d))
 *
 * where rope^T rotates each pair (i, i + d/2) by the negative angle (the
 * transpose of the rotation). lse and out are the forward's outputs for the
 * same q, k, v (lse is required: P is recomputed from it, not stored). The
 * rotated q and k are computed exactly as the forward computes them; the
 * gradient passes the rotation's roundings unchanged (rope^T uses the fp32
 * cos/sin). P and dS enter their products as
 * bf16; every product accumulates in fp32; dq is summed over the key tiles
 * of each query tile in fp32 (once per row, no atomics) and rotated back.
 *
 * All of q, k, v, out, dout, dq, dk, dv are bf16 in the forward's layout
 * (q, out, dout, dq: [total_tokens, n_q_heads, head_dim]; k, v, dk, dv:
 * [total_tokens, n_kv_heads, head_dim]), contiguous device memory, 16-byte
 * aligned; lse is fp32 [n_q_heads, total_tokens]. positions, rope_theta,
 * cu_seqlens, num_seqs, total_tokens, the head counts, head_dim and causal
 * are those of the forward call and obey its rules (a bad cu_seqlens sets
 * GQA_ERR_BAD_SEQLENS in the status word; dk and dv are then not written).
 * dq, dk and dv are overwritten (not accumulated into). workspace: at least
 * gqa_rope_attn_bwd_workspace_size() bytes, 256-byte aligned, contents need
 * not be initialised, not shared by calls that may overlap. Four kernels
 * are queued on `stream` (prologue, dk/dv per key tile, dq per query tile,
 * dq's rotation); the call does not wait. Returns GQA_OK or an
 * error code; on an error nothing has been queued.
 */
size_t gqa_rope_attn_bwd_workspace_size(int num_seqs, int total_tokens, int n_q_heads, int n_kv_heads,
                                        int head_dim);

int gqa_rope_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                      const void* dout, const int32_t* positions, double rope_theta,
                      const int32_t* cu_seqlens, int num_seqs, int total_tokens, int n_q_heads,
                      int n_kv_heads, int head_dim, int causal, void* dq, void* dk, void* dv,
                      void* workspace, size_t workspace_bytes, void* stream);

/* ---- QKV projection with the RoPE epilogue -------------------------------
 *
 * Steps 1 and 2 of the attention module ("Attention from Scratch", section
 * "Attention, the math": Project, then Rotate) for tokens x of the residual
 * stream, with the three bias-free linear layers stacked into one weight:
 *
 *   [q | k | v] = x W_qkv^T,   W_qkv = [W_q; W_k; W_v]
 *   q[t, h, :] = rope(row t of x W_q^T, head h),  k likewise,  v not rotated
 *
 * Feature h * head_dim + c of each projection is column c of head h. RoPE
 * is that of gqa_rope_attn_fwd (feature i rotated with i + d/2 by
 * position * theta^(-2i/d)); the rotation is applied to the fp32
 * accumulator and rounded once to bf16 (no rounding in between).
 *
 *   x          [total_tokens, hidden] bf16
 *   w_qkv      [(n_q_heads + 2 n_kv_heads) head_dim, hidden] bf16, the rows
 *              of W_q, then W_k, then W_v (out_features x in_features)
 *   positions  int32 [total_tokens] or NULL: then each token's index inside
 *              its sequence of cu_seqlens ([num_seqs + 1], as for the
 *              forward; required when positions is NULL)
 *   q          [total_tokens, n_q_heads, head_dim] bf16, rotated
 *   k, v       [total_tokens, n_kv_heads, head_dim] bf16, k rotated
 * All device memory, contiguous, 16-byte aligned; hidden a multiple of 8;
 * head_dim 32, 64 or 128; n_q_heads a multiple of n_kv_heads. workspace: at
 * least gqa_rope_attn_qkv_proj_workspace_size() bytes (the cos/sin table),
 * 256-byte aligned. Two kernels are queued on `stream`; the call does not
 * wait. Returns GQA_OK or an error code; on an error nothing has been queued.
 * The outputs feed gqa_rope_attn_fwd only through its unrotated inputs: q
 * and k leave this call already rotated.
 */
size_t gqa_rope_attn_qkv_proj_workspace_size(int total_tokens, int head_dim);

int gqa_rope_attn_qkv_proj(const void* x, const void* w_qkv, const int32_t* positions, double rope_theta,
                           const int32_t* cu_seqlens, int num_seqs, int total_tokens, int hidden,
                           int n_q_heads, int n_kv_heads, int head_dim, void* q, void* k, void* v,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Measurement aid. Arms the calling thread's next gqa_rope_attn_fwd,
 * gqa_rope_attn_fwd_masked, gqa_rope_attn_decode, gqa_rope_attn_bwd or
 * gqa_rope_attn_qkv_proj call to record three CUDA events
 * (cudaEvent_t passed as void*, any may be NULL) on its stream: before its
 * first kernel, between its first two kernels, and after the second, so
 * that each kernel's duration can be read with cudaEventElapsedTime (the
 * backward's third kernel, the dq rotation, runs after the last event). The
 * arming is consumed by that one call (also when it fails). The caller owns
 * the events. */
void gqa_rope_attn_set_profile_events(void* ev_start, void* ev_mid, void* ev_end);

#ifdef __cplusplus
}
#endif

#endif /* GQA_ROPE_ATTN_H_ */
