"""Float64 CPU oracle for causal grouped-query attention with RoPE'd Q and K.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it. It
shares no code with the CUDA library and imports nothing from it.

What it computes is the plain definition, in the pages' own order of steps
("Attention from Scratch", section "Attention, the math: Grouped-Query
Attention with RoPE'd Q/K", the six-step walk-through of
``GroupedQueryAttention.forward``), with the projections left out because the
inputs are already per-head Q, K, V:

  2. Rotate   -- RoPE on Q and K, never on V ("Embeddings & the Residual
                 Stream", section "Positional information: RoPE, not a learned
                 table": inv_freq[i] = theta^(-2i/d), angle = pos*inv_freq[i],
                 table duplicated as cat([f, f]) and x*cos + rotate_half(x)*sin
                 with rotate_half(x1, x2) = (-x2, x1), i.e. feature i is
                 paired with feature i + d/2).
  3. Share    -- each KV head serves G = n_q/n_kv consecutive query heads
                 (repeat_interleave along the head axis, not repeat).
  4. Score    -- q @ k^T / sqrt(head_dim).
  5. Mask     -- entries above the diagonal set to -inf (causal), then a
                 max-shifted softmax over keys ("Attention from Scratch",
                 section "The compute thread": reduce_max, subtract, exp,
                 reduce_sum, divide).
  6. Gather   -- weights @ v.

plus the natural-log log-sum-exp of each row's scaled, masked scores (not on
the pages; it is the normaliser a backward pass needs).

Packed batches: ``cu_seqlens`` holds prefix sums of the sequence lengths; each
sequence is attended to on its own (no token sees another sequence) and its
positions default to 0..L-1 ("Kohaku-TT" page, Highlights: flash attention with
packed variable-length batches).

Precision. Everything is float64. One quantisation is part of the method and
is modelled on purpose: the rotated Q and K are tensors of the input dtype.
The RoPE page's ``apply_rope`` casts the fp32 cos/sin table to ``x.dtype``
and evaluates ``x * cos + rotate_half(x) * sin`` in that dtype; for bf16
inputs (also the tensor-core operands' type) that is: cos and sin rounded to
bf16, each product rounded to bf16, the sum rounded to bf16, all to nearest
even. With ``operand_rounding=True`` the rotation is evaluated that way, on
the fp32 table the page builds (here: the float64 cos/sin of the float64
angle, rounded once to fp32). With ``operand_rounding=False`` the rotation is
exact float64 and nothing is rounded; the RoPE pins use that form.

Decoding (``gqa_rope_decode``): one new token per sequence against a cache of
the keys and values of every earlier token ("Attention from Scratch", section
"Attention, the math: Grouped-Query Attention with RoPE'd Q/K", the paragraph
on why GQA shrinks the KV cache: one K and one V vector per token and KV head
is kept for every token generated so far). The new token is the last row of
the causal mask, so the step is the forward's last row; the cache holds the
keys after rotation, each at its own position.

Projection (``qkv_rope_projection``): steps 1 and 2 of the same walk-through
for the tokens x of the residual stream: q_proj, k_proj, v_proj are linears
without bias (y = x W^T), q_proj n_q heads wide and k_proj, v_proj n_kv heads
wide, each output split into heads as view(tokens, heads, head_dim); then Q
and K are rotated and V is not.

Masks (``gqa_rope_attention_masked``): the attention kernel of the same
page adds a mask tile to the scaled scores (scores * scale + mask, the mask
holding -inf where a key is hidden), and the "Kohaku-TT" page lists masks
among its flash-attention features. Here: an additive float mask over
in-sequence (query, key) indices, shared by all sequences and heads, added
after the 1/sqrt(d) scaling and combined with the causal mask when asked.

Backward (``gqa_rope_attention_backward``): the gradients of the forward's
output with respect to q, k, v for an upstream gradient dout, i.e. of the
scalar sum(dout * out). It is the training-time counterpart of the forward
(the "Train and Run" page's training loop over SDPA-based attention); the
formulas are the chain rule through the six steps: gather (dV = P^T dO,
dP = dO V^T), softmax (dS = P * (dP - rowsum(dO * O))), score (dQ' = dS K' /
sqrt(d), dK' = dS^T Q' / sqrt(d)), share (the G query heads of a group add
their dK', dV), rotate (the transpose of the rotation: by -angle).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "round_to_bf16",
    "rope_inv_freq",
    "rope_cos_sin",
    "rotate_half",
    "apply_rope",
    "rope_exact_rounded_once",
    "share_kv_heads",
    "score",
    "causal_mask",
    "softmax_with_lse",
    "gather",
    "gqa_rope_attention",
    "brute_force_attention",
    "gqa_rope_decode",
    "rope_backward",
    "gqa_rope_attention_backward",
    "qkv_rope_projection",
    "gqa_rope_attention_masked",
]


# ---------------------------------------------------------------------------
# Rounding
# ---------------------------------------------------------------------------

_BF16_MAX_FINITE_NEXT = 2.0 ** 128  # first magnitude that rounds to inf


def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even) in a
    single rounding, returned as float64.

    bfloat16 has 8 significant bits, exponent range as fp32: normal numbers
    down to 2^-126, subnormals with a fixed quantum of 2^-133.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e with 0.5 <= |m| < 1
    normal = e >= -125  # |x| >= 2^-126
    with np.errstate(over="ignore", invalid="ignore"):
        qn = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
        qs = np.ldexp(np.rint(np.ldexp(x, 133)), -133)
    q = np.where(normal, qn, qs)
    q = np.where(np.abs(q) >= _BF16_MAX_FINITE_NEXT, np.copysign(np.inf, x), q)
    q = np.where(np.isnan(x), np.nan, q)
    q = np.where(np.isinf(x), x, q)
    return q


def _round_to_fp32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# RoPE ("Embeddings & the Residual Stream", section "Positional information:
# RoPE, not a learned table")
# ---------------------------------------------------------------------------

def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """inv_freq[i] = theta^(-2i/head_dim) for i in [0, head_dim/2)."""
    if head_dim % 2:
        raise ValueError("RoPE needs an even head_dim")
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(theta), -(2.0 * i) / float(head_dim))


def rope_cos_sin(positions, head_dim: int, theta: float, table_fp32: bool = False) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin tables of shape [T, head_dim]: angle(pos, i) = pos * inv_freq[i],
    duplicated across the two halves (cat([f, f])) to line up with
    rotate_half. ``table_fp32`` rounds each entry to fp32, as the page's
    table is an fp32 tensor."""
    pos = np.asarray(positions, dtype=np.float64).reshape(-1)
    freqs = np.outer(pos, rope_inv_freq(head_dim, theta))  # [T, d/2]
    emb = np.concatenate([freqs, freqs], axis=-1)  # [T, d]
    c, s = np.cos(emb), np.sin(emb)
    if table_fp32:
        c, s = _round_to_fp32(c), _round_to_fp32(s)
    return c, s


def rotate_half(x: np.ndarray) -> np.ndarray:
    """(x1, x2) -> (-x2, x1) on the two halves of the last axis."""
    h = x.shape[-1] // 2
    return np.concatenate([-x[..., h:], x[..., :h]], axis=-1)


def apply_rope(x: np.ndarray, positions, theta: float, operand_rounding: bool = False) -> np.ndarray:
    """x: [T, H, d] (token-major). Returns x*cos + rotate_half(x)*sin with the
    cos/sin row of each token's position broadcast over heads.

    With ``operand_rounding`` the page's bf16 evaluation: x taken as bf16
    (rounded first; a no-op for bf16 inputs), the fp32 table cast to bf16,
    then x*cos and rotate_half(x)*sin each rounded to bf16 and their sum
    rounded to bf16. A product of two bf16 values has at most 16 significant
    bits, so it is exact in float64 and rounding it here is the page's fp32
    product cast to bf16; a sum of two bf16 values is exact in float64 unless
    the addends' exponents differ by more than 44, and then the sum rounds to
    the larger addend either way."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    c, s = rope_cos_sin(positions, d, theta, table_fp32=operand_rounding)
    c = c[:, None, :]
    s = s[:, None, :]
    if not operand_rounding:
        return x * c + rotate_half(x) * s
    xb = round_to_bf16(x)
    cb, sb = round_to_bf16(c), round_to_bf16(s)
    a = round_to_bf16(xb * cb)
    b = round_to_bf16(rotate_half(xb) * sb)
    return round_to_bf16(a + b)


def rope_exact_rounded_once(x: np.ndarray, positions, theta: float) -> np.ndarray:
    """The rotation of a fused projection epilogue: x (float64, e.g. a
    projection before any rounding) rotated exactly with the fp32 cos/sin
    table and rounded once, to nearest even, to bf16. Each product of a
    float64 value with an fp32 table entry is formed in float64, the sum
    rounded once to float64, then once to bf16."""
    x = np.asarray(x, dtype=np.float64)
    c, s = rope_cos_sin(positions, x.shape[-1], theta, table_fp32=True)
    return round_to_bf16(x * c[:, None, :] + rotate_half(x) * s[:, None, :])


# ---------------------------------------------------------------------------
# GQA sharing ("Attention from Scratch": repeat_interleave keeps the query
# heads of one group adjacent)
# ---------------------------------------------------------------------------

def share_kv_heads(kv: np.ndarray, group_size: int, axis: int = 1) -> np.ndarray:
    """Repeat each KV head ``group_size`` times in place (repeat_interleave):
    query head h reads KV head h // group_size."""
    return np.repeat(kv, group_size, axis=axis)


# ---------------------------------------------------------------------------
# Attention steps ("Attention from Scratch", section "Attention, the math")
# ---------------------------------------------------------------------------

def score(qh: np.ndarray, kh: np.ndarray) -> np.ndarray:
    """Step 4: q @ k^T / sqrt(head_dim) for head-major [H, Tq, d], [H, Tk, d]."""
    d = qh.shape[-1]
    return np.matmul(qh, np.swapaxes(kh, -1, -2)) / math.sqrt(d)


def causal_mask(scores: np.ndarray, query_idx: np.ndarray, key_idx: np.ndarray) -> np.ndarray:
    """Step 5a: key j is visible to query i iff j <= i (indices inside the
    sequence); the rest is filled with -inf."""
    visible = key_idx[None, :] <= query_idx[:, None]
    return np.where(visible[None, :, :], scores, -np.inf)


def softmax_with_lse(scores: np.ndarray):
    """Step 5b: max-shifted softmax over the key axis ("The compute thread":
    reduce_max, subtract, exp, reduce_sum, divide) and the natural-log
    log-sum-exp m + ln(sum exp(s - m)) of each row."""
    m = np.max(scores, axis=-1, keepdims=True)
    e = np.exp(scores - m)
    z = np.sum(e, axis=-1, keepdims=True)
    return e / z, (m + np.log(z))[..., 0]


def gather(weights: np.ndarray, vh: np.ndarray) -> np.ndarray:
    """Step 6: weights @ v."""
    return np.matmul(weights, vh)


# ---------------------------------------------------------------------------
# Forward
# ---------------------------------------------------------------------------

def _check_args(q, k, v, cu_seqlens, n_q_heads, n_kv_heads):
    if q.ndim != 3 or k.ndim != 3 or v.ndim != 3:
        raise ValueError("q, k, v must be [N, heads, d]")
    N, hq, d = q.shape
    if hq != n_q_heads or k.shape != (N, n_kv_heads, d) or v.shape != (N, n_kv_heads, d):
        raise ValueError("shape mismatch")
    if n_q_heads % n_kv_heads:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if cu[0] != 0 or cu[-1] != N or np.any(np.diff(cu) < 0):
        raise ValueError("bad cu_seqlens")
    return N, d, cu


def gqa_rope_attention(q, k, v, cu_seqlens, n_q_heads: int, n_kv_heads: int, rope_theta: float,
                       positions=None, causal: bool = True, operand_rounding: bool = True,
                       query_rows: Optional[Sequence[int]] = None, row_block: int = 1024):
    """Reference forward.

    q: [N, n_q, d], k, v: [N, n_kv, d] (any float dtype; used as float64).
    cu_seqlens: [num_seqs+1] prefix sums. positions: [N] ints or None (then
    the index inside each sequence). Returns (out [N, n_q, d] float64,
    lse [n_q, N] float64). If ``query_rows`` (global token indices) is given,
    only those rows are computed; the others are NaN.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, d, cu = _check_args(q, k, v, cu_seqlens, n_q_heads, n_kv_heads)
    G = n_q_heads // n_kv_heads
    if positions is None:
        pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)] + [np.zeros(0)])
    else:
        pos = np.asarray(positions, dtype=np.int64).reshape(-1)
    out = np.full((N, n_q_heads, d), np.nan)
    lse = np.full((n_q_heads, N), np.nan)
    want = None
    if query_rows is not None:
        want = np.zeros(N, dtype=bool)
        want[np.asarray(query_rows, dtype=np.int64)] = True

    for si in range(len(cu) - 1):
        a, b = int(cu[si]), int(cu[si + 1])
        L = b - a
        if L == 0:
            continue
        rows = np.arange(L) if want is None else np.nonzero(want[a:b])[0]
        if rows.size == 0:
            continue
        # 2. Rotate Q and K (never V) by each token's position.
        qr = apply_rope(q[a:b], pos[a:b], rope_theta, operand_rounding)  # [L, n_q, d]
        kr = apply_rope(k[a:b], pos[a:b], rope_theta, operand_rounding)  # [L, n_kv, d]
        # 3. Share each KV head across its group of query heads.
        ks = share_kv_heads(kr, G, axis=1)  # [L, n_q, d]
        vs = share_kv_heads(v[a:b], G, axis=1)
        # head-major views [H, L, d]
        qh = np.transpose(qr, (1, 0, 2))
        kh = np.transpose(ks, (1, 0, 2))
        vh = np.transpose(vs, (1, 0, 2))
        for r0 in range(0, rows.size, row_block):
            rsel = rows[r0:r0 + row_block]
            kmax = int(rsel.max()) + 1 if causal else L
            scores = score(qh[:, rsel, :], kh[:, :kmax, :])  # 4. Score
            if causal:
                scores = causal_mask(scores, rsel, np.arange(kmax))  # 5. Mask
            w, row_lse = softmax_with_lse(scores)  # 5. Softmax
            o = gather(w, vh[:, :kmax, :])  # 6. Gather, [H, rows, d]
            out[a + rsel, :, :] = np.transpose(o, (1, 0, 2))
            lse[:, a + rsel] = row_lse
    return out, lse


def brute_force_attention(q, k, v, cu_seqlens, n_q_heads: int, n_kv_heads: int, rope_theta: float,
                          positions=None, causal: bool = True):
    """Pure-Python loops with math.cos/sin/exp, no rounding of the rotated
    operands. For tiny inputs only (T <= ~16, d <= ~8)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, hq, d = q.shape
    G = n_q_heads // n_kv_heads
    half = d // 2
    cu = [int(x) for x in cu_seqlens]
    out = [[[0.0] * d for _ in range(hq)] for _ in range(N)]
    lse = [[0.0] * N for _ in range(hq)]

    def rot(vec, p):
        r = [0.0] * d
        for i in range(half):
            ang = p * rope_theta ** (-(2.0 * i) / d)
            c, s = math.cos(ang), math.sin(ang)
            r[i] = vec[i] * c - vec[i + half] * s
            r[i + half] = vec[i + half] * c + vec[i] * s
        return r

    for si in range(len(cu) - 1):
        a, b = cu[si], cu[si + 1]
        for h in range(hq):
            g = h // G
            for i in range(a, b):
                pi = (i - a) if positions is None else int(positions[i])
                qi = rot(list(q[i, h]), pi)
                sc = []
                js = []
                for j in range(a, b):
                    if causal and (j - a) > (i - a):
                        continue
                    pj = (j - a) if positions is None else int(positions[j])
                    kj = rot(list(k[j, g]), pj)
                    sc.append(sum(qi[t] * kj[t] for t in range(d)) / math.sqrt(d))
                    js.append(j)
                mx = max(sc)
                ex = [math.exp(s - mx) for s in sc]
                z = sum(ex)
                for t in range(d):
                    out[i][h][t] = sum(ex[n] * v[js[n], g, t] for n in range(len(js))) / z
                lse[h][i] = mx + math.log(z)
    return np.array(out, dtype=np.float64).reshape(N, hq, d), np.array(lse, dtype=np.float64).reshape(hq, N)


def gqa_rope_decode(q, k_new, v_new, k_cache, v_cache, cache_seqlens, n_q_heads: int, n_kv_heads: int,
                    rope_theta: float, operand_rounding: bool = True):
    """One decoding step for a batch of sequences.

    q: [B, n_q, d] queries of each sequence's new token; k_new, v_new:
    [B, n_kv, d] its key (not rotated yet) and value; k_cache, v_cache:
    [B, max_len, n_kv, d] with rows 0..p-1 holding the rotated keys and the
    values of the earlier tokens of sequence b, p = cache_seqlens[b] (rows
    from p on are not read). The new token sits at position p: its key is
    rotated at p and becomes cache row p, its value too, and its rotated
    query attends to keys 0..p (step 5's causal row of the last token).

    Returns (out [B, n_q, d], lse [n_q, B], k_row [B, n_kv, d],
    v_row [B, n_kv, d]); k_row / v_row are the rows the step appends.
    """
    q = np.asarray(q, dtype=np.float64)
    k_new = np.asarray(k_new, dtype=np.float64)
    v_new = np.asarray(v_new, dtype=np.float64)
    k_cache = np.asarray(k_cache, dtype=np.float64)
    v_cache = np.asarray(v_cache, dtype=np.float64)
    B, hq, d = q.shape
    if hq != n_q_heads or n_q_heads % n_kv_heads:
        raise ValueError("bad head counts")
    if k_new.shape != (B, n_kv_heads, d) or v_new.shape != (B, n_kv_heads, d):
        raise ValueError("shape mismatch")
    if k_cache.shape[0] != B or k_cache.shape[2:] != (n_kv_heads, d) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape mismatch")
    lens = np.asarray(cache_seqlens, dtype=np.int64).reshape(-1)
    if lens.shape != (B,) or np.any(lens < 0) or np.any(lens >= k_cache.shape[1]):
        raise ValueError("bad cache_seqlens")
    G = n_q_heads // n_kv_heads
    out = np.empty((B, n_q_heads, d))
    lse = np.empty((n_q_heads, B))
    k_row = np.empty((B, n_kv_heads, d))
    for b in range(B):
        p = int(lens[b])
        # 2. Rotate the new token's query and key at its position p.
        qr = apply_rope(q[b][None], [p], rope_theta, operand_rounding)[0]      # [n_q, d]
        kr = apply_rope(k_new[b][None], [p], rope_theta, operand_rounding)[0]  # [n_kv, d]
        k_row[b] = kr
        keys = np.concatenate([k_cache[b, :p], kr[None]], axis=0)              # [p+1, n_kv, d]
        vals = np.concatenate([v_cache[b, :p], v_new[b][None]], axis=0)
        # 3. Share each KV head across its group; head-major views.
        kh = np.transpose(share_kv_heads(keys, G, axis=1), (1, 0, 2))          # [n_q, p+1, d]
        vh = np.transpose(share_kv_heads(vals, G, axis=1), (1, 0, 2))
        qh = qr[:, None, :]                                                     # [n_q, 1, d]
        # 4.-6. Score, softmax over the p + 1 visible keys, gather.
        w, row_lse = softmax_with_lse(score(qh, kh))
        out[b] = gather(w, vh)[:, 0, :]
        lse[:, b] = row_lse[:, 0]
    return out, lse, k_row, v_new.copy()


def rope_backward(dx_rot: np.ndarray, positions, theta: float) -> np.ndarray:
    """Gradient through x -> x*cos + rotate_half(x)*sin: the transpose of the
    per-pair rotation, i.e. the rotation by the negative angle:
    dx_i = g_i*cos + g_{i+d/2}*sin, dx_{i+d/2} = g_{i+d/2}*cos - g_i*sin."""
    g = np.asarray(dx_rot, dtype=np.float64)
    d = g.shape[-1]
    c, s = rope_cos_sin(positions, d, theta, table_fp32=False)
    c = c[:, None, :]
    s = s[:, None, :]
    return g * c - rotate_half(g) * s


def gqa_rope_attention_backward(q, k, v, dout, cu_seqlens, n_q_heads: int, n_kv_heads: int, rope_theta: float,
                                positions=None, causal: bool = True, operand_rounding: bool = False):
    """Gradients (dq [N, n_q, d], dk [N, n_kv, d], dv [N, n_kv, d]) of
    sum(dout * out) for the forward above, in float64.

    With ``operand_rounding`` the scores and products use the bf16-rounded
    rotated operands the forward uses, and the rounding is passed through as
    the identity (its derivative is zero almost everywhere; the gradient of the
    unrounded rotation is used instead)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    N, d, cu = _check_args(q, k, v, cu_seqlens, n_q_heads, n_kv_heads)
    if dout.shape != q.shape:
        raise ValueError("dout shape mismatch")
    G = n_q_heads // n_kv_heads
    if positions is None:
        pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)] + [np.zeros(0)])
    else:
        pos = np.asarray(positions, dtype=np.int64).reshape(-1)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    scale = 1.0 / math.sqrt(d)
    for si in range(len(cu) - 1):
        a, b = int(cu[si]), int(cu[si + 1])
        L = b - a
        if L == 0:
            continue
        p = pos[a:b]
        qr = apply_rope(q[a:b], p, rope_theta, operand_rounding)
        kr = apply_rope(k[a:b], p, rope_theta, operand_rounding)
        qh = np.transpose(qr, (1, 0, 2))                                           # [n_q, L, d]
        kh = np.transpose(share_kv_heads(kr, G, axis=1), (1, 0, 2))
        vh = np.transpose(share_kv_heads(v[a:b], G, axis=1), (1, 0, 2))
        doh = np.transpose(dout[a:b], (1, 0, 2))
        scores = score(qh, kh)
        if causal:
            scores = causal_mask(scores, np.arange(L), np.arange(L))
        w, _ = softmax_with_lse(scores)                                            # P [n_q, L, L]
        o = gather(w, vh)
        # gather: out = P V
        dvh = np.matmul(np.swapaxes(w, -1, -2), doh)                               # [n_q, L, d]
        dw = np.matmul(doh, np.swapaxes(vh, -1, -2))                               # dP
        # softmax: dS = P * (dP - sum_j P_ij dP_ij); sum_j P_ij dP_ij = dO_i . O_i
        delta = np.sum(doh * o, axis=-1, keepdims=True)
        ds = w * (dw - delta)
        # score: S = Q' K'^T / sqrt(d)
        dqh = np.matmul(ds, kh) * scale
        dkh = np.matmul(np.swapaxes(ds, -1, -2), qh) * scale
        # share: the G query heads of a group add into their KV head
        dkr = np.transpose(dkh, (1, 0, 2)).reshape(L, n_kv_heads, G, d).sum(axis=2)
        dv[a:b] = np.transpose(dvh, (1, 0, 2)).reshape(L, n_kv_heads, G, d).sum(axis=2)
        # rotate: transpose of the rotation
        dq[a:b] = rope_backward(np.transpose(dqh, (1, 0, 2)), p, rope_theta)
        dk[a:b] = rope_backward(dkr, p, rope_theta)
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Projection ("Attention from Scratch", section "Attention, the math", steps
# 1 Project and 2 Rotate)
# ---------------------------------------------------------------------------

def qkv_rope_projection(x, w_q, w_k, w_v, n_q_heads: int, n_kv_heads: int, rope_theta: float, positions=None,
                        cu_seqlens=None, operand_rounding: bool = False):
    """q = rope(x W_q^T), k = rope(x W_k^T), v = x W_v^T for tokens x [N, C].

    W_q: [n_q * d, C]; W_k, W_v: [n_kv * d, C] (the linear layers' weight
    layout, out_features x in_features). Feature h*d + c of a projection is
    column c of head h. Each token is rotated by positions[t] if given, else
    by its index inside its sequence of ``cu_seqlens`` if given, else by t.
    Returns q [N, n_q, d], k [N, n_kv, d], v [N, n_kv, d] in float64. With
    ``operand_rounding`` the outputs are those of a fused epilogue: the
    rotation takes the fp32 cos/sin table and every output is rounded once,
    to bf16, from its float64 value (no rounding between the projection and
    the rotation; ``rope_exact_rounded_once``)."""
    x = np.asarray(x, dtype=np.float64)
    w_q = np.asarray(w_q, dtype=np.float64)
    w_k = np.asarray(w_k, dtype=np.float64)
    w_v = np.asarray(w_v, dtype=np.float64)
    N, C = x.shape
    d = w_q.shape[0] // n_q_heads
    if w_q.shape != (n_q_heads * d, C) or w_k.shape != (n_kv_heads * d, C) or w_v.shape != (n_kv_heads * d, C):
        raise ValueError("weight shapes must be [heads * head_dim, C]")
    if positions is not None:
        pos = np.asarray(positions, dtype=np.int64).reshape(-1)
    elif cu_seqlens is not None:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)] + [np.zeros(0)])
    else:
        pos = np.arange(N)
    if pos.shape != (N,):
        raise ValueError("one position per token")
    # 1. Project: y = x W^T, then split the features into heads.
    yq = np.matmul(x, w_q.T).reshape(N, n_q_heads, d)
    yk = np.matmul(x, w_k.T).reshape(N, n_kv_heads, d)
    yv = np.matmul(x, w_v.T).reshape(N, n_kv_heads, d)
    # 2. Rotate Q and K, never V.
    if operand_rounding:
        rope = lambda y: rope_exact_rounded_once(y, pos, rope_theta)  # noqa: E731
    else:
        rope = lambda y: apply_rope(y, pos, rope_theta)  # noqa: E731
    q = rope(yq)
    k = rope(yk)
    v = round_to_bf16(yv) if operand_rounding else yv
    return q, k, v
    return q, k, v


# ---------------------------------------------------------------------------
# Additive masks ("Attention from Scratch", section "The compute thread":
# scores * scale + mask)
# ---------------------------------------------------------------------------

def gqa_rope_attention_masked(q, k, v, cu_seqlens, n_q_heads: int, n_kv_heads: int, rope_theta: float, attn_mask,
                              positions=None, causal: bool = False, operand_rounding: bool = True):
    """The forward with an additive mask: score(i, j) = q_i . k_j / sqrt(d) +
    attn_mask[i, j], i and j indices inside the sequence (attn_mask is
    [Lm, Lm] with Lm >= every sequence length, the same for every sequence
    and head; -inf hides a key), then the causal mask if ``causal``, softmax,
    weights @ v. A row whose scores are all -inf has no distribution: its out
    is 0 and its lse -inf. Returns (out [N, n_q, d], lse [n_q, N]) in float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    mask = np.asarray(attn_mask, dtype=np.float64)
    N, d, cu = _check_args(q, k, v, cu_seqlens, n_q_heads, n_kv_heads)
    G = n_q_heads // n_kv_heads
    if positions is None:
        pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)] + [np.zeros(0)])
    else:
        pos = np.asarray(positions, dtype=np.int64).reshape(-1)
    out = np.zeros((N, n_q_heads, d))
    lse = np.full((n_q_heads, N), -np.inf)
    for si in range(len(cu) - 1):
        a, b = int(cu[si]), int(cu[si + 1])
        L = b - a
        if L == 0:
            continue
        if mask.shape[0] < L or mask.shape[1] < L:
            raise ValueError("attn_mask smaller than a sequence")
        qh = np.transpose(apply_rope(q[a:b], pos[a:b], rope_theta, operand_rounding), (1, 0, 2))
        kh = np.transpose(share_kv_heads(apply_rope(k[a:b], pos[a:b], rope_theta, operand_rounding), G, axis=1),
                          (1, 0, 2))
        vh = np.transpose(share_kv_heads(v[a:b], G, axis=1), (1, 0, 2))
        scores = score(qh, kh) + mask[None, :L, :L]
        if causal:
            scores = causal_mask(scores, np.arange(L), np.arange(L))
        m = np.max(scores, axis=-1, keepdims=True)
        live = np.isfinite(m)
        e = np.where(live, np.exp(scores - np.where(live, m, 0.0)), 0.0)
        z = np.sum(e, axis=-1, keepdims=True)
        w = e / np.where(z > 0, z, 1.0)
        out[a:b] = np.transpose(gather(w, vh), (1, 0, 2))
        lse[:, a:b] = np.where(live, m + np.log(np.where(z > 0, z, 1.0)), -np.inf)[..., 0]
    return out, lse
