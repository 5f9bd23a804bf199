"""Fused causal grouped-query attention with RoPE'd Q/K for NVIDIA B200
(sm_100a): a C-ABI CUDA library (include/gqa_rope_attn.h) and this thin
PyTorch-facing binding. PyTorch provides device memory and streams only."""
from __future__ import annotations

from . import _abi
from ._abi import (GqaError, workspace_size, decode_workspace_size, bwd_workspace_size,  # noqa: F401
                   qkv_proj_workspace_size, get_device_status)

__all__ = ["gqa_rope_attention", "gqa_rope_attn_fwd", "gqa_rope_attn_fwd_rotated", "gqa_rope_attn_fwd_masked", "gqa_rope_attn_decode", "gqa_rope_attn_bwd", "gqa_rope_attn_qkv_proj",
           "workspace_size", "decode_workspace_size", "bwd_workspace_size", "qkv_proj_workspace_size",
           "get_device_status", "GqaError", "Workspace"]


def _ptr(t):
    return 0 if t is None else int(t.data_ptr())


def _check(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _check_tensors(named: dict, device) -> None:
    """Every given tensor is a contiguous CUDA tensor on `device`: the library
    receives raw device addresses and cannot tell a host pointer or a
    strided view from a valid operand."""
    for name, t in named.items():
        if t is None:
            continue
        _check(t.is_cuda, f"{name} must be a CUDA tensor")
        _check(t.device == device, f"{name} is on {t.device}, expected {device}")
        _check(t.is_contiguous(), f"{name} must be contiguous")


class Workspace:
    """Reusable device scratch for the library's calls (grown on demand) on
    `device`, by default the current CUDA device."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        import torch
        if self.device is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


def gqa_rope_attn_fwd(q, k, v, cu_seqlens, rope_theta: float, positions=None, causal: bool = True,
                      out=None, lse=None, workspace=None, stream=None, need_lse: bool = True):
    """out, lse = softmax(rope(q) rope(k)^T / sqrt(d) + causal mask) v.

    q: [N, n_q, d], k/v: [N, n_kv, d] CUDA tensors (bf16, or fp32 for fp32
    I/O); cu_seqlens: int32 [num_seqs+1] on the device; positions: int32 [N]
    or None. Returns (out [N, n_q, d] of q's dtype, lse [n_q, N] fp32 or
    None). Raises GqaError on a non-OK status.
    """
    import torch

    _check(q.dim() == 3 and k.dim() == 3, "q must be [N, n_q, d] and k, v [N, n_kv, d]")
    N, nq, d = q.shape
    nkv = k.shape[1]
    if q.dtype == torch.bfloat16:
        dt = _abi.GQA_DTYPE_BF16
    elif q.dtype == torch.float32:
        dt = _abi.GQA_DTYPE_FP32
    else:
        raise TypeError("q must be bfloat16 or float32")
    _check(k.shape == (N, nkv, d) and v.shape == (N, nkv, d), "k and v must be [N, n_kv, d] matching q")
    _check(k.dtype == q.dtype and v.dtype == q.dtype, "q, k and v must share one dtype")
    _check(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 1,
           "cu_seqlens must be a 1-D int32 tensor")
    if positions is not None:
        _check(positions.dtype == torch.int32 and positions.shape == (N,), "positions must be int32 [N]")
    num_seqs = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((nq, N), dtype=torch.float32, device=q.device)
    _check(out.shape == q.shape and out.dtype == q.dtype, "out must match q's shape and dtype")
    if lse is not None:
        _check(lse.shape == (nq, N) and lse.dtype == torch.float32, "lse must be float32 [n_q, N]")
    _check_tensors(dict(q=q, k=k, v=v, cu_seqlens=cu_seqlens, positions=positions, out=out, lse=lse), q.device)
    nbytes = workspace_size(num_seqs, N, nq, nkv, d, dt)
    if workspace is None:
        workspace = Workspace(q.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    _check_tensors(dict(workspace=ws), q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _abi.gqa_rope_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(positions), rope_theta, _ptr(cu_seqlens), num_seqs,
                                N, nq, nkv, d, 1 if causal else 0, dt, _ptr(out), _ptr(lse), _ptr(ws),
                                ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc)
    return out, lse


def gqa_rope_attn_fwd_rotated(q, k, v, cu_seqlens, causal: bool = True, out=None, lse=None, workspace=None,
                              stream=None, need_lse: bool = True):
    """out, lse = softmax(q k^T / sqrt(d) + causal mask) v on q and k that are
    already rotated (e.g. gqa_rope_attn_qkv_proj's outputs): the attention
    steps after the rotation. bf16 CUDA tensors q [N, n_q, d], k/v
    [N, n_kv, d]; cu_seqlens int32 [num_seqs+1]. Returns (out, lse [n_q, N]
    fp32 or None). Raises GqaError on a non-OK status."""
    import torch

    _check(q.dim() == 3 and k.dim() == 3, "q must be [N, n_q, d] and k, v [N, n_kv, d]")
    N, nq, d = q.shape
    nkv = k.shape[1]
    if q.dtype != torch.bfloat16:
        raise TypeError("q must be bfloat16")
    _check(k.shape == (N, nkv, d) and v.shape == (N, nkv, d), "k and v must be [N, n_kv, d] matching q")
    _check(k.dtype == q.dtype and v.dtype == q.dtype, "q, k and v must share one dtype")
    _check(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 1,
           "cu_seqlens must be a 1-D int32 tensor")
    num_seqs = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((nq, N), dtype=torch.float32, device=q.device)
    _check(out.shape == q.shape and out.dtype == q.dtype, "out must match q's shape and dtype")
    if lse is not None:
        _check(lse.shape == (nq, N) and lse.dtype == torch.float32, "lse must be float32 [n_q, N]")
    _check_tensors(dict(q=q, k=k, v=v, cu_seqlens=cu_seqlens, out=out, lse=lse), q.device)
    nbytes = workspace_size(num_seqs, N, nq, nkv, d, _abi.GQA_DTYPE_BF16)
    if workspace is None:
        workspace = Workspace(q.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    _check_tensors(dict(workspace=ws), q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _abi.gqa_rope_attn_fwd_rotated(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), num_seqs, N, nq, nkv, d,
                                        1 if causal else 0, _ptr(out), _ptr(lse), _ptr(ws),
                                        ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc, "gqa_rope_attn_fwd_rotated")
    return out, lse


def gqa_rope_attn_decode(q, k_new, v_new, k_cache, v_cache, cache_seqlens, rope_theta: float, out=None, lse=None,
                         workspace=None, stream=None, need_lse: bool = True):
    """One decoding step: the new token of each sequence b sits at position
    p = cache_seqlens[b]; its key is rotated at p and written, with its
    value, to cache row p; out = softmax(rope(q) . K[0..p]^T / sqrt(d)) V[0..p].

    q: [B, n_q, d]; k_new, v_new: [B, n_kv, d]; k_cache, v_cache:
    [B, max_len, n_kv, d] (rotated keys) -- bf16 CUDA tensors;
    cache_seqlens: int32 [B] on the device. The caches are updated in place.
    Returns (out [B, n_q, d] bf16, lse [n_q, B] fp32 or None). Raises
    GqaError on a non-OK status.
    """
    import torch

    _check(q.dim() == 3 and k_new.dim() == 3 and k_cache.dim() == 4,
           "q must be [B, n_q, d], k_new/v_new [B, n_kv, d], caches [B, max_len, n_kv, d]")
    B, nq, d = q.shape
    nkv = k_new.shape[1]
    Lmax = k_cache.shape[1]
    if any(t.dtype != torch.bfloat16 for t in (q, k_new, v_new, k_cache, v_cache)):
        raise TypeError("decode tensors must be bfloat16")
    _check(k_new.shape == (B, nkv, d) and v_new.shape == (B, nkv, d), "k_new and v_new must be [B, n_kv, d]")
    _check(k_cache.shape == (B, Lmax, nkv, d) and v_cache.shape == k_cache.shape,
           "k_cache and v_cache must be [B, max_len, n_kv, d]")
    _check(cache_seqlens.dtype == torch.int32 and cache_seqlens.shape == (B,), "cache_seqlens must be int32 [B]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((nq, B), dtype=torch.float32, device=q.device)
    _check(out.shape == q.shape and out.dtype == q.dtype, "out must match q's shape and dtype")
    if lse is not None:
        _check(lse.shape == (nq, B) and lse.dtype == torch.float32, "lse must be float32 [n_q, B]")
    _check_tensors(dict(q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache,
                        cache_seqlens=cache_seqlens, out=out, lse=lse), q.device)
    nbytes = decode_workspace_size(B, Lmax, nq, nkv, d)
    if workspace is None:
        workspace = Workspace(q.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    _check_tensors(dict(workspace=ws), q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _abi.gqa_rope_attn_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(cache_seqlens), rope_theta, B, Lmax, nq, nkv, d, _ptr(out), _ptr(lse),
                                   _ptr(ws), ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc, "gqa_rope_attn_decode")
    return out, lse


def gqa_rope_attn_bwd(q, k, v, out, lse, dout, cu_seqlens, rope_theta: float, positions=None, causal: bool = True,
                      dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of sum(dout * out) for out, lse =
    gqa_rope_attn_fwd(q, k, v, cu_seqlens, rope_theta, positions, causal).

    q, out, dout: [N, n_q, d]; k, v: [N, n_kv, d] -- bf16 CUDA tensors; lse:
    fp32 [n_q, N], the forward's; cu_seqlens and positions as for the
    forward. Returns bf16 dq [N, n_q, d], dk and dv [N, n_kv, d] (written
    into dq/dk/dv when given). Raises GqaError on a non-OK status.
    """
    import torch

    _check(q.dim() == 3 and k.dim() == 3, "q must be [N, n_q, d] and k, v [N, n_kv, d]")
    N, nq, d = q.shape
    nkv = k.shape[1]
    if any(t.dtype != torch.bfloat16 for t in (q, k, v, out, dout)):
        raise TypeError("q, k, v, out and dout must be bfloat16")
    _check(k.shape == (N, nkv, d) and v.shape == (N, nkv, d), "k and v must be [N, n_kv, d] matching q")
    _check(out.shape == q.shape and dout.shape == q.shape, "out and dout must match q's shape")
    _check(lse.shape == (nq, N) and lse.dtype == torch.float32, "lse must be float32 [n_q, N]")
    _check(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 1,
           "cu_seqlens must be a 1-D int32 tensor")
    if positions is not None:
        _check(positions.dtype == torch.int32 and positions.shape == (N,), "positions must be int32 [N]")
    num_seqs = cu_seqlens.numel() - 1
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check(dq.shape == q.shape and dq.dtype == q.dtype, "dq must match q's shape and dtype")
    _check(dk.shape == k.shape and dk.dtype == k.dtype and dv.shape == v.shape and dv.dtype == v.dtype,
           "dk and dv must match k's and v's shapes and dtype")
    _check_tensors(dict(q=q, k=k, v=v, out=out, lse=lse, dout=dout, cu_seqlens=cu_seqlens, positions=positions,
                        dq=dq, dk=dk, dv=dv), q.device)
    nbytes = bwd_workspace_size(num_seqs, N, nq, nkv, d)
    if workspace is None:
        workspace = Workspace(q.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    _check_tensors(dict(workspace=ws), q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _abi.gqa_rope_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(positions),
                                rope_theta, _ptr(cu_seqlens), num_seqs, N, nq, nkv, d, 1 if causal else 0,
                                _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc, "gqa_rope_attn_bwd")
    return dq, dk, dv


def gqa_rope_attn_qkv_proj(x, w_qkv, n_q_heads: int, n_kv_heads: int, rope_theta: float, cu_seqlens=None,
                           positions=None, q=None, k=None, v=None, workspace=None, stream=None):
    """q, k, v = rope(x W_q^T), rope(x W_k^T), x W_v^T split into heads, with
    W_qkv = [W_q; W_k; W_v] ([(n_q + 2 n_kv) d, C] bf16) and x [N, C] bf16
    CUDA tensors. Each token is rotated by positions[t] (int32 [N]) or, when
    positions is None, by its index inside its sequence of cu_seqlens.
    Returns bf16 q [N, n_q, d], k and v [N, n_kv, d]. Raises GqaError on a
    non-OK status.
    """
    import torch

    _check(x.dim() == 2 and w_qkv.dim() == 2, "x must be [N, C] and w_qkv [(n_q + 2 n_kv) d, C]")
    if x.dtype != torch.bfloat16 or w_qkv.dtype != torch.bfloat16:
        raise TypeError("x and w_qkv must be bfloat16")
    N, C = x.shape
    heads = n_q_heads + 2 * n_kv_heads
    _check(w_qkv.shape[1] == C and w_qkv.shape[0] % heads == 0, "w_qkv must be [(n_q + 2 n_kv) d, C]")
    d = w_qkv.shape[0] // heads
    _check(positions is not None or cu_seqlens is not None, "give positions or cu_seqlens")
    if positions is not None:
        _check(positions.dtype == torch.int32 and positions.shape == (N,), "positions must be int32 [N]")
    if cu_seqlens is not None:
        _check(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 1,
               "cu_seqlens must be a 1-D int32 tensor")
    num_seqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    q = torch.empty((N, n_q_heads, d), dtype=torch.bfloat16, device=x.device) if q is None else q
    k = torch.empty((N, n_kv_heads, d), dtype=torch.bfloat16, device=x.device) if k is None else k
    v = torch.empty((N, n_kv_heads, d), dtype=torch.bfloat16, device=x.device) if v is None else v
    _check(q.shape == (N, n_q_heads, d) and k.shape == (N, n_kv_heads, d) and v.shape == (N, n_kv_heads, d),
           "q, k, v must be [N, n_q, d], [N, n_kv, d], [N, n_kv, d]")
    _check(all(t.dtype == torch.bfloat16 for t in (q, k, v)), "q, k, v must be bfloat16")
    _check_tensors(dict(x=x, w_qkv=w_qkv, positions=positions, cu_seqlens=cu_seqlens, q=q, k=k, v=v), x.device)
    nbytes = qkv_proj_workspace_size(N, d)
    if workspace is None:
        workspace = Workspace(x.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    _check_tensors(dict(workspace=ws), x.device)
    if stream is None:
        stream = torch.cuda.current_stream(x.device).cuda_stream
    rc = _abi.gqa_rope_attn_qkv_proj(_ptr(x), _ptr(w_qkv), _ptr(positions), rope_theta, _ptr(cu_seqlens), num_seqs,
                                     N, C, n_q_heads, n_kv_heads, d, _ptr(q), _ptr(k), _ptr(v), _ptr(ws),
                                     ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc, "gqa_rope_attn_qkv_proj")
    return q, k, v


def gqa_rope_attn_fwd_masked(q, k, v, cu_seqlens, rope_theta: float, mask, positions=None, causal: bool = False,
                             out=None, lse=None, workspace=None, stream=None):
    """out, lse of softmax(rope(q) rope(k)^T / sqrt(d) + mask [+ causal mask]) v.

    mask: bf16 [Lm, ld] CUDA tensor (ld >= Lm, a multiple of 8; a contiguous
    [Lm, Lm] tensor needs Lm a multiple of 8) over in-sequence (query, key)
    indices, shared by every sequence and head, -inf hiding a key; Lm must
    be at least the longest sequence. Other arguments as for
    gqa_rope_attn_fwd (bf16 only). Rows that see no key get out 0 and lse
    -inf. Raises GqaError on a non-OK status.
    """
    import torch

    _check(q.dim() == 3 and k.dim() == 3, "q must be [N, n_q, d] and k, v [N, n_kv, d]")
    N, nq, d = q.shape
    nkv = k.shape[1]
    if any(t.dtype != torch.bfloat16 for t in (q, k, v, mask)):
        raise TypeError("q, k, v and mask must be bfloat16")
    _check(k.shape == (N, nkv, d) and v.shape == (N, nkv, d), "k and v must be [N, n_kv, d] matching q")
    _check(mask.dim() == 2 and mask.stride(1) == 1, "mask must be a 2-D tensor with unit column stride")
    mask_len, ld = mask.shape[0], mask.stride(0)
    _check(mask.shape[1] >= mask_len and ld % 8 == 0, "mask must be [Lm, >= Lm] with a row stride divisible by 8")
    _check(cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1 and cu_seqlens.numel() >= 1,
           "cu_seqlens must be a 1-D int32 tensor")
    if positions is not None:
        _check(positions.dtype == torch.int32 and positions.shape == (N,), "positions must be int32 [N]")
    num_seqs = cu_seqlens.numel() - 1
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((nq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(out.shape == q.shape and out.dtype == q.dtype, "out must match q's shape and dtype")
    _check(lse.shape == (nq, N) and lse.dtype == torch.float32, "lse must be float32 [n_q, N]")
    _check_tensors(dict(q=q, k=k, v=v, cu_seqlens=cu_seqlens, positions=positions, out=out, lse=lse), q.device)
    _check(mask.is_cuda and mask.device == q.device, "mask must be a CUDA tensor on q's device")
    nbytes = workspace_size(num_seqs, N, nq, nkv, d, _abi.GQA_DTYPE_BF16)
    if workspace is None:
        workspace = Workspace(q.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    _check_tensors(dict(workspace=ws), q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _abi.gqa_rope_attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(positions), rope_theta, _ptr(cu_seqlens),
                                       num_seqs, N, nq, nkv, d, 1 if causal else 0, _ptr(mask), mask_len, ld,
                                       _ptr(out), _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc, "gqa_rope_attn_fwd_masked")
    return out, lse


def _autograd_function():
    """The torch.autograd.Function over the library's forward and backward
    (built on first use, so that importing the package needs no torch)."""
    global _GqaRopeAttention
    if _GqaRopeAttention is not None:
        return _GqaRopeAttention
    import torch

    class GqaRopeAttention(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, cu_seqlens, rope_theta, positions, causal):
            out, lse = gqa_rope_attn_fwd(q, k, v, cu_seqlens, rope_theta, positions=positions, causal=causal)
            ctx.save_for_backward(q, k, v, out, lse, cu_seqlens)
            ctx.positions = positions
            ctx.rope_theta = rope_theta
            ctx.causal = causal
            ctx.mark_non_differentiable(lse)
            return out, lse

        @staticmethod
        def backward(ctx, dout, _dlse):
            q, k, v, out, lse, cu = ctx.saved_tensors
            dq, dk, dv = gqa_rope_attn_bwd(q, k, v, out, lse, dout.contiguous(), cu, ctx.rope_theta,
                                           positions=ctx.positions, causal=ctx.causal)
            return dq, dk, dv, None, None, None, None

    _GqaRopeAttention = GqaRopeAttention
    return GqaRopeAttention


_GqaRopeAttention = None
# dtypes both library calls under gqa_rope_attention accept
_AUTOGRAD_DTYPES = ("bfloat16",)


def gqa_rope_attention(q, k, v, cu_seqlens, rope_theta: float, positions=None, causal: bool = True):
    """softmax(rope(q) rope(k)^T / sqrt(d) + causal mask) v with gradients:
    out = gqa_rope_attn_fwd(...) in the forward pass, and dq, dk, dv from
    gqa_rope_attn_bwd (which reuses the forward's out and lse) in the
    backward pass. bf16 q, k, v [N, heads, d]; returns out (lse is kept for
    the backward and not returned). The backward takes bf16 only, so other
    dtypes are refused here, before the forward runs."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if str(t.dtype).replace("torch.", "") not in _AUTOGRAD_DTYPES:
            raise TypeError(f"gqa_rope_attention: {name} must be bfloat16 (the backward is bf16 only), got {t.dtype}")
    out, _ = _autograd_function().apply(q, k, v, cu_seqlens, rope_theta, positions, causal)
    return out
