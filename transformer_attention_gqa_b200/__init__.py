"""Fused causal grouped-query attention with RoPE'd Q/K for NVIDIA B200
(sm_100a): a C-ABI CUDA library (include/gqa_rope_attn.h) and this thin
PyTorch-facing binding. PyTorch provides device memory and streams only."""
from __future__ import annotations

from . import _abi
from ._abi import GqaError, workspace_size, decode_workspace_size, get_device_status  # noqa: F401

__all__ = ["gqa_rope_attn_fwd", "gqa_rope_attn_decode", "workspace_size", "decode_workspace_size",
           "get_device_status", "GqaError", "Workspace"]


def _ptr(t):
    return 0 if t is None else int(t.data_ptr())


class Workspace:
    """Reusable device scratch for gqa_rope_attn_fwd (grown on demand)."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        import torch
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

    N, nq, d = q.shape
    nkv = k.shape[1]
    if q.dtype == torch.bfloat16:
        dt = _abi.GQA_DTYPE_BF16
    elif q.dtype == torch.float32:
        dt = _abi.GQA_DTYPE_FP32
    else:
        raise TypeError("q must be bfloat16 or float32")
    for t in (q, k, v, cu_seqlens) + ((positions,) if positions is not None else ()):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    num_seqs = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((nq, N), dtype=torch.float32, device=q.device)
    nbytes = workspace_size(num_seqs, N, nq, nkv, d, dt)
    if workspace is None:
        workspace = Workspace(q.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _abi.gqa_rope_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(positions), rope_theta, _ptr(cu_seqlens), num_seqs,
                                N, nq, nkv, d, 1 if causal else 0, dt, _ptr(out), _ptr(lse), _ptr(ws),
                                ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc)
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

    B, nq, d = q.shape
    nkv = k_new.shape[1]
    Lmax = k_cache.shape[1]
    for t in (q, k_new, v_new, k_cache, v_cache, cache_seqlens):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    if any(t.dtype != torch.bfloat16 for t in (q, k_new, v_new, k_cache, v_cache)):
        raise TypeError("decode tensors must be bfloat16")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((nq, B), dtype=torch.float32, device=q.device)
    nbytes = decode_workspace_size(B, Lmax, nq, nkv, d)
    if workspace is None:
        workspace = Workspace(q.device)
    ws = workspace.get(nbytes) if isinstance(workspace, Workspace) else workspace
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    rc = _abi.gqa_rope_attn_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(cache_seqlens), rope_theta, B, Lmax, nq, nkv, d, _ptr(out), _ptr(lse),
                                   _ptr(ws), ws.numel() * ws.element_size(), stream)
    if rc != _abi.GQA_OK:
        raise GqaError(rc, "gqa_rope_attn_decode")
    return out, lse
