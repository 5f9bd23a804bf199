"""ctypes binding of the C ABI declared in include/gqa_rope_attn.h.

Argument marshalling only: every step of the computation runs in the CUDA
library. Loading fails loudly when the library has not been built."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libgqa_rope_attn.so")

GQA_DTYPE_BF16 = 0
GQA_DTYPE_FP32 = 1

GQA_OK = 0
GQA_ERR_INVALID_ARG = 1
GQA_ERR_UNSUPPORTED = 2
GQA_ERR_CUDA = 3
GQA_ERR_BAD_SEQLENS = 4
GQA_ERR_TIMEOUT = 5
GQA_ERR_WORKSPACE = 6
GQA_ERR_NOALLOC_LIMIT = 7
NOALLOC_SCRATCH_BYTES = 32 << 20

EXPORTED = (
    "gqa_rope_attn_workspace_size",
    "gqa_rope_attn_fwd",
    "gqa_rope_attn_get_device_status",
    "gqa_rope_attn_strerror",
    "gqa_rope_attn_abi_version",
    "gqa_rope_attn_last_launch_count",
    "gqa_rope_attn_set_profile_events",
    "gqa_rope_attn_fwd_noalloc",
    "gqa_rope_attn_decode_workspace_size",
    "gqa_rope_attn_decode",
    "gqa_rope_attn_bwd_workspace_size",
    "gqa_rope_attn_bwd",
    "gqa_rope_attn_qkv_proj_workspace_size",
    "gqa_rope_attn_qkv_proj",
    "gqa_rope_attn_fwd_masked",
    "gqa_rope_attn_fwd_rotated",
)

_lib = None


class GqaError(RuntimeError):
    def __init__(self, code: int, where: str = "gqa_rope_attn_fwd"):
        self.code = code
        super().__init__(f"{where} failed: {code} ({strerror(code)})")


def load() -> ctypes.CDLL:
    """Load the library (once). Raises if it is missing: there is no
    fallback implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with `python -m transformer_attention_gqa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    c_int, c_size, c_void, c_double = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_double
    lib.gqa_rope_attn_workspace_size.restype = c_size
    lib.gqa_rope_attn_workspace_size.argtypes = [c_int] * 6
    lib.gqa_rope_attn_fwd.restype = c_int
    lib.gqa_rope_attn_fwd.argtypes = [c_void, c_void, c_void, c_void, c_double, c_void, c_int, c_int, c_int, c_int,
                                      c_int, c_int, c_int, c_void, c_void, c_void, c_size, c_void]
    lib.gqa_rope_attn_get_device_status.restype = c_int
    lib.gqa_rope_attn_get_device_status.argtypes = [c_void]
    lib.gqa_rope_attn_strerror.restype = ctypes.c_char_p
    lib.gqa_rope_attn_strerror.argtypes = [c_int]
    lib.gqa_rope_attn_abi_version.restype = c_int
    lib.gqa_rope_attn_abi_version.argtypes = []
    lib.gqa_rope_attn_last_launch_count.restype = c_int
    lib.gqa_rope_attn_last_launch_count.argtypes = []
    lib.gqa_rope_attn_fwd_noalloc.restype = c_int
    lib.gqa_rope_attn_fwd_noalloc.argtypes = [c_void, c_void, c_void, c_void, c_double, c_void, c_int, c_int, c_int,
                                              c_int, c_int, c_int, c_int, c_void, c_void, c_void]
    lib.gqa_rope_attn_decode_workspace_size.restype = c_size
    lib.gqa_rope_attn_decode_workspace_size.argtypes = [c_int] * 5
    lib.gqa_rope_attn_decode.restype = c_int
    lib.gqa_rope_attn_decode.argtypes = [c_void, c_void, c_void, c_void, c_void, c_void, c_double, c_int, c_int,
                                         c_int, c_int, c_int, c_void, c_void, c_void, c_size, c_void]
    lib.gqa_rope_attn_bwd_workspace_size.restype = c_size
    lib.gqa_rope_attn_bwd_workspace_size.argtypes = [c_int] * 5
    lib.gqa_rope_attn_bwd.restype = c_int
    lib.gqa_rope_attn_bwd.argtypes = [c_void, c_void, c_void, c_void, c_void, c_void, c_void, c_double, c_void,
                                      c_int, c_int, c_int, c_int, c_int, c_int, c_void, c_void, c_void, c_void,
                                      c_size, c_void]
    lib.gqa_rope_attn_qkv_proj_workspace_size.restype = c_size
    lib.gqa_rope_attn_qkv_proj_workspace_size.argtypes = [c_int, c_int]
    lib.gqa_rope_attn_qkv_proj.restype = c_int
    lib.gqa_rope_attn_qkv_proj.argtypes = [c_void, c_void, c_void, c_double, c_void, c_int, c_int, c_int, c_int,
                                           c_int, c_int, c_void, c_void, c_void, c_void, c_size, c_void]
    lib.gqa_rope_attn_fwd_masked.restype = c_int
    lib.gqa_rope_attn_fwd_masked.argtypes = [c_void, c_void, c_void, c_void, c_double, c_void, c_int, c_int, c_int,
                                             c_int, c_int, c_int, c_void, c_int, c_int, c_void, c_void, c_void,
                                             c_size, c_void]
    lib.gqa_rope_attn_fwd_rotated.restype = c_int
    lib.gqa_rope_attn_fwd_rotated.argtypes = [c_void, c_void, c_void, c_void, c_int, c_int, c_int, c_int, c_int,
                                              c_int, c_void, c_void, c_void, c_size, c_void]
    lib.gqa_rope_attn_set_profile_events.restype = None
    lib.gqa_rope_attn_set_profile_events.argtypes = [c_void, c_void, c_void]
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().gqa_rope_attn_strerror(int(code)).decode()


def workspace_size(num_seqs: int, total_tokens: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                   dtype: int = GQA_DTYPE_BF16) -> int:
    return int(load().gqa_rope_attn_workspace_size(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim, dtype))


def gqa_rope_attn_fwd(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads, n_kv_heads,
                      head_dim, causal, dtype, out, lse, workspace, workspace_bytes, stream) -> int:
    """Raw call with integer device addresses (0 for NULL); returns the status."""
    return int(load().gqa_rope_attn_fwd(q, k, v, positions, float(rope_theta), cu_seqlens, int(num_seqs),
                                        int(total_tokens), int(n_q_heads), int(n_kv_heads), int(head_dim),
                                        int(causal), int(dtype), out, lse, workspace, int(workspace_bytes), stream))


def gqa_rope_attn_fwd_rotated(q, k, v, cu_seqlens, num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim, causal,
                              out, lse, workspace, workspace_bytes, stream) -> int:
    """Raw call of the forward on already rotated q and k; integer device
    addresses, 0 for NULL; returns the status."""
    return int(load().gqa_rope_attn_fwd_rotated(q, k, v, cu_seqlens, int(num_seqs), int(total_tokens),
                                                int(n_q_heads), int(n_kv_heads), int(head_dim), int(causal), out, lse,
                                                workspace, int(workspace_bytes), stream))


def gqa_rope_attn_fwd_noalloc(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,
                              n_kv_heads, head_dim, causal, dtype, out, lse, stream) -> int:
    """Raw call of the no-allocation entry point (scratch built into the
    library); integer device addresses, 0 for NULL; returns the status."""
    return int(load().gqa_rope_attn_fwd_noalloc(q, k, v, positions, float(rope_theta), cu_seqlens, int(num_seqs),
                                                int(total_tokens), int(n_q_heads), int(n_kv_heads), int(head_dim),
                                                int(causal), int(dtype), out, lse, stream))


def decode_workspace_size(batch: int, max_cache_len: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> int:
    return int(load().gqa_rope_attn_decode_workspace_size(batch, max_cache_len, n_q_heads, n_kv_heads, head_dim))


def gqa_rope_attn_decode(q, k_new, v_new, k_cache, v_cache, cache_seqlens, rope_theta, batch, max_cache_len,
                         n_q_heads, n_kv_heads, head_dim, out, lse, workspace, workspace_bytes, stream) -> int:
    """Raw call of the decoding step; integer device addresses (0 for NULL);
    returns the status."""
    return int(load().gqa_rope_attn_decode(q, k_new, v_new, k_cache, v_cache, cache_seqlens, float(rope_theta),
                                           int(batch), int(max_cache_len), int(n_q_heads), int(n_kv_heads),
                                           int(head_dim), out, lse, workspace, int(workspace_bytes), stream))


def bwd_workspace_size(num_seqs: int, total_tokens: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> int:
    return int(load().gqa_rope_attn_bwd_workspace_size(num_seqs, total_tokens, n_q_heads, n_kv_heads, head_dim))


def gqa_rope_attn_bwd(q, k, v, out, lse, dout, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,
                      n_kv_heads, head_dim, causal, dq, dk, dv, workspace, workspace_bytes, stream) -> int:
    """Raw call of the backward; integer device addresses (0 for NULL);
    returns the status."""
    return int(load().gqa_rope_attn_bwd(q, k, v, out, lse, dout, positions, float(rope_theta), cu_seqlens,
                                        int(num_seqs), int(total_tokens), int(n_q_heads), int(n_kv_heads),
                                        int(head_dim), int(causal), dq, dk, dv, workspace, int(workspace_bytes),
                                        stream))


def qkv_proj_workspace_size(total_tokens: int, head_dim: int) -> int:
    return int(load().gqa_rope_attn_qkv_proj_workspace_size(total_tokens, head_dim))


def gqa_rope_attn_qkv_proj(x, w_qkv, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, hidden, n_q_heads,
                           n_kv_heads, head_dim, q, k, v, workspace, workspace_bytes, stream) -> int:
    """Raw call of the QKV projection with the RoPE epilogue; integer device
    addresses (0 for NULL); returns the status."""
    return int(load().gqa_rope_attn_qkv_proj(x, w_qkv, positions, float(rope_theta), cu_seqlens, int(num_seqs),
                                             int(total_tokens), int(hidden), int(n_q_heads), int(n_kv_heads),
                                             int(head_dim), q, k, v, workspace, int(workspace_bytes), stream))


def gqa_rope_attn_fwd_masked(q, k, v, positions, rope_theta, cu_seqlens, num_seqs, total_tokens, n_q_heads,
                             n_kv_heads, head_dim, causal, mask, mask_len, mask_ld, out, lse, workspace,
                             workspace_bytes, stream) -> int:
    """Raw call of the forward with an additive mask; integer device
    addresses (0 for NULL); returns the status."""
    return int(load().gqa_rope_attn_fwd_masked(q, k, v, positions, float(rope_theta), cu_seqlens, int(num_seqs),
                                               int(total_tokens), int(n_q_heads), int(n_kv_heads), int(head_dim),
                                               int(causal), mask, int(mask_len), int(mask_ld), out, lse, workspace,
                                               int(workspace_bytes), stream))


def get_device_status(stream=None) -> int:
    return int(load().gqa_rope_attn_get_device_status(stream))


def abi_version() -> int:
    return int(load().gqa_rope_attn_abi_version())


def last_launch_count() -> int:
    return int(load().gqa_rope_attn_last_launch_count())


def set_profile_events(ev_start=None, ev_mid=None, ev_end=None) -> None:
    """Arm the next call on this thread to record the given cudaEvent_t
    handles (ints) around its first two kernels."""
    load().gqa_rope_attn_set_profile_events(ev_start, ev_mid, ev_end)
