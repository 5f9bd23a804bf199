"""CPU-only checks of the C ABI: the library loads, exports every function
include/gqa_rope_attn.h declares, and rejects bad arguments on the host
before any CUDA call (no GPU is touched here)."""
import os
import re
import subprocess

import pytest

from transformer_attention_gqa_b200 import _abi
from transformer_attention_gqa_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build()
    _abi.load()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(gqa_rope_attn_\w+)\s*\(", text)
    return sorted(set(names))


def test_exports_every_declared_function():
    decl = declared_functions()
    assert "gqa_rope_attn_fwd" in decl and len(decl) >= 5
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gqa_rope_attn_\w+)", out))
    assert set(decl) <= exported, set(decl) - exported
    lib = _abi.load()
    for name in decl:
        assert hasattr(lib, name)
    assert set(_abi.EXPORTED) == set(decl)


def test_abi_version_and_strerror():
    assert _abi.abi_version() == 1
    for code in range(7):
        assert isinstance(_abi.strerror(code), str) and _abi.strerror(code)
    assert _abi.strerror(99) == "unknown status"


def test_workspace_size():
    ws = _abi.workspace_size(1, 8192, 32, 8, 128)
    # at least the RoPE'd K (n_kv * N * d * 2) and the bf16 cos/sin table (N * d/2 * 4)
    assert ws >= 8 * 8192 * 128 * 2 + 8192 * 64 * 4
    assert ws % 256 == 0
    assert _abi.workspace_size(1, 8192, 32, 8, 128, _abi.GQA_DTYPE_FP32) > ws
    assert _abi.workspace_size(1, 8192, 32, 8, 96) == 0
    assert _abi.workspace_size(1, 8192, 30, 8, 128) == 0
    assert _abi.workspace_size(1, 8192, 256, 1, 128) == 0  # group of 256 heads
    assert _abi.workspace_size(-1, 8192, 32, 8, 128) == 0
    assert _abi.workspace_size(2, 100, 4, 2, 64) < _abi.workspace_size(2, 200, 4, 2, 64)


A = 4096  # fake, 256-byte aligned "device" addresses; never dereferenced by these checks


def call(**kw):
    args = dict(q=A, k=A, v=A, positions=0, rope_theta=1e4, cu_seqlens=A, num_seqs=1, total_tokens=128,
                n_q_heads=4, n_kv_heads=2, head_dim=64, causal=1, dtype=0, out=A, lse=0, workspace=0,
                workspace_bytes=0, stream=None)
    args.update(kw)
    return _abi.gqa_rope_attn_fwd(**args)


def test_host_rejections_before_any_cuda_call():
    E = _abi
    assert call(total_tokens=0) == E.GQA_OK  # no-op
    assert call(total_tokens=-1) == E.GQA_ERR_INVALID_ARG
    assert call(n_q_heads=6, n_kv_heads=4) == E.GQA_ERR_INVALID_ARG
    assert call(n_kv_heads=0) == E.GQA_ERR_INVALID_ARG
    assert call(causal=2) == E.GQA_ERR_INVALID_ARG
    assert call(dtype=7) == E.GQA_ERR_INVALID_ARG
    assert call(rope_theta=0.0) == E.GQA_ERR_INVALID_ARG
    assert call(rope_theta=float("nan")) == E.GQA_ERR_INVALID_ARG
    assert call(head_dim=96) == E.GQA_ERR_UNSUPPORTED
    assert call(n_q_heads=256, n_kv_heads=1) == E.GQA_ERR_UNSUPPORTED
    assert call(num_seqs=0) == E.GQA_ERR_INVALID_ARG
    assert call(q=0) == E.GQA_ERR_INVALID_ARG
    assert call(out=0) == E.GQA_ERR_INVALID_ARG
    assert call(cu_seqlens=0) == E.GQA_ERR_INVALID_ARG
    assert call(k=A + 8) == E.GQA_ERR_INVALID_ARG  # misaligned
    assert call(lse=A + 2) == E.GQA_ERR_INVALID_ARG
    # every argument fine but the workspace
    assert call() == E.GQA_ERR_WORKSPACE
    need = _abi.workspace_size(1, 128, 4, 2, 64)
    assert call(workspace=A, workspace_bytes=need - 1) == E.GQA_ERR_WORKSPACE
    assert call(workspace=A + 16, workspace_bytes=need) == E.GQA_ERR_WORKSPACE
    assert _abi.last_launch_count() == 0


def test_rotated_forward_host_rejections_before_any_cuda_call():
    E = _abi

    def rot(**kw):
        args = dict(q=A, k=A, v=A, cu_seqlens=A, num_seqs=1, total_tokens=128, n_q_heads=4, n_kv_heads=2,
                    head_dim=64, causal=1, out=A, lse=0, workspace=0, workspace_bytes=0, stream=None)
        args.update(kw)
        return _abi.gqa_rope_attn_fwd_rotated(**args)

    assert rot(total_tokens=0) == E.GQA_OK
    assert rot(total_tokens=-1) == E.GQA_ERR_INVALID_ARG
    assert rot(n_q_heads=6, n_kv_heads=4) == E.GQA_ERR_INVALID_ARG
    assert rot(causal=3) == E.GQA_ERR_INVALID_ARG
    assert rot(head_dim=48) == E.GQA_ERR_UNSUPPORTED
    assert rot(n_q_heads=256, n_kv_heads=1) == E.GQA_ERR_UNSUPPORTED
    assert rot(num_seqs=0) == E.GQA_ERR_INVALID_ARG
    assert rot(k=0) == E.GQA_ERR_INVALID_ARG
    assert rot(v=A + 4) == E.GQA_ERR_INVALID_ARG
    assert rot() == E.GQA_ERR_WORKSPACE
    need = _abi.workspace_size(1, 128, 4, 2, 64)
    assert rot(workspace=A, workspace_bytes=need - 1) == E.GQA_ERR_WORKSPACE
    assert _abi.last_launch_count() == 0


def test_product_path_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(ImportError):
        _abi.load()


def test_decode_workspace_size():
    ws = _abi.decode_workspace_size(32, 4097, 32, 8, 128)
    assert ws > 0 and ws % 256 == 0
    # partial outputs of at least one key range per (sequence, KV head)
    assert ws >= 32 * 8 * 4 * 128 * 4
    assert _abi.decode_workspace_size(32, 4097, 32, 8, 96) == 0      # head_dim
    assert _abi.decode_workspace_size(32, 4097, 32, 1, 128) == 0     # group of 32 > 16
    assert _abi.decode_workspace_size(32, 4097, 30, 8, 128) == 0     # not a multiple
    assert _abi.decode_workspace_size(32, 0, 32, 8, 128) == 0        # empty cache
    assert _abi.decode_workspace_size(-1, 4097, 32, 8, 128) == 0
    assert _abi.decode_workspace_size(0, 4097, 32, 8, 128) > 0       # empty batch: a no-op still accepted


def dcall(**kw):
    args = dict(q=A, k_new=A, v_new=A, k_cache=A, v_cache=A, cache_seqlens=A, rope_theta=1e4, batch=4,
                max_cache_len=100, n_q_heads=8, n_kv_heads=2, head_dim=64, out=A, lse=0, workspace=A,
                workspace_bytes=1 << 30, stream=None)
    args.update(kw)
    return _abi.gqa_rope_attn_decode(**args)


def test_decode_host_rejections_before_any_cuda_call():
    E = _abi
    assert dcall(batch=0) == E.GQA_OK  # no-op
    assert dcall(batch=-1) == E.GQA_ERR_INVALID_ARG
    assert dcall(max_cache_len=0) == E.GQA_ERR_INVALID_ARG
    assert dcall(n_q_heads=6, n_kv_heads=4) == E.GQA_ERR_INVALID_ARG
    assert dcall(rope_theta=0.0) == E.GQA_ERR_INVALID_ARG
    assert dcall(rope_theta=float("nan")) == E.GQA_ERR_INVALID_ARG
    assert dcall(head_dim=96) == E.GQA_ERR_UNSUPPORTED
    assert dcall(n_q_heads=64, n_kv_heads=2) == E.GQA_ERR_UNSUPPORTED  # group of 32
    assert dcall(batch=70000) == E.GQA_ERR_UNSUPPORTED
    assert dcall(q=0) == E.GQA_ERR_INVALID_ARG
    assert dcall(k_cache=0) == E.GQA_ERR_INVALID_ARG
    assert dcall(cache_seqlens=0) == E.GQA_ERR_INVALID_ARG
    assert dcall(out=A + 8) == E.GQA_ERR_INVALID_ARG      # 16-byte alignment
    assert dcall(lse=A + 2) == E.GQA_ERR_INVALID_ARG      # 4-byte alignment
    assert dcall(workspace=0) == E.GQA_ERR_WORKSPACE
    assert dcall(workspace=A + 16) == E.GQA_ERR_WORKSPACE  # 256-byte alignment
    assert dcall(workspace_bytes=16) == E.GQA_ERR_WORKSPACE


def test_bwd_workspace_size():
    ws = _abi.bwd_workspace_size(1, 8192, 32, 8, 128)
    assert ws % 256 == 0
    # at least K' (n_kv * N * d * 2), Q' (N * n_q * d * 2) and the fp32 dq accumulator (N * n_q * d * 4)
    assert ws >= 8 * 8192 * 128 * 2 + 8192 * 32 * 128 * 6
    assert _abi.bwd_workspace_size(1, 8192, 32, 8, 96) == 0
    assert _abi.bwd_workspace_size(1, 8192, 30, 8, 128) == 0
    assert _abi.bwd_workspace_size(1, 8192, 256, 1, 128) == 0
    assert _abi.bwd_workspace_size(-1, 8192, 32, 8, 128) == 0
    assert _abi.bwd_workspace_size(2, 100, 4, 2, 64) < _abi.bwd_workspace_size(2, 200, 4, 2, 64)


def bcall(**kw):
    args = dict(q=A, k=A, v=A, out=A, lse=A, dout=A, positions=0, rope_theta=1e4, cu_seqlens=A, num_seqs=1,
                total_tokens=128, n_q_heads=4, n_kv_heads=2, head_dim=64, causal=1, dq=A, dk=A, dv=A, workspace=0,
                workspace_bytes=0, stream=None)
    args.update(kw)
    return _abi.gqa_rope_attn_bwd(**args)


def test_bwd_host_rejections_before_any_cuda_call():
    E = _abi
    assert bcall(total_tokens=0) == E.GQA_OK  # no-op
    assert bcall(total_tokens=-1) == E.GQA_ERR_INVALID_ARG
    assert bcall(n_q_heads=6, n_kv_heads=4) == E.GQA_ERR_INVALID_ARG
    assert bcall(causal=2) == E.GQA_ERR_INVALID_ARG
    assert bcall(rope_theta=-1.0) == E.GQA_ERR_INVALID_ARG
    assert bcall(head_dim=80) == E.GQA_ERR_UNSUPPORTED
    assert bcall(n_q_heads=256, n_kv_heads=1) == E.GQA_ERR_UNSUPPORTED
    assert bcall(num_seqs=0) == E.GQA_ERR_INVALID_ARG
    for name in ("q", "k", "v", "out", "lse", "dout", "cu_seqlens", "dq", "dk", "dv"):
        assert bcall(**{name: 0}) == E.GQA_ERR_INVALID_ARG, name
    for name in ("q", "k", "v", "out", "dout", "dq", "dk", "dv"):
        assert bcall(**{name: A + 8}) == E.GQA_ERR_INVALID_ARG, name  # 16-byte alignment
    assert bcall(lse=A + 2) == E.GQA_ERR_INVALID_ARG
    assert bcall(positions=A + 2) == E.GQA_ERR_INVALID_ARG
    assert bcall() == E.GQA_ERR_WORKSPACE
    need = _abi.bwd_workspace_size(1, 128, 4, 2, 64)
    assert bcall(workspace=A, workspace_bytes=need - 1) == E.GQA_ERR_WORKSPACE
    assert bcall(workspace=A + 16, workspace_bytes=need) == E.GQA_ERR_WORKSPACE
    assert _abi.last_launch_count() == 0


def test_qkv_proj_workspace_size():
    ws = _abi.qkv_proj_workspace_size(8192, 128)
    assert ws >= 8192 * 64 * 8 and ws % 256 == 0
    assert _abi.qkv_proj_workspace_size(8192, 96) == 0
    assert _abi.qkv_proj_workspace_size(-1, 128) == 0


def pcall(**kw):
    args = dict(x=A, w_qkv=A, positions=0, rope_theta=1e4, cu_seqlens=A, num_seqs=1, total_tokens=128, hidden=256,
                n_q_heads=4, n_kv_heads=2, head_dim=64, q=A, k=A, v=A, workspace=0, workspace_bytes=0, stream=None)
    args.update(kw)
    return _abi.gqa_rope_attn_qkv_proj(**args)


def test_qkv_proj_host_rejections_before_any_cuda_call():
    E = _abi
    assert pcall(total_tokens=0) == E.GQA_OK  # no-op
    assert pcall(total_tokens=-1) == E.GQA_ERR_INVALID_ARG
    assert pcall(hidden=0) == E.GQA_ERR_INVALID_ARG
    assert pcall(n_q_heads=6, n_kv_heads=4) == E.GQA_ERR_INVALID_ARG
    assert pcall(rope_theta=float("inf")) == E.GQA_ERR_INVALID_ARG
    assert pcall(head_dim=96) == E.GQA_ERR_UNSUPPORTED
    assert pcall(hidden=100) == E.GQA_ERR_UNSUPPORTED  # rows not 16-byte aligned
    for name in ("x", "w_qkv", "q", "k", "v"):
        assert pcall(**{name: 0}) == E.GQA_ERR_INVALID_ARG, name
        assert pcall(**{name: A + 8}) == E.GQA_ERR_INVALID_ARG, name
    assert pcall(cu_seqlens=0) == E.GQA_ERR_INVALID_ARG        # neither positions nor cu_seqlens
    assert pcall(cu_seqlens=0, positions=A) == E.GQA_ERR_WORKSPACE  # positions alone are enough
    assert pcall(positions=A + 2) == E.GQA_ERR_INVALID_ARG
    assert pcall() == E.GQA_ERR_WORKSPACE
    need = _abi.qkv_proj_workspace_size(128, 64)
    assert pcall(workspace=A, workspace_bytes=need - 1) == E.GQA_ERR_WORKSPACE
    assert _abi.last_launch_count() == 0


def mcall(**kw):
    args = dict(q=A, k=A, v=A, positions=0, rope_theta=1e4, cu_seqlens=A, num_seqs=1, total_tokens=128,
                n_q_heads=4, n_kv_heads=2, head_dim=64, causal=0, mask=A, mask_len=128, mask_ld=128, out=A, lse=0,
                workspace=0, workspace_bytes=0, stream=None)
    args.update(kw)
    return _abi.gqa_rope_attn_fwd_masked(**args)


def test_masked_host_rejections_before_any_cuda_call():
    E = _abi
    assert mcall(total_tokens=0) == E.GQA_OK
    assert mcall(mask_len=0) == E.GQA_ERR_INVALID_ARG
    assert mcall(mask_ld=100) == E.GQA_ERR_INVALID_ARG       # < mask_len
    assert mcall(mask_ld=132) == E.GQA_ERR_INVALID_ARG       # not a multiple of 8
    assert mcall(mask=0) == E.GQA_ERR_INVALID_ARG
    assert mcall(mask=A + 8) == E.GQA_ERR_INVALID_ARG
    assert mcall(causal=3) == E.GQA_ERR_INVALID_ARG
    assert mcall(head_dim=48) == E.GQA_ERR_UNSUPPORTED
    assert mcall() == E.GQA_ERR_WORKSPACE
    assert _abi.last_launch_count() == 0
