"""The Python binding rejects tensors the C library could not use (host
tensors, mismatched shapes or dtypes) before any library call: the library
takes raw device addresses and cannot tell a host pointer from a device one.
CPU only."""
import pytest
import torch

import transformer_attention_gqa_b200 as g


def _fwd_args(N=16, nq=4, nkv=2, d=32, dtype=torch.bfloat16):
    return (torch.zeros(N, nq, d, dtype=dtype), torch.zeros(N, nkv, d, dtype=dtype),
            torch.zeros(N, nkv, d, dtype=dtype), torch.tensor([0, N], dtype=torch.int32))


def test_fwd_rejects_host_tensors():
    q, k, v, cu = _fwd_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        g.gqa_rope_attn_fwd(q, k, v, cu, 1e4)


@pytest.mark.parametrize("bad", ["k_shape", "v_dtype", "cu_dtype", "positions", "out_shape", "lse_dtype", "q_dim"])
def test_fwd_rejects_inconsistent_arguments(bad):
    q, k, v, cu = _fwd_args()
    kw = {}
    if bad == "k_shape":
        k = torch.zeros(16, 2, 64, dtype=torch.bfloat16)
    elif bad == "v_dtype":
        v = v.float()
    elif bad == "cu_dtype":
        cu = cu.long()
    elif bad == "positions":
        kw["positions"] = torch.zeros(15, dtype=torch.int32)
    elif bad == "out_shape":
        kw["out"] = torch.zeros(16, 4, 16, dtype=torch.bfloat16)
    elif bad == "lse_dtype":
        kw["lse"] = torch.zeros(4, 16, dtype=torch.float64)
    elif bad == "q_dim":
        q = q[0]
    with pytest.raises(ValueError):
        g.gqa_rope_attn_fwd(q, k, v, cu, 1e4, **kw)


def test_fwd_rejects_other_dtypes():
    q, k, v, cu = _fwd_args(dtype=torch.float16)
    with pytest.raises(TypeError):
        g.gqa_rope_attn_fwd(q, k, v, cu, 1e4)


def _dec_args(B=3, L=10, nq=8, nkv=2, d=64):
    bf = torch.bfloat16
    return (torch.zeros(B, nq, d, dtype=bf), torch.zeros(B, nkv, d, dtype=bf), torch.zeros(B, nkv, d, dtype=bf),
            torch.zeros(B, L, nkv, d, dtype=bf), torch.zeros(B, L, nkv, d, dtype=bf),
            torch.zeros(B, dtype=torch.int32))


def test_decode_rejects_host_tensors():
    with pytest.raises(ValueError, match="CUDA tensor"):
        g.gqa_rope_attn_decode(*_dec_args(), 1e4)


@pytest.mark.parametrize("bad", ["cache_shape", "lens_dtype", "lens_shape", "knew_shape", "out_shape"])
def test_decode_rejects_inconsistent_arguments(bad):
    q, kn, vn, kc, vc, lens = _dec_args()
    kw = {}
    if bad == "cache_shape":
        vc = torch.zeros(3, 11, 2, 64, dtype=torch.bfloat16)
    elif bad == "lens_dtype":
        lens = lens.long()
    elif bad == "lens_shape":
        lens = torch.zeros(4, dtype=torch.int32)
    elif bad == "knew_shape":
        kn = torch.zeros(3, 1, 64, dtype=torch.bfloat16)
    elif bad == "out_shape":
        kw["out"] = torch.zeros(3, 8, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        g.gqa_rope_attn_decode(q, kn, vn, kc, vc, lens, 1e4, **kw)


def test_decode_rejects_other_dtypes():
    q, kn, vn, kc, vc, lens = _dec_args()
    with pytest.raises(TypeError):
        g.gqa_rope_attn_decode(q.float(), kn, vn, kc, vc, lens, 1e4)


def _bwd_args(N=16, nq=4, nkv=2, d=32):
    bf = torch.bfloat16
    q, k, v, cu = _fwd_args(N, nq, nkv, d)
    return q, k, v, torch.zeros(N, nq, d, dtype=bf), torch.zeros(nq, N), torch.zeros(N, nq, d, dtype=bf), cu


def test_bwd_rejects_host_tensors():
    q, k, v, out, lse, dout, cu = _bwd_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        g.gqa_rope_attn_bwd(q, k, v, out, lse, dout, cu, 1e4)


@pytest.mark.parametrize("bad", ["lse_shape", "lse_dtype", "dout_shape", "dk_shape", "positions"])
def test_bwd_rejects_inconsistent_arguments(bad):
    q, k, v, out, lse, dout, cu = _bwd_args()
    kw = {}
    if bad == "lse_shape":
        lse = torch.zeros(16, 4)
    elif bad == "lse_dtype":
        lse = lse.double()
    elif bad == "dout_shape":
        dout = dout[:8]
    elif bad == "dk_shape":
        kw["dk"] = torch.zeros(16, 4, 32, dtype=torch.bfloat16)
    elif bad == "positions":
        kw["positions"] = torch.zeros(16, dtype=torch.int64)
    with pytest.raises(ValueError):
        g.gqa_rope_attn_bwd(q, k, v, out, lse, dout, cu, 1e4, **kw)


def test_bwd_rejects_other_dtypes():
    q, k, v, out, lse, dout, cu = _bwd_args()
    with pytest.raises(TypeError):
        g.gqa_rope_attn_bwd(q.float(), k.float(), v.float(), out.float(), lse, dout.float(), cu, 1e4)


def test_qkv_proj_rejects_host_tensors_and_bad_shapes():
    bf = torch.bfloat16
    x = torch.zeros(16, 64, dtype=bf)
    w = torch.zeros((4 + 2 * 2) * 32, 64, dtype=bf)
    cu = torch.tensor([0, 16], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        g.gqa_rope_attn_qkv_proj(x, w, 4, 2, 1e4, cu_seqlens=cu)
    with pytest.raises(ValueError):
        g.gqa_rope_attn_qkv_proj(x, w[:, :32], 4, 2, 1e4, cu_seqlens=cu)  # C mismatch
    with pytest.raises(ValueError):
        g.gqa_rope_attn_qkv_proj(x, w[:250], 4, 2, 1e4, cu_seqlens=cu)    # rows not heads x d
    with pytest.raises(ValueError):
        g.gqa_rope_attn_qkv_proj(x, w, 4, 2, 1e4)                          # no positions, no cu_seqlens
    with pytest.raises(TypeError):
        g.gqa_rope_attn_qkv_proj(x.float(), w, 4, 2, 1e4, cu_seqlens=cu)


def test_masked_rejects_host_tensors_and_bad_masks():
    q, k, v, cu = _fwd_args()
    bf = torch.bfloat16
    with pytest.raises(TypeError):
        g.gqa_rope_attn_fwd_masked(q, k, v, cu, 1e4, torch.zeros(16, 16))          # fp32 mask
    with pytest.raises(ValueError):
        g.gqa_rope_attn_fwd_masked(q, k, v, cu, 1e4, torch.zeros(16, 12, dtype=bf))  # fewer columns than rows
    with pytest.raises(ValueError):
        g.gqa_rope_attn_fwd_masked(q, k, v, cu, 1e4, torch.zeros(12, 12, dtype=bf))  # row stride 12
    with pytest.raises(ValueError, match="CUDA tensor"):
        g.gqa_rope_attn_fwd_masked(q, k, v, cu, 1e4, torch.zeros(16, 16, dtype=bf))
