"""GPU parity of the QKV projection with the RoPE epilogue
(gqa_rope_attn_qkv_proj, through the C ABI) against the float64 oracle
(``qkv_rope_projection``) on the same seeded bf16 inputs.

Tolerance, from the arithmetic: the kernel accumulates x W^T in fp32 (for C
up to 4096 and unit-scale outputs, errors of order 1e-5) and rounds each
rotated output once to bf16 (at most 2^-9 relative, 2^-8 allowing the fp32
error to cross a rounding midpoint); per element
|gpu - ref| <= 2^-8 |ref| + 1e-4 max|ref|."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc
from tests.conftest import gpu_available
from transformer_attention_gqa_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

# (sequence lengths, hidden, n_q, n_kv, d, theta): ragged token tails; the
# Llama-3-8B layer's widths (4096 -> 32/8 heads of 128); feature counts that
# end inside a 256-wide tile (6/2 heads of 64 = 640 features); d = 32; a
# hidden size that is not a multiple of 64.
CASES = {
    "llama_widths": ((200, 77), 4096, 32, 8, 128, 5e5),
    "nano_ragged_features": ((300,), 384, 6, 2, 64, 1e4),
    "d32": ((130, 1, 60), 256, 8, 4, 32, 1e4),
    "hidden_tail": ((70,), 200, 4, 2, 32, 1e4),  # the last 64-wide block of C is partly past the rows
}


def run(inp, positions=None):
    import torch
    import transformer_attention_gqa_b200 as g

    bf = torch.bfloat16
    x = torch.from_numpy(inp.x).to(bf).cuda()
    w = torch.from_numpy(inp.w_qkv).to(bf).cuda()
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    pos = None if positions is None else torch.from_numpy(np.ascontiguousarray(positions, np.int32)).cuda()
    q, k, v = g.gqa_rope_attn_qkv_proj(x, w, inp.n_q_heads, inp.n_kv_heads, inp.rope_theta, cu_seqlens=cu,
                                       positions=pos)
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    return [t.float().cpu().numpy().astype(np.float64) for t in (q, k, v)]


def oracle(inp, positions=None):
    f = inp.n_q_heads * inp.head_dim
    fk = inp.n_kv_heads * inp.head_dim
    w = inp.w_qkv
    return orc.qkv_rope_projection(inp.x, w[:f], w[f:f + fk], w[f + fk:], inp.n_q_heads, inp.n_kv_heads,
                                   inp.rope_theta, positions=positions, cu_seqlens=inp.cu_seqlens)


def compare(got, ref, what):
    for name, a, b in zip("qkv", got, ref):
        assert np.all(np.isfinite(a)), f"{what} {name}: non-finite"
        bound = 2.0 ** -8 * np.abs(b) + 1e-4 * np.abs(b).max()
        bad = np.abs(a - b) > bound
        assert not bad.any(), f"{what} {name}: {bad.sum()} elements off, max err {np.abs(a - b).max():.3e}"


@pytest.mark.parametrize("name", sorted(CASES))
def test_projection_against_oracle(name):
    lens, C, nq, nkv, d, theta = CASES[name]
    inp = wl.make_projection_inputs(lens, C, nq, nkv, d, rope_theta=theta, seed=7)
    compare(run(inp), oracle(inp), name)


def test_projection_explicit_positions():
    inp = wl.make_projection_inputs((100, 50), 512, 8, 2, 64, seed=8)
    pos = np.random.default_rng(9).integers(0, 100000, size=150).astype(np.int32)
    compare(run(inp, positions=pos), oracle(inp, positions=pos), "positions")
