"""GPU parity of the backward (gqa_rope_attn_bwd, through the C ABI) against
the float64 oracle's backward on the same seeded, bf16-rounded inputs; the
forward's own out and lse feed the backward, as in training.

Tolerance, from the arithmetic: the kernel rounds P and dS to bf16 (relative
2^-9 each) before their products, reads the forward's bf16 out for Delta, and
writes bf16 gradients (relative 2^-9). The products sum O(100-1000) terms of
either sign (dS sums to zero over the keys of a row), so the rounding errors
average instead of adding up, and each gradient stays within a few 2^-9
of its own scale: max |gpu - ref| <= 3e-2 * max |ref| and
mean |gpu - ref| <= 1e-2 * mean |ref|, per gradient."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc
from tests.conftest import gpu_available
from tests import gpu_helpers as H
from transformer_attention_gqa_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

MAX_REL = 3e-2
MEAN_REL = 1e-2

# (sequence lengths, n_q, n_kv, d, causal, theta): several key and query tiles
# with ragged tails; G = 1, 3 (padded packing), 4, 8, 128 (one token per
# query tile); an empty and a one-token sequence; MQA; non-causal.
CASES = {
    "g4_d64": ((300,), 8, 2, 64, True, 1e4),
    "varlen_g3_d32": ((70, 1, 0, 130, 257), 6, 2, 32, True, 1e4),
    "llama_heads_d128": ((256, 200), 32, 8, 128, True, 5e5),
    "mqa_g8_d128": ((200,), 8, 1, 128, True, 1e4),
    "noncausal_g1_d64": ((150, 40), 8, 8, 64, False, 1e4),
    "g128_d32": ((9,), 128, 1, 32, True, 1e4),
}


def run_bwd(inp, dout, positions=None):
    import torch
    import transformer_attention_gqa_b200 as g

    w = inp.workload
    q, k, v, cu, _ = H.to_device(inp)
    pos = None if positions is None else torch.from_numpy(np.ascontiguousarray(positions, np.int32)).cuda()
    out, lse = g.gqa_rope_attn_fwd(q, k, v, cu, w.rope_theta, positions=pos, causal=w.causal)
    do = torch.from_numpy(dout).to(torch.bfloat16).cuda()
    dq, dk, dv = g.gqa_rope_attn_bwd(q, k, v, out, lse, do, cu, w.rope_theta, positions=pos, causal=w.causal)
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    return [t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv)]


def oracle_bwd(inp, dout, positions=None):
    w = inp.workload
    return orc.gqa_rope_attention_backward(inp.q, inp.k, inp.v, dout, inp.cu_seqlens, w.n_q_heads, w.n_kv_heads,
                                           w.rope_theta, positions=positions, causal=w.causal,
                                           operand_rounding=True)


def compare_grads(got, ref, what):
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        assert np.all(np.isfinite(a)), f"{what} {name}: non-finite"
        err = np.abs(a - b)
        scale_max, scale_mean = np.abs(b).max(), np.abs(b).mean()
        assert err.max() <= MAX_REL * scale_max, f"{what} {name}: max {err.max():.3e} vs scale {scale_max:.3e}"
        assert err.mean() <= MEAN_REL * scale_mean, f"{what} {name}: mean {err.mean():.3e} vs {scale_mean:.3e}"


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_against_oracle(name):
    lens, nq, nkv, d, causal, theta = CASES[name]
    inp = wl.make_custom(lens, nq, nkv, d, rope_theta=theta, causal=causal, seed=5, name=name)
    dout = wl.make_grad_output(inp)
    compare_grads(run_bwd(inp, dout), oracle_bwd(inp, dout), name)


def test_backward_explicit_positions():
    inp = wl.make_custom((100, 90), 8, 2, 64, seed=6, name="positions")
    rng = np.random.default_rng(3)
    pos = (inp.positions + rng.integers(0, 4000, size=inp.positions.shape)).astype(np.int32)
    dout = wl.make_grad_output(inp)
    compare_grads(run_bwd(inp, dout, positions=pos), oracle_bwd(inp, dout, positions=pos), "positions")


def test_backward_dv_column_sums_at_full_size():
    """Llama-3-8B-shaped T = 8192 (too large for the oracle's backward): the
    softmax rows sum to one, so per KV head the keys' dv sum to the sum of
    dout over every token and every query head of the group."""
    inp = wl.make_inputs(wl.WORKLOADS["llama8b"])
    w = inp.workload
    dout = wl.make_grad_output(inp)
    _, _, dv = run_bwd(inp, dout)
    G = w.n_q_heads // w.n_kv_heads
    want = dout.astype(np.float64).reshape(-1, w.n_kv_heads, G, w.head_dim).sum(axis=(0, 2))
    got = dv.sum(axis=0)
    assert np.abs(got - want).max() <= 1e-2 * np.abs(want).max() + 1.0
