"""GPU parity of the forward with an additive mask (gqa_rope_attn_fwd_masked,
through the C ABI) against the float64 oracle (``gqa_rope_attention_masked``)
on the same seeded bf16 inputs and bf16 mask values, at the forward's bar
(out max-abs <= 2e-2 and mean-abs <= 2e-3; lse |d| / max(|lse|, 1) <= 1e-4),
rows that see no key compared exactly (out 0, lse -inf)."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc
from tests.conftest import gpu_available
from tests import gpu_helpers as H
from transformer_attention_gqa_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

# (sequence lengths, n_q, n_kv, d, causal, share of hidden entries, rows hidden entirely)
CASES = {
    "causal_holes_g4_d128": ((300, 77), 32, 8, 128, True, 0.3, ()),
    "full_holes_varlen_g3_d64": ((150, 1, 40), 6, 2, 64, False, 0.5, (3,)),
    "dead_rows_g1_d32": ((140,), 4, 4, 32, True, 0.2, (0, 5, 139)),
    # the nano shapes of the benchmark's masked_nano workload (16 x 512 tokens, G = 3, d = 64)
    "nano_shapes_g3_d64": ((512,) * 16, 6, 2, 64, True, 0.0, ()),
    # one long sequence at the Llama-3-8B head layout: 16 KV tiles per q-tile row, 512 work items
    "long_2048_g4_d128": ((2048,), 32, 8, 128, True, 0.1, ()),
}


def _mask(seed, Lm, holes, dead):
    rng = np.random.default_rng(seed)
    Lp = (Lm + 7) // 8 * 8  # row stride a multiple of 8
    m = wl.to_bf16_values((rng.standard_normal((Lp, Lp)) * 2.0).astype(np.float32)).astype(np.float64)
    m[rng.random((Lp, Lp)) < holes] = -np.inf
    for i in dead:
        m[i, :] = -np.inf
    return m


@pytest.mark.parametrize("name", sorted(CASES))
def test_masked_forward_against_oracle(name):
    import torch
    import transformer_attention_gqa_b200 as g

    lens, nq, nkv, d, causal, holes, dead = CASES[name]
    inp = wl.make_custom(lens, nq, nkv, d, causal=causal, seed=11, name=name)
    mask = _mask(12, max(lens), holes, dead)
    q, k, v, cu, _ = H.to_device(inp)
    mt = torch.from_numpy(mask.astype(np.float32)).to(torch.bfloat16).cuda()
    out, lse = g.gqa_rope_attn_fwd_masked(q, k, v, cu, inp.workload.rope_theta, mt, causal=causal)
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    ro, rl = orc.gqa_rope_attention_masked(inp.q, inp.k, inp.v, inp.cu_seqlens, nq, nkv, inp.workload.rope_theta,
                                           mask, causal=causal)
    dead_rows = ~np.isfinite(rl)
    assert np.array_equal(dead_rows, ~np.isfinite(l)), "rows that see no key"
    assert np.all(o[np.transpose(dead_rows)] == 0)
    live = ~dead_rows
    err = np.abs(o - ro)
    assert err.max() <= H.OUT_MAX_ABS and err.mean() <= H.OUT_MEAN_ABS
    rel = np.abs(l[live] - rl[live]) / np.maximum(np.abs(rl[live]), 1.0)
    assert rel.max() <= H.LSE_REL


def test_zero_mask_equals_the_forward():
    import torch
    import transformer_attention_gqa_b200 as g

    inp = wl.make_custom((200, 57), 8, 2, 64, causal=True, seed=13)
    q, k, v, cu, _ = H.to_device(inp)
    mt = torch.zeros((200, 200), dtype=torch.bfloat16, device="cuda")
    out_m, lse_m = g.gqa_rope_attn_fwd_masked(q, k, v, cu, 1e4, mt, causal=True)
    out_f, lse_f = g.gqa_rope_attn_fwd(q, k, v, cu, 1e4, causal=True)
    torch.cuda.synchronize()
    assert (out_m.float() - out_f.float()).abs().max().item() <= 2e-2
    assert ((lse_m - lse_f).abs() / lse_f.abs().clamp(min=1.0)).max().item() <= 1e-5


def test_mask_with_a_wider_row_stride():
    """A mask whose rows are longer than mask_len (ld > Lm): only the first
    Lm columns of each row are read."""
    import torch
    import transformer_attention_gqa_b200 as g

    lens = (120, 9)
    inp = wl.make_custom(lens, 8, 2, 64, causal=True, seed=14, name="wide_ld")
    mask = _mask(15, 120, 0.2, ())                        # [120, 120]
    wide = np.full((mask.shape[0], mask.shape[1] + 16), np.nan)
    wide[:, : mask.shape[1]] = mask                       # never-read columns hold NaN
    q, k, v, cu, _ = H.to_device(inp)
    mt = torch.from_numpy(wide.astype(np.float32)).to(torch.bfloat16).cuda()
    out, lse = g.gqa_rope_attn_fwd_masked(q, k, v, cu, inp.workload.rope_theta, mt, causal=True)
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    ro, rl = orc.gqa_rope_attention_masked(inp.q, inp.k, inp.v, inp.cu_seqlens, 8, 2, inp.workload.rope_theta, mask,
                                           causal=True)
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    err = np.abs(o - ro)
    assert err.max() <= H.OUT_MAX_ABS and err.mean() <= H.OUT_MEAN_ABS
