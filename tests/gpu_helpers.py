"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs and compare with the float64 oracle."""
from __future__ import annotations

import numpy as np

import oracle.gqa_oracle as orc
from transformer_attention_gqa_b200 import workloads as wl

# Parity bar: bf16 (or fp32) outputs max-abs <= 2e-2 and mean-abs <= 2e-3;
# LSE relative error <= 1e-4, measured as |d| / max(|lse|, 1) because a row
# whose only key gives a score of 0 has lse = 0.
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
LSE_REL = 1e-4


def to_device(inp: "wl.Inputs", positions: bool = False):
    import torch

    dt = torch.float32 if inp.workload.io_dtype == "fp32" else torch.bfloat16
    q = torch.from_numpy(inp.q).to(dt).cuda()
    k = torch.from_numpy(inp.k).to(dt).cuda()
    v = torch.from_numpy(inp.v).to(dt).cuda()
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    pos = torch.from_numpy(inp.positions).cuda() if positions else None
    return q, k, v, cu, pos


def run_gpu(inp, positions=None, causal=None, need_lse=True):
    """Returns (out float64 [N, n_q, d], lse float64 [n_q, N] or None)."""
    import torch
    import transformer_attention_gqa_b200 as g

    w = inp.workload
    q, k, v, cu, _ = to_device(inp)
    pos = None if positions is None else torch.from_numpy(np.ascontiguousarray(positions, np.int32)).cuda()
    out, lse = g.gqa_rope_attn_fwd(q, k, v, cu, w.rope_theta, positions=pos,
                                   causal=w.causal if causal is None else causal, need_lse=need_lse)
    torch.cuda.synchronize()
    st = g.get_device_status()
    assert st == 0, f"device status {st}"
    o = out.float().cpu().numpy().astype(np.float64)
    l = None if lse is None else lse.cpu().numpy().astype(np.float64)
    return o, l


def oracle(inp, positions=None, causal=None, rows=None, operand_rounding=True, row_block=1024):
    w = inp.workload
    return orc.gqa_rope_attention(inp.q, inp.k, inp.v, inp.cu_seqlens, w.n_q_heads, w.n_kv_heads, w.rope_theta,
                                  positions=positions, causal=w.causal if causal is None else causal,
                                  operand_rounding=operand_rounding, query_rows=rows, row_block=row_block)


def compare(out, lse, ref_out, ref_lse, rows=None, what=""):
    if rows is not None:
        out, ref_out = out[rows], ref_out[rows]
        if lse is not None:
            lse, ref_lse = lse[:, rows], ref_lse[:, rows]
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    err = np.abs(out - ref_out)
    assert err.max() <= OUT_MAX_ABS, f"{what}: out max-abs {err.max():.3e}"
    assert err.mean() <= OUT_MEAN_ABS, f"{what}: out mean-abs {err.mean():.3e}"
    stats = {"out_max_abs": float(err.max()), "out_mean_abs": float(err.mean())}
    if lse is not None:
        rel = np.abs(lse - ref_lse) / np.maximum(np.abs(ref_lse), 1.0)
        assert rel.max() <= LSE_REL, f"{what}: lse rel {rel.max():.3e}"
        stats["lse_rel"] = float(rel.max())
        with np.errstate(divide="ignore", invalid="ignore"):
            stats["lse_rel_plain"] = float(np.max(np.abs(lse - ref_lse) / np.abs(ref_lse)))
    return stats
