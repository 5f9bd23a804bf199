"""GPU parity of the forward on already rotated q and k
(gqa_rope_attn_fwd_rotated, through the C ABI).

* Given the rotated, bf16-rounded q and k that the oracle's apply_rope
  produces (the rounding the fused forward is pinned to bit for bit), the
  call must reproduce the fused forward on the unrotated inputs exactly:
  the attention kernel then sees the same operands.
* Against the oracle: attention on rotated inputs is the oracle's forward at
  position 0 for every token, where the rotation is the identity (cos 0 = 1,
  sin 0 = 0; pinned by the oracle's own RoPE tests).
* The pages' module chain, project -> rotate -> attend ("Attention from
  Scratch", section "Attention, the math", steps 1-2 and 4-6): the GPU
  projection with the RoPE epilogue feeding this call, against the oracle's
  projection feeding its attention, at the forward's bar."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc
from tests.conftest import gpu_available
from tests import gpu_helpers as H
from transformer_attention_gqa_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

CASES = [
    # (seq_lens, n_q, n_kv, d, theta, causal)
    ([300, 0, 77], 32, 8, 128, 5e5, True),
    ([129, 1, 400], 6, 2, 64, 1e4, True),
    ([513], 4, 4, 32, 1e4, True),
    ([200, 90], 14, 2, 64, 1e6, False),
    ([257], 128, 1, 32, 1e4, True),
]


def _rotated(inp):
    w = inp.workload
    pos = np.concatenate([np.arange(b - a) for a, b in zip(inp.cu_seqlens[:-1], inp.cu_seqlens[1:])])
    qr = orc.apply_rope(inp.q, pos, w.rope_theta, operand_rounding=True)
    kr = orc.apply_rope(inp.k, pos, w.rope_theta, operand_rounding=True)
    return qr, kr


def _run_rotated(qr, kr, v, cu, causal):
    import torch
    import transformer_attention_gqa_b200 as g

    bf = torch.bfloat16
    q = torch.from_numpy(qr.astype(np.float32)).to(bf).cuda()
    k = torch.from_numpy(kr.astype(np.float32)).to(bf).cuda()
    vv = torch.from_numpy(np.asarray(v, np.float32)).to(bf).cuda()
    cud = torch.from_numpy(np.asarray(cu, np.int32)).cuda()
    out, lse = g.gqa_rope_attn_fwd_rotated(q, k, vv, cud, causal=causal)
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0]}-q{c[1]}-kv{c[2]}-d{c[3]}-c{int(c[5])}" for c in CASES])
def test_rotated_inputs_reproduce_the_fused_forward_bit_for_bit(case):
    lens, nq, nkv, d, theta, causal = case
    inp = wl.make_custom(lens, nq, nkv, d, theta, causal=causal, seed=sum(lens) + 3 * nq)
    fused_out, fused_lse = H.run_gpu(inp)
    qr, kr = _rotated(inp)
    out, lse = _run_rotated(qr, kr, inp.v, inp.cu_seqlens, causal)
    assert np.array_equal(out, fused_out)
    assert np.array_equal(lse, fused_lse)
    zero = np.zeros(inp.workload.total_tokens, np.int32)
    ref_out, ref_lse = orc.gqa_rope_attention(qr, kr, inp.v, inp.cu_seqlens, nq, nkv, theta, positions=zero,
                                              causal=causal)
    H.compare(out, lse, ref_out, ref_lse, what=f"rotated {case}")


@pytest.mark.parametrize("lens, C, nq, nkv, d", [((200, 77), 4096, 32, 8, 128), ((300, 45), 384, 6, 2, 64)])
def test_projection_feeds_the_rotated_forward(lens, C, nq, nkv, d):
    """The GPU chain against the oracle chain. The two projections may round
    a few elements to neighbouring bf16 values (fp32 against float64
    accumulation), which moves the scores: the attention step is therefore
    checked at the forward's bar on the GPU projection's own outputs, and
    the end-to-end LSE within the score perturbation those roundings cause
    (log-sum-exp moves by at most the largest change of a row's scores),
    computed from the two sets of operands."""
    import torch
    import transformer_attention_gqa_b200 as g

    theta = 5e5 if d == 128 else 1e4
    inp = wl.make_projection_inputs(lens, C, nq, nkv, d, rope_theta=theta, seed=17)
    bf = torch.bfloat16
    x = torch.from_numpy(inp.x).to(bf).cuda()
    w = torch.from_numpy(inp.w_qkv).to(bf).cuda()
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    q, k, v = g.gqa_rope_attn_qkv_proj(x, w, nq, nkv, theta, cu_seqlens=cu)
    out, lse = g.gqa_rope_attn_fwd_rotated(q, k, v, cu)
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    out = out.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    gq, gk, gv = (t.float().cpu().numpy().astype(np.float64) for t in (q, k, v))
    zero = np.zeros(sum(lens), np.int32)
    # the attention step on the GPU projection's outputs
    ref_out, ref_lse = orc.gqa_rope_attention(gq, gk, gv, inp.cu_seqlens, nq, nkv, theta, positions=zero)
    H.compare(out, lse, ref_out, ref_lse, what="rotated forward on the projection's outputs")
    # the chain end to end
    f, fk = nq * d, nkv * d
    wq = inp.w_qkv
    rq, rk, rv = orc.qkv_rope_projection(inp.x, wq[:f], wq[f:f + fk], wq[f + fk:], nq, nkv, theta,
                                         cu_seqlens=inp.cu_seqlens, operand_rounding=True)
    chain_out, chain_lse = orc.gqa_rope_attention(rq, rk, rv, inp.cu_seqlens, nq, nkv, theta, positions=zero)
    H.compare(out, None, chain_out, None, what="projection -> rotated forward, out")
    G = nq // nkv
    ds = np.zeros((nq, sum(lens)))
    for a, b in zip(inp.cu_seqlens[:-1], inp.cu_seqlens[1:]):
        for h in range(nq):
            s1 = gq[a:b, h] @ gk[a:b, h // G].T
            s2 = rq[a:b, h] @ rk[a:b, h // G].T
            dlt = np.tril(np.abs(s1 - s2)) / np.sqrt(d)
            ds[h, a:b] = dlt.max(axis=1)
    err = np.abs(lse - chain_lse)
    assert np.all(err <= ds + H.LSE_REL * np.maximum(np.abs(chain_lse), 1.0)), \
        f"chain lse: {err.max():.3e} vs score change {ds.max():.3e}"
