"""The autograd binding (``gqa_rope_attention``) on the CPU: the library's
two calls are replaced by float64 oracle stand-ins, so that only the
binding's plumbing is under test (what it saves, what reaches the backward
call, what it returns to autograd). CPU only; the GPU path of the same
function is in tests/test_gpu_backward_autograd.py."""
import numpy as np
import pytest
import torch

import oracle.gqa_oracle as orc
import transformer_attention_gqa_b200 as g


@pytest.fixture
def oracle_library(monkeypatch):
    calls = {}

    def fwd(q, k, v, cu, theta, positions=None, causal=True, **kw):
        o, l = orc.gqa_rope_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), cu.numpy(),
                                      q.shape[1], k.shape[1], theta, positions=positions, causal=causal,
                                      operand_rounding=False)
        calls["fwd"] = (theta, positions, causal)
        return torch.from_numpy(o).to(q.dtype), torch.from_numpy(l).float()

    def bwd(q, k, v, out, lse, dout, cu, theta, positions=None, causal=True, **kw):
        r = orc.gqa_rope_attention_backward(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                            dout.double().numpy(), cu.numpy(), q.shape[1], k.shape[1], theta,
                                            positions=positions, causal=causal)
        calls["bwd"] = (theta, positions, causal, out.shape, lse.shape, dout.is_contiguous())
        return tuple(torch.from_numpy(x).to(q.dtype) for x in r)

    monkeypatch.setattr(g, "gqa_rope_attn_fwd", fwd)
    monkeypatch.setattr(g, "gqa_rope_attn_bwd", bwd)
    monkeypatch.setattr(g, "_AUTOGRAD_DTYPES", ("float64",))  # the stand-ins work in float64
    return calls


@pytest.mark.parametrize("causal", [True, False])
def test_gradients_flow_through_the_binding(oracle_library, causal):
    rng = np.random.default_rng(0)
    lens = (5, 1, 7)
    N, nq, nkv, d = sum(lens), 4, 2, 8
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    q, k, v = (torch.tensor(rng.standard_normal((N, h, d)), dtype=torch.float64, requires_grad=True)
               for h in (nq, nkv, nkv))
    dout = torch.tensor(rng.standard_normal((N, nq, d)), dtype=torch.float64)
    out = g.gqa_rope_attention(q, k, v, cu, 1e4, causal=causal)
    (out * dout).sum().backward()
    ref = orc.gqa_rope_attention_backward(q.detach().numpy(), k.detach().numpy(), v.detach().numpy(), dout.numpy(),
                                          cu.numpy(), nq, nkv, 1e4, causal=causal)
    for t, r in zip((q, k, v), ref):
        assert np.max(np.abs(t.grad.numpy() - r)) < 1e-12
    theta, pos, c, oshape, lshape, contiguous = oracle_library["bwd"]
    assert theta == 1e4 and pos is None and c == causal and contiguous
    assert oshape == (N, nq, d) and lshape == (nq, N)


def test_non_contiguous_upstream_gradient_is_made_contiguous(oracle_library):
    rng = np.random.default_rng(1)
    N, nq, nkv, d = 6, 2, 1, 8
    cu = torch.tensor([0, N], dtype=torch.int32)
    q, k, v = (torch.tensor(rng.standard_normal((N, h, d)), dtype=torch.float64, requires_grad=True)
               for h in (nq, nkv, nkv))
    out = g.gqa_rope_attention(q, k, v, cu, 1e4)
    big = torch.tensor(rng.standard_normal((N, nq, 2 * d)), dtype=torch.float64)
    out.backward(big[..., ::2])  # a strided view
    assert oracle_library["bwd"][5]


def test_dtypes_the_backward_cannot_take_are_refused_before_the_forward(monkeypatch):
    called = []
    monkeypatch.setattr(g, "gqa_rope_attn_fwd", lambda *a, **kw: called.append(1))
    cu = torch.tensor([0, 4], dtype=torch.int32)
    q, k, v = (torch.zeros((4, 2, 8), dtype=torch.float32, requires_grad=True) for _ in range(3))
    with pytest.raises(TypeError, match="bfloat16"):
        g.gqa_rope_attention(q, k, v, cu, 1e4)
    assert not called
