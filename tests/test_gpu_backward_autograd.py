"""The autograd binding (``gqa_rope_attention``) on the GPU: out.backward()
runs the library's backward on the forward's saved out and lse; the
gradients match the float64 oracle's backward at the backward's bar
(tests/test_gpu_backward.py)."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc
from tests.conftest import gpu_available
from transformer_attention_gqa_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]


def test_autograd_gradients_match_the_oracle():
    import torch
    import transformer_attention_gqa_b200 as g

    inp = wl.make_custom((130, 70), 8, 2, 64, seed=21, name="autograd")
    w = inp.workload
    bf = torch.bfloat16
    q, k, v = (torch.from_numpy(a).to(bf).cuda().requires_grad_(True) for a in (inp.q, inp.k, inp.v))
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    dout = wl.make_grad_output(inp)
    out = g.gqa_rope_attention(q, k, v, cu, w.rope_theta)
    out.backward(torch.from_numpy(dout).to(bf).cuda())
    torch.cuda.synchronize()
    assert g.get_device_status() == 0
    ref = orc.gqa_rope_attention_backward(inp.q, inp.k, inp.v, dout, inp.cu_seqlens, w.n_q_heads, w.n_kv_heads,
                                          w.rope_theta, operand_rounding=True)
    for name, t, r in zip(("dq", "dk", "dv"), (q, k, v), ref):
        a = t.grad.float().cpu().numpy().astype(np.float64)
        err = np.abs(a - r)
        assert err.max() <= 3e-2 * np.abs(r).max() and err.mean() <= 1e-2 * np.abs(r).mean(), name
