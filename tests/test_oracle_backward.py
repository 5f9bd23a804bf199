"""Pins of the oracle's backward (CPU), each independent of its code:
central finite differences of the (separately pinned) forward, float64 torch
autograd through a torch formulation of the same forward written here, and
the closed form of single-key rows. Planted mistakes in a private copy of the
backward (a dropped term, a wrong sign of the rotation's transpose, a wrong
head map, a missing scale) must each fail a pin."""
import importlib.util
import math
import os

import numpy as np
import pytest

import oracle.gqa_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _inputs(seed, lens=(3, 2), nq=4, nkv=2, d=8):
    rng = np.random.default_rng(seed)
    n = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return (rng.standard_normal((n, nq, d)), rng.standard_normal((n, nkv, d)), rng.standard_normal((n, nkv, d)),
            rng.standard_normal((n, nq, d)), cu)


def pin_finite_differences(m, causal=True):
    q, k, v, dout, cu = _inputs(1)
    nq, nkv, theta = q.shape[1], k.shape[1], 100.0
    dq, dk, dv = m.gqa_rope_attention_backward(q, k, v, dout, cu, nq, nkv, theta, causal=causal)

    def loss(q_, k_, v_):
        o, _ = orc.gqa_rope_attention(q_, k_, v_, cu, nq, nkv, theta, causal=causal, operand_rounding=False)
        return float(np.sum(o * dout))

    eps = 1e-6
    for arr, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += eps
            fp = loss(*args)
            args[which][idx] -= 2 * eps
            fm = loss(*args)
            num[idx] = (fp - fm) / (2 * eps)
        assert np.max(np.abs(num - grad)) < 1e-6, f"finite differences, input {which}"


def _torch_reference(q, k, v, dout, cu, nq, nkv, theta, causal=True):
    """Float64 torch autograd of: rotate q and k by each token's in-sequence
    position (feature i with i + d/2), repeat each KV head over its group,
    scaled scores, causal mask, softmax, weighted sum."""
    import torch

    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    d = q.shape[-1]
    h = d // 2
    inv = theta ** (-torch.arange(h, dtype=torch.float64) * 2.0 / d)
    outs = []
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        ang = torch.arange(b - a, dtype=torch.float64)[:, None] * inv[None, :]
        c, sn = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]

        def rot(x):
            x1, x2 = x[..., :h], x[..., h:]
            return torch.cat([x1 * c - x2 * sn, x2 * c + x1 * sn], dim=-1)

        qr = rot(tq[a:b]).transpose(0, 1)
        kr = rot(tk[a:b]).repeat_interleave(nq // nkv, dim=1).transpose(0, 1)
        vr = tv[a:b].repeat_interleave(nq // nkv, dim=1).transpose(0, 1)
        sc = qr @ kr.transpose(-1, -2) / math.sqrt(d)
        if causal:
            mask = torch.ones(b - a, b - a, dtype=torch.bool).tril()
            sc = sc.masked_fill(~mask, float("-inf"))
        outs.append((torch.softmax(sc, dim=-1) @ vr).transpose(0, 1))
    out = torch.cat(outs, dim=0)
    (out * torch.tensor(dout, dtype=torch.float64)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def pin_torch_autograd(m):
    for causal in (True, False):
        q, k, v, dout, cu = _inputs(2, lens=(7, 1, 12), nq=6, nkv=2, d=16)
        got = m.gqa_rope_attention_backward(q, k, v, dout, cu, 6, 2, 1e4, causal=causal)
        ref = _torch_reference(q, k, v, dout, cu, 6, 2, 1e4, causal=causal)
        for g, r in zip(got, ref):
            assert np.max(np.abs(g - r)) < 1e-10, "torch autograd"


def pin_single_key_rows(m):
    """Sequences of one token: softmax over one key is constant, so dq = dk = 0
    and dv = the group's sum of dout."""
    q, k, v, dout, _ = _inputs(3, lens=(1, 1, 1), nq=6, nkv=3, d=8)
    dq, dk, dv = m.gqa_rope_attention_backward(q, k, v, dout, [0, 1, 2, 3], 6, 3, 1e4)
    assert np.max(np.abs(dq)) < 1e-14 and np.max(np.abs(dk)) < 1e-14, "single key: dq, dk"
    assert np.max(np.abs(dv - dout.reshape(3, 3, 2, 8).sum(axis=2))) < 1e-14, "single key: dv"


PINS = [pin_finite_differences, pin_torch_autograd, pin_single_key_rows]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_backward_pins(pin):
    pin(orc)


def test_backward_with_operand_rounding_is_close_to_exact():
    q, k, v, dout, cu = _inputs(4, lens=(20,), nq=4, nkv=2, d=32)
    q, k, v = orc.round_to_bf16(q), orc.round_to_bf16(k), orc.round_to_bf16(v)
    ex = orc.gqa_rope_attention_backward(q, k, v, dout, cu, 4, 2, 1e4, operand_rounding=False)
    rd = orc.gqa_rope_attention_backward(q, k, v, dout, cu, 4, 2, 1e4, operand_rounding=True)
    for a, b in zip(ex, rd):
        assert np.max(np.abs(a - b)) < 0.05 * max(1.0, np.max(np.abs(a)))


MUTATIONS = {
    "no_delta": ("ds = w * (dw - delta)", "ds = w * dw"),
    "rotation_not_transposed": ("return g * c - rotate_half(g) * s", "return g * c + rotate_half(g) * s"),
    "repeat_head_map": ("reshape(L, n_kv_heads, G, d).sum(axis=2)\n        dv[a:b]",
                        "reshape(L, G, n_kv_heads, d).sum(axis=1)\n        dv[a:b]"),
    "missing_scale": ("dqh = np.matmul(ds, kh) * scale", "dqh = np.matmul(ds, kh)"),
    "dv_not_transposed": ("dvh = np.matmul(np.swapaxes(w, -1, -2), doh)", "dvh = np.matmul(w, doh)"),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_backward_mistakes_are_caught(name):
    src = open(os.path.join(ROOT, "oracle", "gqa_oracle.py")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, name
    spec = importlib.util.spec_from_loader("_oracle_bwd_mut", loader=None)
    m = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), "_oracle_bwd_mut", "exec"), m.__dict__)
    failed = 0
    for pin in PINS:
        try:
            pin(m)
        except AssertionError:
            failed += 1
    assert failed >= 1, f"mutation {name} not caught"
