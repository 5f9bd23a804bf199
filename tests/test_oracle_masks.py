"""Pins of the oracle's additive masks (``gqa_rope_attention_masked``), CPU
only, each independent of its code: the causal mask written as an additive
0/-inf mask reproduces the (separately pinned) causal forward; a zero mask
reproduces the unmasked forward; a constant added to a row leaves out
unchanged and shifts lse by that constant; a row left with one visible key
returns that key's value and its score (closed form); torch's scaled dot
product attention with the same float mask agrees. Planted mistakes (mask
transposed, added before the scaling, ignored) must each fail a pin."""
import importlib.util
import math
import os

import numpy as np
import pytest

import oracle.gqa_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _inputs(seed, lens=(6, 1, 9), nq=4, nkv=2, d=8):
    rng = np.random.default_rng(seed)
    n = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    return rng.standard_normal((n, nq, d)), rng.standard_normal((n, nkv, d)), rng.standard_normal((n, nkv, d)), cu


def pin_causal_as_additive(m):
    q, k, v, cu = _inputs(1)
    Lm = 9
    add = np.where(np.tril(np.ones((Lm, Lm))) > 0, 0.0, -np.inf)
    a = m.gqa_rope_attention_masked(q, k, v, cu, 4, 2, 1e4, add, causal=False, operand_rounding=False)
    b = orc.gqa_rope_attention(q, k, v, cu, 4, 2, 1e4, causal=True, operand_rounding=False)
    assert np.max(np.abs(a[0] - b[0])) < 1e-13 and np.max(np.abs(a[1] - b[1])) < 1e-13, "causal as additive"


def pin_zero_mask(m):
    q, k, v, cu = _inputs(2)
    for causal in (True, False):
        a = m.gqa_rope_attention_masked(q, k, v, cu, 4, 2, 1e4, np.zeros((9, 9)), causal=causal)
        b = orc.gqa_rope_attention(q, k, v, cu, 4, 2, 1e4, causal=causal)
        assert np.max(np.abs(a[0] - b[0])) < 1e-13 and np.max(np.abs(a[1] - b[1])) < 1e-13, "zero mask"


def pin_row_shift(m):
    q, k, v, cu = _inputs(3)
    rng = np.random.default_rng(4)
    base = rng.standard_normal((9, 9))
    c = rng.standard_normal(9) * 3
    a = m.gqa_rope_attention_masked(q, k, v, cu, 4, 2, 1e4, base, causal=True)
    b = m.gqa_rope_attention_masked(q, k, v, cu, 4, 2, 1e4, base + c[:, None], causal=True)
    assert np.max(np.abs(a[0] - b[0])) < 1e-12, "row shift: out"
    pos = np.concatenate([np.arange(L) for L in (6, 1, 9)])
    assert np.max(np.abs(b[1] - a[1] - c[pos][None, :])) < 1e-12, "row shift: lse"


def pin_single_visible_key(m):
    """Row i sees only key j(i) = (3 i + 1) mod L (an asymmetric pattern):
    out = v[j(i)], lse = q_i' . k_j' / sqrt(d) + mask value there."""
    rng = np.random.default_rng(5)
    L, nq, nkv, d = 7, 2, 1, 8
    q, k, v = rng.standard_normal((L, nq, d)), rng.standard_normal((L, nkv, d)), rng.standard_normal((L, nkv, d))
    mask = np.full((L, L), -np.inf)
    j = (3 * np.arange(L) + 1) % L
    bias = rng.standard_normal(L)
    mask[np.arange(L), j] = bias
    o, l = m.gqa_rope_attention_masked(q, k, v, [0, L], nq, nkv, 1e4, mask, operand_rounding=False)
    pos = np.arange(L)
    qr, kr = orc.apply_rope(q, pos, 1e4), orc.apply_rope(k, pos, 1e4)
    for i in range(L):
        for h in range(nq):
            assert np.max(np.abs(o[i, h] - v[j[i], 0])) < 1e-13, "single key: out"
            want = float(np.dot(qr[i, h], kr[j[i], 0])) / math.sqrt(d) + bias[i]
            assert abs(l[h, i] - want) < 1e-12, "single key: lse"


def pin_torch_sdpa_float_mask(m):
    import torch
    import torch.nn.functional as F

    rng = np.random.default_rng(6)
    L, nq, nkv, d = 11, 4, 2, 16
    q, k, v = rng.standard_normal((L, nq, d)), rng.standard_normal((L, nkv, d)), rng.standard_normal((L, nkv, d))
    mask = rng.standard_normal((L, L)) * 2
    mask[rng.random((L, L)) < 0.3] = -np.inf
    np.fill_diagonal(mask, 0.0)  # every row keeps a key
    o, _ = m.gqa_rope_attention_masked(q, k, v, [0, L], nq, nkv, 1e4, mask, operand_rounding=False)
    pos = np.arange(L)
    qr = torch.tensor(orc.apply_rope(q, pos, 1e4)).transpose(0, 1)
    kr = torch.tensor(orc.apply_rope(k, pos, 1e4)).repeat_interleave(nq // nkv, dim=1).transpose(0, 1)
    vr = torch.tensor(v).repeat_interleave(nq // nkv, dim=1).transpose(0, 1)
    ref = F.scaled_dot_product_attention(qr, kr, vr, attn_mask=torch.tensor(mask)).transpose(0, 1).numpy()
    assert np.max(np.abs(o - ref)) < 1e-12, "torch sdpa with a float mask"


PINS = [pin_causal_as_additive, pin_zero_mask, pin_row_shift, pin_single_visible_key, pin_torch_sdpa_float_mask]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_mask_pins(pin):
    pin(orc)


def test_fully_masked_row_is_zero_with_lse_minus_inf():
    q, k, v, cu = _inputs(7, lens=(5,))
    mask = np.zeros((5, 5))
    mask[2, :] = -np.inf
    o, l = orc.gqa_rope_attention_masked(q, k, v, cu, 4, 2, 1e4, mask)
    assert np.all(o[2] == 0) and np.all(np.isneginf(l[:, 2]))
    assert np.all(np.isfinite(o)) and np.sum(np.isneginf(l)) == 4


MUTATIONS = {
    "mask_transposed": ("scores = score(qh, kh) + mask[None, :L, :L]",
                        "scores = score(qh, kh) + mask[None, :L, :L].transpose(0, 2, 1)"),
    "mask_before_scaling": ("scores = score(qh, kh) + mask[None, :L, :L]",
                            "scores = score(qh, kh) + mask[None, :L, :L] / math.sqrt(d)"),
    "mask_ignored": ("scores = score(qh, kh) + mask[None, :L, :L]", "scores = score(qh, kh)"),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mask_mistakes_are_caught(name):
    src = open(os.path.join(ROOT, "oracle", "gqa_oracle.py")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, name
    spec = importlib.util.spec_from_loader("_oracle_mask_mut", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), "_oracle_mask_mut", "exec"), mod.__dict__)
    failed = 0
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            failed += 1
    assert failed >= 1, f"mutation {name} not caught"
