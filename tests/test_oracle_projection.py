"""Pins of the oracle's projection + RoPE (``qkv_rope_projection``), CPU only,
each independent of its code: float64 torch through the linear layers'
own convention (F.linear: y = x W^T) and a rotation written here; selection
(permutation) weights, which reduce the projection to a known re-indexing
of x; brute-force dot products at position 0, where the rotation is the
identity, and for V, which is never rotated. Planted mistakes in a private
copy of the oracle (a transposed weight, a wrong head split, a rotated V, an
unrotated K, ignored positions) must each fail a pin."""
import importlib.util
import os

import numpy as np
import pytest

import oracle.gqa_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _weights(rng, C, nq, nkv, d):
    return (rng.standard_normal((nq * d, C)), rng.standard_normal((nkv * d, C)), rng.standard_normal((nkv * d, C)))


def pin_torch_linear(m):
    """F.linear, view(tokens, heads, d), rotation of feature i with i + d/2
    by the in-sequence position (cos/sin in torch), V left alone."""
    import torch
    import torch.nn.functional as F

    rng = np.random.default_rng(1)
    lens, C, nq, nkv, d, theta = (5, 1, 7), 24, 6, 2, 8, 500.0
    N = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    x = rng.standard_normal((N, C))
    wq, wk, wv = _weights(rng, C, nq, nkv, d)
    got = m.qkv_rope_projection(x, wq, wk, wv, nq, nkv, theta, cu_seqlens=cu)
    tx = torch.tensor(x, dtype=torch.float64)
    pos = torch.cat([torch.arange(L, dtype=torch.float64) for L in lens])
    h = d // 2
    ang = pos[:, None] * theta ** (-torch.arange(h, dtype=torch.float64) * 2.0 / d)[None, :]
    c, s = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]

    def rot(y):
        return torch.cat([y[..., :h] * c - y[..., h:] * s, y[..., h:] * c + y[..., :h] * s], dim=-1)

    ref = (rot(F.linear(tx, torch.tensor(wq)).view(N, nq, d)), rot(F.linear(tx, torch.tensor(wk)).view(N, nkv, d)),
           F.linear(tx, torch.tensor(wv)).view(N, nkv, d))
    for name, a, b in zip("qkv", got, ref):
        assert np.max(np.abs(a - b.numpy())) < 1e-12, f"torch linear: {name}"


def pin_selection_weights(m):
    """W with one 1 per row, at column perm[j]: projected feature j is
    x[:, perm[j]], so q = rope(x[:, perm_q] split into heads) and v =
    x[:, perm_v] split into heads."""
    rng = np.random.default_rng(2)
    N, nq, nkv, d, theta = 9, 4, 2, 8, 1e4
    C = nq * d
    x = rng.standard_normal((N, C))
    perms = [rng.permutation(C)[: nh * d] for nh in (nq, nkv, nkv)]
    ws = []
    for perm in perms:
        w = np.zeros((len(perm), C))
        w[np.arange(len(perm)), perm] = 1.0
        ws.append(w)
    pos = rng.integers(0, 3000, size=N)
    q, k, v = m.qkv_rope_projection(x, *ws, nq, nkv, theta, positions=pos)
    assert np.max(np.abs(q - orc.apply_rope(x[:, perms[0]].reshape(N, nq, d), pos, theta))) < 1e-12, "selection q"
    assert np.max(np.abs(k - orc.apply_rope(x[:, perms[1]].reshape(N, nkv, d), pos, theta))) < 1e-12, "selection k"
    assert np.max(np.abs(v - x[:, perms[2]].reshape(N, nkv, d))) < 1e-15, "selection v"


def _brute_projection(x, w, heads, d):
    N, C = x.shape
    out = np.zeros((N, heads, d))
    for n in range(N):
        for f in range(heads * d):
            out[n, f // d, f % d] = sum(x[n, c] * w[f, c] for c in range(C))
    return out


def pin_brute_force_at_position_zero(m):
    """At position 0 every angle is 0, so q and k are the plain projections;
    V is the plain projection at any position."""
    rng = np.random.default_rng(3)
    N, C, nq, nkv, d = 3, 5, 2, 1, 4
    x = rng.standard_normal((N, C))
    wq, wk, wv = _weights(rng, C, nq, nkv, d)
    q, k, v = m.qkv_rope_projection(x, wq, wk, wv, nq, nkv, 1e4, positions=np.zeros(N, dtype=np.int64))
    assert np.max(np.abs(q - _brute_projection(x, wq, nq, d))) < 1e-12, "brute q"
    assert np.max(np.abs(k - _brute_projection(x, wk, nkv, d))) < 1e-12, "brute k"
    _, _, v2 = m.qkv_rope_projection(x, wq, wk, wv, nq, nkv, 1e4, positions=np.array([7, 90, 1234]))
    assert np.max(np.abs(v2 - _brute_projection(x, wv, nkv, d))) < 1e-12, "brute v"


def pin_positions_source(m):
    """Explicit positions override the in-sequence index: shifting every
    position by s rotates each pair by s * inv_freq more."""
    rng = np.random.default_rng(4)
    N, C, nq, nkv, d, theta = 6, 8, 2, 1, 4, 100.0
    x = rng.standard_normal((N, C))
    wq, wk, wv = _weights(rng, C, nq, nkv, d)
    cu = np.array([0, 4, 6])
    a = m.qkv_rope_projection(x, wq, wk, wv, nq, nkv, theta, cu_seqlens=cu)
    b = m.qkv_rope_projection(x, wq, wk, wv, nq, nkv, theta, positions=np.array([0, 1, 2, 3, 0, 1]))
    for u, w in zip(a, b):
        assert np.max(np.abs(u - w)) < 1e-15, "in-sequence index"
    c = m.qkv_rope_projection(x, wq, wk, wv, nq, nkv, theta, positions=np.array([0, 1, 2, 3, 0, 1]) + 5)
    inv = theta ** (-np.arange(d // 2) * 2.0 / d)
    z0 = a[1][..., : d // 2] + 1j * a[1][..., d // 2:]
    z1 = c[1][..., : d // 2] + 1j * c[1][..., d // 2:]
    assert np.max(np.abs(z1 - z0 * np.exp(1j * 5 * inv))) < 1e-12, "shifted positions"


PINS = [pin_torch_linear, pin_selection_weights, pin_brute_force_at_position_zero, pin_positions_source]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_projection_pins(pin):
    pin(orc)


def test_operand_rounding_rounds_once_to_bf16():
    rng = np.random.default_rng(5)
    x = orc.round_to_bf16(rng.standard_normal((7, 16)))
    wq, wk, wv = (orc.round_to_bf16(w) for w in _weights(rng, 16, 2, 1, 8))
    ex = orc.qkv_rope_projection(x, wq, wk, wv, 2, 1, 1e4)
    rd = orc.qkv_rope_projection(x, wq, wk, wv, 2, 1, 1e4, operand_rounding=True)
    for a, b in zip(ex, rd):
        assert np.array_equal(orc.round_to_bf16(b), b)  # bf16 values
        assert np.all(np.abs(a - b) <= 2.0 ** -8 * np.abs(a) + 1e-30)  # within one rounding


MUTATIONS = {
    "weight_not_transposed": ("yq = np.matmul(x, w_q.T)", "yq = np.matmul(x, w_q)"),
    "head_split_transposed": ("np.matmul(x, w_k.T).reshape(N, n_kv_heads, d)",
                              "np.matmul(x, w_k.T).reshape(N, d, n_kv_heads).transpose(0, 2, 1)"),
    "v_rotated": ("v = round_to_bf16(yv) if operand_rounding else yv",
                  "v = rope(yv)"),
    "k_not_rotated": ("k = rope(yk)", "k = yk"),
    "positions_ignored": ("pos = np.asarray(positions, dtype=np.int64).reshape(-1)\n    elif",
                          "pos = np.arange(N)\n    elif"),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_projection_mistakes_are_caught(name):
    src = open(os.path.join(ROOT, "oracle", "gqa_oracle.py")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, name
    spec = importlib.util.spec_from_loader("_oracle_proj_mut", loader=None)
    m = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), "_oracle_proj_mut", "exec"), m.__dict__)
    failed = 0
    for pin in PINS:
        try:
            pin(m)
        except (AssertionError, ValueError):
            failed += 1
    assert failed >= 1, f"mutation {name} not caught"
