"""Pins for the float64 oracle: values and properties fixed by the pages and by
mathematics, each independent of the oracle's own code. A plausible mistake in
the oracle (dropped term, wrong sign or index, transposed operand, wrong head
map, wrong scale, off-by-one mask) fails at least one of these; the planted
mistakes in ``test_oracle_mutations.py`` show which.
"""
import math

import numpy as np
import pytest

import oracle.gqa_oracle as orc
from transformer_attention_gqa_b200 import workloads as wl


def _rng(seed=0):
    return np.random.default_rng(seed)


def _bf16(x):
    return wl.to_bf16_values(np.asarray(x, np.float32)).astype(np.float64)


def _seq_positions(cu):
    return np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)])


# ---------------------------------------------------------------------------
# bf16 rounding vs a library routine (torch's RN-even fp32 -> bf16)
# ---------------------------------------------------------------------------

def pin_bf16_rounding(m=orc):
    r = _rng(1)
    x = np.concatenate([
        r.standard_normal(20000).astype(np.float32),
        (r.standard_normal(2000) * 1e30).astype(np.float32),
        (r.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormal range
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 3.0e38, -3.4e38, 0.0, -0.0], np.float32),
    ])
    # exact ties of bf16 built from fp32 bit patterns: low 16 bits = 0x8000
    bits = (r.integers(0, 2 ** 14, 2000, dtype=np.uint32) << 16 | np.uint32(0x8000)) + np.uint32(0x3F000000)
    ties = bits.view(np.float32)
    x = np.concatenate([x, ties])
    lib = wl.to_bf16_values(x).astype(np.float64)
    got = m.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, lib, equal_nan=True)


def test_bf16_rounding_matches_torch():
    pin_bf16_rounding()


# ---------------------------------------------------------------------------
# RoPE pins
# ---------------------------------------------------------------------------

def pin_inv_freq(golden, m=orc):
    for case in golden["rope_inv_freq"]:
        got = m.rope_inv_freq(case["head_dim"], case["theta"])
        assert np.allclose(got, case["inv_freq"], rtol=1e-14, atol=0)


def test_inv_freq_worked_values(golden):
    pin_inv_freq(golden)


def pin_rope_worked_example(golden, m=orc):
    for case in golden["rope_rotation"]:
        x = np.array(case["x"], np.float64).reshape(1, 1, -1)
        got = m.apply_rope(x, [case["position"]], case["theta"], operand_rounding=False)[0, 0]
        exp = []
        for f1, a1, c1, f2, a2, c2 in case["expected_terms"]:
            exp.append(c1 * getattr(math, f1)(a1) + c2 * getattr(math, f2)(a2))
        assert np.allclose(got, exp, rtol=0, atol=1e-14)


def test_rope_worked_example(golden):
    pin_rope_worked_example(golden)


def pin_rope_norm(m=orc):
    r = _rng(2)
    for d in (2, 8, 64, 128):
        x = r.standard_normal((50, 3, d))
        pos = r.integers(0, 100000, 50)
        y = m.apply_rope(x, pos, 500000.0)
        # each (i, i + d/2) pair is rotated: its 2-norm is kept, so is the whole norm
        h = d // 2
        pn_x = x[..., :h] ** 2 + x[..., h:] ** 2
        pn_y = y[..., :h] ** 2 + y[..., h:] ** 2
        assert np.allclose(pn_x, pn_y, rtol=1e-12, atol=1e-12)
        assert np.allclose(np.linalg.norm(x, axis=-1), np.linalg.norm(y, axis=-1), rtol=1e-12)


def test_rope_preserves_pair_norms():
    pin_rope_norm()


def pin_rope_identity_at_zero(m=orc):
    r = _rng(3)
    x = _bf16(r.standard_normal((7, 2, 64)))
    for rounding in (False, True):
        y = m.apply_rope(x, np.zeros(7, np.int64), 10000.0, operand_rounding=rounding)
        assert np.array_equal(y, x)


def test_rope_identity_at_position_zero():
    pin_rope_identity_at_zero()


def pin_rope_relative(m=orc):
    """rope(q, a) . rope(k, b) depends only on a - b."""
    r = _rng(4)
    d = 64
    q = r.standard_normal((20, 1, d))
    k = r.standard_normal((20, 1, d))
    a = r.integers(0, 5000, 20)
    b = r.integers(0, 5000, 20)
    c = r.integers(-3000, 3000, 20)
    lhs = np.sum(m.apply_rope(q, a, 1e4) * m.apply_rope(k, b, 1e4), axis=-1)
    rhs = np.sum(m.apply_rope(q, a + c, 1e4) * m.apply_rope(k, b + c, 1e4), axis=-1)
    assert np.allclose(lhs, rhs, rtol=1e-9, atol=1e-9)
    # and it does depend on a - b (not a constant)
    rhs2 = np.sum(m.apply_rope(q, a + 1, 1e4) * m.apply_rope(k, b, 1e4), axis=-1)
    assert not np.allclose(lhs, rhs2, rtol=1e-6, atol=1e-6)


def test_rope_relative_position():
    pin_rope_relative()


def pin_rope_basis_closed_form(m=orc):
    """rope(e_i, p): component i = cos(p*w_i), component i+d/2 = sin(p*w_i),
    nothing else; for i = 0 the angle is exactly p radians."""
    d = 16
    theta = 10000.0
    for p in (0, 1, 7, 1234):
        for i in range(d // 2):
            e = np.zeros((1, 1, d))
            e[0, 0, i] = 1.0
            y = m.apply_rope(e, [p], theta)[0, 0]
            w = theta ** (-(2.0 * i) / d) if i else 1.0
            exp = np.zeros(d)
            exp[i] = math.cos(p * w)
            exp[i + d // 2] = math.sin(p * w)
            assert np.allclose(y, exp, atol=1e-13)
            # the second half maps to (-sin, cos)
            e2 = np.zeros((1, 1, d))
            e2[0, 0, i + d // 2] = 1.0
            y2 = m.apply_rope(e2, [p], theta)[0, 0]
            exp2 = np.zeros(d)
            exp2[i] = -math.sin(p * w)
            exp2[i + d // 2] = math.cos(p * w)
            assert np.allclose(y2, exp2, atol=1e-13)


def test_rope_basis_closed_form():
    pin_rope_basis_closed_form()


def _table(pos, d, theta):
    """fp32 cos/sin of the float64 angle pos * theta^(-2i/d), duplicated over
    the two halves (the RoPE page's table), written out here on its own."""
    i = np.arange(d // 2, dtype=np.float64)
    ang = np.asarray(pos, np.float64)[:, None] * theta ** (-2.0 * i / d)
    ang = np.concatenate([ang, ang], axis=-1)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def pin_rope_operand_rounding(m=orc):
    """Rounded rotation: bf16-representable and within the error of its
    roundings of the exact rotation: cos/sin and the two products each to
    bf16 (unit roundoff u = 2^-8), the sum to bf16 (u of the result), plus
    the fp32 table's error."""
    r = _rng(5)
    x = _bf16(r.standard_normal((300, 2, 128)))
    pos = r.integers(0, 8192, 300)
    ex = m.apply_rope(x, pos, 5e5, operand_rounding=False)
    ro = m.apply_rope(x, pos, 5e5, operand_rounding=True)
    assert np.array_equal(ro, _bf16(ro))
    c, s = (t.astype(np.float64)[:, None, :] for t in _table(pos, 128, 5e5))
    u = 2.0 ** -8
    y = orc.rotate_half(x)
    err = np.abs(ro - ex)
    bound = u * np.abs(ex) + 2.1 * u * (np.abs(x * c) + np.abs(y * s)) + 4e-7 * (np.abs(x) + np.abs(y))
    assert np.all(err <= bound + 1e-30)


def pin_rope_bf16_matches_torch(m=orc):
    """The rounded rotation is, bit for bit, the RoPE page's apply_rope run by
    torch on bf16 CPU tensors (cos and sin cast to bf16, x * cos +
    rotate_half(x) * sin in bf16): inputs over a wide range of scales, with
    cancelling pairs, zeros and position 0."""
    import torch

    r = _rng(6)
    T, H, d, theta = 400, 3, 64, 5e5
    x = r.standard_normal((T, H, d)) * np.exp2(r.integers(-20, 21, (T, H, d)))
    x[:5] = 0.0
    x[5:40, :, d // 2:] = x[5:40, :, : d // 2]  # pairs (v, v): x*cos and x*sin cancel near 45 degrees
    x = _bf16(x)
    pos = r.integers(0, 100000, T)
    pos[:10] = 0
    cos, sin = (torch.from_numpy(t)[:, None, :].to(torch.bfloat16) for t in _table(pos, d, theta))
    xt = torch.from_numpy(x).to(torch.bfloat16)
    rot = torch.cat((-xt[..., d // 2:], xt[..., : d // 2]), dim=-1)
    ref = (xt * cos + rot * sin).double().numpy()
    got = m.apply_rope(x, pos, theta, operand_rounding=True)
    assert np.array_equal(got, ref)


def test_rope_bf16_matches_torch():
    pin_rope_bf16_matches_torch()


def test_rope_operand_rounding_bound():
    pin_rope_operand_rounding()


# ---------------------------------------------------------------------------
# Attention pins
# ---------------------------------------------------------------------------

def pin_worked_attention(golden, m=orc):
    c = golden["attention"][0]
    q = np.array(c["q"]).reshape(2, 1, 2)
    k = np.array(c["k"]).reshape(2, 1, 2)
    v = np.array(c["v"]).reshape(2, 1, 2)
    out, lse = m.gqa_rope_attention(q, k, v, [0, 2], 1, 1, 1e4, positions=np.zeros(2, np.int64),
                                    operand_rounding=False)
    assert np.allclose(out[:, 0, :], c["out"], atol=1e-12)
    assert np.allclose(lse[0], c["lse"], atol=1e-12)


def test_worked_attention_example(golden):
    pin_worked_attention(golden)


def pin_first_row(m=orc):
    """Row 0 of every causal sequence (and T=1) sees only key 0: out = v_0 of
    its KV head, lse = s_00."""
    r = _rng(6)
    lens = [1, 5, 9]
    N = sum(lens)
    hq, hk, d = 6, 2, 16
    q, k, v = r.standard_normal((N, hq, d)), r.standard_normal((N, hk, d)), r.standard_normal((N, hk, d))
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, lse = m.gqa_rope_attention(q, k, v, cu, hq, hk, 1e4, operand_rounding=False)
    for a in cu[:-1]:
        for h in range(hq):
            g = h // (hq // hk)
            assert np.allclose(out[a, h], v[a, g], atol=1e-13)
            # position 0: RoPE is the identity
            assert abs(lse[h, a] - float(q[a, h] @ k[a, g]) / math.sqrt(d)) < 1e-12


def test_first_row_returns_v0():
    pin_first_row()


def pin_identical_keys(m=orc):
    """All-zero positions make RoPE the identity; identical keys then give
    equal scores, so causal row r is the mean of v_0..v_r and
    lse_r = s + ln(r+1). q = 0 gives the same prefix mean for any K."""
    r = _rng(7)
    T, hq, hk, d = 12, 4, 2, 8
    q = r.standard_normal((T, hq, d))
    k = np.repeat(r.standard_normal((1, hk, d)), T, axis=0)
    v = r.standard_normal((T, hk, d))
    out, lse = m.gqa_rope_attention(q, k, v, [0, T], hq, hk, 1e4, positions=np.zeros(T, np.int64),
                                    operand_rounding=False)
    for h in range(hq):
        g = h // 2
        for i in range(T):
            assert np.allclose(out[i, h], v[: i + 1, g].mean(axis=0), atol=1e-13)
            s = float(q[i, h] @ k[0, g]) / math.sqrt(d)
            assert abs(lse[h, i] - (s + math.log(i + 1))) < 1e-12
    q0 = np.zeros_like(q)
    k2 = r.standard_normal((T, hk, d))
    out, lse = m.gqa_rope_attention(q0, k2, v, [0, T], hq, hk, 1e4, operand_rounding=False)
    for h in range(hq):
        for i in range(T):
            assert np.allclose(out[i, h], v[: i + 1, h // 2].mean(axis=0), atol=1e-13)
            assert abs(lse[h, i] - math.log(i + 1)) < 1e-12


def test_identical_keys_prefix_mean():
    pin_identical_keys()


def pin_gqa_equals_mha(m=orc):
    """GQA == MHA on K/V replicated with repeat_interleave; it differs from
    plain repeat (tile) when G > 1 and n_kv > 1; n_kv == n_q is MHA."""
    r = _rng(8)
    T, hq, hk, d = 10, 6, 2, 8
    q = r.standard_normal((T, hq, d))
    k = r.standard_normal((T, hk, d))
    v = r.standard_normal((T, hk, d))
    o1, l1 = m.gqa_rope_attention(q, k, v, [0, T], hq, hk, 1e4, operand_rounding=False)
    kr = np.stack([k[:, h // 3] for h in range(hq)], axis=1)
    vr = np.stack([v[:, h // 3] for h in range(hq)], axis=1)
    o2, l2 = m.gqa_rope_attention(q, kr, vr, [0, T], hq, hq, 1e4, operand_rounding=False)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)
    kt = np.concatenate([k] * 3, axis=1)  # "repeat": head h reads kv head h % n_kv
    vt = np.concatenate([v] * 3, axis=1)
    o3, _ = m.gqa_rope_attention(q, kt, vt, [0, T], hq, hq, 1e4, operand_rounding=False)
    assert not np.allclose(o1, o3, atol=1e-3)


def test_gqa_equals_mha_repeat_interleave():
    pin_gqa_equals_mha()


def pin_brute_force(m=orc):
    r = _rng(9)
    for lens, hq, hk, d, causal in [([5], 2, 1, 4, True), ([3, 6], 4, 2, 6, True), ([4, 1, 7], 3, 3, 8, False)]:
        N = sum(lens)
        cu = np.concatenate([[0], np.cumsum(lens)])
        q, k, v = r.standard_normal((N, hq, d)), r.standard_normal((N, hk, d)), r.standard_normal((N, hk, d))
        pos = r.integers(0, 50, N)
        for p in (None, pos):
            ob, lb = orc.brute_force_attention(q, k, v, cu, hq, hk, 1e4, positions=p, causal=causal)
            o, l = m.gqa_rope_attention(q, k, v, cu, hq, hk, 1e4, positions=p, causal=causal, operand_rounding=False)
            assert np.allclose(o, ob, atol=1e-12, rtol=0)
            assert np.allclose(l, lb, atol=1e-12, rtol=0)


def test_brute_force_agreement():
    pin_brute_force()


def pin_torch_sdpa(m=orc):
    """Independent library: torch CPU float64 SDPA with enable_gqa on the
    oracle's own rotated Q/K; LSE against scipy's logsumexp of torch scores."""
    import torch
    import torch.nn.functional as F
    from scipy.special import logsumexp

    r = _rng(10)
    for T, hq, hk, d, theta, causal in [(64, 8, 2, 32, 1e4, True), (48, 6, 3, 64, 5e5, False), (33, 7, 1, 16, 1e6, True)]:
        q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d))
        o, l = m.gqa_rope_attention(q, k, v, [0, T], hq, hk, theta, causal=causal, operand_rounding=False)
        pos = np.arange(T)
        qr = torch.from_numpy(m.apply_rope(q, pos, theta)).permute(1, 0, 2)[None]
        kr = torch.from_numpy(m.apply_rope(k, pos, theta)).permute(1, 0, 2)[None]
        vt = torch.from_numpy(v).permute(1, 0, 2)[None]
        ot = F.scaled_dot_product_attention(qr, kr, vt, is_causal=causal, enable_gqa=True)[0].permute(1, 0, 2).numpy()
        assert np.allclose(o, ot, atol=1e-10, rtol=0)
        kk = torch.repeat_interleave(kr, hq // hk, dim=1)
        sc = (qr @ kk.transpose(-1, -2))[0].numpy() / math.sqrt(d)
        if causal:
            sc = np.where(np.tril(np.ones((T, T), bool))[None], sc, -np.inf)
        assert np.allclose(l, logsumexp(sc, axis=-1), atol=1e-10, rtol=0)


def test_torch_sdpa_cross_check():
    pin_torch_sdpa()


def pin_varlen(m=orc):
    """A packed batch equals each sequence run alone (positions restart); a
    shuffled sequence order permutes the outputs."""
    r = _rng(11)
    lens = [7, 1, 12, 4]
    hq, hk, d = 4, 2, 8
    seqs = [(r.standard_normal((L, hq, d)), r.standard_normal((L, hk, d)), r.standard_normal((L, hk, d))) for L in lens]

    def pack(order):
        q = np.concatenate([seqs[i][0] for i in order])
        k = np.concatenate([seqs[i][1] for i in order])
        v = np.concatenate([seqs[i][2] for i in order])
        cu = np.concatenate([[0], np.cumsum([lens[i] for i in order])])
        return q, k, v, cu

    q, k, v, cu = pack([0, 1, 2, 3])
    o, l = m.gqa_rope_attention(q, k, v, cu, hq, hk, 1e4, operand_rounding=False)
    for i, L in enumerate(lens):
        oi, li = m.gqa_rope_attention(*seqs[i], [0, L], hq, hk, 1e4, operand_rounding=False)
        assert np.allclose(o[cu[i]:cu[i + 1]], oi, atol=1e-13)
        assert np.allclose(l[:, cu[i]:cu[i + 1]], li, atol=1e-13)
    order = [2, 0, 3, 1]
    q2, k2, v2, cu2 = pack(order)
    o2, _ = m.gqa_rope_attention(q2, k2, v2, cu2, hq, hk, 1e4, operand_rounding=False)
    for j, i in enumerate(order):
        assert np.allclose(o2[cu2[j]:cu2[j + 1]], o[cu[i]:cu[i + 1]], atol=1e-13)


def test_varlen_packing():
    pin_varlen()


def pin_causal_last_row(m=orc):
    """The last causal row sees every key: it equals the non-causal last row;
    earlier rows differ."""
    r = _rng(12)
    T, hq, hk, d = 16, 2, 1, 8
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d))
    oc, lc = m.gqa_rope_attention(q, k, v, [0, T], hq, hk, 1e4, causal=True, operand_rounding=False)
    on, ln = m.gqa_rope_attention(q, k, v, [0, T], hq, hk, 1e4, causal=False, operand_rounding=False)
    assert np.allclose(oc[-1], on[-1], atol=1e-13) and np.allclose(lc[:, -1], ln[:, -1], atol=1e-13)
    assert not np.allclose(oc[0], on[0], atol=1e-6)


def test_causal_last_row():
    pin_causal_last_row()


def pin_query_rows_subset(m=orc):
    r = _rng(13)
    T, hq, hk, d = 40, 4, 2, 16
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hk, d)), r.standard_normal((T, hk, d))
    o, l = m.gqa_rope_attention(q, k, v, [0, 25, 40], hq, hk, 1e4)
    rows = [0, 3, 24, 25, 39]
    o2, l2 = m.gqa_rope_attention(q, k, v, [0, 25, 40], hq, hk, 1e4, query_rows=rows, row_block=2)
    assert np.allclose(o2[rows], o[rows], atol=1e-13) and np.allclose(l2[:, rows], l[:, rows], atol=1e-13)


def test_query_rows_subset_matches_full():
    pin_query_rows_subset()


def test_workload_shapes():
    w = wl.WORKLOADS["varlen"]
    assert list(w.seq_lens) == [3494, 2632, 2125, 1152, 1305, 229, 367, 130, 770, 3343, 837]
    assert w.total_tokens == 16384
    assert abs(wl.WORKLOADS["llama8b"].flops() - 549.755813888e9) < 1e3
    inp = wl.make_inputs(wl.WORKLOADS["tiny"])
    assert inp.q.shape == (128, 4, 32) and inp.k.shape == (128, 2, 32)
    assert np.array_equal(inp.q, wl.to_bf16_values(inp.q))
