"""Pins of the oracle's decoding step (CPU). The step is the last causal row
of the forward ("Attention from Scratch", the KV-cache paragraph of section
"Attention, the math: Grouped-Query Attention with RoPE'd Q/K"), so it is
checked against the separately pinned forward, against brute-force loops, and
against the closed form of a cache-less first token."""
import math

import numpy as np
import pytest

import oracle.gqa_oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _bf16(x):
    return orc.round_to_bf16(np.asarray(x, dtype=np.float64))


def _sequences(rng, lens, nq, nkv, d):
    """Raw per-token q, k, v of B sequences of lengths p_b + 1 (bf16 values)."""
    return [(_bf16(rng.standard_normal((p + 1, nq, d))), _bf16(rng.standard_normal((p + 1, nkv, d))),
             _bf16(rng.standard_normal((p + 1, nkv, d)))) for p in lens]


def _decode_inputs(seqs, lens, nkv, d, theta, rounding, max_len):
    B = len(lens)
    nq = seqs[0][0].shape[1]
    q = np.stack([s[0][-1] for s in seqs])
    k_new = np.stack([s[1][-1] for s in seqs])
    v_new = np.stack([s[2][-1] for s in seqs])
    kc = np.full((B, max_len, nkv, d), np.nan)  # rows >= p must not be read
    vc = np.full((B, max_len, nkv, d), np.nan)
    for b, p in enumerate(lens):
        kc[b, :p] = orc.apply_rope(seqs[b][1][:p], np.arange(p), theta, rounding)
        vc[b, :p] = seqs[b][2][:p]
    return q, k_new, v_new, kc, vc


@pytest.mark.parametrize("rounding", [True, False])
def test_decode_is_last_row_of_forward(rounding):
    rng = np.random.default_rng(11)
    lens = [5, 0, 17, 1]
    nq, nkv, d, theta = 6, 2, 16, 1e4
    seqs = _sequences(rng, lens, nq, nkv, d)
    q, kn, vn, kc, vc = _decode_inputs(seqs, lens, nkv, d, theta, rounding, max_len=20)
    out, lse, k_row, v_row = orc.gqa_rope_decode(q, kn, vn, kc, vc, lens, nq, nkv, theta, operand_rounding=rounding)
    for b, p in enumerate(lens):
        qs, ks, vs = seqs[b]
        fo, fl = orc.gqa_rope_attention(qs, ks, vs, [0, p + 1], nq, nkv, theta, operand_rounding=rounding)
        np.testing.assert_allclose(out[b], fo[p], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, b], fl[:, p], rtol=0, atol=1e-12)
        np.testing.assert_array_equal(k_row[b], orc.apply_rope(ks[p:p + 1], [p], theta, rounding)[0])
        np.testing.assert_array_equal(v_row[b], vs[p])


def test_decode_matches_brute_force_loops():
    rng = np.random.default_rng(12)
    lens = [3, 6]
    nq, nkv, d, theta = 4, 2, 8, 100.0
    seqs = _sequences(rng, lens, nq, nkv, d)
    q, kn, vn, kc, vc = _decode_inputs(seqs, lens, nkv, d, theta, False, max_len=8)
    out, lse, _, _ = orc.gqa_rope_decode(q, kn, vn, kc, vc, lens, nq, nkv, theta, operand_rounding=False)
    for b, p in enumerate(lens):
        qs, ks, vs = seqs[b]
        bo, bl = orc.brute_force_attention(qs, ks, vs, [0, p + 1], nq, nkv, theta)
        np.testing.assert_allclose(out[b], bo[p], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, b], bl[:, p], rtol=0, atol=1e-12)


def test_first_token_closed_form():
    """Empty cache: position 0 rotates nothing, the only key is the token's
    own, so out = v_new of the head's KV group and lse = q.k / sqrt(d)."""
    rng = np.random.default_rng(13)
    B, nq, nkv, d = 3, 8, 2, 32
    q = _bf16(rng.standard_normal((B, nq, d)))
    kn = _bf16(rng.standard_normal((B, nkv, d)))
    vn = _bf16(rng.standard_normal((B, nkv, d)))
    kc = np.full((B, 4, nkv, d), np.nan)
    out, lse, k_row, _ = orc.gqa_rope_decode(q, kn, vn, kc, kc, [0] * B, nq, nkv, 5e5)
    G = nq // nkv
    for b in range(B):
        for h in range(nq):
            np.testing.assert_array_equal(out[b, h], vn[b, h // G])
            assert abs(lse[h, b] - float(q[b, h] @ kn[b, h // G]) / math.sqrt(d)) < 1e-12
    np.testing.assert_array_equal(k_row, kn)


def test_decode_rejects_positions_outside_the_cache():
    z = np.zeros((1, 2, 8))
    with pytest.raises(ValueError):
        orc.gqa_rope_decode(z, z[:, :1], z[:, :1], np.zeros((1, 4, 1, 8)), np.zeros((1, 4, 1, 8)), [4], 2, 1, 1e4)
