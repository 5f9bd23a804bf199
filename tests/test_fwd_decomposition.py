"""The forward kernel's online softmax, restated in numpy with its exact
update rules and checked against the oracle (``gqa_rope_attention``,
float64, exact rotation) on the CPU:

* work items = (sequence, packed q-tile of tq = 128 / G tokens x the G query
  heads of one KV head); an item visits KV tiles 0 .. ceil(t_end / 128) - 1
  with t_end = min(t0 + tq, L) for causal attention, else L;
* every 128-key tile is split into two column halves (keys [0, 64) and
  [64, 128) of the tile), one thread each; at d <= 64 each half keeps its
  own running max m_h, sum l_h and partial output O_h, so the two halves
  never exchange anything; at d = 128 (``shared``) the halves share one
  running max (their tile maxima exchanged once per tile) and one O;
* per half and tile: keys past the row's last visible key get -inf; the
  first tile sets m_h to the half's max; later tiles use the running max and
  redo the tile with the new max (O_h and l_h scaled by 2^((m_h - m') s))
  only when the tile's max exceeds m_h by more than 8 / s (2^8 in p);
  a half that has seen no visible key keeps m_h = -inf and bias 0, so its
  p are 0;
* the epilogue: m = max(m_a, m_b), a_h = 2^((m_h - m) s) (0 for m_h = -inf),
  out = (a_a O_a + a_b O_b) / (a_a l_a + a_b l_b),
  lse = (m s + log2(a_a l_a + a_b l_b)) ln 2, with s = log2(e) / sqrt(d)
  (with a shared max: a_a = a_b = 1).

The masked form of the kernel adds mask[query, key] * sqrt(d) to every raw
score of a visible key before the causal / length bound; a row that sees no
key at all then gets out = 0 and lse = -inf. It is checked against
``gqa_rope_attention_masked`` with masks that have holes, fully masked rows
and fully masked first tiles.

Planted mistakes in the model (the halves combined without their weights, a
redo without the rescale) are shown to fail the comparison. CPU only."""
import math

import numpy as np
import pytest

import oracle.gqa_oracle as orc

BM = BN = 128
HALF = BN // 2


def kernel_model(q, k, v, cu, nq, nkv, theta, causal, plant=None, stats=None, shared=False, mask=None):
    N, _, d = q.shape
    G = nq // nkv
    tq = BM // G
    pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)])
    qr, kr = orc.apply_rope(q, pos, theta), orc.apply_rope(k, pos, theta)
    s = math.log2(math.e) / math.sqrt(d)
    thr = 8.0 / s
    out = np.full((N, nq, d), np.nan)
    lse = np.full((nq, N), np.nan)
    for si in range(len(cu) - 1):
        a, L = int(cu[si]), int(cu[si + 1] - cu[si])
        for qi in range((L + tq - 1) // tq):
            t0 = qi * tq
            t_end = min(t0 + tq, L) if causal else L
            ntiles = (t_end + BN - 1) // BN
            for kvh in range(nkv):
                rows = np.arange(tq * G)
                tok = t0 + rows // G
                h = kvh * G + rows % G
                valid = tok < L
                tokc = np.minimum(tok, L - 1)
                last_key = tok if causal else np.full_like(tok, L - 1)
                qrow = qr[a + tokc, h]                       # [R, d]
                m = np.full((2, rows.size), -np.inf)
                l = np.zeros((2, rows.size))
                o = np.zeros((2, rows.size, d))
                for j in range(ntiles):
                    sc, vt = [], []
                    for hf in range(2):
                        keys = j * BN + hf * HALF + np.arange(HALF)
                        kc = np.minimum(keys, L - 1)         # keys past L: any finite row (masked below)
                        t = qrow @ kr[a + kc, kvh].T         # [R, 64]
                        if mask is not None:                 # keys past L read 0 (hidden below)
                            mv = np.where(keys[None, :] < L, mask[np.minimum(tokc, mask.shape[0] - 1)][:, kc], 0.0)
                            t = t + mv * math.sqrt(d)
                        sc.append(np.where(keys[None, :] > last_key[:, None], -np.inf, t))
                        vt.append(v[a + kc, kvh])            # [64, d]
                    mh = [x.max(axis=1) for x in sc]
                    if shared:                               # both halves see both tile maxima
                        mh = [np.maximum(mh[0], mh[1])] * 2
                    for hf in range(2):
                        if j == 0:
                            m[hf] = mh[hf]
                        else:
                            need = mh[hf] > m[hf] + thr
                            if stats is not None:
                                stats["redo"] += int(need.sum())
                            with np.errstate(invalid="ignore"):
                                alpha = np.where(need, np.exp2((m[hf] - mh[hf]) * s), 1.0)
                            if plant != "redo without rescale":
                                o[hf] *= alpha[:, None]
                                l[hf] *= alpha
                            m[hf] = np.where(need, mh[hf], m[hf])
                        if stats is not None:
                            stats["neg_inf_half"] += int((valid & (m[hf] == -np.inf)).sum())
                        bias = np.where(m[hf] == -np.inf, 0.0, -m[hf] * s)
                        p = np.exp2(sc[hf] * s + bias[:, None])
                        l[hf] += p.sum(axis=1)
                        o[hf] += p @ vt[hf]
                if shared:
                    assert np.array_equal(m[0], m[1])
                mrow = m.max(axis=0)
                if plant == "halves unweighted":
                    wgt = np.ones((2, rows.size))
                else:
                    with np.errstate(invalid="ignore"):
                        wgt = np.where(m == -np.inf, 0.0, np.exp2((m - mrow[None, :]) * s))
                lrow = (wgt * l).sum(axis=0)
                seen = mrow > -np.inf                        # a row that saw no key: out 0, lse -inf
                with np.errstate(invalid="ignore", divide="ignore"):
                    orow = np.where(seen[:, None], (wgt[:, :, None] * o).sum(axis=0) / lrow[:, None], 0.0)
                for r in np.nonzero(valid)[0]:
                    out[a + tok[r], h[r]] = orow[r]
                    lse[h[r], a + tok[r]] = (mrow[r] * s + math.log2(lrow[r])) * math.log(2.0) if seen[r] else -np.inf
    return out, lse


def _inputs(lens, nq, nkv, d, seed, k_ramp=0.0):
    rng = np.random.default_rng(seed)
    N = sum(lens)
    q = rng.standard_normal((N, nq, d))
    k = rng.standard_normal((N, nkv, d))
    v = rng.standard_normal((N, nkv, d))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    if k_ramp:
        # scores that grow along the keys, so later tiles raise the running max
        for i in range(len(lens)):
            t = np.arange(lens[i])
            k[cu[i]:cu[i + 1]] += k_ramp * (t / max(lens[i], 1))[:, None, None] * np.sign(q[cu[i]:cu[i + 1], :nkv])
    return q, k, v, cu


CASES = [
    # lens, nq, nkv, d, causal
    ([1, 70, 130, 257], 8, 2, 32, True),     # G = 4 (tq = 32): ragged tails, tiles with one visible half
    ([5, 200], 6, 2, 16, True),              # G = 3 (tq = 42, two padding rows per tile)
    ([90, 300], 4, 4, 16, False),            # G = 1, full attention: keys past L masked per half
    ([129], 14, 2, 16, True),                # G = 7 (tq = 18)
]


@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("lens,nq,nkv,d,causal", CASES)
def test_half_softmax_matches_oracle(lens, nq, nkv, d, causal, shared):
    q, k, v, cu = _inputs(lens, nq, nkv, d, seed=sum(lens) + nq)
    stats = {"redo": 0, "neg_inf_half": 0}
    out, lse = kernel_model(q, k, v, cu, nq, nkv, 1e4, causal, stats=stats, shared=shared)
    ref_out, ref_lse = orc.gqa_rope_attention(q, k, v, cu, nq, nkv, 1e4, causal=causal, operand_rounding=False)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13, atol=1e-13)
    if causal and not shared:
        # rows below token 64 see no key of the first tile's upper half
        assert stats["neg_inf_half"] > 0


@pytest.mark.parametrize("shared", [False, True])
def test_redo_path_taken_and_exact(shared):
    q, k, v, cu = _inputs([600, 300], 8, 2, 32, seed=7, k_ramp=12.0)
    stats = {"redo": 0, "neg_inf_half": 0}
    out, lse = kernel_model(q, k, v, cu, 8, 2, 1e4, True, stats=stats, shared=shared)
    ref_out, ref_lse = orc.gqa_rope_attention(q, k, v, cu, 8, 2, 1e4, operand_rounding=False)
    assert stats["redo"] > 0
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("plant,k_ramp", [("halves unweighted", 0.0), ("redo without rescale", 12.0)])
def test_planted_mistakes_fail(plant, k_ramp):
    q, k, v, cu = _inputs([600, 300], 8, 2, 32, seed=7, k_ramp=k_ramp)
    out, lse = kernel_model(q, k, v, cu, 8, 2, 1e4, True, plant=plant)
    ref_out, ref_lse = orc.gqa_rope_attention(q, k, v, cu, 8, 2, 1e4, operand_rounding=False)
    err = max(np.nanmax(np.abs(out - ref_out)), np.nanmax(np.abs(lse - ref_lse)))
    assert not err < 1e-3


def _masked_case(seed, lens, nq, nkv, d, causal, holes, dead_rows=(), dead_prefix=0):
    rng = np.random.default_rng(seed)
    N = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v = (rng.standard_normal((N, h, d)) for h in (nq, nkv, nkv))
    Lm = max(lens)
    mask = rng.standard_normal((Lm, Lm)) * 2.0
    mask[rng.random((Lm, Lm)) < holes] = -np.inf
    for i in dead_rows:
        mask[i, :] = -np.inf
    if dead_prefix:
        mask[:, :dead_prefix] = -np.inf  # every row's first keys hidden
    return q, k, v, cu, mask


MASKED_CASES = {
    "holes_causal_g4": dict(seed=1, lens=(300,), nq=8, nkv=2, d=32, causal=True, holes=0.3),
    "holes_full_varlen_g3": dict(seed=2, lens=(150, 1, 40), nq=6, nkv=2, d=32, causal=False, holes=0.5),
    "dead_rows": dict(seed=3, lens=(140,), nq=4, nkv=4, d=32, causal=True, holes=0.2, dead_rows=(0, 5, 139)),
    "dead_first_tile": dict(seed=4, lens=(260,), nq=2, nkv=1, d=64, causal=False, holes=0.1, dead_prefix=200),
}


@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("name", sorted(MASKED_CASES))
def test_masked_form_matches_oracle(name, shared):
    c = dict(MASKED_CASES[name])
    q, k, v, cu, mask = _masked_case(**c)
    ref_o, ref_l = orc.gqa_rope_attention_masked(q, k, v, cu, c["nq"], c["nkv"], 1e4, mask, causal=c["causal"],
                                                 operand_rounding=False)
    got_o, got_l = kernel_model(q, k, v, cu, c["nq"], c["nkv"], 1e4, c["causal"], shared=shared, mask=mask)
    assert np.max(np.abs(got_o - ref_o)) < 1e-10
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l))
    assert np.max(np.abs(got_l[fin] - ref_l[fin])) < 1e-10
    if c.get("dead_rows"):
        assert (~fin).any()
