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

Planted mistakes in the model (the halves combined without their weights, a
redo without the rescale) are shown to fail the comparison. CPU only."""
import math

import numpy as np
import pytest

import oracle.gqa_oracle as orc

BM = BN = 128
HALF = BN // 2


def kernel_model(q, k, v, cu, nq, nkv, theta, causal, plant=None, stats=None, shared=False):
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
                orow = (wgt[:, :, None] * o).sum(axis=0) / lrow[:, None]
                for r in np.nonzero(valid)[0]:
                    out[a + tok[r], h[r]] = orow[r]
                    lse[h[r], a + tok[r]] = (mrow[r] * s + math.log2(lrow[r])) * math.log(2.0)
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
