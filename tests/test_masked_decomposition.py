"""The masked attention kernel's algorithm, restated in numpy with its exact
update rules and checked against the oracle (``gqa_rope_attention_masked``,
float64, no rounding): per packed q-tile (tq = 128 / G tokens x G heads) and
128-key tile, the raw scores plus mask * sqrt(d), the causal / length bound
(columns past tok, or past L, hidden), the running max (O rescaled only when
the max grows from a finite value), exponent bias 0 while a row has seen no
visible key, and out = 0, lse = -inf for a row that never does. Cases include
masks with holes, fully masked rows, and rows whose first key tiles are fully
masked. CPU only."""
import math

import numpy as np
import pytest

import oracle.gqa_oracle as orc

BM = BN = 128


def kernel_model(q, k, v, cu, nq, nkv, theta, mask, causal):
    N, _, d = q.shape
    G = nq // nkv
    tq = BM // G
    pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)])
    qr, kr = orc.apply_rope(q, pos, theta), orc.apply_rope(k, pos, theta)
    sl2 = math.log2(math.e) / math.sqrt(d)
    out = np.zeros((N, nq, d))
    lse = np.full((nq, N), -np.inf)
    for s in range(len(cu) - 1):
        a, L = int(cu[s]), int(cu[s + 1] - cu[s])
        for qi in range((L + tq - 1) // tq):
            t0 = qi * tq
            t_end = min(t0 + tq, L) if causal else L
            nkv_tiles = (t_end + BN - 1) // BN
            for kvh in range(nkv):
                for r in range(tq * G):
                    tt, hin = divmod(r, G)
                    tok = t0 + tt
                    if tok >= L:
                        continue
                    h = kvh * G + hin
                    last_key = tok if causal else L - 1
                    m, l, o = -np.inf, 0.0, np.zeros(d)
                    for j in range(nkv_tiles):
                        keys = j * BN + np.arange(BN)
                        inb = keys < L
                        kk = np.clip(keys, 0, L - 1)
                        sc = kr[a + kk, kvh] @ qr[a + tok, h]
                        sc = sc + np.where(inb, mask[tok, kk], 0.0) * math.sqrt(d)
                        sc = np.where(keys - j * BN > last_key - j * BN, -np.inf, sc)
                        mx = sc.max()
                        m_new = max(m, mx)
                        if j > 0 and m != -np.inf and m_new > m:
                            alpha = 2.0 ** ((m - m_new) * sl2)
                            o *= alpha
                            l *= alpha
                        m = m_new
                        bias = 0.0 if m == -np.inf else -m * sl2
                        p = np.exp2(sc * sl2 + bias)
                        l += p.sum()
                        o = o + p @ np.where(inb[:, None], v[a + kk, kvh], 0.0)
                    if m != -np.inf and l > 0:
                        out[a + tok, h] = o / l
                        lse[h, a + tok] = (m * sl2 + math.log2(l)) * math.log(2.0)
    return out, lse


def _case(seed, lens, nq, nkv, d, causal, holes, dead_rows=(), dead_prefix=0):
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


CASES = {
    "holes_causal_g4": dict(seed=1, lens=(300,), nq=8, nkv=2, d=32, causal=True, holes=0.3),
    "holes_full_varlen_g3": dict(seed=2, lens=(150, 1, 40), nq=6, nkv=2, d=32, causal=False, holes=0.5),
    "dead_rows": dict(seed=3, lens=(140,), nq=4, nkv=4, d=32, causal=True, holes=0.2, dead_rows=(0, 5, 139)),
    "dead_first_tile": dict(seed=4, lens=(260,), nq=2, nkv=1, d=64, causal=False, holes=0.1, dead_prefix=200),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_masked_kernel_algorithm_reproduces_the_oracle(name):
    c = dict(CASES[name])
    q, k, v, cu, mask = _case(**c)
    ref_o, ref_l = orc.gqa_rope_attention_masked(q, k, v, cu, c["nq"], c["nkv"], 1e4, mask, causal=c["causal"],
                                                 operand_rounding=False)
    got_o, got_l = kernel_model(q, k, v, cu, c["nq"], c["nkv"], 1e4, mask, c["causal"])
    assert np.max(np.abs(got_o - ref_o)) < 1e-10
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l))
    assert np.max(np.abs(got_l[fin] - ref_l[fin])) < 1e-10
    if c.get("dead_rows"):
        assert (~fin).any()
