"""The tensor-core decoding kernel's algorithm, restated in numpy with its
update rules and checked against the oracle (``gqa_rope_decode``) before
the kernel runs on a GPU:

* key ranges of kps keys (whole 128-key tiles, about 256 ranges over the
  batch), one per CTA, merged by the combine kernel's rule;
* keys in the rows of the products: per tile S^T = K Q^T (128 keys x the G
  heads) and O^T += V^T P^T (features x heads), so the G heads of a KV head
  are columns and no row is padding;
* per 128-key tile and head: scores masked past the range (selected to
  -inf, so NaN cache rows there never count), the head's max over the
  tile's keys, the running max set by the first tile and moved only when a
  score exceeds it by more than 2^8 in p (O and l then rescaled),
  p = 2^((s - m) log2(e) / sqrt(d));
* the range's last tile fixed up in shared memory: the new token's rotated
  key and value in row pos, V rows past the range zeroed, so that the cache
  rows there (NaN in the tests) never reach a product with a nonzero weight.
CPU only."""
import math

import numpy as np
import pytest

import oracle.gqa_oracle as orc

KT = 128


def layout(B, Lmax, nkv, target=256):
    tiles = -(-Lmax // KT)
    want = max(1, min(tiles, -(-target // (B * nkv))))
    tps = -(-tiles // want)
    return tps * KT, -(-tiles // tps)  # kps, splits


def kernel_model(q, k_new, v_new, k_cache, v_cache, lens, nq, nkv, theta):
    B, _, d = q.shape
    Lmax = k_cache.shape[1]
    G = nq // nkv
    sl2 = math.log2(math.e) / math.sqrt(d)
    thr = 8.0 / sl2
    kps, splits = layout(B, Lmax, nkv)
    out = np.zeros((B, nq, d))
    lse = np.zeros((nq, B))
    kc, vc = k_cache.copy(), v_cache.copy()
    flat_k = k_cache.reshape(-1, nkv, d)
    flat_v = v_cache.reshape(-1, nkv, d)
    for b in range(B):
        pos = int(lens[b])
        qr = orc.apply_rope(q[b][None], [pos], theta, operand_rounding=True)[0]
        kr = orc.apply_rope(k_new[b][None], [pos], theta, operand_rounding=True)[0]
        for h in range(nkv):
            Q = qr[h * G:(h + 1) * G]  # [G, d]: the heads are the MMA's N
            parts = []
            for split in range(splits):
                k0 = split * kps
                k1 = min(k0 + kps, pos + 1)
                if k0 >= k1:
                    parts.append(None)
                    continue
                ntiles = -(-(k1 - k0) // KT)
                m = np.full(G, -np.inf)
                l = np.zeros(G)
                oT = np.zeros((d, G))
                for j in range(ntiles):
                    t0 = k0 + j * KT
                    idx = b * Lmax + t0 + np.arange(KT)  # rows of the cache maps (may run into b + 1)
                    ok_rows = idx < flat_k.shape[0]      # past the cache's end: zero fill
                    K = np.where(ok_rows[:, None], flat_k[np.minimum(idx, flat_k.shape[0] - 1), h], 0.0)
                    V = np.where(ok_rows[:, None], flat_v[np.minimum(idx, flat_v.shape[0] - 1), h], 0.0)
                    nvalid = min(KT, k1 - t0)
                    if j == ntiles - 1:  # fix-up of the last tile
                        if k0 <= pos < k1:
                            K[pos - t0] = kr[h]
                            V[pos - t0] = v_new[b, h]
                        V[nvalid:] = 0.0
                    with np.errstate(invalid="ignore"):
                        ST = K @ Q.T  # [KT, G]; NaN in K rows past the range
                    valid = np.arange(KT) < nvalid
                    ST = np.where(valid[:, None], ST, -np.inf)
                    mx = ST.max(axis=0)  # per head, over the tile's keys
                    need = mx > m + thr
                    if need.any():
                        m_new = np.where(need, mx, m)
                        if j > 0:
                            alpha = np.where(need, np.exp2((m - m_new) * sl2), 1.0)
                            oT *= alpha[None, :]
                            l *= alpha
                        m = m_new
                    PT = np.exp2(ST * sl2 - (m * sl2)[None, :])  # [KT, G]
                    l += PT.sum(axis=0)
                    oT += V.T @ PT
                parts.append((m * sl2, l, oT.T))
            # combine: per head, over the ranges holding a visible key
            used = [pt for pt in parts if pt is not None]
            for g in range(G):
                M = max(pt[0][g] for pt in used)
                L = sum(pt[1][g] * 2.0 ** (pt[0][g] - M) for pt in used)
                acc = sum(pt[2][g] * 2.0 ** (pt[0][g] - M) for pt in used)
                out[b, h * G + g] = acc / L
                lse[h * G + g, b] = (M + math.log2(L)) * math.log(2.0)
            kc[b, pos, h] = kr[h]
            vc[b, pos, h] = v_new[b, h]
    return out, lse, kc, vc


def _inputs(lens, Lmax, nq, nkv, d, seed):
    rng = np.random.default_rng(seed)
    B = len(lens)
    bf = lambda a: orc.round_to_bf16(a)
    q = bf(rng.standard_normal((B, nq, d)))
    k_new = bf(rng.standard_normal((B, nkv, d)))
    v_new = bf(rng.standard_normal((B, nkv, d)))
    k_cache = bf(rng.standard_normal((B, Lmax, nkv, d)))
    v_cache = bf(rng.standard_normal((B, Lmax, nkv, d)))
    for b, p in enumerate(lens):  # rows from p on must not be read
        k_cache[b, p:] = np.nan
        v_cache[b, p:] = np.nan
    return q, k_new, v_new, k_cache, v_cache, np.asarray(lens)


@pytest.mark.parametrize("lens, Lmax, nq, nkv, d", [
    ((0, 1, 127, 128, 129, 300), 310, 12, 4, 32),  # G = 3; an empty cache, tile edges
    ((300, 2047, 5), 2100, 16, 2, 64),             # G = 8; several ranges per sequence
    ((129, 400), 513, 16, 1, 32),                  # G = 16
    ((77,), 128, 4, 4, 64),                        # G = 1
])
def test_kernel_model_matches_the_oracle(lens, Lmax, nq, nkv, d):
    theta = 1e4
    q, kn, vn, kc, vc, L = _inputs(lens, Lmax, nq, nkv, d, seed=sum(lens) + nq)
    out, lse, kc2, vc2 = kernel_model(q, kn, vn, kc, vc, L, nq, nkv, theta)
    ro, rl, krow, vrow = orc.gqa_rope_decode(q, kn, vn, kc, vc, L, nq, nkv, theta)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(out - ro)) < 1e-10 * max(1.0, np.abs(ro).max())
    assert np.max(np.abs(lse - rl)) < 1e-10 * max(1.0, np.abs(rl).max())
    for b, p in enumerate(L):
        assert np.array_equal(kc2[b, p], krow[b]) and np.array_equal(vc2[b, p], vrow[b])


def test_growing_scores_take_the_rescale_path():
    """Keys whose scores grow along the cache move the running max by more
    than the threshold in later tiles (O rescaled), and the result still
    matches the oracle."""
    lens, Lmax, nq, nkv, d = (500, 260), 520, 8, 2, 64
    q, kn, vn, kc, vc, L = _inputs(lens, Lmax, nq, nkv, d, seed=3)
    ramp = (1.0 + np.arange(Lmax) / 40.0)[None, :, None, None]
    kc = orc.round_to_bf16(kc * ramp)
    out, lse, _, _ = kernel_model(q, kn, vn, kc, vc, L, nq, nkv, 1e4)
    ro, rl, _, _ = orc.gqa_rope_decode(q, kn, vn, kc, vc, L, nq, nkv, 1e4)
    assert np.max(np.abs(out - ro)) < 1e-10 * np.abs(ro).max()
    assert np.max(np.abs(lse - rl)) < 1e-10 * np.abs(rl).max()


def test_planted_mistake_is_caught():
    """Without the V fix-up the NaN rows past the range reach the weighted
    sum through zero weights."""
    lens, Lmax, nq, nkv, d = (70,), 128, 4, 2, 32
    q, kn, vn, kc, vc, L = _inputs(lens, Lmax, nq, nkv, d, seed=9)
    with np.errstate(invalid="ignore"):
        PT = np.zeros((KT, 1))
        V = vc[0, 0:128, 0]  # rows 70.. are NaN
        assert np.isnan(V.T @ PT).any()
