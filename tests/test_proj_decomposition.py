"""The projection kernel's tiling and epilogue, restated in numpy and checked
against the oracle (float64, no rounding): tiles of 128 tokens x 256 output
features of x W_qkv^T, walked by persistent CTAs (CTA b takes tiles b,
b + grid, ...; tile t covers features (t % n_tiles_n) * 256 and tokens
(t / n_tiles_n) * 128; its accumulator alternates with the CTA's tile
count); a tile holds 256 / d whole heads; head index
n0 / d + hd selects q (< n_q), k (< n_q + n_kv) or v, and a tile past the
last head stops there; q and k heads are rotated pairwise (i, i + d/2) from
the accumulator. This pins the index arithmetic of csrc/proj_kernel.cuh on
the CPU. CPU only."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc

BM, BN = 128, 256


def persistent_tiles(N, F, grid):
    """(CTA, local tile index i, accumulator i & 1, n0, m0) in issue order."""
    n_tiles_n = (F + BN - 1) // BN
    n_tiles = n_tiles_n * ((N + BM - 1) // BM)
    for b in range(min(grid, n_tiles)):
        for i, t in enumerate(range(b, n_tiles, grid)):
            yield b, i, i & 1, (t % n_tiles_n) * BN, (t // n_tiles_n) * BM


def decomposed_projection(x, w, nq, nkv, d, pos, theta, grid=148):
    N, C = x.shape
    F = w.shape[0]
    heads = nq + 2 * nkv
    q, k, v = np.zeros((N, nq, d)), np.zeros((N, nkv, d)), np.zeros((N, nkv, d))
    half = d // 2
    inv = theta ** (-np.arange(half) * 2.0 / d)
    for _, _, _, n0, m0 in persistent_tiles(N, F, grid):
        wt = np.zeros((BN, C))
        rows = min(BN, F - n0)
        wt[:rows] = w[n0:n0 + rows]  # rows past F are zero-filled
        xt = np.zeros((BM, C))
        toks = min(BM, N - m0)
        xt[:toks] = x[m0:m0 + toks]
        acc = xt @ wt.T
        for hd in range(BN // d):
            head = n0 // d + hd
            if head >= heads:
                break
            blk = acc[:toks, hd * d:(hd + 1) * d]
            t = np.arange(m0, m0 + toks)
            if head < nq + nkv:
                ang = pos[t][:, None] * inv[None, :]
                c, s = np.cos(ang), np.sin(ang)
                lo, hi = blk[:, :half], blk[:, half:]
                out = np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=1)
                if head < nq:
                    q[t, head] = out
                else:
                    k[t, head - nq] = out
            else:
                v[t, head - nq - nkv] = blk
    return q, k, v


CASES = [((300,), 96, 6, 2, 64), ((200, 77), 64, 8, 2, 128), ((130, 1, 60), 40, 8, 4, 32), ((5,), 16, 1, 1, 128)]


@pytest.mark.parametrize("lens,C,nq,nkv,d", CASES)
def test_projection_decomposition_reproduces_the_oracle(lens, C, nq, nkv, d):
    rng = np.random.default_rng(sum(lens) + C)
    N = sum(lens)
    x = rng.standard_normal((N, C))
    w = rng.standard_normal(((nq + 2 * nkv) * d, C))
    cu = np.concatenate([[0], np.cumsum(lens)])
    pos = np.concatenate([np.arange(L) for L in lens])
    f, fk = nq * d, nkv * d
    ref = orc.qkv_rope_projection(x, w[:f], w[f:f + fk], w[f + fk:], nq, nkv, 1e4, cu_seqlens=cu)
    got = decomposed_projection(x, w, nq, nkv, d, pos, 1e4)
    for name, a, b in zip("qkv", ref, got):
        assert np.max(np.abs(a - b)) <= 1e-10 * np.max(np.abs(a)), name


@pytest.mark.parametrize("N,F,grid", [(8192, 6144, 148), (300, 512, 148), (5, 256, 148), (1000, 1280, 3)])
def test_persistent_tiles_cover_each_tile_once(N, F, grid):
    seen = {}
    for b, i, acc, n0, m0 in persistent_tiles(N, F, grid):
        assert (n0, m0) not in seen
        seen[(n0, m0)] = b
        assert acc == i % 2
    assert len(seen) == ((F + BN - 1) // BN) * ((N + BM - 1) // BM)
