"""The backward kernels' work decomposition, restated in numpy and checked
against the oracle's backward in float64 (no rounding).

dK' and dV (csrc/bwd_kernel.cuh): one work item per (sequence, 128-key tile,
KV head); each item visits the packed query tiles (tq = 128 / G tokens x G
heads) from floor(k0 / tq) (causal) or 0 to the sequence's last; a key row j
sees packed column r iff r >= (k0 + j - t0) * G (causal) and k0 + j < L;
rows past the sequence and padding rows carry lse = +inf and Delta = 0; dV
and dK' accumulate per item.

dQ' (csrc/bwd_q_kernel.cuh): one work item per (sequence, query tile, KV
head); each item visits the key tiles below ceil(t_end / 128), t_end =
min(t0 + tq, L) (causal) or L; packed row r sees key c of tile j iff
j * 128 + c <= t0 + r / G (causal) or < L; dQ' is summed over the item's
key tiles and written once per valid row.

This pins the index arithmetic on the CPU (the products themselves run on
tensor cores there). CPU only."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc

BM = BN = 128


def decomposed_backward(q, k, v, dout, cu, nq, nkv, theta, causal):
    N, _, d = q.shape
    G = nq // nkv
    tq = BM // G
    rows = tq * G
    out, lse = orc.gqa_rope_attention(q, k, v, cu, nq, nkv, theta, causal=causal, operand_rounding=False)
    pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)])
    qr = orc.apply_rope(q, pos, theta)
    kr = orc.apply_rope(k, pos, theta)
    delta = np.einsum("thc,thc->ht", dout, out)
    lse2 = lse * np.log2(np.e)
    sl2 = np.log2(np.e) / np.sqrt(d)
    dq_acc = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    r_idx = np.arange(BM)
    tt, hin = r_idx // G, r_idx % G
    for s in range(len(cu) - 1):
        seq_start, L = int(cu[s]), int(cu[s + 1] - cu[s])
        for l in range((L + BN - 1) // BN):
            k0 = l * BN
            qi0 = k0 // tq if causal else 0
            nt = (L + tq - 1) // tq - qi0
            assert nt >= 1
            keys = seq_start + k0 + np.arange(BN)
            in_n = keys < N  # TMA fills rows past the tensor with zeros
            for kvh in range(nkv):
                Kt = np.where(in_n[:, None], kr[np.minimum(keys, N - 1), kvh], 0.0)
                Vt = np.where(in_n[:, None], v[np.minimum(keys, N - 1), kvh], 0.0)
                dVt = np.zeros((BN, d))
                dKt = np.zeros((BN, d))
                for i in range(nt):
                    t0 = (qi0 + i) * tq
                    toks = seq_start + t0 + tt
                    loaded = (r_idx < rows) & (toks < N)
                    valid = (r_idx < rows) & (t0 + tt < L)
                    heads = kvh * G + hin
                    tc = np.minimum(toks, N - 1)
                    Qt = np.where(loaded[:, None], qr[tc, heads], 0.0)
                    dOt = np.where(loaded[:, None], dout[tc, heads], 0.0)
                    st_l2 = np.where(valid, lse2[heads, tc], np.inf)
                    st_d = np.where(valid, delta[heads, tc], 0.0)
                    key_in_seq = k0 + np.arange(BN)
                    bound = np.minimum(BM, np.maximum(0, (key_in_seq - t0) * G)) if causal else 0
                    r_lo = np.where(key_in_seq >= L, BM, bound)
                    visible = r_idx[None, :] >= r_lo[:, None]
                    PT = np.where(visible, np.exp2((Kt @ Qt.T) * sl2 - st_l2[None, :]), 0.0)
                    dST = PT * ((Vt @ dOt.T) - st_d[None, :])
                    dVt += PT @ dOt
                    dKt += dST @ Qt
                ok = key_in_seq < L
                dv[keys[ok], kvh] = dVt[ok]
                dk[keys[ok], kvh] = dKt[ok] / np.sqrt(d)
    # dQ': query-tile items, the forward's packing
    written = np.zeros(q.shape[:2], dtype=int)
    for s in range(len(cu) - 1):
        seq_start, L = int(cu[s]), int(cu[s + 1] - cu[s])
        for l in range((L + tq - 1) // tq):
            t0 = l * tq
            t_end = min(t0 + tq, L) if causal else L
            nkt = (t_end + BN - 1) // BN
            toks = seq_start + t0 + tt
            loaded = (r_idx < rows) & (toks < N)
            valid = (r_idx < rows) & (t0 + tt < L)
            tc = np.minimum(toks, N - 1)
            last_key = (t0 + tt) if causal else np.full(BM, L - 1)
            for kvh in range(nkv):
                heads = kvh * G + hin
                Qt = np.where(loaded[:, None], qr[tc, heads], 0.0)
                dOt = np.where(loaded[:, None], dout[tc, heads], 0.0)
                st_l2 = np.where(valid, lse2[heads, tc], np.inf)
                st_d = np.where(valid, delta[heads, tc], 0.0)
                dQt = np.zeros((BM, d))
                for j in range(nkt):
                    keys = seq_start + j * BN + np.arange(BN)
                    in_n = keys < N
                    Kt = np.where(in_n[:, None], kr[np.minimum(keys, N - 1), kvh], 0.0)
                    Vt = np.where(in_n[:, None], v[np.minimum(keys, N - 1), kvh], 0.0)
                    visible = (j * BN + np.arange(BN))[None, :] <= last_key[:, None]
                    P = np.where(visible, np.exp2((Qt @ Kt.T) * sl2 - st_l2[:, None]), 0.0)
                    dS = P * ((dOt @ Vt.T) - st_d[:, None])
                    dQt += dS @ Kt
                for r in np.nonzero(valid)[0]:
                    dq_acc[seq_start + t0 + tt[r], heads[r]] = dQt[r]
                    written[seq_start + t0 + tt[r], heads[r]] += 1
    assert np.all(written == 1)  # every (token, head) row written exactly once
    return (orc.rope_backward(dq_acc / np.sqrt(d), pos, theta), orc.rope_backward(dk, pos, theta), dv)


CASES = [((200,), 4, 1, 32, True), ((70, 1, 130, 257), 6, 2, 32, True), ((150, 40), 8, 8, 32, False),
         ((300,), 12, 4, 64, True), ((129, 5), 2, 2, 32, True), ((9,), 128, 1, 32, True)]


@pytest.mark.parametrize("lens,nq,nkv,d,causal", CASES)
def test_decomposition_reproduces_the_oracle(lens, nq, nkv, d, causal):
    rng = np.random.default_rng(sum(lens) + nq)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(cu[-1])
    q = rng.standard_normal((N, nq, d))
    k = rng.standard_normal((N, nkv, d))
    v = rng.standard_normal((N, nkv, d))
    do = rng.standard_normal((N, nq, d))
    ref = orc.gqa_rope_attention_backward(q, k, v, do, cu, nq, nkv, 1e4, causal=causal)
    got = decomposed_backward(q, k, v, do, cu, nq, nkv, 1e4, causal)
    for name, a, b in zip(("dq", "dk", "dv"), ref, got):
        assert np.max(np.abs(a - b)) <= 1e-10 * np.max(np.abs(a)), name
