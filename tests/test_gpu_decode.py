"""GPU parity of the decoding step (through the C ABI) against the float64
oracle's decoding step, on seeded caches whose unused rows hold NaN (they
must never be read). Small shapes are compared in full; the Llama-3-8B- and
Qwen2.5-3B-shaped batches run at full size (the launch configuration the
benchmark times) and are compared on sampled sequences. The appended cache
row must equal the oracle's rotated, bf16-rounded key bit for bit."""
import numpy as np
import pytest

import oracle.gqa_oracle as orc
from tests.conftest import gpu_available
from tests import gpu_helpers as H
from transformer_attention_gqa_b200 import workloads as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]


def _dev(inp):
    import torch

    bf = torch.bfloat16
    return dict(q=torch.from_numpy(inp.q).to(bf).cuda(), k_new=torch.from_numpy(inp.k_new).to(bf).cuda(),
                v_new=torch.from_numpy(inp.v_new).to(bf).cuda(), k_cache=torch.from_numpy(inp.k_cache).to(bf).cuda(),
                v_cache=torch.from_numpy(inp.v_cache).to(bf).cuda(),
                lens=torch.from_numpy(inp.cache_seqlens).cuda())


def _run(inp, t=None, workspace=None):
    import torch
    import transformer_attention_gqa_b200 as g

    t = t or _dev(inp)
    out, lse = g.gqa_rope_attn_decode(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["lens"],
                                      inp.workload.rope_theta, workspace=workspace)
    torch.cuda.synchronize()
    st = g.get_device_status()
    assert st == 0, f"device status {st}"
    return t, out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _oracle(inp, seqs=None):
    w = inp.workload
    sel = np.arange(w.batch) if seqs is None else np.asarray(seqs)
    return orc.gqa_rope_decode(inp.q[sel], inp.k_new[sel], inp.v_new[sel], inp.k_cache[sel], inp.v_cache[sel],
                               inp.cache_seqlens[sel], w.n_q_heads, w.n_kv_heads, w.rope_theta), sel


def _check(inp, t, out, lse, seqs=None, what=""):
    (ro, rl, rk, rv), sel = _oracle(inp, seqs)
    H.compare(out[sel].reshape(-1, out.shape[-1]), lse[:, sel], ro.reshape(-1, ro.shape[-1]), rl, what=what)
    kc = t["k_cache"].float().cpu().numpy()
    vc = t["v_cache"].float().cpu().numpy()
    for i, b in enumerate(sel):
        p = int(inp.cache_seqlens[b])
        assert np.array_equal(kc[b, p], rk[i]), f"{what}: appended key row of sequence {b}"
        assert np.array_equal(vc[b, p], rv[i]), f"{what}: appended value row of sequence {b}"
        assert np.array_equal(kc[b, :p], inp.k_cache[b, :p]) and np.array_equal(vc[b, :p], inp.v_cache[b, :p])
        assert np.all(np.isnan(kc[b, p + 1:])) and np.all(np.isnan(vc[b, p + 1:])), f"{what}: rows after p"


def test_decode_small_in_full():
    inp = wl.make_decode_inputs(wl.DECODE_WORKLOADS["decode_small"])
    t, out, lse = _run(inp)
    _check(inp, t, out, lse, what="decode_small")


CASES = [
    # (cache lens, max_len, n_q, n_kv, d, theta)
    ((0,), 1, 4, 4, 32, 1e4),
    ((0, 5, 17), 40, 8, 8, 128, 5e5),
    ((63, 64, 65, 127, 128, 129), 130, 12, 4, 64, 1e4),
    ((1000, 3, 2047), 2048, 16, 1, 128, 1e4),
    ((700, 701), 800, 14, 2, 64, 1e6),
    ((300,), 1024, 6, 2, 32, 1e4),
    ((4095, 2, 4000, 1), 4096, 32, 4, 128, 5e5),
    ((5000,), 6000, 16, 16, 64, 1e4),
]


@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0][:3]}-M{c[1]}-q{c[2]}-kv{c[3]}-d{c[4]}" for c in CASES])
def test_decode_shapes(case):
    lens, L, nq, nkv, d, theta = case
    w = wl.DecodeWorkload("case", tuple(lens), L, nq, nkv, d, theta, seed=sum(lens) + nq)
    inp = wl.make_decode_inputs(w)
    t, out, lse = _run(inp)
    _check(inp, t, out, lse, what=str(case))


@pytest.mark.parametrize("name", ["decode_llama8b", "decode_qwen3b"])
def test_decode_full_size_sampled(name):
    w = wl.DECODE_WORKLOADS[name]
    inp = wl.make_decode_inputs(w)
    t, out, lse = _run(inp)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    seqs = [0, 1, w.batch // 2, w.batch - 1]
    _check(inp, t, out, lse, seqs=seqs, what=name)


def test_decode_ragged_batch():
    lens = wl.DECODE_WORKLOADS["decode_ragged"].cache_lens[:12]
    w = wl.DecodeWorkload("ragged12", lens, max(lens) + 3, 32, 8, 128, 5e5, seed=5)
    inp = wl.make_decode_inputs(w)
    t, out, lse = _run(inp)
    _check(inp, t, out, lse, what="ragged")


def test_decode_bad_length_sets_status_and_skips_that_sequence():
    import torch
    import transformer_attention_gqa_b200 as g

    w = wl.DecodeWorkload("bad", (10, 20, 30), 32, 8, 2, 64, 1e4, seed=3)
    inp = wl.make_decode_inputs(w)
    t = _dev(inp)
    t["lens"] = torch.tensor([10, 32, 30], dtype=torch.int32, device="cuda")  # 32 is outside the cache
    out = torch.full_like(t["q"], 7.0)
    g.gqa_rope_attn_decode(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["lens"], 1e4, out=out)
    torch.cuda.synchronize()
    assert g.get_device_status() == 4
    assert g.get_device_status() == 0
    assert torch.all(out[1] == 7.0)
    o = out.float().cpu().numpy().astype(np.float64)
    (ro, _, _, _), _ = _oracle(inp, seqs=[0, 2])
    H.compare(o[[0, 2]].reshape(-1, 64), None, ro.reshape(-1, 64), None, what="bad-length neighbours")


def test_decode_workspace_reuse_with_garbage():
    import torch
    import transformer_attention_gqa_b200 as g

    ws = g.Workspace(torch.device("cuda"))
    for rep, name in enumerate(["decode_small", "decode_small"]):
        inp = wl.make_decode_inputs(wl.DECODE_WORKLOADS[name], seed=40 + rep)
        w = inp.workload
        buf = ws.get(g.decode_workspace_size(w.batch, w.max_cache_len, w.n_q_heads, w.n_kv_heads, w.head_dim))
        buf.fill_(0xFF)  # NaN patterns everywhere
        t, out, lse = _run(inp, workspace=ws)
        _check(inp, t, out, lse, what=f"reuse {rep}")


def test_decode_timeout_is_reported_and_the_context_stays_usable(monkeypatch):
    """Failure detection without a fault: with the test hook set, the first
    K/V tile of every key range is never loaded; each CTA's bounded wait (2 s)
    runs out, the CTA drains what it issued and exits, and the status word
    reads GQA_ERR_TIMEOUT. The next call must then be correct."""
    import torch
    import transformer_attention_gqa_b200 as g

    w = wl.DecodeWorkload("timeout", (100, 5), 128, 8, 2, 64, 1e4, seed=12)
    inp = wl.make_decode_inputs(w)
    t = _dev(inp)
    monkeypatch.setenv("GQA_ROPE_ATTN_TEST_DROP_FIRST_LOAD", "1")
    g.gqa_rope_attn_decode(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["lens"], w.rope_theta)
    torch.cuda.synchronize()
    assert g.get_device_status() == 5
    monkeypatch.delenv("GQA_ROPE_ATTN_TEST_DROP_FIRST_LOAD")
    t2, out, lse = _run(inp)
    _check(inp, t2, out, lse, what="after a timeout")
