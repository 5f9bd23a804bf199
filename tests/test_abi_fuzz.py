"""Argument fuzzing of the C ABI on the host: random sizes, head counts,
flags and null / misaligned / aligned fake pointers for every compute entry
point. Each call must return a documented status code and never crash;
calls that pass the host checks stop at the first CUDA call with
GQA_ERR_CUDA or GQA_ERR_UNSUPPORTED, because the child process sees no GPU
(CUDA_VISIBLE_DEVICES is emptied): no fuzzed call, with its fake pointers,
can reach a kernel launch, on any machine. Run in a child process so that a
crash is a test failure rather than the end of the test run. CPU only."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, ROOT)
from hypothesis import given, settings, strategies as st, HealthCheck
from transformer_attention_gqa_b200 import _abi

_abi.load()
CODES = set(range(8))
ptr = st.sampled_from([0, 4096, 4096 + 2, 4096 + 8, 1 << 20])
small = st.integers(min_value=-3, max_value=300)
heads = st.integers(min_value=-1, max_value=260)
dims = st.sampled_from([-1, 0, 16, 32, 48, 64, 96, 128, 256])
flags = st.integers(min_value=-1, max_value=2)
theta = st.sampled_from([1e4, 0.0, -1.0, float("inf"), float("nan"), 5e5])
size = st.sampled_from([0, 16, 1 << 20, 1 << 40])
cfg = settings(max_examples=150, deadline=None, suppress_health_check=list(HealthCheck))

@cfg
@given(ptr, ptr, ptr, ptr, theta, ptr, small, small, heads, heads, dims, flags, flags, ptr, ptr, ptr, size)
def fwd(q, k, v, pos, th, cu, ns, n, hq, hk, d, causal, dt, out, lse, ws, wb):
    assert _abi.gqa_rope_attn_fwd(q, k, v, pos, th, cu, ns, n, hq, hk, d, causal, dt, out, lse, ws, wb, None) in CODES

@cfg
@given(ptr, ptr, ptr, ptr, theta, ptr, small, small, heads, heads, dims, flags, flags, ptr, ptr)
def fwd_noalloc(q, k, v, pos, th, cu, ns, n, hq, hk, d, causal, dt, out, lse):
    assert _abi.gqa_rope_attn_fwd_noalloc(q, k, v, pos, th, cu, ns, n, hq, hk, d, causal, dt, out, lse, None) in CODES

@cfg
@given(ptr, ptr, ptr, ptr, small, small, heads, heads, dims, flags, ptr, ptr, ptr, size)
def fwd_rotated(q, k, v, cu, ns, n, hq, hk, d, causal, out, lse, ws, wb):
    assert _abi.gqa_rope_attn_fwd_rotated(q, k, v, cu, ns, n, hq, hk, d, causal, out, lse, ws, wb, None) in CODES

@cfg
@given(ptr, ptr, ptr, ptr, ptr, ptr, theta, small, small, heads, heads, dims, ptr, ptr, ptr, size)
def dec(q, kn, vn, kc, vc, lens, th, b, lm, hq, hk, d, out, lse, ws, wb):
    assert _abi.gqa_rope_attn_decode(q, kn, vn, kc, vc, lens, th, b, lm, hq, hk, d, out, lse, ws, wb, None) in CODES

@cfg
@given(ptr, ptr, ptr, ptr, ptr, ptr, ptr, theta, ptr, small, small, heads, heads, dims, flags, ptr, ptr, ptr, ptr, size)
def bwd(q, k, v, o, lse, do, pos, th, cu, ns, n, hq, hk, d, causal, dq, dk, dv, ws, wb):
    assert _abi.gqa_rope_attn_bwd(q, k, v, o, lse, do, pos, th, cu, ns, n, hq, hk, d, causal, dq, dk, dv, ws, wb,
                                  None) in CODES

@cfg
@given(ptr, ptr, ptr, theta, ptr, small, small, small, heads, heads, dims, ptr, ptr, ptr, ptr, size)
def proj(x, w, pos, th, cu, ns, n, c, hq, hk, d, q, k, v, ws, wb):
    assert _abi.gqa_rope_attn_qkv_proj(x, w, pos, th, cu, ns, n, c, hq, hk, d, q, k, v, ws, wb, None) in CODES

@cfg
@given(ptr, ptr, ptr, ptr, theta, ptr, small, small, heads, heads, dims, flags, ptr, small, small, ptr, ptr, ptr, size)
def masked(q, k, v, pos, th, cu, ns, n, hq, hk, d, causal, m, ml, ld, out, lse, ws, wb):
    assert _abi.gqa_rope_attn_fwd_masked(q, k, v, pos, th, cu, ns, n, hq, hk, d, causal, m, ml, ld, out, lse, ws, wb,
                                         None) in CODES

for f in (fwd, fwd_noalloc, fwd_rotated, dec, bwd, proj, masked):
    f()
print("fuzz ok")
"""


def test_abi_argument_fuzzing_never_crashes():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], capture_output=True, text=True,
                       timeout=600, env=env)
    assert r.returncode == 0 and "fuzz ok" in r.stdout, (r.returncode, r.stdout[-2000:], r.stderr[-3000:])
