"""The kernel evaluates a quarter of its exponentials with a polynomial on
the FMA pipe. These CPU checks re-derive the polynomial, check the constants
the kernel compiles in, and bound the error of the kernel's fp32 evaluation
(emulated here step by step in float32) against exact 2^x."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "transformer_attention_gqa_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def header_coeffs():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    return [float(v) for v in re.findall(r"kExp2C\d = ([0-9.eE+-]+)f;", text)]


def test_header_matches_fit():
    g = _gen()
    c, err = g.remez_rel()
    assert err < 3e-6
    h = header_coeffs()
    assert len(h) == len(c) == 5
    assert np.array_equal(np.float32(h), np.float32(c))
    assert open(os.path.join(CSRC, "exp2_poly.cuh")).read() == g.header_text()


def exp2_fma_emulated(x):
    """float32 step-by-step copy of the kernel's evaluation."""
    f32 = np.float32
    c = [f32(v) for v in header_coeffs()]
    x = np.maximum(np.asarray(x, f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    f = (x - (t - f32(12582912.0)).astype(f32)).astype(f32)
    p = (c[4] * f + c[3]).astype(f32)  # fmaf rounds once; the float32 products here round twice,
    p = (p * f + c[2]).astype(f32)     # which only loosens the bound checked below
    p = (p * f + c[1]).astype(f32)
    p = (p * f + c[0]).astype(f32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_fp32_evaluation_error_bound():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), np.arange(-125, 9, dtype=np.float64)])
    x32 = x.astype(np.float32)
    got = exp2_fma_emulated(x32).astype(np.float64)
    ref = np.exp2(x32.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 4e-6, rel.max()
    # clamped region and -inf (masked scores) give a negligible positive value
    tiny = exp2_fma_emulated(np.array([-np.inf, -1e30, -200.0], np.float32))
    assert np.all(tiny > 0) and np.all(tiny <= 2.0 ** -124)


def test_bf16_pack_rounds_to_nearest():
    import torch
    rng = np.random.default_rng(0)
    p = np.abs(rng.standard_normal(100000)).astype(np.float32) * np.float32(10.0)
    packed = ((p.view(np.uint32).astype(np.uint64) + 0x8000) >> 16).astype(np.uint16)
    ref = torch.from_numpy(p).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ties = (p.view(np.uint32) & 0xFFFF) == 0x8000
    assert np.array_equal(packed[~ties], ref[~ties])
