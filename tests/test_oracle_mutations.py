"""Planted mistakes, on the CPU, in a private copy of the oracle: each one
must make at least one pin fail. This shows the pins can tell a wrong oracle
from a right one (a dropped term, a wrong sign or index, a transposed
operand, a wrong head map, a wrong scale, an off-by-one mask)."""
import importlib.util
import math
import os

import numpy as np
import pytest

import tests.test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fresh_oracle():
    spec = importlib.util.spec_from_file_location("_oracle_copy", os.path.join(ROOT, "oracle", "gqa_oracle.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _all_pins(m, golden):
    checks = [
        lambda: pins.pin_inv_freq(golden, m),
        lambda: pins.pin_rope_worked_example(golden, m),
        lambda: pins.pin_rope_norm(m),
        lambda: pins.pin_rope_identity_at_zero(m),
        lambda: pins.pin_rope_relative(m),
        lambda: pins.pin_rope_basis_closed_form(m),
        lambda: pins.pin_rope_operand_rounding(m),
        lambda: pins.pin_rope_bf16_matches_torch(m),
        lambda: pins.pin_worked_attention(golden, m),
        lambda: pins.pin_first_row(m),
        lambda: pins.pin_identical_keys(m),
        lambda: pins.pin_gqa_equals_mha(m),
        lambda: pins.pin_brute_force(m),
        lambda: pins.pin_torch_sdpa(m),
        lambda: pins.pin_varlen(m),
        lambda: pins.pin_causal_last_row(m),
    ]
    failed = 0
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    return failed


def _mut_rotate_sign(m):
    h = lambda x: x.shape[-1] // 2
    m.rotate_half = lambda x: np.concatenate([x[..., h(x):], -x[..., :h(x)]], axis=-1)


def _mut_interleaved_pairs(m):
    def rot(x):
        y = np.empty_like(x)
        y[..., 0::2] = -x[..., 1::2]
        y[..., 1::2] = x[..., 0::2]
        return y
    orig = m.rope_cos_sin

    def cs(positions, head_dim, theta, table_fp32=False):
        c, s = orig(positions, head_dim, theta, table_fp32)
        hh = head_dim // 2
        return np.repeat(c[:, :hh], 2, axis=1), np.repeat(s[:, :hh], 2, axis=1)
    m.rotate_half = rot
    m.rope_cos_sin = cs


def _mut_inv_freq_exponent(m):
    m.rope_inv_freq = lambda d, theta: np.power(float(theta), -np.arange(d // 2, dtype=np.float64) / float(d))


def _mut_share_repeat(m):
    m.share_kv_heads = lambda kv, g, axis=1: np.concatenate([kv] * g, axis=axis)


def _mut_scale_1_over_d(m):
    m.score = lambda qh, kh: np.matmul(qh, np.swapaxes(kh, -1, -2)) / qh.shape[-1]


def _mut_mask_strict(m):
    def cm(scores, qi, ki):
        vis = ki[None, :] < qi[:, None]
        vis[:, 0] = True
        return np.where(vis[None], scores, -np.inf)
    m.causal_mask = cm


def _mut_lse_drops_max(m):
    def sl(scores):
        mx = np.max(scores, axis=-1, keepdims=True)
        e = np.exp(scores - mx)
        z = np.sum(e, axis=-1, keepdims=True)
        return e / z, np.log(z)[..., 0]
    m.softmax_with_lse = sl


def _mut_transposed_scores(m):
    def sc(qh, kh):
        s = np.matmul(qh, np.swapaxes(kh, -1, -2)) / math.sqrt(qh.shape[-1])
        if s.shape[-1] == s.shape[-2]:
            return np.swapaxes(s, -1, -2)
        return s
    m.score = sc


def _mut_rope_on_v(m):
    orig = m.gather

    def g(w, vh):
        H, T, d = vh.shape
        v = np.transpose(vh, (1, 0, 2))
        vr = m.apply_rope(v, np.arange(T), 1e4)
        return orig(w, np.transpose(vr, (1, 0, 2)))
    m.gather = g


def _mut_no_normalise(m):
    def sl(scores):
        mx = np.max(scores, axis=-1, keepdims=True)
        e = np.exp(scores - mx)
        z = np.sum(e, axis=-1, keepdims=True)
        return e, (mx + np.log(z))[..., 0]
    m.softmax_with_lse = sl


MUTATIONS = {
    "rotate_half sign": _mut_rotate_sign,
    "interleaved pairs": _mut_interleaved_pairs,
    "inv_freq exponent": _mut_inv_freq_exponent,
    "repeat instead of repeat_interleave": _mut_share_repeat,
    "1/d scale": _mut_scale_1_over_d,
    "strict causal mask": _mut_mask_strict,
    "lse drops max": _mut_lse_drops_max,
    "transposed scores": _mut_transposed_scores,
    "rope on V": _mut_rope_on_v,
    "softmax not normalised": _mut_no_normalise,
}


# Planted mistakes in the rounded rotation, made in the oracle's source text.
SOURCE_MUTATIONS = {
    "cos/sin left in fp32": ("cb, sb = round_to_bf16(c), round_to_bf16(s)", "cb, sb = c, s"),
    "products not rounded": ("a = round_to_bf16(xb * cb)", "a = xb * cb"),
    "one rounding of the whole rotation": ("return round_to_bf16(a + b)",
                                           "return round_to_bf16(xb * c + rotate_half(xb) * s)"),
    "sum left unrounded": ("return round_to_bf16(a + b)", "return a + b"),
}


def _source_mutant(old, new):
    src = open(os.path.join(ROOT, "oracle", "gqa_oracle.py")).read()
    assert src.count(old) == 1, old
    spec = importlib.util.spec_from_loader("_oracle_src_mut", loader=None)
    m = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), "_oracle_src_mut", "exec"), m.__dict__)
    return m


@pytest.mark.parametrize("name", sorted(SOURCE_MUTATIONS))
def test_planted_rounding_mistake_is_caught(name, golden):
    m = _source_mutant(*SOURCE_MUTATIONS[name])
    assert _all_pins(m, golden) >= 1, f"no pin caught the planted mistake: {name}"


def test_unmutated_copy_passes_all_pins(golden):
    assert _all_pins(_fresh_oracle(), golden) == 0


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, golden):
    m = _fresh_oracle()
    MUTATIONS[name](m)
    assert _all_pins(m, golden) >= 1, f"no pin caught the planted mistake: {name}"
