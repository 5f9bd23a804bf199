"""Seeded synthetic inputs for causal GQA + RoPE attention.

This module is shared by the tests, the benchmark and the float64 oracle's
checks. It only draws random numbers and lays them out; it holds none of the
attention or RoPE arithmetic. Every array it returns is a plain NumPy array, so
nothing here touches a GPU.

The five named workloads follow the shapes used throughout the pages' model
family (the "Attention from Scratch" page's GQA module with n_head query heads
sharing n_kv_groups key/value heads; the "Embeddings & the Residual Stream"
page's RoPE with theta = 500000 for the nano config) scaled to Llama-3-8B /
Qwen2.5-0.5B head layouts:

  tiny      B=1,  T=128,  n_q=4,  n_kv=2, d=32,  theta=1e4, fp32 I/O
  nano      B=16, T=512,  n_q=6,  n_kv=2, d=64,  theta=1e4
  qwen05b   B=4,  T=2048, n_q=14, n_kv=2, d=64,  theta=1e6, K scaled by 0.5
  llama8b   B=1,  T=8192, n_q=32, n_kv=8, d=128, theta=5e5
  varlen    16384 packed tokens, lengths ~ U{64..4096} (seed 0, last one
            truncated), n_q=32, n_kv=8, d=128, theta=5e5

Decoding workloads (one new token per sequence against a KV cache of
rotated keys; the "Kohaku-TT" page times a Qwen2.5-3B greedy decode):

  decode_llama8b  B=32, 4096 cached tokens each, n_q=32, n_kv=8, d=128,
                  theta=5e5 (537 MB of K and V read per step)
  decode_qwen3b   B=64, 8192 cached tokens each, n_q=16, n_kv=2, d=128,
                  theta=1e6 (Qwen2.5-3B head layout; 537 MB per step)
  decode_ragged   B=64, cached lengths ~ U{1..8191} (seed 5), n_q=32,
                  n_kv=8, d=128, theta=5e5
  decode_small    B=5, lengths 0, 1, 63, 64, 190 in a 200-row cache,
                  n_q=12, n_kv=4, d=64, theta=1e4
The cache holds standard-normal bf16 values in the rows before each
sequence's length (a rotation keeps that distribution, so no RoPE is applied
here) and NaN in the rows after it, which the step must never read.

Recipe: ``numpy.random.default_rng(seed)`` draws ``standard_normal`` float32
arrays in the order q, k, v; values are then rounded to bfloat16 (round to
nearest even, done by ``torch.Tensor.to(torch.bfloat16)``) because the kernel's
tensor-core operands are bf16. The tiny workload keeps fp32 buffers that hold
those bf16-representable values. Positions restart at 0 for every sequence.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "varlen_lengths",
    "make_inputs",
    "make_custom",
    "to_bf16_values",
    "DecodeWorkload",
    "DECODE_WORKLOADS",
    "DecodeInputs",
    "make_decode_inputs",
]


@dataclass(frozen=True)
class Workload:
    name: str
    seq_lens: tuple
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_theta: float
    causal: bool = True
    io_dtype: str = "bf16"  # "bf16" or "fp32"
    k_scale: float = 1.0
    seed: int = 0
    description: str = ""

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens)

    @property
    def group_size(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def flops(self) -> float:
        """Metric convention: 4*Tq*Tk*d per query head, halved when causal.

        For a packed batch this is summed per sequence: sum_i 4*L_i^2*d*n_q/2.
        """
        tot = 0.0
        for L in self.seq_lens:
            f = 4.0 * L * L * self.head_dim * self.n_q_heads
            tot += f / 2.0 if self.causal else f
        return tot

    def exps(self) -> float:
        """Exponentials by the same convention: one per (query, key, head)
        pair, T^2/2 pairs per head when causal (summed per sequence)."""
        tot = 0.0
        for L in self.seq_lens:
            e = float(L) * L * self.n_q_heads
            tot += e / 2.0 if self.causal else e
        return tot

    def io_bytes(self) -> int:
        """Algorithmic HBM bytes: read q, k, v once; write out once, lse once."""
        el = 4 if self.io_dtype == "fp32" else 2
        n = self.total_tokens
        d = self.head_dim
        qo = 2 * n * self.n_q_heads * d * el
        kv = 2 * n * self.n_kv_heads * d * el
        lse = n * self.n_q_heads * 4
        pos = n * 4
        return qo + kv + lse + pos


def varlen_lengths(total: int = 16384, lo: int = 64, hi: int = 4096, seed: int = 0) -> List[int]:
    """Sequence lengths drawn uniformly from lo..hi inclusive until they cover
    ``total`` tokens; the last one is truncated so the sum is exactly total."""
    rng = np.random.default_rng(seed)
    out: List[int] = []
    s = 0
    while s < total:
        x = int(rng.integers(lo, hi, endpoint=True))
        x = min(x, total - s)
        out.append(x)
        s += x
    return out


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", (128,), 4, 2, 32, 1e4, io_dtype="fp32", seed=0,
                     description="B=1 T=128 n_q=4 n_kv=2 d=32 theta=1e4 fp32 I/O causal"),
    "nano": Workload("nano", (512,) * 16, 6, 2, 64, 1e4, seed=1,
                     description="B=16 T=512 n_q=6 n_kv=2 d=64 theta=1e4 bf16 causal"),
    "qwen05b": Workload("qwen05b", (2048,) * 4, 14, 2, 64, 1e6, k_scale=0.5, seed=2,
                        description="B=4 T=2048 n_q=14 n_kv=2 d=64 theta=1e6 K*0.5 bf16 causal"),
    "llama8b": Workload("llama8b", (8192,), 32, 8, 128, 5e5, seed=3,
                        description="B=1 T=8192 n_q=32 n_kv=8 d=128 theta=5e5 bf16 causal"),
    "varlen": Workload("varlen", tuple(varlen_lengths()), 32, 8, 128, 5e5, seed=4,
                       description="packed 16384 tokens, L~U{64..4096} seed 0, n_q=32 n_kv=8 d=128 theta=5e5 causal"),
}


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even) and return
    them as float32. Uses torch's conversion; this is input preparation, not
    part of the method."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


@dataclass
class Inputs:
    workload: Workload
    q: np.ndarray  # [N, n_q, d] float32 holding bf16-representable values
    k: np.ndarray  # [N, n_kv, d]
    v: np.ndarray  # [N, n_kv, d]
    cu_seqlens: np.ndarray  # [num_seqs+1] int32
    positions: np.ndarray  # [N] int32, restarting at 0 per sequence
    extra: dict = field(default_factory=dict)


def _cu_and_positions(seq_lens):
    cu = np.zeros(len(seq_lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(seq_lens, dtype=np.int64)).astype(np.int32)
    pos = np.concatenate([np.arange(L, dtype=np.int32) for L in seq_lens]) if len(seq_lens) else np.zeros(0, np.int32)
    if pos.size == 0:
        pos = np.zeros(0, dtype=np.int32)
    return cu, pos


def make_custom(seq_lens, n_q_heads: int, n_kv_heads: int, head_dim: int, rope_theta: float = 1e4,
                causal: bool = True, seed: int = 0, k_scale: float = 1.0, io_dtype: str = "bf16",
                name: str = "custom") -> Inputs:
    w = Workload(name, tuple(int(x) for x in seq_lens), n_q_heads, n_kv_heads, head_dim, float(rope_theta),
                 causal=causal, io_dtype=io_dtype, k_scale=k_scale, seed=seed)
    return make_inputs(w)


def make_inputs(w: Workload, seed: Optional[int] = None) -> Inputs:
    rng = np.random.default_rng(w.seed if seed is None else seed)
    n = w.total_tokens
    d = w.head_dim
    q = rng.standard_normal((n, w.n_q_heads, d), dtype=np.float32)
    k = rng.standard_normal((n, w.n_kv_heads, d), dtype=np.float32)
    v = rng.standard_normal((n, w.n_kv_heads, d), dtype=np.float32)
    if w.k_scale != 1.0:
        k = (k * np.float32(w.k_scale)).astype(np.float32)
    q, k, v = to_bf16_values(q), to_bf16_values(k), to_bf16_values(v)
    cu, pos = _cu_and_positions(w.seq_lens)
    return Inputs(w, q, k, v, cu, pos)


def make_grad_output(inp: Inputs, seed: int = 1) -> np.ndarray:
    """Seeded upstream gradient dL/dout for the backward: standard normal
    values rounded to bf16, shape [N, n_q, d] like out."""
    w = inp.workload
    rng = np.random.default_rng(w.seed * 7919 + seed)
    return to_bf16_values(rng.standard_normal((w.total_tokens, w.n_q_heads, w.head_dim), dtype=np.float32))


@dataclass
class ProjectionInputs:
    x: np.ndarray       # [N, C] float32 holding bf16 values
    w_qkv: np.ndarray   # [(n_q + 2 n_kv) d, C] float32 holding bf16 values: rows of W_q, W_k, W_v
    cu_seqlens: np.ndarray
    positions: np.ndarray
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_theta: float


def make_projection_inputs(seq_lens, hidden: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                           rope_theta: float = 1e4, seed: int = 0) -> ProjectionInputs:
    """Seeded tokens x ~ N(0, 1) and stacked q/k/v projection weights ~
    N(0, 1/hidden) (the scale of randomly initialised linear layers, so the
    projections are of unit scale), both rounded to bf16."""
    rng = np.random.default_rng(seed)
    n = int(sum(seq_lens))
    f = (n_q_heads + 2 * n_kv_heads) * head_dim
    x = to_bf16_values(rng.standard_normal((n, hidden), dtype=np.float32))
    w = to_bf16_values(rng.standard_normal((f, hidden), dtype=np.float32) / np.float32(np.sqrt(hidden)))
    cu, pos = _cu_and_positions(seq_lens)
    return ProjectionInputs(x, w, cu, pos, n_q_heads, n_kv_heads, head_dim, float(rope_theta))


# ---------------------------------------------------------------- decoding

@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    cache_lens: tuple  # tokens already cached per sequence (the new token's position)
    max_cache_len: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    rope_theta: float
    seed: int = 0
    description: str = ""

    @property
    def batch(self) -> int:
        return len(self.cache_lens)

    def kv_bytes(self) -> int:
        """K and V bytes one step must read: p + 1 rows (p cached, one new)
        of n_kv heads x d bf16 each, per sequence."""
        return int(sum(p + 1 for p in self.cache_lens)) * self.n_kv_heads * self.head_dim * 2 * 2

    def step_bytes(self) -> int:
        """Algorithmic HBM bytes of one step: the K/V rows read, q / k_new /
        v_new read, the appended K/V rows and out written, lse written."""
        B, nq, nkv, d = self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim
        return self.kv_bytes() + B * (nq + 2 * nkv) * d * 2 + B * (2 * nkv + nq) * d * 2 + B * nq * 4

    def flops(self) -> float:
        """Scores and weighted sum: 4 * (p + 1) * d per query head."""
        return float(sum(4.0 * (p + 1) * self.head_dim * self.n_q_heads for p in self.cache_lens))


def _ragged_lens(n: int, lo: int, hi: int, seed: int) -> tuple:
    rng = np.random.default_rng(seed)
    return tuple(int(x) for x in rng.integers(lo, hi, size=n, endpoint=True))


DECODE_WORKLOADS: Dict[str, DecodeWorkload] = {
    "decode_llama8b": DecodeWorkload("decode_llama8b", (4096,) * 32, 4097, 32, 8, 128, 5e5, seed=6,
                                     description="B=32 cache 4096 n_q=32 n_kv=8 d=128 theta=5e5 bf16"),
    "decode_qwen3b": DecodeWorkload("decode_qwen3b", (8192,) * 64, 8193, 16, 2, 128, 1e6, seed=7,
                                    description="B=64 cache 8192 n_q=16 n_kv=2 d=128 theta=1e6 bf16"),
    "decode_ragged": DecodeWorkload("decode_ragged", _ragged_lens(64, 1, 8191, 5), 8192, 32, 8, 128, 5e5,
                                    seed=8, description="B=64 cache ~U{1..8191} n_q=32 n_kv=8 d=128 theta=5e5 bf16"),
    "decode_small": DecodeWorkload("decode_small", (0, 1, 63, 64, 190), 200, 12, 4, 64, 1e4, seed=9,
                                   description="B=5 cache 0,1,63,64,190 of 200 n_q=12 n_kv=4 d=64 theta=1e4 bf16"),
}


@dataclass
class DecodeInputs:
    workload: DecodeWorkload
    q: np.ndarray        # [B, n_q, d] float32 holding bf16 values
    k_new: np.ndarray    # [B, n_kv, d]
    v_new: np.ndarray    # [B, n_kv, d]
    k_cache: np.ndarray  # [B, max_len, n_kv, d]; NaN from each sequence's length on
    v_cache: np.ndarray
    cache_seqlens: np.ndarray  # [B] int32


def make_decode_inputs(w: DecodeWorkload, seed: Optional[int] = None, nan_tail: bool = True) -> DecodeInputs:
    rng = np.random.default_rng(w.seed if seed is None else seed)
    B, L, nq, nkv, d = w.batch, w.max_cache_len, w.n_q_heads, w.n_kv_heads, w.head_dim
    q = to_bf16_values(rng.standard_normal((B, nq, d), dtype=np.float32))
    kn = to_bf16_values(rng.standard_normal((B, nkv, d), dtype=np.float32))
    vn = to_bf16_values(rng.standard_normal((B, nkv, d), dtype=np.float32))
    kc = np.full((B, L, nkv, d), np.nan if nan_tail else 0.0, dtype=np.float32)
    vc = np.full((B, L, nkv, d), np.nan if nan_tail else 0.0, dtype=np.float32)
    for b, p in enumerate(w.cache_lens):
        kc[b, :p] = to_bf16_values(rng.standard_normal((p, nkv, d), dtype=np.float32))
        vc[b, :p] = to_bf16_values(rng.standard_normal((p, nkv, d), dtype=np.float32))
    lens = np.asarray(w.cache_lens, dtype=np.int32)
    return DecodeInputs(w, q, kn, vn, kc, vc, lens)
