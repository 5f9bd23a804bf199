"""The no-allocation entry point, gqa_rope_attn_fwd_noalloc.

Some callers cannot allocate device memory: code running as a plug-in of a
host application that owns every device allocation, or latency-critical
callers that cannot afford the device-wide synchronisation of
cudaMalloc/cudaFree. This entry point takes the same inputs and outputs as
gqa_rope_attn_fwd but keeps its scratch in a fixed-size device array inside
the library, so the caller passes no workspace. These tests call it through
the C ABI and compare it with the regular entry point. (This file is named
so that pytest collects it last.)"""
import numpy as np
import pytest

from tests.conftest import gpu_available
from tests import gpu_helpers as H
from transformer_attention_gqa_b200 import _abi
from transformer_attention_gqa_b200 import workloads as wl


def test_rejects_shapes_beyond_the_builtin_buffer():
    # 16384 tokens x 8 KV heads x d 128 needs ~42 MB of scratch > 32 MiB
    need = _abi.workspace_size(11, 16384, 32, 8, 128)
    assert need > _abi.NOALLOC_SCRATCH_BYTES
    A = 4096  # fake aligned addresses: the call returns before touching them
    rc = _abi.gqa_rope_attn_fwd_noalloc(A, A, A, 0, 5e5, A, 11, 16384, 32, 8, 128, 1, 0, A, 0, None)
    assert rc == _abi.GQA_ERR_NOALLOC_LIMIT
    assert "no-allocation" in _abi.strerror(rc)
    # invalid arguments keep their usual codes, still before any CUDA call
    assert _abi.gqa_rope_attn_fwd_noalloc(A, A, A, 0, 1e4, A, 1, 128, 4, 2, 96, 1, 0, A, 0, None) == \
        _abi.GQA_ERR_UNSUPPORTED
    assert _abi.gqa_rope_attn_fwd_noalloc(0, 0, 0, 0, 1e4, 0, 1, 0, 4, 2, 64, 1, 0, 0, 0, None) == _abi.GQA_OK


def _run(inp, noalloc, ws=None):
    import torch

    w = inp.workload
    q, k, v, cu, _ = H.to_device(inp)
    out = torch.empty_like(q)
    lse = torch.empty((w.n_q_heads, w.total_tokens), dtype=torch.float32, device="cuda")
    dt = _abi.GQA_DTYPE_FP32 if w.io_dtype == "fp32" else _abi.GQA_DTYPE_BF16
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, w.rope_theta, cu.data_ptr(), w.num_seqs, w.total_tokens,
            w.n_q_heads, w.n_kv_heads, w.head_dim, 1 if w.causal else 0, dt, out.data_ptr(), lse.data_ptr())
    stream = torch.cuda.current_stream().cuda_stream
    if noalloc:
        rc = _abi.gqa_rope_attn_fwd_noalloc(*args, stream)
    else:
        rc = _abi.gqa_rope_attn_fwd(*args, ws.data_ptr(), ws.numel(), stream)
    assert rc == _abi.GQA_OK, _abi.strerror(rc)
    torch.cuda.synchronize()
    assert _abi.get_device_status() == 0
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.gpu
@pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")
def test_noalloc_matches_regular_entry_point_on_two_calls():
    """Both entry points run the same deterministic kernels on the same
    inputs, so their outputs must be identical bit for bit; the first shape
    needs the larger scratch, so the second call runs over its leftovers."""
    import torch

    shapes = [wl.make_custom([900, 700], 16, 4, 128, 5e5, seed=41),
              wl.make_custom([640, 33, 90], 12, 4, 64, 1e4, seed=42)]
    sizes = [_abi.workspace_size(s.workload.num_seqs, s.workload.total_tokens, s.workload.n_q_heads,
                                 s.workload.n_kv_heads, s.workload.head_dim) for s in shapes]
    assert sizes[0] > sizes[1] and max(sizes) <= _abi.NOALLOC_SCRATCH_BYTES
    for inp, size in zip(shapes, sizes):  # two calls in a row
        ws = torch.empty(size, dtype=torch.uint8, device="cuda")
        ref_out, ref_lse = _run(inp, noalloc=False, ws=ws)
        out, lse = _run(inp, noalloc=True)
        assert np.array_equal(out, ref_out) and np.array_equal(lse, ref_lse)
        orc_out, orc_lse = H.oracle(inp)
        H.compare(out, lse, orc_out, orc_lse, what="no-alloc vs oracle")
