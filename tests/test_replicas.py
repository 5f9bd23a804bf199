"""The multi-process path on CPU: two gloo ranks, replica seeds, the
max-over-ranks timing reduction the benchmark uses, and the oracle run
independently per replica (the path has no data-path collective)."""
import os
import socket

import numpy as np
import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from transformer_attention_gqa_b200 import replicas, workloads as wl
    import oracle.gqa_oracle as orc

    replicas.init("gloo", timeout_s=60)
    r, w, lr = replicas.env_rank()
    assert (r, w, lr) == (rank, world, rank)
    # each replica computes its own batch; nothing is exchanged
    inp = wl.make_inputs(wl.Workload("rep", (40, 24), 4, 2, 16, 1e4), seed=replicas.replica_seed(7, rank))
    out, lse = orc.gqa_rope_attention(inp.q, inp.k, inp.v, inp.cu_seqlens, 4, 2, 1e4)
    replicas.barrier()
    t = replicas.max_over_ranks([1.0 + rank, 10.0 - rank])
    results[rank] = (t, float(np.sum(out)), replicas.replica_seed(7, rank))
    replicas.shutdown()


def test_two_gloo_ranks():
    import torch.multiprocessing as mp

    port = _free_port()
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(2, port, results), nprocs=2, join=True)
    assert results[0][0] == results[1][0] == [2.0, 10.0]
    assert results[0][2] != results[1][2]
    assert results[0][1] != results[1][1]  # different replica batches


def test_single_process_is_a_noop():
    from transformer_attention_gqa_b200 import replicas

    os.environ.pop("WORLD_SIZE", None)
    replicas.init("gloo")
    assert replicas.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
