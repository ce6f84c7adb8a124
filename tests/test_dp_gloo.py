"""Data-parallel host logic on CPU: two gloo ranks, each with its own token
shard, sum their per-rank gradients with dora_weight_decomposed_b200.dp and
must get the gradients of the whole batch. The per-rank gradients come from
the CPU oracle (no GPU here); on GPUs bench.py runs the same exchange over
NCCL after the library's backward.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

from dora_weight_decomposed_b200.dp import token_shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, T, q):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from dora_inputs import make_inputs, workload
    from dora_weight_decomposed_b200.dp import allreduce_gradients, token_shard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = workload("c2", d_out=48, d_in=40, r=8, T=T)
        inp = make_inputs(wl)
        a, b = token_shard(T, rank, world)
        W0, A, B, m, s = (inp[k] for k in ("W0", "A", "B", "m", "s"))
        local = oracle.backward(inp["dy"][a:b], inp["x"][a:b], W0, A, B, m, s)
        dm, dA, dB = (torch.from_numpy(np.ascontiguousarray(local[k])) for k in ("dm", "dA", "dB"))
        allreduce_gradients(dm, dA, dB)
        full = oracle.backward(inp["dy"], inp["x"], W0, A, B, m, s)
        errs = {k: float(np.max(np.abs(v.numpy() - full[k])) / max(1e-30, np.max(np.abs(full[k]))))
                for k, v in (("dm", dm), ("dA", dA), ("dB", dB))}
        errs["dx"] = float(np.max(np.abs(local["dx"] - full["dx"][a:b])))
        q.put((rank, errs, (a, b)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T", [10, 7])
def test_two_rank_gradient_sum_matches_full_batch(T):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, T, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shards = sorted(r[2] for r in results)
    assert shards[0][0] == 0 and shards[0][1] == shards[1][0] and shards[1][1] == T
    for rank, errs, _ in results:
        for k, e in errs.items():
            assert e <= 1e-12, f"rank {rank} {k}: {e}"


def test_token_shard_covers_batch():
    for T in (0, 1, 5, 4096, 4097):
        for world in (1, 2, 3, 8):
            spans = [token_shard(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        token_shard(4, 2, 2)
