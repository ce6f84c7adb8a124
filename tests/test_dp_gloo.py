"""Data-parallel host logic on CPU: gloo ranks, each with its own token
shard, sum their per-rank gradients with dora_weight_decomposed_b200.dp and
must get the gradients of the whole batch. The per-rank gradients come from
the CPU oracle (no GPU here); on GPUs bench.py runs the same exchange over
NCCL after the library's backward. With four ranks the per-rank gradients are
rounded to bf16 as the library stores them: the sum must then be rounded only
once (float32 all-reduce), not once per hop as a bf16 all-reduce would.
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


def _bf16_rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from dora_inputs import make_inputs, round_to_bf16, workload
    from dora_weight_decomposed_b200.dp import allreduce_gradients, token_shard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T = 64
        wl = workload("c2", d_out=48, d_in=40, r=8, T=T)
        inp = make_inputs(wl)
        W0, A, B, m, s = (inp[k] for k in ("W0", "A", "B", "m", "s"))
        per_rank = []
        for q_rank in range(world):  # every rank's bf16 gradients, to form the exact sum here
            a, b = token_shard(T, q_rank, world)
            gr = oracle.backward(inp["dy"][a:b], inp["x"][a:b], W0, A, B, m, s)
            per_rank.append({k: round_to_bf16(gr[k]).astype(np.float64) for k in ("dA", "dB")} |
                            {"dm": gr["dm"].astype(np.float32).astype(np.float64)})
        mine = per_rank[rank]
        dm = torch.from_numpy(mine["dm"].astype(np.float32))
        dA = torch.from_numpy(mine["dA"].astype(np.float32)).to(torch.bfloat16)
        dB = torch.from_numpy(mine["dB"].astype(np.float32)).to(torch.bfloat16)
        allreduce_gradients(dm, dA, dB)
        res = {}
        for k, t in (("dm", dm), ("dA", dA), ("dB", dB)):
            exact = sum(p[k] for p in per_rank)
            mag = sum(np.abs(p[k]) for p in per_rank)
            u = 2.0 ** -8 if k != "dm" else 2.0 ** -24
            got = t.float().numpy().astype(np.float64)
            # one rounding to the storage type + float32 summation of `world` terms
            bound = u * np.abs(exact) + world * 2.0 ** -24 * mag
            res[k] = float(np.max(np.abs(got - exact) / np.maximum(bound, 1e-300)))
            # what a bf16 sum in ring order would give: a rounding after every addition
            if k != "dm":
                acc = per_rank[0][k]
                for p in per_rank[1:]:
                    acc = round_to_bf16(acc + p[k]).astype(np.float64)
                res[k + "_bf16_ring_worst"] = float(np.max(np.abs(acc - exact) / np.maximum(bound, 1e-300)))
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_four_rank_bf16_gradients_are_rounded_once():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 4
    procs = [ctx.Process(target=_bf16_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, res in results:
        for k in ("dm", "dA", "dB"):
            assert res[k] <= 1.0, f"rank {rank} {k}: error {res[k]:.2f} x the one-rounding bound"
        # The test can tell the two apart: rounding at every hop leaves the bound somewhere.
        assert max(res["dA_bf16_ring_worst"], res["dB_bf16_ring_worst"]) > 1.0
