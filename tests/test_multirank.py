"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks check the
per-rank seeding (independent batches) and the max-over-ranks timing reduction
that turns per-rank step times into one whole-job throughput."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q_out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from exact_tiled_attention_29_b200.inputs import WORKLOADS, make_qkv
        w = WORKLOADS["tiny"]
        q, _, _ = make_qkv(w, seed=bench.rank_seed(w, rank))
        # every rank reports a different step time; all must agree on the max
        local = [1.0 + rank, 10.0 - rank]
        got = bench.max_over_ranks(local)
        value = bench.throughput_tflops(w, world, got[0])
        q_out.put((rank, float(q_checksum(q)), got, value))
    finally:
        dist.destroy_process_group()


def q_checksum(t):
    return t.float().sum().item()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, c0, g0, v0), (r1, c1, g1, v1) = res
    assert g0 == g1 == [2.0, 10.0]
    assert v0 == v1
    assert c0 != c1  # independent batches per rank
    from exact_tiled_attention_29_b200.inputs import WORKLOADS
    import bench
    assert v0 == pytest.approx(2 * WORKLOADS["tiny"].flops() / 2.0e-3 / 1e12)


def test_single_process_reduction_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]
