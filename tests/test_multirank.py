"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks check the
per-rank seeding, the max-over-ranks timing reduction that turns per-rank
step times into one whole-job throughput, and that splitting one problem's
KV-head groups over the ranks needs no exchange: each rank's oracle result on
its heads, gathered, equals the oracle on the whole problem bit for bit
("FlashAttention-2: expose enough parallel work" on the independence of
(batch, head) problems)."""

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


def _shard_worker(rank, world, port, q_out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from exact_tiled_attention_29_b200.inputs import Workload, bf16_bits, make_qkv
        w = Workload("shard", 2, 4, 2, 96, 80, 64, True, seed=11)   # GQA, Nq != Nk, causal
        q, k, v = make_qkv(w, seed=bench.rank_seed(w, rank))
        o, lse = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal, w.softmax_scale)
        # gather every rank's head slice (the benchmark itself gathers nothing)
        o_all = [torch.empty(o.shape, dtype=torch.float64) for _ in range(world)]
        l_all = [torch.empty(lse.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(o_all, torch.from_numpy(o))
        dist.all_gather(l_all, torch.from_numpy(lse))
        if rank == 0:
            q_out.put((torch.cat(o_all, dim=2).numpy(), torch.cat(l_all, dim=1).numpy()))
    finally:
        dist.destroy_process_group()


def test_head_groups_split_over_two_ranks_reassemble_the_whole_problem():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    o_got, l_got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import numpy as np
    import oracle
    from exact_tiled_attention_29_b200.inputs import (Workload, bf16_bits, global_workload,
                                                      make_global_qkv, make_qkv)
    w = Workload("shard", 2, 4, 2, 96, 80, 64, True, seed=11)
    g = global_workload(w, 2)
    assert (g.Hq, g.Hkv) == (8, 4)
    qg, kg, vg = make_global_qkv(w, 2)
    assert qg.shape == (2, 96, 8, 64) and kg.shape == (2, 80, 4, 64)
    # rank 0's slice is the single-GPU workload's own inputs
    assert torch.equal(qg[:, :, :4], make_qkv(w)[0])
    o_ref, l_ref = oracle.attention(bf16_bits(qg), bf16_bits(kg), bf16_bits(vg), g.causal, g.softmax_scale)
    assert np.array_equal(o_got, o_ref)
    assert np.array_equal(np.isneginf(l_got), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    assert np.array_equal(l_got[fin], l_ref[fin])


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
