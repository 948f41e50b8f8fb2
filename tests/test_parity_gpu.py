"""GPU forward pass vs the fp64 oracle, element by element, through the C ABI.

Every case runs under both schedules: one thread block per unit
(``fa2_forward``) and stream-K over a workspace (``fa2_forward_ws``), which on
a 148-SM GPU splits the units of every workload here that has more than one
unit's worth of iterations per SM or fewer units than SMs.

Tolerances (on every compared row): O max-abs <= 2e-2 and mean-abs <= 2e-3,
LSE max-abs <= 1e-3, no NaN/Inf where the oracle is finite.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_29_b200.inputs import WORKLOADS, Workload, bf16_bits, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module")
def fa2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_29_b200 as m
    return m


@pytest.fixture(params=["units", "streamk"])
def sched(request):
    return request.param


def run_gpu(fa2, q, k, v, causal, scale, guard=0, sched="units"):
    """Run the C-ABI forward on copies of q, k, v; O and LSE are carved out of
    NaN-filled buffers with `guard` poisoned elements on both sides.  Under
    stream-K the workspace starts filled with NaN: it is scratch and must not
    leak into the result."""
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev).contiguous() for t in (q, k, v))
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    g_o = guard * d  # keep 16-byte alignment of the O view
    o_buf = torch.full((B * Nq * Hq * d + 2 * g_o,), float("nan"), dtype=torch.bfloat16, device=dev)
    l_buf = torch.full((B * Hq * Nq + 2 * max(guard, 4),), float("nan"), dtype=torch.float32, device=dev)
    gl = max(guard, 4)
    o = o_buf[g_o:g_o + B * Nq * Hq * d].view(B, Nq, Hq, d)
    lse = l_buf[gl:gl + B * Hq * Nq].view(B, Hq, Nq)
    ws = None
    if sched == "units":
        st = fa2.fa2_forward(qd, kd, vd, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                             torch.cuda.current_stream())
    else:
        ws = fa2.alloc_workspace(B, Hq, Hkv, Nq, Nk, d, causal, dev)
        ws.fill_(0xFF)  # every float in it reads as NaN
        st = fa2.fa2_forward_ws(qd, kd, vd, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, ws,
                                ws.numel(), torch.cuda.current_stream())
    assert st == 0, fa2.fa2_status_string(st)
    torch.cuda.synchronize()
    assert fa2.fa2_debug_status(None) == 0
    if guard:
        assert torch.isnan(o_buf[:g_o].float()).all() and torch.isnan(o_buf[-g_o:].float()).all(), \
            "O guard band overwritten"
    assert torch.isnan(l_buf[:gl]).all() and torch.isnan(l_buf[-gl:]).all(), "LSE guard band overwritten"
    return o.float().cpu().numpy(), lse.cpu().numpy()


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """o_* [B,R,Hq,d], lse_* [B,Hq,R] on the same rows."""
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), np.isneginf(lse_ref)), f"{what}: -inf pattern of LSE"
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite O"
    assert not np.isnan(lse_gpu).any(), f"{what}: NaN LSE"
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= O_MAX, f"{what}: O max-abs {err.max():.3g}"
    assert err.mean() <= O_MEAN, f"{what}: O mean-abs {err.mean():.3g}"
    if fin.any():
        lerr = np.abs(lse_gpu[fin] - lse_ref[fin]).max()
        assert lerr <= LSE_MAX, f"{what}: LSE max-abs {lerr:.3g}"
    return float(err.max()), float(err.mean())


def check_case(fa2, w: Workload, rows=None, scale=None, guard=0, sched="units"):
    q, k, v = make_qkv(w)
    scale = w.softmax_scale if scale is None else scale
    o_gpu, lse_gpu = run_gpu(fa2, q, k, v, w.causal, scale, guard=guard, sched=sched)
    o_ref, lse_ref = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal, scale,
                                      rows=rows)
    if rows is not None:
        o_gpu, lse_gpu = o_gpu[:, rows], lse_gpu[:, :, rows]
    return compare(o_gpu, lse_gpu, o_ref, lse_ref, what=f"{w.name}/{sched}")


# ---- the five specified workloads, in the launch configuration the benchmark times ----

def test_tiny_all_rows(fa2, sched):
    check_case(fa2, WORKLOADS["tiny"], guard=8, sched=sched)


def test_noncausal_2k_all_rows(fa2, sched):
    check_case(fa2, WORKLOADS["noncausal_2k"], sched=sched)


@pytest.mark.parametrize("name", ["causal_8k", "long_32k", "gqa_4k"])
def test_full_size_sampled_rows(fa2, name, sched):
    w = WORKLOADS[name]
    idx = list(WORKLOADS).index(name)
    rows = sample_rows(w, 1024, seed=idx)
    check_case(fa2, w, rows=rows, sched=sched)


# ---- ragged and odd sizes, both head dims, Nq != Nk in both directions ----

ODD = [1, 17, 127, 129, 1000]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(n, n) for n in ODD] + [(17, 1000), (1000, 17), (129, 127),
                                                            (127, 129), (1, 1000), (300, 1)])
def test_odd_sizes(fa2, d, causal, nq, nk, sched):
    w = Workload(f"odd{nq}x{nk}", 2, 4, 2, nq, nk, d, causal, seed=nq * 7 + nk)
    check_case(fa2, w, guard=8, sched=sched)


@pytest.mark.parametrize("scale", [0.0, -0.0883883, 0.5])
def test_scale_values(fa2, scale, sched):
    w = Workload("scale", 1, 2, 1, 300, 300, 128, True, seed=3)
    check_case(fa2, w, scale=scale, sched=sched)


def test_large_scores_outliers_d64(fa2, sched):
    w = Workload("outl64", 1, 2, 2, 2048, 2048, 64, True, seed=5, outlier_frac=0.01, outlier_scale=8.0)
    check_case(fa2, w, sched=sched)


@pytest.mark.parametrize("d", [64, 128])
def test_one_long_unit_cut_into_many_pieces(fa2, d, sched):
    # one query block against 64k keys: stream-K cuts the single unit at every
    # SM's range boundary and merges ~148 partials
    w = Workload("longkv", 1, 1, 1, 256, 65536, d, False, seed=21)
    check_case(fa2, w, sched=sched)


def test_causal_more_queries_than_keys_streamk_rows(fa2, sched):
    # Nq > Nk causal: leading query blocks see no key (empty units written
    # outside the stream-K ranges) while the rest are split
    w = Workload("nq>nk", 2, 3, 1, 3000, 1100, 128, True, seed=22)
    check_case(fa2, w, guard=8, sched=sched)


# ---- closed forms on the GPU ----

def test_causal_row0_is_v0_bitwise(fa2, sched):
    w = Workload("row0", 2, 4, 2, 384, 384, 128, True, seed=9)
    q, k, v = make_qkv(w)
    o, lse = run_gpu(fa2, q, k, v, True, w.softmax_scale, sched=sched)
    vv = v.float().numpy()
    for hq in range(4):
        assert np.array_equal(o[:, 0, hq], vv[:, 0, hq // 2]), "row 0 must be exactly V[0]"
    qk = np.einsum("bhc,bhc->bh", q.double().numpy()[:, 0], np.repeat(k.double().numpy()[:, 0], 2, axis=1))
    assert np.abs(lse[:, :, 0] - w.softmax_scale * qk).max() < 1e-3


def test_zero_query_gives_mean_of_visible_v(fa2, sched):
    w = Workload("q0", 1, 2, 2, 260, 260, 64, True, seed=10)
    q, k, v = make_qkv(w)
    q = torch.zeros_like(q)
    o, lse = run_gpu(fa2, q, k, v, True, w.softmax_scale, sched=sched)
    vv = v.double().numpy()
    csum = np.cumsum(vv, axis=1) / np.arange(1, 261)[None, :, None, None]
    assert np.abs(o - csum).max() < 2e-2
    assert np.abs(lse - np.log(np.arange(1, 261))[None, None, :]).max() < 1e-3


# ---- structural properties ----

def test_gqa_equals_repeated_heads_bitwise(fa2, sched):
    w = Workload("gqa", 2, 8, 2, 700, 700, 128, True, seed=12)
    q, k, v = make_qkv(w)
    o1, l1 = run_gpu(fa2, q, k, v, True, w.softmax_scale, sched=sched)
    o2, l2 = run_gpu(fa2, q, k.repeat_interleave(4, dim=2), v.repeat_interleave(4, dim=2), True,
                     w.softmax_scale, sched=sched)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_deterministic_across_runs(fa2, sched):
    # stream-K merges the pieces of a split unit in their order in the unit,
    # whichever CTA finishes last, so it is deterministic too
    w = Workload("det", 2, 4, 4, 1500, 1500, 128, True, seed=13)
    q, k, v = make_qkv(w)
    outs = [run_gpu(fa2, q, k, v, True, w.softmax_scale, sched=sched) for _ in range(3)]
    for o, l in outs[1:]:
        assert np.array_equal(o, outs[0][0]) and np.array_equal(l, outs[0][1])


def test_torch_convenience_wrapper(fa2):
    w = Workload("wrap", 1, 4, 2, 333, 444, 64, False, seed=14)
    q, k, v = make_qkv(w)
    o, lse = fa2.attention(q.cuda(), k.cuda(), v.cuda(), causal=False)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), False, w.softmax_scale)
    compare(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, what="wrapper")


def test_streamk_matches_units_closely(fa2):
    # same arithmetic per key tile; only the split units' merge rounds differently
    w = Workload("sk_vs_u", 2, 16, 16, 4096, 4096, 128, True, seed=23)
    q, k, v = make_qkv(w)
    o1, l1 = run_gpu(fa2, q, k, v, True, w.softmax_scale, sched="units")
    o2, l2 = run_gpu(fa2, q, k, v, True, w.softmax_scale, sched="streamk")
    assert np.abs(o1 - o2).max() <= 1.6e-2
    assert np.abs(l1 - l2).max() <= 1e-4


def test_workspace_reused_across_calls_and_shapes(fa2):
    # one workspace, sized for the largest problem, serves calls of different
    # shapes ordered on one stream
    dev = torch.device("cuda")
    shapes = [Workload("r1", 2, 16, 16, 4096, 4096, 128, True, seed=24),
              Workload("r2", 1, 4, 2, 1000, 3000, 64, False, seed=25),
              Workload("r3", 2, 16, 16, 4096, 4096, 128, True, seed=24)]
    need = max(fa2.fa2_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal) for w in shapes)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=dev)
    outs = []
    for w in shapes:
        q, k, v = (t.to(dev) for t in make_qkv(w))
        o, lse = fa2.attention(q, k, v, causal=w.causal, workspace=ws)
        outs.append((o.float().cpu().numpy(), lse.cpu().numpy()))
    torch.cuda.synchronize()
    assert fa2.fa2_debug_status(None) == 0
    assert np.array_equal(outs[0][0], outs[2][0]) and np.array_equal(outs[0][1], outs[2][1])
    w = shapes[1]
    q, k, v = make_qkv(w)
    o_ref, l_ref = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal, w.softmax_scale)
    compare(outs[1][0], outs[1][1], o_ref, l_ref, what="reused workspace")


def test_small_workspace_is_refused(fa2):
    w = Workload("small_ws", 2, 16, 16, 4096, 4096, 128, True, seed=26)
    dev = torch.device("cuda")
    need = fa2.fa2_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal)
    assert need > 0
    q, k, v = (t.to(dev) for t in make_qkv(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(need - 256, dtype=torch.uint8, device=dev)
    st = fa2.fa2_forward_ws(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                            w.softmax_scale, ws, ws.numel(), torch.cuda.current_stream())
    assert st == 10


# ---- the persistent whole-unit schedule fa2_forward takes with >= 2 units per SM ----

@pytest.mark.parametrize("w", [
    Workload("pu_d64", 4, 16, 16, 2048, 2048, 64, False, seed=71),          # 512 units, d = 64
    Workload("pu_nq_gt_nk", 8, 8, 4, 3000, 1500, 64, True, seed=72),        # 768 units, leading ones empty
    Workload("pu_gqa_ragged", 3, 24, 6, 1900, 1900, 128, True, seed=73),    # 576 units, ragged tail
])
def test_persistent_units_schedule(fa2, w):
    st, units, _, _, _ = fa2.fa2_launch_plan(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)
    assert st == 0 and units >= 2 * torch.cuda.get_device_properties(0).multi_processor_count
    rows = sample_rows(w, 300, seed=74)
    check_case(fa2, w, rows=rows)


# ---- fa2_forward_auto: the schedule the library picks ----

@pytest.mark.parametrize("w", [
    Workload("auto_shortq", 1, 4, 4, 256, 8192, 128, False, seed=41),   # split-KV
    Workload("auto_units", 2, 8, 4, 2048, 2048, 64, True, seed=42),     # whole units
    Workload("auto_long_unit", 1, 1, 1, 300, 20000, 64, True, seed=43),
])
def test_auto_equals_the_schedule_it_picks(fa2, w):
    dev = torch.device("cuda")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    st, split, cu, cs = fa2.fa2_schedule_choice(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, sms)
    assert st == 0
    q, k, v = make_qkv(w)
    picked = run_gpu(fa2, q, k, v, w.causal, w.softmax_scale, sched="streamk" if split else "units")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    ws = fa2.alloc_workspace(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, dev)
    o, lse = fa2.attention(qd, kd, vd, causal=w.causal, workspace=ws, schedule="auto")
    o0 = torch.empty_like(qd)
    l0 = torch.empty_like(lse)
    st = fa2.fa2_forward_auto(qd, kd, vd, o0, l0, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                              w.softmax_scale, None, 0, torch.cuda.current_stream())
    assert st == 0
    torch.cuda.synchronize()
    assert fa2.fa2_debug_status(None) == 0
    # bit for bit the schedule it picked; with no workspace, whole units
    assert np.array_equal(o.float().cpu().numpy(), picked[0]) and np.array_equal(lse.cpu().numpy(), picked[1])
    units = run_gpu(fa2, q, k, v, w.causal, w.softmax_scale, sched="units")
    assert np.array_equal(o0.float().cpu().numpy(), units[0]) and np.array_equal(l0.cpu().numpy(), units[1])
    if w.name == "auto_shortq":
        assert split == 1
    if w.name == "auto_units":
        assert split == 0


def test_half_units_compute_the_same_bits(fa2):
    # 512 units on a 148-SM GPU: the last 68 run as single-tile halves on two
    # CTAs each.  A query tile's arithmetic does not depend on its partner
    # tile, so every batch element equals, bit for bit, its own launch (128
    # units: one block per unit, no halves).
    w = Workload("halves", 4, 16, 16, 2048, 2048, 128, False, seed=75)
    dev = torch.device("cuda")
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    st, start, units = fa2.fa2_persistent_plan(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, sms)
    assert st == 0
    if not any(u >> 13 for u in units):
        pytest.skip("no half units on this SM count")
    q, k, v = (t.to(dev) for t in make_qkv(w))
    o, lse = fa2.attention(q, k, v, causal=w.causal)
    for b in range(w.B):
        ob, lb = fa2.attention(q[b:b + 1].contiguous(), k[b:b + 1].contiguous(), v[b:b + 1].contiguous(),
                               causal=w.causal)
        assert torch.equal(o[b:b + 1], ob) and torch.equal(lse[b:b + 1], lb)
    torch.cuda.synchronize()
    assert fa2.fa2_debug_status(None) == 0


def test_more_units_than_the_plan_table(fa2):
    # 9216 units (> 8192, the plan table's size): the persistent blocks deal
    # units round robin, heaviest first, instead of following a host plan
    w = Workload("rr_units", 72, 16, 16, 2048, 2048, 64, True, seed=76)
    st, start, units = fa2.fa2_persistent_plan(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, 148)
    assert st == 8  # FA2_ERR_SIZE: no table
    rows = sample_rows(w, 48, seed=77)
    check_case(fa2, w, rows=rows)
