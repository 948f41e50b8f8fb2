"""Backward pass on the GPU vs the fp64 oracle (gradients from the definition).

Tolerance, derived from the arithmetic: P and dS enter the tensor cores as
bf16 (relative rounding 2^-9), are accumulated in fp32, and dS also carries
the forward's bf16 O through D = dO . O.  Each gradient is compared relative
to its own scale: max |err| <= 3e-2 * max |ref| and mean |err| <= 1e-2 *
mean |ref|, with no NaN or Inf.  Where a gradient vanishes exactly (a row that
sees one key has dS = P (dP - D) = 0) the GPU's dP - D is a rounding residue,
so the scales have floors: 1e-3 for the max and 1e-4 for the mean.

Row by row as well: every gradient row (one key's dK / dV, one query's dQ, d
values) whose largest element is at least a tenth of the tensor's largest is
held to its own scale, max |err_row| <= 1.5e-2 * max |ref_row| for dK and dV
(each a sum of bf16 products with fp32 accumulation: a few units of 2^-9)
and 3e-2 for dQ, whose dS = P (dP - D) loses relative precision where dP and
D = dO . O (O rounded to bf16) nearly cancel.  Rows smaller than that are the
ones whose gradient (nearly) vanishes; the tensor-wide bound covers them.
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_29_b200.inputs import Workload, bf16_bits, make_qkv

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 3e-2, 1e-2
ROW_REL = {"dQ": 3e-2, "dK": 1.5e-2, "dV": 1.5e-2}
ROW_MIN = 0.1  # rows checked on their own scale: max |ref_row| >= ROW_MIN * max |ref|


def check_rows(tag, name, a, r):
    big = max(np.abs(r).max(), 1e-3)
    err = np.abs(a - r).max(axis=-1)
    rmax = np.abs(r).max(axis=-1)
    sel = rmax >= ROW_MIN * big
    if sel.any():
        worst = (err[sel] / rmax[sel]).max()
        assert worst <= ROW_REL[name], f"{tag} {name}: row-relative error {worst:.3g}"


@pytest.fixture(scope="module")
def fa2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_29_b200 as m
    return m


def grads_gpu(fa2, q, k, v, g, causal, scale):
    dev = torch.device("cuda")
    qd, kd, vd, gd = (t.to(dev) for t in (q, k, v, g))
    o, lse = fa2.attention(qd, kd, vd, causal=causal, softmax_scale=scale)
    dq, dk, dv = fa2.attention_backward(qd, kd, vd, o, lse, gd, causal=causal, softmax_scale=scale)
    torch.cuda.synchronize()
    assert fa2.fa2_debug_status(None) == 0
    return [t.float().cpu().numpy() for t in (dq, dk, dv)]


def check(fa2, w, scale=None):
    q, k, v = make_qkv(w)
    g = torch.randn(q.shape, generator=torch.Generator().manual_seed(w.seed + 99)).to(torch.bfloat16)
    scale = w.softmax_scale if scale is None else scale
    got = grads_gpu(fa2, q, k, v, g, w.causal, scale)
    ref = oracle.backward(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(g), w.causal, scale)
    for name, a, r in zip(("dQ", "dK", "dV"), got, ref):
        assert np.isfinite(a).all(), f"{w.name}: non-finite {name}"
        err = np.abs(a - r)
        big = max(np.abs(r).max(), 1e-3)
        assert err.max() <= MAX_REL * big, f"{w.name} {name}: max err {err.max():.3g} vs scale {big:.3g}"
        assert err.mean() <= MEAN_REL * max(np.abs(r).mean(), 1e-4), \
            f"{w.name} {name}: mean err {err.mean():.3g} vs mean {np.abs(r).mean():.3g}"
        check_rows(w.name, name, a, r)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(256, 256), (300, 300), (129, 700), (700, 129), (1, 200), (1000, 1000)])
def test_backward_vs_oracle(fa2, d, causal, nq, nk):
    check(fa2, Workload(f"bwd{nq}x{nk}", 2, 4, 2, nq, nk, d, causal, seed=nq * 5 + nk + d))


def test_backward_gqa_and_scale(fa2):
    check(fa2, Workload("bwd_gqa", 1, 8, 2, 512, 512, 128, True, seed=51), scale=0.2)
    check(fa2, Workload("bwd_neg", 1, 2, 2, 384, 384, 64, False, seed=52), scale=-0.1)


def test_backward_deterministic_dk_dv(fa2):
    # dK and dV are summed in tensor memory in a fixed order: bitwise repeatable
    w = Workload("bwd_det", 2, 4, 2, 640, 640, 128, True, seed=53)
    q, k, v = make_qkv(w)
    g = torch.randn(q.shape, generator=torch.Generator().manual_seed(54)).to(torch.bfloat16)
    a = grads_gpu(fa2, q, k, v, g, True, w.softmax_scale)
    b = grads_gpu(fa2, q, k, v, g, True, w.softmax_scale)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


@pytest.mark.parametrize("window", [(0, 0), (127, 0), (300, -1), (200, 100), (-1, 50)])
@pytest.mark.parametrize("d", [64, 128])
def test_backward_local_window(fa2, window, d):
    w = Workload("bwd_loc", 2, 4, 2, 700, 650, d, False, seed=60 + d)
    q, k, v = make_qkv(w)
    g = torch.randn(q.shape, generator=torch.Generator().manual_seed(61)).to(torch.bfloat16)
    dev = torch.device("cuda")
    qd, kd, vd, gd = (t.to(dev) for t in (q, k, v, g))
    o, lse = fa2.attention(qd, kd, vd, window=window)
    got = [t.float().cpu().numpy()
           for t in fa2.attention_backward(qd, kd, vd, o, lse, gd, window=window)]
    torch.cuda.synchronize()
    assert fa2.fa2_debug_status(None) == 0
    ref = oracle.backward(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(g), False,
                          w.softmax_scale, window=window)
    for name, a, r in zip(("dQ", "dK", "dV"), got, ref):
        assert np.isfinite(a).all(), f"{window} non-finite {name}"
        err = np.abs(a - r)
        big = max(np.abs(r).max(), 1e-3)
        assert err.max() <= MAX_REL * big, f"{window} {name}: max err {err.max():.3g} vs {big:.3g}"
        assert err.mean() <= MEAN_REL * max(np.abs(r).mean(), 1e-4), f"{window} {name}: mean err"
        check_rows(str(window), name, a, r)


@pytest.mark.parametrize("name,b,hk", [("causal_8k", 1, 5), ("gqa_4k", 2, 3)])
def test_backward_full_size_one_group(fa2, name, b, hk):
    # The full-size problem exactly as the benchmark times it, checked on one
    # (batch, KV head) slice: dK and dV of a KV head depend only on its group
    # of query heads, and dQ of a query head only on its KV head, so the
    # slice's gradients are the oracle's on the sliced problem.
    from exact_tiled_attention_29_b200.inputs import WORKLOADS
    w = WORKLOADS[name]
    q, k, v = make_qkv(w)
    g = torch.randn(q.shape, generator=torch.Generator().manual_seed(w.seed + 99)).to(torch.bfloat16)
    got = grads_gpu(fa2, q, k, v, g, w.causal, w.softmax_scale)
    grp = w.Hq // w.Hkv
    hs = slice(hk * grp, (hk + 1) * grp)
    qs, gs = q[b:b + 1, :, hs].contiguous(), g[b:b + 1, :, hs].contiguous()
    ks, vs = k[b:b + 1, :, hk:hk + 1].contiguous(), v[b:b + 1, :, hk:hk + 1].contiguous()
    ref = oracle.backward(bf16_bits(qs), bf16_bits(ks), bf16_bits(vs), bf16_bits(gs), w.causal, w.softmax_scale)
    sl = [got[0][b:b + 1, :, hs], got[1][b:b + 1, :, hk:hk + 1], got[2][b:b + 1, :, hk:hk + 1]]
    for nm, a, r in zip(("dQ", "dK", "dV"), sl, ref):
        assert np.isfinite(a).all(), f"{name}: non-finite {nm}"
        err = np.abs(a - r)
        big = max(np.abs(r).max(), 1e-3)
        assert err.max() <= MAX_REL * big, f"{name} {nm}: max err {err.max():.3g} vs scale {big:.3g}"
        assert err.mean() <= MEAN_REL * max(np.abs(r).mean(), 1e-4), f"{name} {nm}: mean err"
        check_rows(name, nm, a, r)
