"""Local (sliding-window) attention on the GPU vs the fp64 oracle.

fa2_forward_local(window_left, window_right): key j visible to row i iff
g - left <= j <= g + right with g = i + Nk - Nq.  Same tolerances as the
other parity tests; the limits (-1, 0) and (-1, -1) must equal fa2_forward's
causal and full results bit for bit (same kernel, same tiles).
"""

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_29_b200.inputs import (EXTRA_WORKLOADS, Workload, bf16_bits, make_qkv,
                                                  sample_rows)

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module")
def fa2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_29_b200 as m
    return m


def run_local(fa2, q, k, v, window, scale):
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, Hq, Nq), float("nan"), dtype=torch.float32, device=dev)
    st = fa2.fa2_forward_local(qd, kd, vd, o, lse, B, Hq, Hkv, Nq, Nk, d, window[0], window[1],
                               scale, torch.cuda.current_stream())
    assert st == 0, fa2.fa2_status_string(st)
    torch.cuda.synchronize()
    assert fa2.fa2_debug_status(None) == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def run_plain(fa2, q, k, v, causal, scale):
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    o = torch.empty_like(qd)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    st = fa2.fa2_forward(qd, kd, vd, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                         torch.cuda.current_stream())
    assert st == 0
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), lse.cpu().numpy()


def compare(o, lse, o_ref, lse_ref, what):
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref)), f"{what}: -inf pattern of LSE"
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    err = np.abs(o - o_ref)
    assert err.max() <= O_MAX, f"{what}: O max-abs {err.max():.3g}"
    assert err.mean() <= O_MEAN, f"{what}: O mean-abs {err.mean():.3g}"
    fin = np.isfinite(lse_ref)
    if fin.any():
        assert np.abs(lse[fin] - lse_ref[fin]).max() <= LSE_MAX, f"{what}: LSE"


WINDOWS = [(0, 0), (127, 0), (128, 0), (300, -1), (-1, 300), (256, 256), (1000, 5), (5000, 5000)]
SHAPES = [(300, 300), (1000, 1000), (129, 1000), (1000, 129)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("nq,nk", SHAPES)
@pytest.mark.parametrize("window", WINDOWS)
def test_local_vs_oracle(fa2, d, nq, nk, window):
    w = Workload(f"loc{nq}x{nk}", 2, 4, 2, nq, nk, d, False, seed=nq + 3 * nk + d)
    q, k, v = make_qkv(w)
    o, lse = run_local(fa2, q, k, v, window, w.softmax_scale)
    o_ref, l_ref = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), False,
                                    w.softmax_scale, window=window)
    compare(o, lse, o_ref, l_ref, f"{w.name} window {window} d{d}")


def test_window_limits_equal_causal_and_full_bitwise(fa2):
    w = Workload("lim", 2, 8, 2, 1500, 1500, 128, False, seed=40)
    q, k, v = make_qkv(w)
    o_c, l_c = run_plain(fa2, q, k, v, True, w.softmax_scale)
    o_w, l_w = run_local(fa2, q, k, v, (-1, 0), w.softmax_scale)
    assert np.array_equal(o_c, o_w) and np.array_equal(l_c, l_w)
    o_f, l_f = run_plain(fa2, q, k, v, False, w.softmax_scale)
    o_w, l_w = run_local(fa2, q, k, v, (-1, -1), w.softmax_scale)
    assert np.array_equal(o_f, o_w) and np.array_equal(l_f, l_w)
    # widths beyond every key are no bound at all
    o_w, l_w = run_local(fa2, q, k, v, (1 << 20, 1 << 20), w.softmax_scale)
    assert np.array_equal(o_f, o_w) and np.array_equal(l_f, l_w)


def test_diagonal_window_is_v_of_the_diagonal_key(fa2):
    # width (0, 0): each row sees only its diagonal key, so O = V[g] exactly
    w = Workload("diag", 1, 4, 2, 700, 500, 128, False, seed=41)
    q, k, v = make_qkv(w)
    o, lse = run_local(fa2, q, k, v, (0, 0), w.softmax_scale)
    vv = v.float().numpy()
    for i in range(w.Nq):
        g = i + w.Nk - w.Nq
        for hq in range(w.Hq):
            if 0 <= g < w.Nk:
                assert np.array_equal(o[0, i, hq], vv[0, g, hq // 2])
            else:
                assert np.all(o[0, i, hq] == 0) and np.isneginf(lse[0, hq, i])


def test_local_8k_sampled_rows(fa2):
    w = EXTRA_WORKLOADS["local_8k"]
    q, k, v = make_qkv(w)
    window = (w.window_left, 0 if w.causal else w.window_right)
    o, lse = run_local(fa2, q, k, v, window, w.softmax_scale)
    rows = sample_rows(w, 1024, seed=7)
    o_ref, l_ref = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal,
                                    w.softmax_scale, rows=rows, window=(w.window_left, w.window_right))
    compare(o[:, rows], lse[:, :, rows], o_ref, l_ref, "local_8k")
