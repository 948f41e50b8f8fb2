"""fa2_forward_static_ws: stream-K with the library's fixed scratch array.

Collected last on purpose (file name), and independent of every other test:
it must pass alone and after the rest of the suite.  On the GPU it is
compared, bit for bit, with fa2_forward_ws on a caller workspace (the same
kernels and schedule) over two calls in a row with different inputs, and
within the parity tolerance with fa2_forward; the device's free memory must
not change across the calls.  On the CPU, validation and the capacity rule.
"""

import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_29_b200 as fa2
from exact_tiled_attention_29_b200.inputs import Workload, make_qkv

BLOCK_M = 128


def call_static(q, k, v, o, lse, w, stream=None):
    return fa2.fa2_forward_static_ws(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                                     w.softmax_scale, stream)


def test_static_validation_before_any_cuda_call():
    w = Workload("v", 1, 2, 1, 5, 7, 128, True, seed=0)
    args = dict(q=16, k=32, v=48, o=64, lse=80)
    assert call_static(0, 32, 48, 64, 80, w) == 1
    assert fa2.fa2_forward_static_ws(16, 32, 48, 64, 80, 1, 3, 2, 5, 7, 128, 1, 0.1, None) == 2
    assert fa2.fa2_forward_static_ws(16, 32, 48, 64, 80, 1, 2, 1, 5, 7, 96, 1, 0.1, None) == 3
    assert fa2.fa2_forward_static_ws(16, 32, 48, 64, 80, 1, 2, 1, 5, 7, 128, 1, math.nan, None) == 5
    # misaligned q / o (16 bytes) or lse (4 bytes): refused before the device is touched
    assert fa2.fa2_forward_static_ws(24, 32, 48, 64, 80, 1, 2, 1, 5, 7, 128, 1, 0.1, None) == 4
    assert fa2.fa2_forward_static_ws(16, 32, 48, 72, 80, 1, 2, 1, 5, 7, 128, 1, 0.1, None) == 4
    assert fa2.fa2_forward_static_ws(16, 32, 48, 64, 82, 1, 2, 1, 5, 7, 128, 1, 0.1, None) == 4
    if not torch.cuda.is_available():
        assert call_static(args["q"], args["k"], args["v"], args["o"], args["lse"], w) == 6


def test_static_capacity_covers_this_gpu_class():
    # two fp32 partials of 2 x 128 x (d + 3) floats per SM: 156 SMs fit at d = 128, 157 do not
    for d in (64, 128):
        st, _, G, ws = fa2.fa2_streamk_plan(1, 1, 1, 256, 1 << 20, d, 0, 156)
        assert st == 0 and G == 156 and ws <= fa2.FA2_STATIC_WS_BYTES
    st, _, G, ws = fa2.fa2_streamk_plan(1, 1, 1, 256, 1 << 20, 128, 0, 157)
    assert st == 0 and ws > fa2.FA2_STATIC_WS_BYTES


@pytest.mark.gpu
def test_static_matches_caller_workspace_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    shapes = [Workload("na1", 2, 16, 16, 4096, 4096, 128, True, seed=31),   # many split units
              Workload("na2", 1, 4, 2, 256, 30000, 64, False, seed=32)]     # short query, long keys
    for w in shapes:
        inputs = [tuple(t.to(dev) for t in make_qkv(Workload(w.name, w.B, w.Hq, w.Hkv, w.Nq, w.Nk,
                                                                w.d, w.causal, seed=w.seed + i)))
                  for i in range(2)]
        outs = [(torch.empty_like(q), torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev))
                for q, _, _ in inputs]
        # first call on the device (looks the array up), then the measured pair
        assert call_static(*inputs[0], *outs[0], w, stream) == 0
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        for (q, k, v), (o, lse) in zip(inputs, outs):
            assert call_static(q, k, v, o, lse, w, stream) == 0
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free1 == free0, "the allocation-free call changed the device's free memory"
        assert fa2.fa2_debug_status(None) == 0
        ws = fa2.alloc_workspace(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, dev)
        for (q, k, v), (o, lse) in zip(inputs, outs):
            o_ws, l_ws = torch.empty_like(o), torch.empty_like(lse)
            st = fa2.fa2_forward_ws(q, k, v, o_ws, l_ws, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                                    w.causal, w.softmax_scale, ws, ws.numel(), stream)
            assert st == 0
            o_u, l_u = torch.empty_like(o), torch.empty_like(lse)
            st = fa2.fa2_forward(q, k, v, o_u, l_u, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                                 w.softmax_scale, stream)
            assert st == 0
            torch.cuda.synchronize()
            assert torch.equal(o, o_ws) and torch.equal(lse, l_ws)
            assert (o.float() - o_u.float()).abs().max().item() <= 1.6e-2
            assert (lse - l_u).abs().max().item() <= 1e-4
        assert fa2.fa2_debug_status(None) == 0
