"""One process calling the library on two GPUs in turn.

Kernel set-up (the raised dynamic shared-memory limit, the register check)
is a per-device property; a call on the second device must launch as well as
the first.  The same inputs on both devices give bit-identical results (the
kernels are deterministic).  Skipped unless the process sees two devices.
"""

import pytest
import torch

from exact_tiled_attention_29_b200.inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu


def _forward_on(fa2, dev, q, k, v, w):
    with torch.cuda.device(dev):
        qd, kd, vd = (t.to(dev) for t in (q, k, v))
        o = torch.empty_like(qd)
        lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
        st = fa2.fa2_forward(qd, kd, vd, o, lse, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                             w.softmax_scale, torch.cuda.current_stream(dev))
        assert st == 0, fa2.fa2_status_string(st)
        ws = torch.empty(fa2.fa2_backward_workspace_size(w.B, w.Hq, w.Nq, w.d), dtype=torch.uint8,
                         device=dev)
        g = torch.ones_like(qd)
        dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
        st = fa2.fa2_backward(qd, kd, vd, o, lse, g, dq, dk, dv, w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d,
                              w.causal, w.softmax_scale, ws, ws.numel(), torch.cuda.current_stream(dev))
        assert st == 0, fa2.fa2_status_string(st)
        torch.cuda.synchronize(dev)
        return o.cpu(), lse.cpu(), dk.cpu(), dv.cpu()


def test_second_device_gets_its_own_setup():
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two CUDA devices")
    import exact_tiled_attention_29_b200 as fa2
    w = Workload("two_dev", 1, 4, 2, 700, 700, 128, True, seed=5)
    q, k, v = make_qkv(w)
    r0 = _forward_on(fa2, torch.device("cuda", 0), q, k, v, w)
    r1 = _forward_on(fa2, torch.device("cuda", 1), q, k, v, w)
    for a, b in zip(r0, r1):
        assert torch.equal(a, b)
