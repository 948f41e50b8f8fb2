"""The FMA-pipe exp2 option of the forward kernel, built and checked on the GPU.

The library is built a second time with FA2_EMU_PAIRS=2 (two of every sixteen
pairs of exponentials in an unmasked tile go through the Cody-Waite + cubic
polynomial on the FMA pipe instead of the MUFU; see tests/test_exp2_poly.py
for the polynomial against numpy) and compared with the fp64 oracle on the
sampled rows of the full-size causal workloads, at the same tolerances as the
default build.  ("FlashAttention 2: Three Places the Chip Was Still Waiting",
section 2.1: non-matmul work priced against matmul work; the option moves some
of it from the unit that computes exponentials to the one that multiplies.)
"""

import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_29_b200 import build as cuda_build
from exact_tiled_attention_29_b200.inputs import WORKLOADS, bf16_bits, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3


@pytest.fixture(scope="module")
def emu_lib(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = str(tmp_path_factory.mktemp("emu") / "libfa2_emu2.so")
    flags = [f for f in cuda_build.NVCC_FLAGS if f != "-v" and f != "-Xptxas"]
    cmd = [cuda_build.nvcc(), *flags, "-DFA2_EMU_PAIRS=2", "-o", out, *cuda_build.SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    lib = ctypes.CDLL(out, mode=os.RTLD_LOCAL)
    lib.fa2_forward.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 7 + [ctypes.c_float, ctypes.c_void_p]
    lib.fa2_forward.restype = ctypes.c_int
    lib.fa2_debug_status.argtypes = [ctypes.c_void_p]
    lib.fa2_debug_status.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("name", ["causal_8k", "long_32k"])
def test_emulated_exp2_parity(emu_lib, name):
    w = WORKLOADS[name]
    dev = torch.device("cuda")
    q, k, v = make_qkv(w)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    st = emu_lib.fa2_forward(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
                             w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, int(w.causal), w.softmax_scale, None)
    assert st == 0
    torch.cuda.synchronize()
    assert emu_lib.fa2_debug_status(None) == 0
    rows = sample_rows(w, 1024, seed=list(WORKLOADS).index(name))
    o_ref, lse_ref = oracle.attention(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal, w.softmax_scale,
                                      rows=rows)
    o_gpu = o.float().cpu().numpy()[:, rows]
    lse_gpu = lse.cpu().numpy()[:, :, rows]
    err = np.abs(o_gpu - o_ref)
    assert np.isfinite(o_gpu).all()
    assert err.max() <= O_MAX, err.max()
    assert err.mean() <= O_MEAN, err.mean()
    assert np.abs(lse_gpu - lse_ref).max() <= LSE_MAX
