"""ctypes binding of ``libfa2.so`` (the C ABI declared in ``include/fa2.h``).

Argument marshalling only: every step of the attention forward pass runs in
the CUDA library.  Importing this module loads the in-tree library and raises
``ImportError`` if it is missing -- there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa2.so")

FA2_OK = 0
STATUS_NAMES = {
    0: "FA2_OK", 1: "FA2_ERR_NULL_POINTER", 2: "FA2_ERR_BAD_SHAPE", 3: "FA2_ERR_HEAD_DIM",
    4: "FA2_ERR_ALIGNMENT", 5: "FA2_ERR_SCALE", 6: "FA2_ERR_DEVICE", 7: "FA2_ERR_LAUNCH",
    8: "FA2_ERR_SIZE", 9: "FA2_ERR_BUILD", 10: "FA2_ERR_WORKSPACE", 11: "FA2_ERR_WINDOW",
}
SITE_NAMES = {
    1: "Q_LOADED", 2: "KV_LOADED", 3: "KV_FREE", 4: "S_READY", 5: "P_READY", 6: "STATS_READY",
    7: "O_RESCALED", 8: "O_FINAL", 9: "FINAL_STATS", 10: "MMA_DRAIN", 11: "LOAD_DRAIN",
    13: "SMEM_ALIGN", 15: "SELFTEST",
}
FA2_SITE_SELFTEST = 15
FA2_STATIC_WS_BYTES = 40 << 20  # the library's fixed stream-K scratch per device (fa2.h)


class FA2Error(RuntimeError):
    def __init__(self, status: int, where: str = "fa2_forward"):
        self.status = status
        super().__init__(f"{where} failed with status {status} ({fa2_status_string(status)})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m exact_tiled_attention_29_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, ci, cf, cll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
    lib.fa2_forward.argtypes = [vp, vp, vp, vp, vp] + [ci] * 7 + [cf, vp]
    lib.fa2_forward.restype = ci
    lib.fa2_forward_ws.argtypes = [vp, vp, vp, vp, vp] + [ci] * 7 + [cf, vp, cll, vp]
    lib.fa2_forward_ws.restype = ci
    lib.fa2_forward_auto.argtypes = [vp, vp, vp, vp, vp] + [ci] * 7 + [cf, vp, cll, vp]
    lib.fa2_forward_auto.restype = ci
    lib.fa2_forward_local.argtypes = [vp, vp, vp, vp, vp] + [ci] * 8 + [cf, vp]
    lib.fa2_forward_local.restype = ci
    lib.fa2_forward_static_ws.argtypes = [vp, vp, vp, vp, vp] + [ci] * 7 + [cf, vp]
    lib.fa2_forward_static_ws.restype = ci
    lib.fa2_backward.argtypes = [vp] * 9 + [ci] * 7 + [cf, vp, cll, vp]
    lib.fa2_backward.restype = ci
    lib.fa2_backward_local.argtypes = [vp] * 9 + [ci] * 8 + [cf, vp, cll, vp]
    lib.fa2_backward_local.restype = ci
    lib.fa2_backward_workspace_size.argtypes = [ci] * 4
    lib.fa2_backward_workspace_size.restype = cll
    lib.fa2_workspace_size.argtypes = [ci] * 7
    lib.fa2_workspace_size.restype = cll
    lib.fa2_status_string.argtypes = [ci]
    lib.fa2_status_string.restype = ctypes.c_char_p
    lib.fa2_debug_status.argtypes = [vp]
    lib.fa2_debug_status.restype = ci
    lib.fa2_selftest_timeout.argtypes = [vp, cll]
    lib.fa2_selftest_timeout.restype = ci
    lib.fa2_num_blocks.argtypes = [ci, ci, ci, ci]
    lib.fa2_num_blocks.restype = cll
    ip = ctypes.POINTER(ci)
    lib.fa2_launch_plan.argtypes = [ci] * 6 + [ip] * 4
    lib.fa2_launch_plan.restype = ci
    llp = ctypes.POINTER(cll)
    lib.fa2_streamk_plan.argtypes = [ci] * 8 + [llp, ip, llp]
    lib.fa2_streamk_plan.restype = ci
    lib.fa2_persistent_plan.argtypes = [ci] * 8 + [ip, ip, ci]
    lib.fa2_persistent_plan.restype = ci
    lib.fa2_schedule_choice.argtypes = [ci] * 8 + [ip, llp, llp]
    lib.fa2_schedule_choice.restype = ci
    return lib


_lib = _load()


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


# ---- the C ABI, one function per entry point, same names ----

def fa2_forward(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale, stream) -> int:
    """Enqueue the forward pass; pointers may be ints or tensors.  Returns the status code."""
    return int(_lib.fa2_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq),
                                int(Hkv), int(Nq), int(Nk), int(d), int(bool(causal)),
                                float(softmax_scale), _stream(stream)))


def fa2_forward_local(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, window_left, window_right,
                      softmax_scale, stream) -> int:
    """Local (sliding-window) attention; -1 leaves a side open.  Returns the status code."""
    return int(_lib.fa2_forward_local(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B),
                                      int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                      int(window_left), int(window_right), float(softmax_scale),
                                      _stream(stream)))


def fa2_forward_ws(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale, workspace,
                   workspace_bytes, stream) -> int:
    """Stream-K variant over a caller-provided workspace.  Returns the status code."""
    return int(_lib.fa2_forward_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq),
                                   int(Hkv), int(Nq), int(Nk), int(d), int(bool(causal)),
                                   float(softmax_scale), _ptr(workspace), int(workspace_bytes),
                                   _stream(stream)))


def fa2_forward_auto(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale, workspace,
                     workspace_bytes, stream) -> int:
    """Whole units or stream-K, as the library's cost model picks (workspace may be None)."""
    return int(_lib.fa2_forward_auto(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq),
                                     int(Hkv), int(Nq), int(Nk), int(d), int(bool(causal)),
                                     float(softmax_scale), _ptr(workspace), int(workspace_bytes),
                                     _stream(stream)))


def fa2_forward_static_ws(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale,
                          stream) -> int:
    """Stream-K with the library's fixed scratch array; calls must not overlap."""
    return int(_lib.fa2_forward_static_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B),
                                          int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                          int(bool(causal)), float(softmax_scale),
                                          _stream(stream)))


def fa2_backward(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale,
                 workspace, workspace_bytes, stream) -> int:
    """Gradients dq, dk, dv of the forward pass (fp32 scratch in `workspace`).  Returns the status."""
    return int(_lib.fa2_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                 _ptr(dk), _ptr(dv), int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                 int(bool(causal)), float(softmax_scale), _ptr(workspace),
                                 int(workspace_bytes), _stream(stream)))


def fa2_backward_local(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, window_left,
                       window_right, softmax_scale, workspace, workspace_bytes, stream) -> int:
    """Gradients of fa2_forward_local (same window).  Returns the status."""
    return int(_lib.fa2_backward_local(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                       _ptr(dq), _ptr(dk), _ptr(dv), int(B), int(Hq), int(Hkv),
                                       int(Nq), int(Nk), int(d), int(window_left), int(window_right),
                                       float(softmax_scale), _ptr(workspace), int(workspace_bytes),
                                       _stream(stream)))


def fa2_backward_workspace_size(B, Hq, Nq, d) -> int:
    return int(_lib.fa2_backward_workspace_size(int(B), int(Hq), int(Nq), int(d)))


def fa2_workspace_size(B, Hq, Hkv, Nq, Nk, d, causal) -> int:
    return int(_lib.fa2_workspace_size(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                       int(bool(causal))))


def fa2_streamk_plan(B, Hq, Hkv, Nq, Nk, d, causal, num_sms):
    """(status, total_iters, ctas, workspace_bytes)."""
    t, g, w = ctypes.c_longlong(0), ctypes.c_int(0), ctypes.c_longlong(0)
    st = _lib.fa2_streamk_plan(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                               int(bool(causal)), int(num_sms), ctypes.byref(t), ctypes.byref(g),
                               ctypes.byref(w))
    return int(st), t.value, g.value, w.value


def fa2_schedule_choice(B, Hq, Hkv, Nq, Nk, d, causal, num_sms):
    """(status, split, cost_units, cost_split): fa2_forward_auto's choice."""
    sp, cu, cs = ctypes.c_int(0), ctypes.c_longlong(0), ctypes.c_longlong(0)
    st = _lib.fa2_schedule_choice(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                  int(bool(causal)), int(num_sms), ctypes.byref(sp), ctypes.byref(cu),
                                  ctypes.byref(cs))
    return int(st), sp.value, cu.value, cs.value


def fa2_persistent_plan(B, Hq, Hkv, Nq, Nk, d, causal, num_sms, capacity=1 << 14):
    """(status, start, units): block c of the persistent launch runs
    units[start[c]:start[c + 1]] in that order."""
    start = (ctypes.c_int * (num_sms + 1))()
    units = (ctypes.c_int * capacity)()
    st = _lib.fa2_persistent_plan(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                                  int(bool(causal)), int(num_sms), start, units, int(capacity))
    if st != 0:
        return int(st), [], []
    n = start[num_sms]
    return 0, list(start), list(units[:n])


def fa2_status_string(status: int) -> str:
    return _lib.fa2_status_string(int(status)).decode()


def fa2_debug_status(stream=None) -> int:
    return int(_lib.fa2_debug_status(_stream(stream)))


def fa2_selftest_timeout(stream, limit_ns: int) -> int:
    return int(_lib.fa2_selftest_timeout(_stream(stream), int(limit_ns)))


def fa2_num_blocks(B: int, H: int, N: int, rows_per_block: int) -> int:
    return int(_lib.fa2_num_blocks(int(B), int(H), int(N), int(rows_per_block)))


def fa2_launch_plan(B, Hq, Hkv, Nq, Nk, d):
    """(status, grid_blocks, threads_per_block, smem_bytes, rows_per_block)."""
    out = [ctypes.c_int(0) for _ in range(4)]
    st = _lib.fa2_launch_plan(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d),
                              *[ctypes.byref(x) for x in out])
    return (int(st), *[x.value for x in out])


# ---- torch convenience: allocate outputs with torch, then call the C ABI ----

def alloc_workspace(B, Hq, Hkv, Nq, Nk, d, causal, device):
    """A uint8 CUDA tensor large enough for ``fa2_forward_ws`` (scratch: no
    initialisation needed; reusable by later calls ordered on one stream)."""
    import torch

    n = fa2_workspace_size(B, Hq, Hkv, Nq, Nk, d, causal)
    if n < 0:
        raise FA2Error(2, "fa2_workspace_size")
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def attention(q, k, v, causal: bool = False, softmax_scale: float | None = None, out=None,
              lse=None, stream=None, workspace=None, window=None, schedule: str = "streamk"):
    """O, LSE for bf16 CUDA tensors q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] (contiguous).

    Outputs are allocated with torch unless given; the work is one call to
    ``fa2_forward`` on ``stream`` (default: torch's current stream), or, when
    ``workspace`` -- a CUDA tensor from ``alloc_workspace`` -- is given, to
    ``fa2_forward_ws`` (stream-K schedule; ``schedule="streamk"``) or
    ``fa2_forward_auto`` (the library picks; ``schedule="auto"``), or to
    ``fa2_forward_local`` when ``window`` = (left, right) is given (causal then
    narrows the right side to 0).
    """
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D bf16 CUDA tensor")
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if v.shape != k.shape or Bk != B or dk != d:
        raise ValueError("k and v must be [B, Nk, Hkv, d] with q's B and d")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    if window is not None:
        if workspace is not None:
            raise ValueError("the local-window path has no stream-K variant")
        wl, wr = int(window[0]), int(window[1])
        if causal:  # j <= g and j <= g + wr (wr >= 0) is j <= g
            wr = 0
        st = fa2_forward_local(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, wl, wr, softmax_scale,
                               stream)
        where = "fa2_forward_local"
    elif workspace is None:
        st = fa2_forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale, stream)
        where = "fa2_forward"
    elif schedule == "auto":
        st = fa2_forward_auto(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale,
                              workspace, workspace.numel() * workspace.element_size(), stream)
        where = "fa2_forward_auto"
    elif schedule == "streamk":
        st = fa2_forward_ws(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, causal, softmax_scale,
                            workspace, workspace.numel() * workspace.element_size(), stream)
        where = "fa2_forward_ws"
    else:
        raise ValueError(f"schedule must be 'streamk' or 'auto', not {schedule!r}")
    if st != FA2_OK:
        raise FA2Error(st, where)
    return out, lse


def attention_backward(q, k, v, o, lse, dout, causal: bool = False,
                       softmax_scale: float | None = None, stream=None, workspace=None, window=None):
    """dq, dk, dv for bf16 CUDA tensors (layouts as ``attention``) given the
    forward's o and lse and the upstream gradient dout; one call to
    ``fa2_backward``.  ``workspace`` (uint8 CUDA tensor of at least
    ``fa2_backward_workspace_size`` bytes) is allocated with torch if absent."""
    import torch

    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    if workspace is None:
        workspace = torch.empty(fa2_backward_workspace_size(B, Hq, Nq, d), dtype=torch.uint8,
                                device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = workspace.numel() * workspace.element_size()
    if window is not None:
        wl, wr = int(window[0]), int(window[1])
        if causal:
            wr = 0
        st = fa2_backward_local(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, wl, wr,
                                softmax_scale, workspace, nbytes, stream)
    else:
        st = fa2_backward(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal,
                          softmax_scale, workspace, nbytes, stream)
    if st != FA2_OK:
        raise FA2Error(st, "fa2_backward")
    return dq, dk, dv
