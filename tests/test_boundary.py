"""The C-ABI library: it loads, exports every entry point its header declares,
and validates arguments before touching CUDA (so these run without a GPU)."""

import json
import math
import os
import re

import pytest

import exact_tiled_attention_29_b200 as fa2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa2.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "worked_counts.json")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(fa2_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("fa2_forward", "fa2_status_string", "fa2_debug_status"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import ctypes
    lib = ctypes.CDLL(fa2.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"declared in fa2.h but not exported: {missing}"


GOOD = dict(q=16, k=32, v=48, o=64, lse=80, B=1, Hq=2, Hkv=1, Nq=5, Nk=7, d=128, causal=1,
            softmax_scale=0.125, stream=None)


def call(**over):
    a = dict(GOOD, **over)
    return fa2.fa2_forward(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                           a["Nq"], a["Nk"], a["d"], a["causal"], a["softmax_scale"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=0), 1), (dict(k=0), 1), (dict(v=0), 1), (dict(o=0), 1), (dict(lse=0), 1),
    (dict(B=0), 2), (dict(Hq=0), 2), (dict(Hkv=0), 2), (dict(Nq=0), 2), (dict(Nk=-3), 2),
    (dict(Hq=3, Hkv=2), 2),
    (dict(d=96), 3), (dict(d=256), 3), (dict(d=0), 3),
    (dict(q=24), 4), (dict(o=72), 4), (dict(lse=82), 4),
    (dict(softmax_scale=math.nan), 5), (dict(softmax_scale=math.inf), 5),
    (dict(B=1 << 20, Nq=1 << 20, Hq=1 << 10, Hkv=1 << 10), 8),
])
def test_validation_status_codes(over, code):
    assert call(**over) == code
    assert fa2.fa2_status_string(code) not in ("", "unknown status")


def test_local_window_validation():
    args = (16, 32, 48, 64, 80, 1, 2, 1, 5, 7, 128)
    assert fa2.fa2_forward_local(*args, -2, 0, 0.1, None) == 11
    assert fa2.fa2_forward_local(*args, 0, -5, 0.1, None) == 11
    assert fa2.fa2_forward_local(0, 32, 48, 64, 80, 1, 2, 1, 5, 7, 128, 3, 0, 0.1, None) == 1
    assert fa2.fa2_forward_local(16, 32, 48, 64, 80, 1, 2, 1, 5, 7, 80, 3, 0, 0.1, None) == 3


def test_backward_validation():
    ok = dict(q=16, k=32, v=48, o=64, lse=80, dout=96, dq=112, dk=128, dv=144, B=1, Hq=2, Hkv=1,
              Nq=5, Nk=7, d=128, causal=1, scale=0.1, ws=160, wsb=1 << 20)

    def call(**over):
        a = dict(ok, **over)
        return fa2.fa2_backward(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], a["dq"], a["dk"],
                                a["dv"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"],
                                a["causal"], a["scale"], a["ws"], a["wsb"], None)
    assert call(dout=0) == 1 and call(ws=0) == 1
    assert call(Hq=3, Hkv=2) == 2 and call(d=96) == 3 and call(dq=120) == 4 and call(lse=81) == 4
    assert call(scale=math.inf) == 5 and call(wsb=16) == 10
    assert fa2.fa2_backward_workspace_size(1, 2, 5, 128) >= 4 * 5 * 2 * 128
    assert fa2.fa2_backward_workspace_size(1, 2, 5, 80) == -1


def test_valid_arguments_reach_the_device_check_only():
    import torch
    st = call()
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; the launch path is covered by the GPU tests")
    assert st == 6  # no sm_100 device on this host


def test_status_strings():
    for code in range(12):
        assert isinstance(fa2.fa2_status_string(code), str)
    assert fa2.fa2_status_string(12345) == "unknown status"


def test_launch_plan_matches_design():
    # 256 query rows (two 128-row tiles) per block; grid over (query block, head, batch)
    cases = {(1, 2, 2, 256, 256, 64): 2, (4, 16, 16, 2048, 2048, 128): 512,
             (2, 16, 16, 8192, 8192, 128): 1024, (1, 2, 2, 32768, 32768, 128): 256,
             (4, 32, 8, 4096, 4096, 128): 2048, (1, 1, 1, 1, 1, 64): 1, (3, 5, 5, 257, 9, 128): 30}
    for (B, Hq, Hkv, Nq, Nk, d), blocks in cases.items():
        st, grid, threads, smem, rows = fa2.fa2_launch_plan(B, Hq, Hkv, Nq, Nk, d)
        assert st == 0 and grid == blocks and threads == 512 and rows == 256
        assert 0 < smem <= 232448
    assert fa2.fa2_launch_plan(1, 3, 2, 4, 4, 128)[0] == 2
    assert fa2.fa2_launch_plan(1, 2, 2, 4, 4, 80)[0] == 3


def test_worked_grid_counts_from_the_pages():
    gold = json.load(open(GOLDEN))
    g = gold["fa1_grid"]
    assert fa2.fa2_num_blocks(g["B"], g["H"], g["N"], g["rows_per_block"]) == g["blocks"]
    assert g["sms"] - g["blocks"] == g["idle_sms"]
    assert round(100 * g["idle_sms"] / g["sms"]) == g["idle_pct_rounded"]

    g = gold["fa2_grid"]
    blocks = fa2.fa2_num_blocks(g["B"], g["H"], g["N"], g["rows_per_block"])
    assert blocks == g["blocks"]
    sms = gold["fa1_grid"]["sms"]
    assert round(blocks / sms, 1) == g["waves_rounded_1dp"]
    last = blocks - (blocks // sms) * sms
    assert last == g["last_wave_blocks"] and sms - last == g["idle_in_last_wave"]
    waves = math.ceil(blocks / sms)
    assert round(100 * (sms - last) / (waves * sms), 1) == g["idle_time_pct_rounded_1dp"]

    g = gold["single_head_blocks"]
    assert fa2.fa2_num_blocks(g["B"], g["H"], g["N"], g["rows_per_block"]) == g["blocks"]

    g = gold["divisions"]
    qblocks = fa2.fa2_num_blocks(1, 1, g["N"], g["rows_per_block"])
    assert qblocks == g["fa2_divisions"]            # one division per query block
    assert qblocks * qblocks == g["fa1_rescales"]   # every query block sweeps every key block
    assert fa2.fa2_num_blocks(0, 1, 1, 1) == -1
