"""Host-side bookkeeping (no GPU): window FLOP counts, the sampled-row FLOP
count of the CPU baseline, and the profile-validity hash of the kernels."""

import itertools

import pytest

import bench
from exact_tiled_attention_29_b200.inputs import EXTRA_WORKLOADS, WORKLOADS, Workload


def brute_pairs(w):
    n = 0
    for i in range(w.Nq):
        g = i + w.Nk - w.Nq
        for j in range(w.Nk):
            if w.causal and j > g:
                continue
            if w.window_left >= 0 and j < g - w.window_left:
                continue
            if w.window_right >= 0 and j > g + w.window_right:
                continue
            n += 1
    return n


@pytest.mark.parametrize("nq,nk,causal,wl,wr", [
    (37, 37, True, 5, -1), (20, 50, False, 3, 4), (50, 20, True, -1, -1), (33, 33, False, 0, 0),
    (16, 40, True, 100, -1), (40, 16, False, -1, 2),
])
def test_visible_pairs_counts_every_visible_key(nq, nk, causal, wl, wr):
    w = Workload("c", 1, 1, 1, nq, nk, 8, causal, window_left=wl, window_right=wr)
    assert w.visible_pairs() == brute_pairs(w)
    if w.windowed:
        assert w.flops() == 4.0 * w.d * w.visible_pairs()


def test_sampled_flops_agree_with_the_workload_count():
    for w in [EXTRA_WORKLOADS["local_8k"].with_(Nq=300, Nk=300),
              Workload("c", 2, 3, 1, 200, 260, 16, True),
              Workload("n", 1, 2, 2, 100, 90, 16, False, window_left=7, window_right=3)]:
        all_rows = list(range(w.Nq))
        assert bench.sample_flops(w, all_rows) == pytest.approx(4.0 * w.d * w.B * w.Hq * brute_pairs(w))


def test_headline_flops_definition():
    w = WORKLOADS["causal_8k"]
    assert w.flops() == 4.0 * 2 * 16 * 8192 * 8192 * 128 / 2


def test_kernel_hash_ignores_comments_only():
    src = "int a; // note\n/* block\n comment */\nint b;\n\n"
    assert bench._code_only(src) == "int a;\nint b;"
    assert bench._code_only(src.replace("note", "other words")) == bench._code_only(src)
    assert bench._code_only(src.replace("int b", "int c")) != bench._code_only(src)
    assert len(bench.kernel_source_hash()) == 16


def test_committed_profiles_carry_the_lookup_header():
    # bench.py reads `traffic` from these headers; each names the kernel
    # source it was taken on and its DRAM bytes per launch
    import os
    import re
    prof = os.path.join(os.path.dirname(bench.__file__), "profiles")
    names = [n for n in os.listdir(prof) if n.endswith(".md")]
    assert any(n.startswith("fa2_fwd_kernel_causal_8k") for n in names)
    for n in names:
        text = open(os.path.join(prof, n)).read()
        assert re.search(r"kernel_source_sha256_16:\s*[0-9a-f]{16}\b", text), n
        assert re.search(r"dram_bytes_per_launch:\s*[0-9]+", text), n
        assert "--clock-control none" in text, n
