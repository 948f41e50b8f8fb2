"""Host logic of the stream-K schedule (no GPU): the plan the library reports,
and a model of the per-CTA piece walk checked for the properties the kernel
relies on -- every K/V-tile iteration of every unit is run exactly once, the
pieces of a split unit agree on their count and order, no two pieces share a
partial buffer, and a CTA holds at most two pieces of split units.

The schedule cuts cost positions, not iterations: a unit with n > 0 K/V
tiles costs UNIT_COST + n positions (its fixed pipeline and epilogue cost
first, then one position per iteration), so SMs that get many short units get
fewer iterations."""

import math

import pytest

import exact_tiled_attention_29_b200 as fa2

ROWS_PER_CTA, BLOCK_M, BLOCK_N = 256, 128, 128
UNIT_COST = 2  # the kernel's fixed cost per unit, in iterations


def kv_tiles_for(Nq, Nk, causal, r0):
    if r0 >= Nq:
        return 0
    nkt = -(-Nk // BLOCK_N)
    if not causal:
        return nkt
    rlast = min(r0 + BLOCK_M - 1, Nq - 1)
    lim = rlast + Nk - Nq  # last key visible to the tile's last row (bottom-right causal)
    if lim < 0:
        return 0
    return min(lim // BLOCK_N + 1, nkt)


def unit_tiles(Nq, Nk, causal, qb):
    return max(kv_tiles_for(Nq, Nk, causal, qb * ROWS_PER_CTA),
               kv_tiles_for(Nq, Nk, causal, qb * ROWS_PER_CTA + BLOCK_M))


def model_plan(B, Hq, Nq, Nk, d, causal, sms):
    """(iterations, CTAs, workspace bytes, summed cost)."""
    nq = -(-Nq // ROWS_PER_CTA)
    ns = [unit_tiles(Nq, Nk, causal, qb) for qb in range(nq)]
    iters = sum(B * Hq * n for n in ns)
    cost = sum(B * Hq * (n + UNIT_COST) for n in ns if n > 0)
    G = min(iters, sms)
    piece = 4 * 2 * BLOCK_M * (d + 3)
    ws = 2 * G * piece if G > 1 else 0
    return iters, G, ws, cost


def units_in_order(B, Hq, Nq, Nk, causal):
    """(round r, flat (batch, head) index k, tiles n) heaviest first."""
    nq = -(-Nq // ROWS_PER_CTA)
    for r in range(nq):
        n = unit_tiles(Nq, Nk, causal, nq - 1 - r)
        for k in range(B * Hq):
            yield r, k, n


def pieces_of_cta(c, G, T, units):
    """The pieces CTA c runs, in unit order: the iterations of each unit whose
    positions fall in [floor(cT/G), floor((c+1)T/G)).  Entries are
    (unit, jb, je, position of iteration 0, n)."""
    lo, hi = c * T // G, (c + 1) * T // G
    out, s = [], 0
    for u, (r, k, n) in enumerate(units):
        if n == 0:
            continue
        base = s + UNIT_COST
        jb, je = max(0, lo - base), min(n, hi - base)
        if jb < je:
            out.append((u, jb, je, base, n))
        s += n + UNIT_COST
    return out


def split_info(c_of_start, G, T, s_u, n, jb):
    """(split, slot, npieces, index) from the range boundaries B_c = floor(cT/G), c = 1..G-1."""
    bounds = [c * T // G for c in range(1, G)]
    inside = [c for c, bc in zip(range(1, G), bounds) if s_u < bc <= s_u + n - 1]
    if not inside:
        return 0, 0, 1, 0
    c_first, c_last = inside[0], inside[-1]
    before = [c for c, bc in zip(range(1, G), bounds) if bc <= s_u + jb]
    ci = before[-1] if before else 0
    index = 0 if ci < c_first else min(ci, c_last) - c_first + 1
    return 1, c_first - 1, c_last - c_first + 2, index


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, sms
    (2, 16, 16, 8192, 8192, 128, 1, 148),
    (4, 16, 16, 2048, 2048, 128, 0, 148),
    (1, 2, 2, 32768, 32768, 128, 1, 148),
    (4, 32, 8, 4096, 4096, 128, 1, 148),
    (1, 2, 2, 256, 256, 64, 1, 148),
    (1, 1, 1, 256, 65536, 128, 0, 148),   # one unit, cut into 148 pieces
    (3, 5, 5, 1000, 777, 64, 1, 7),       # Nq > Nk: units with no visible key
    (1, 1, 1, 1, 1, 64, 0, 148),
    (2, 3, 1, 1500, 3000, 128, 1, 16),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,sms", CASES)
def test_plan_matches_model(B, Hq, Hkv, Nq, Nk, d, causal, sms):
    st, T, G, ws = fa2.fa2_streamk_plan(B, Hq, Hkv, Nq, Nk, d, causal, sms)
    assert st == 0
    assert (T, G, ws) == model_plan(B, Hq, Nq, Nk, d, causal, sms)[:3]
    if causal == 0:
        assert T == B * Hq * -(-Nq // ROWS_PER_CTA) * -(-Nk // BLOCK_N)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,sms", CASES)
def test_piece_walk_covers_every_iteration_once(B, Hq, Hkv, Nq, Nk, d, causal, sms):
    units = list(units_in_order(B, Hq, Nq, Nk, causal))
    iters, G, _, T = model_plan(B, Hq, Nq, Nk, d, causal, sms)
    if G == 0:
        return
    seen = {}
    buffers = set()
    for c in range(G):
        ps = pieces_of_cta(c, G, T, units)
        split_pieces = 0
        for pos, (u, jb, je, s_u, n) in enumerate(ps):
            for j in range(jb, je):
                assert (u, j) not in seen
                seen[(u, j)] = c
            split, slot, npieces, index = split_info(c, G, T, s_u, n, jb)
            if not split:
                assert (jb, je) == (0, n)
                continue
            split_pieces += 1
            # piece `index` runs on CTA slot + index; piece 0 is that CTA's last
            # piece, every other piece its CTA's first
            assert slot + index == c
            if index == 0:
                assert pos == len(ps) - 1
            else:
                assert pos == 0
            buf = 2 * (slot + index) + (1 if index == 0 else 0)
            assert buf not in buffers
            buffers.add(buf)
            assert 0 <= buf < 2 * G
        assert split_pieces <= 2
    total = sum(n for _, _, n in units)
    assert len(seen) == total == iters


def test_plan_validation():
    assert fa2.fa2_streamk_plan(1, 3, 2, 4, 4, 128, 0, 148)[0] == 2
    assert fa2.fa2_streamk_plan(1, 2, 2, 4, 4, 80, 0, 148)[0] == 3
    assert fa2.fa2_streamk_plan(1, 2, 2, 4, 4, 128, 0, 0)[0] == 2


def test_one_unit_workspace_is_modest():
    # the partial buffers grow with the SM count, not with the unit length
    st, T, G, ws = fa2.fa2_streamk_plan(1, 1, 1, 256, 1 << 20, 128, 0, 148)
    assert st == 0 and G == 148 and T == (1 << 20) // 128
    assert ws == 2 * 148 * 4 * 2 * 128 * 131
    assert ws < 48 * 2**20


GOOD = dict(q=16, k=32, v=48, o=64, lse=80, B=1, Hq=2, Hkv=1, Nq=5, Nk=7, d=128, causal=1,
            softmax_scale=0.125, ws=4096, ws_bytes=1 << 20, stream=None)


def call_ws(**over):
    a = dict(GOOD, **over)
    return fa2.fa2_forward_ws(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                              a["Nq"], a["Nk"], a["d"], a["causal"], a["softmax_scale"], a["ws"],
                              a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(ws=0), 1), (dict(q=0), 1), (dict(B=0), 2), (dict(d=96), 3), (dict(ws=4100), 4),
    (dict(softmax_scale=math.nan), 5), (dict(ws_bytes=-1), 10),
])
def test_forward_ws_validation(over, code):
    assert call_ws(**over) == code


def test_workspace_size_rejects_bad_shapes():
    assert fa2.fa2_workspace_size(0, 1, 1, 1, 1, 128, 0) == -1
    assert fa2.fa2_workspace_size(1, 3, 2, 1, 1, 128, 0) == -1


def persistent_units_of_cta(c, G, U):
    """Units CTA c takes when whole units are dealt round robin, alternating
    direction each wave (the kernel's persistent-units schedule)."""
    out, w = [], 0
    while True:
        u = w * G + ((G - 1 - c) if (w & 1) else c)
        if u >= U:
            return out
        out.append(u)
        w += 1


@pytest.mark.parametrize("B,Hq,Nq,causal,G", [(2, 16, 8192, 1, 148), (4, 16, 2048, 0, 148),
                                              (4, 32, 4096, 1, 148), (1, 3, 5000, 1, 7)])
def test_persistent_units_deal_every_unit_once_and_pair_heavy_with_light(B, Hq, Nq, causal, G):
    units = list(units_in_order(B, Hq, Nq, Nq, causal))
    U = len(units)
    dealt = [persistent_units_of_cta(c, G, U) for c in range(G)]
    flat = sorted(u for d in dealt for u in d)
    assert flat == list(range(U))
    loads = [sum(units[u][2] for u in d) for d in dealt]
    # a CTA's load differs from the mean by less than one unit of the heaviest size
    assert max(loads) - min(loads) <= max(n for _, _, n in units)
