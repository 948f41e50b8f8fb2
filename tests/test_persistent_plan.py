"""The plan of persistent whole units (host logic, no GPU): every unit with a
visible key runs exactly once (whole, or as its two single-tile halves), the
planned work of the blocks is balanced to within one unit, a last wave that
would fill at most half the blocks is dealt as half units, and the blocks
running at the same moment share few heads (the property that keeps their K
and V in L2)."""

import pytest

import exact_tiled_attention_29_b200 as fa2

ROWS = 256   # query rows per unit
BLOCK = 128  # keys per K/V tile
UNIT_COST = 2
UNIT_BITS = 13  # an entry is u, or u + 1 << 13 (first query tile only), or u + 2 << 13 (second)


def decode(e):
    return e & ((1 << UNIT_BITS) - 1), e >> UNIT_BITS


def unit_tiles(nq, nk, causal, qb):
    """K/V tiles a unit of two 128-row query tiles needs (bottom-right causal)."""
    r0 = qb * ROWS
    if r0 >= nq:
        return 0
    last_row = min(r0 + ROWS - 1, nq - 1)
    last_key = min(nk - 1, last_row + nk - nq) if causal else nk - 1
    return 0 if last_key < 0 else last_key // BLOCK + 1


SHAPES = [
    # (B, Hq, Hkv, N, causal): the workloads the benchmark times and a few more
    (2, 16, 16, 8192, True),
    (4, 16, 16, 2048, False),
    (4, 32, 8, 4096, True),
    (1, 40, 8, 3000, True),
    (3, 6, 2, 5000, False),
]


def plan(B, Hq, Hkv, N, causal, sms=148):
    st, start, units = fa2.fa2_persistent_plan(B, Hq, Hkv, N, N, 128, causal, sms)
    assert st == 0, fa2.fa2_status_string(st)
    return start, units


@pytest.mark.parametrize("B,Hq,Hkv,N,causal", SHAPES)
def test_every_unit_once(B, Hq, Hkv, N, causal):
    start, units = plan(B, Hq, Hkv, N, causal)
    n_qblk = (N + ROWS - 1) // ROWS
    rounds = sum(1 for qb in range(n_qblk) if unit_tiles(N, N, causal, qb) > 0)
    seen = {}
    for e in units:
        u, half = decode(e)
        seen.setdefault(u, []).append(half)
    assert sorted(seen) == list(range(rounds * B * Hq))
    assert all(sorted(h) in ([0], [1, 2]) for h in seen.values())
    assert start[0] == 0 and all(a <= b for a, b in zip(start, start[1:])) and start[-1] == len(units)


@pytest.mark.parametrize("B,Hq,Hkv,N,causal", SHAPES)
def test_planned_work_balanced_within_one_unit(B, Hq, Hkv, N, causal):
    start, units = plan(B, Hq, Hkv, N, causal)
    HB = B * Hq
    n_qblk = (N + ROWS - 1) // ROWS

    def cost(e):
        u, half = decode(e)
        n = unit_tiles(N, N, causal, n_qblk - 1 - u // HB)
        return n + UNIT_COST if half == 0 else n * 5 // 8 + UNIT_COST

    loads = [sum(cost(u) for u in units[start[c]:start[c + 1]]) for c in range(len(start) - 1)]
    assert max(loads) - min(loads) <= max(cost(u) for u in units)
    if causal:
        # units of many sizes: the light tail evens the blocks out to a few percent
        assert max(loads) <= 1.04 * sum(loads) / len(loads) + UNIT_COST


def footprint(lists, cost, tiles, HB, Hq, grp):
    """Average over time of the K/V tiles the running units stream: per KV head,
    the longest K/V range among its running units."""
    events = []
    for lst in lists:
        t = 0
        for u in lst:
            events.append((t, t + cost(u), u % HB, tiles(u)))
            t += cost(u)
    times = sorted({a for a, _, _, _ in events})
    total = 0
    for t0 in times[::5]:
        span = {}
        for a, b, k, n in events:
            if a <= t0 < b:
                kv = (k // Hq, (k % Hq) // grp)
                span[kv] = max(span.get(kv, 0), n)
        total += sum(span.values())
    return total / len(times[::5])


@pytest.mark.parametrize("B,Hq,Hkv,N", [(2, 16, 16, 8192), (4, 32, 8, 4096)])
def test_concurrent_units_share_kv(B, Hq, Hkv, N):
    # replay the plan in time; compare the K/V footprint of the running units
    # with dealing the same units round robin, heaviest first (snake order)
    G = 148
    start, units = plan(B, Hq, Hkv, N, True, sms=G)
    HB, n_qblk, grp = B * Hq, N // ROWS, Hq // Hkv
    tiles = lambda u: unit_tiles(N, N, True, n_qblk - 1 - u // HB)
    cost = lambda u: tiles(u) + UNIT_COST
    planned = [units[start[c]:start[c + 1]] for c in range(G)]
    n = n_qblk * HB
    rr = [[w * G + (G - 1 - c if w % 2 else c) for w in range((n + G - 1) // G)
           if w * G + (G - 1 - c if w % 2 else c) < n] for c in range(G)]
    f_plan = footprint(planned, cost, tiles, HB, Hq, grp)
    f_rr = footprint(rr, cost, tiles, HB, Hq, grp)
    assert f_plan <= 0.7 * f_rr, (f_plan, f_rr)


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,sms", [(4, 16, 16, 2048, False, 148), (3, 6, 2, 5000, False, 148),
                                                   (2, 16, 16, 8192, True, 148), (4, 16, 16, 2048, False, 132)])
def test_last_wave_in_halves(B, Hq, Hkv, N, causal, sms):
    # R units left after the full waves: dealt as 2R half units when 2R <= SMs,
    # one per block; otherwise no halves at all
    start, units = plan(B, Hq, Hkv, N, causal, sms=sms)
    n_qblk = (N + ROWS - 1) // ROWS
    n_units = B * Hq * sum(1 for qb in range(n_qblk) if unit_tiles(N, N, causal, qb) > 0)
    rest = n_units % sms
    halves = [e for e in units if decode(e)[1]]
    if 2 * rest <= sms:
        assert len(halves) == 2 * rest
        for c in range(sms):  # a block gets at most one half, after its whole units
            mine = [decode(e)[1] for e in units[start[c]:start[c + 1]]]
            n_halves = sum(1 for h in mine if h)
            assert n_halves <= 1
            if n_halves:
                assert mine[-1] != 0
    else:
        assert not halves


def test_plan_limits_and_validation():
    assert fa2.fa2_persistent_plan(1, 3, 2, 512, 512, 128, 1, 148)[0] == 2      # Hq % Hkv
    assert fa2.fa2_persistent_plan(1, 2, 2, 512, 512, 128, 1, 161)[0] == 8      # more SMs than the table
    assert fa2.fa2_persistent_plan(64, 64, 64, 65536, 65536, 128, 0, 148)[0] == 8  # more units than the table
