"""fa2_forward_auto's choice between whole units and split-KV (host logic, no
GPU): the two prices it reports follow the model below, and it takes split-KV
exactly for the shapes where one block per unit leaves most SMs idle -- a
short query against long keys -- and never for the specified workloads,
where whole units measured faster.

Model (in K/V-tile iterations of one block; a unit costs UNIT_COST + its
tiles): whole units = longest-first list scheduling over the SMs, or the
rounded-up average once there are at least two units per SM; split-KV =
the rounded-up average over min(iterations, SMs) blocks plus MERGE_COST.
Split-KV is chosen when there are fewer than two units per SM and
MARGIN x its price is below the whole-unit price."""

import heapq

import pytest

import exact_tiled_attention_29_b200 as fa2
from exact_tiled_attention_29_b200.inputs import EXTRA_WORKLOADS, WORKLOADS

from test_streamk_plan import UNIT_COST, model_plan, unit_tiles, ROWS_PER_CTA

MARGIN, MERGE_COST = 1.5, 4


def model_choice(B, Hq, Nq, Nk, d, causal, sms):
    iters, G, _, T = model_plan(B, Hq, Nq, Nk, d, causal, sms)
    if G == 0:
        return 0, 0, 0
    nq = -(-Nq // ROWS_PER_CTA)
    costs = [n + UNIT_COST for qb in range(nq) for n in [unit_tiles(Nq, Nk, causal, qb)] if n > 0
             for _ in range(B * Hq)]
    split_price = -(-T // G) + MERGE_COST
    if len(costs) >= 2 * sms:
        return 0, -(-T // sms), split_price
    loads = [0] * sms
    for c in sorted(costs, reverse=True):
        heapq.heapreplace(loads, loads[0] + c)
    units_price = max(loads)
    return int(MARGIN * split_price < units_price), units_price, split_price


SHAPES = [
    (1, 16, 256, 32768, 128, 0),   # short query vs long keys
    (1, 1, 256, 1 << 20, 128, 0),  # one unit, a million keys
    (2, 4, 700, 9000, 64, 1),
    (1, 2, 512, 512, 64, 1),       # tiny: too little work to split
    (4, 8, 2048, 2048, 128, 0),
    (1, 40, 3000, 3000, 128, 1),
]


@pytest.mark.parametrize("B,Hq,Nq,Nk,d,causal", SHAPES)
@pytest.mark.parametrize("sms", [148, 132, 16])
def test_choice_matches_model(B, Hq, Nq, Nk, d, causal, sms):
    st, split, cu, cs = fa2.fa2_schedule_choice(B, Hq, Hq, Nq, Nk, d, causal, sms)
    assert st == 0
    assert (split, cu, cs) == model_choice(B, Hq, Nq, Nk, d, causal, sms)


def test_split_only_where_units_starve_the_gpu():
    w = EXTRA_WORKLOADS["shortq_32k"]
    st, split, cu, cs = fa2.fa2_schedule_choice(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, 148)
    assert st == 0 and split == 1 and cu > 5 * cs
    for name, w in WORKLOADS.items():
        st, split, _, _ = fa2.fa2_schedule_choice(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal, 148)
        assert st == 0 and split == 0, name


def test_choice_validation():
    assert fa2.fa2_schedule_choice(1, 3, 2, 256, 256, 128, 0, 148)[0] == 2  # Hq % Hkv
    assert fa2.fa2_schedule_choice(1, 2, 2, 256, 256, 80, 0, 148)[0] == 3   # head dim
    assert fa2.fa2_schedule_choice(1, 2, 2, 256, 256, 128, 0, 0)[0] == 2    # no SMs
