"""The GEMV's division of work among thread blocks (lutq_gemv_plan), checked
on the host: every unit is taken exactly once, every strip is whole in one
block or split between exactly two (the exchange of split halves at the end
of lutq_gemv relies on that), and no block is asked for more than the SMs.
The unit-to-block map below restates the one the header documents."""
import pytest

import dequant_gemv_group_b200 as lq


def blocks_units(plan, S, G):
    """Yield (block, strip, group) for every unit the plan assigns."""
    C = plan["C"]
    U = S * G
    for c in range(C):
        if plan["kind"] == 0:
            s0, ga, W = 0, 0, G
            if plan["align"]:
                v0, v1 = G * (c * S // C), G * ((c + 1) * S // C)
            else:
                v0, v1 = c * U // C, (c + 1) * U // C
        elif c < plan["Cm"]:
            s0, ga, W, v0, v1 = c, 0, G - plan["T"], 0, G - plan["T"]
        else:
            s0 = (c - plan["Cm"]) * plan["nh"]
            ga, W, v0 = G - plan["T"], plan["T"], 0
            v1 = min(plan["nh"], S - s0) * plan["T"] if s0 < S else 0
        for v in range(v0, v1):
            yield c, s0 + v // W, ga + v % W


SHAPES = [(32, 128), (128, 1024), (1024, 8192), (2400, 8192), (4096, 14336), (5120, 8192),
          (14336, 4096), (8192, 28672), (28672, 8192), (32 * 149, 128 * 3), (32 * 75, 128 * 2)]


@pytest.mark.parametrize("sms", [148, 132, 8, 1])
@pytest.mark.parametrize("n,k", SHAPES)
def test_plan_covers_every_unit_once(n, k, sms):
    S, G = n // 32, k // 128
    plan = lq.lutq_gemv_plan(n, k, sms)
    assert 1 <= plan["C"] <= min(sms, 512)
    seen = {}
    strips = {}
    for c, s, g in blocks_units(plan, S, G):
        assert 0 <= s < S and 0 <= g < G
        assert (s, g) not in seen
        seen[(s, g)] = c
        strips.setdefault(s, set()).add(c)
    assert len(seen) == S * G
    for s, cs in strips.items():
        assert len(cs) <= 2
        if len(cs) == 1:
            # a strip in one block is whole there, which the plan allows only
            # with full windows
            assert plan["kind"] == 0


def test_plan_kinds_for_the_benchmark_shapes():
    # whole strips for the Llama-3-8B down projection (128 strips < 148 SMs,
    # the split halves would cost more than the 13% they balance)
    assert lq.lutq_gemv_plan(4096, 14336, 148) == dict(C=128, kind=0, align=1, Cm=0, T=0, nh=0)
    # equal unit ranges over all SMs when strips outnumber them
    assert lq.lutq_gemv_plan(14336, 4096, 148)["C"] == 148
    assert lq.lutq_gemv_plan(14336, 4096, 148)["align"] == 0
    # main and helper blocks for a narrow, deep matrix
    p = lq.lutq_gemv_plan(2400, 8192, 148)
    assert p["kind"] == 1 and p["Cm"] == 75 and p["nh"] == 2


def test_plan_rejects_bad_arguments():
    with pytest.raises(lq.LutqError):
        lq.lutq_gemv_plan(33, 128, 148)
    with pytest.raises(lq.LutqError):
        lq.lutq_gemv_plan(32, 128, 0)
