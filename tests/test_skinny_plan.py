"""The skinny-M GEMM planner (host logic, no GPU): gdit_debug_skinny_plan.

The kernel's shared memory holds, from a 1024-byte boundary, `stages` chunks
of four 64-column boxes of 16 mt activation rows and of 8 nu weight rows
(128-byte rows), the cross-warp partial sums (4 sets of mt x nu fragments of
32 lanes x 16 bytes) and one 8-byte barrier per stage, within 226 KB.  The
planner takes, among row blocks mt in {1, 2, 3, 5} and units 1 .. max(mt),
the plans with at least 2 stages and at most one item per SM, the one whose
CTA streams the fewest bytes (rows of its item times K, plus a fixed 64 KB per
item); shapes of more than 160 rows, or with N not a multiple of 8 or K not a
multiple of 64, are not skinny.
"""

import pytest

import flow_matching_dit_b200 as fm

SMEM = 227 * 1024 - 1024
MAX_UNITS = {1: 16, 2: 16, 3: 12, 5: 7}


def layout(mt, nu, stages):
    stage = 4 * (16 * mt + 8 * nu) * 128
    red = 4 * mt * nu * 32 * 16
    return 1024 + stages * stage + red + 8 * stages, stage, red


def brute_force(M, N, K, sms):
    best = None
    for mt in (1, 2, 3, 5):
        nrb = -(-M // (16 * mt))
        for nu in range(1, MAX_UNITS[mt] + 1):
            items = nrb * -(-(N // 8) // nu)
            _, stage, red = layout(mt, nu, 0)
            stages = min(8, (SMEM - 1024 - red - 64) // stage)
            if stages < 2 or items > sms:
                continue
            cost = (min(16 * mt, M) + 8 * nu) * K * 2 + 64 * 1024
            if best is None or cost < best[0]:
                best = (cost, mt, nu, stages, items)
    return best


DIT = [(1024, 1024), (3072, 1024), (4096, 1024), (1024, 4096)]     # Q/O, QKV, FF1, FF2 (N, K)
TINY = [(128, 128), (384, 128), (512, 128), (128, 512)]


@pytest.mark.parametrize("B", range(1, 10))
@pytest.mark.parametrize("shape", DIT + TINY)
def test_plans_fit_and_are_the_cheapest(B, shape):
    N, K = shape
    M = 17 * B
    plan = fm.debug_skinny_plan(M, N, K, 148)
    ref = brute_force(M, N, K, 148)
    if ref is None:
        assert plan is None
        return
    assert plan is not None
    _, mt, nu, stages, items = ref
    assert (plan["mt"], plan["nu"], plan["stages"], plan["ctas"]) == (mt, nu, stages, items)
    smem, _, _ = layout(mt, nu, stages)
    assert plan["smem_bytes"] == smem <= SMEM
    assert plan["ctas"] <= 148 and plan["stages"] >= 2


def test_known_choices():
    # eight samples' rows: the 1024-wide linears in 32-row blocks of 5 units (130 CTAs)
    assert fm.debug_skinny_plan(136, 1024, 1024) == {"mt": 2, "nu": 5, "stages": 5, "ctas": 130,
                                                     "smem_bytes": 205864}
    # FF1 at 136 rows: one round only with 48-row blocks of 11 units, on a 2-stage ring
    assert fm.debug_skinny_plan(136, 4096, 1024) == {"mt": 3, "nu": 11, "stages": 2, "ctas": 141,
                                                     "smem_bytes": 1024 + 2 * 4 * (48 + 88) * 128 + 4 * 3 * 11 * 512 + 16}
    # 153 rows (nine samples): FF1 in two 80-row blocks of 7 units, one CTA per SM
    p = fm.debug_skinny_plan(153, 4096, 1024)
    assert (p["mt"], p["nu"], p["ctas"]) == (5, 7, 148)
    # a single 16-row block of a few units when there are few rows
    p = fm.debug_skinny_plan(34, 1024, 1024)
    assert p["mt"] == 1 and p["ctas"] <= 148


@pytest.mark.parametrize("M,N,K", [(161, 1024, 1024), (0, 1024, 1024), (136, 1020, 1024), (136, 1024, 1000)])
def test_shapes_outside_the_kernel_are_refused(M, N, K):
    assert fm.debug_skinny_plan(M, N, K) is None


def test_fewer_sms_give_fewer_items():
    for sms in (16, 32, 74, 132):
        p = fm.debug_skinny_plan(68, 1024, 1024, sms)
        ref = brute_force(68, 1024, 1024, sms)
        if ref is None:
            assert p is None
        else:
            assert p["ctas"] == ref[4] <= sms
