"""Which calls run the whole K-step loop as the persistent kernel (host logic,
no GPU): gdit_debug_small_plan.

One sample, or up to 4 with one group of num_sms / B CTAs per sample, when a
sample's N = H + 1 tokens fit the loop's shared buffers (N <= 32), each group
has a CTA per head, and the phase tables of all samples fit; the grouped
instantiation runs for several samples or when a CTA has more than 4 units of
8 features in some linear (num_sms / B CTAs over N / 8 units).
"""

import dataclasses

import pytest

import flow_matching_dit_b200 as fm
import synth

FULL = synth.GEOM_FULL
TINY = synth.GEOM_TINY


@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_full_geometry_up_to_four_samples(B):
    p = fm.debug_small_plan(FULL, B)
    assert p == {"group_ctas": 148 // B, "grouped": B > 1}


@pytest.mark.parametrize("B", [5, 6, 8, 32, 256])
def test_five_samples_and_more_take_the_per_layer_kernels(B):
    assert fm.debug_small_plan(FULL, B) is None


def test_long_horizon_does_not_fit_the_loop():
    # H = 50: 51 tokens per sample, more than the loop's 32 rows
    assert fm.debug_small_plan(dataclasses.replace(FULL, action_horizon=50), 1) is None


def test_flag_turns_the_loop_off():
    assert fm.debug_small_plan(FULL, 1, flags=fm.GDIT_FLAG_NO_SMALL) is None


def test_tiny_geometry():
    assert fm.debug_small_plan(TINY, 1) == {"group_ctas": 148, "grouped": False}
    assert fm.debug_small_plan(TINY, 3) == {"group_ctas": 49, "grouped": True}


def test_fewer_sms():
    # 74 SMs at B = 1: FF1's 512 units make 7 per CTA, more than one pass of 4
    assert fm.debug_small_plan(FULL, 1, num_sms=74) == {"group_ctas": 74, "grouped": True}
    # 4 groups of 15 CTAs cannot give each of the 16 heads a CTA
    assert fm.debug_small_plan(FULL, 4, num_sms=60) is None
    assert fm.debug_small_plan(FULL, 3, num_sms=60) == {"group_ctas": 20, "grouped": True}


def test_phase_tables_bound_the_steps():
    # 150 phases per step and sample; the tables hold 20864 phases
    assert fm.debug_small_plan(FULL, 4, num_steps=34) is not None
    assert fm.debug_small_plan(FULL, 4, num_steps=35) is None
    assert fm.debug_small_plan(FULL, 1, num_steps=139) is not None
    assert fm.debug_small_plan(FULL, 1, num_steps=140) is None


def test_bad_arguments_raise():
    with pytest.raises(fm.GditError):
        fm.debug_small_plan(FULL, 0)
