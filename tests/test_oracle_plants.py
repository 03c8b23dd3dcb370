"""Planted controls, on the CPU: each deliberately broken build of the oracle
must turn the pin that covers it red.  These mirror the pages' six planted
controls for the seam (TensorFold PR #1433, step-1 body: a stage on the
peer's half, a gather writing its own half twice, an argmax and a pick that
tie to the higher id, an argmax that does not flag, a pick whose flag test is
dropped) plus three for the arithmetic (bias dropped, nibbles swapped, GLU
orientation swapped) and two for the adjacent steps (a residual add rounded to
bf16, an embedding bound taken from the shard's width) and two for the merged
top two (a second place that skips ties, a merge that keeps the winning part's
second).  Only the oracle is ever broken; no broken kernel is
built or run."""
import pytest

import oracle
import oracle_checks as C

PLANTS = {
    1: [C.check_spans, C.check_split_equals_whole_mlp],
    2: [C.check_gather, C.check_split_equals_whole_mlp],
    3: [C.check_argmax_bruteforce],
    4: [C.check_pick_truth_table],
    5: [C.check_argmax_bruteforce],
    6: [C.check_pick_truth_table],
    7: [C.check_hand_cases, C.check_vs_numpy_matmul, C.check_dequant_closed_forms],
    8: [C.check_hand_cases, C.check_one_hot],
    9: [C.check_glu],
    10: [C.check_residual_add],
    11: [C.check_embed_rows],
    12: [C.check_qmm8],
    13: [C.check_top2_hand, C.check_top2_bruteforce],
    14: [C.check_top2_merge_split],
}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_plant_goes_red(plant):
    bad = oracle.load(plant=plant)
    for check in PLANTS[plant]:
        with pytest.raises(AssertionError):
            check(bad)


def test_unplanted_passes_the_same_checks(orc):
    for checks in PLANTS.values():
        for check in checks:
            check(orc)
