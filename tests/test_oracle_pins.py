"""The oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

import oracle_checks as C


@pytest.mark.parametrize("check", C.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_every_oracle_function_has_a_pin_entry():
    import oracle
    names = {"bf16_rne", "dequant", "qmm_rows", "glu", "gather_rows", "argmax_rows", "pick",
             "half_rows", "top2_gap", "residual_add", "embed_rows", "qmm8_rows", "top2_rows", "top2_merge"}
    assert names <= set(oracle.PINS)
    assert "parity unpinned" in oracle.PINS["end_to_end_on_real_weights"]
