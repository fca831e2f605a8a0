"""The refresh schedule's BSGS plans, derived from the butterfly structure
alone, against the oracle's plans read off the factored matrices' nonzero
diagonals."""
import pytest

from rns_ckks_polynomial_b200 import refresh


@pytest.mark.parametrize("n", [64, 256, 2048])
@pytest.mark.parametrize("depth", [1, 2, 3, 4])
def test_plans_match_the_oracle(orc, n, depth):
    if depth > (n // 2).bit_length() - 1:
        pytest.skip("more levels than stages")
    S = n // 2
    cts, stc = refresh.factored_plans(n, depth)
    assert cts == [orc.bsgs_plan(F, S) for F in orc.factored_coeff_to_slot(n, depth)]
    assert stc == [orc.bsgs_plan(F, S) for F in orc.factored_slot_to_coeff(n, depth)]
    from oracle import boot
    assert refresh.plan_rotations(cts + stc, n) == boot.factored_rotation_amounts(n, depth)
    assert refresh.stage_groups(n, depth) == orc.stage_groups(n, depth)
