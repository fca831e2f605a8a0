"""A few slips from the mutation sweep (tests/mutation_sweep.py), one per
layer of the oracle, each planted in a temporary copy and run against the pin
expected to catch it.  The full sweep plants every slip and runs the whole pin
suite; it takes about a quarter of an hour and is run by hand."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import mutation_sweep  # noqa: E402

SAMPLE = [
    0,   # NTT twiddle index
    13,  # key inner product without the automorphism
    15,  # ModDown without P^-1
    22,  # rescale subtracts the wrong way
]


def test_sweep_entries_apply():
    """Every slip's text occurs in the oracle, so the sweep plants what it says."""
    import tempfile
    for i in range(len(mutation_sweep.MUTATIONS)):
        with tempfile.TemporaryDirectory() as d:
            mutation_sweep.plant(i, d)


@pytest.mark.parametrize("index", SAMPLE)
def test_planted_slip_is_caught(index):
    caught, first = mutation_sweep.run(index, targeted=True, timeout=600)
    assert caught, "slip %r passed its pin" % mutation_sweep.MUTATIONS[index][0]
    assert first.split("[")[0] == mutation_sweep.MUTATIONS[index][5]
