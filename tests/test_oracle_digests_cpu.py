"""The oracle's outputs on small seeded cases against the digests that
tests/golden/make_oracle_digests.py stored.  A mismatch means the oracle's
arithmetic changed: the pins decide whether the change is right, and the
digests are then rewritten by that script in the same commit.  The second
run uses one OpenMP thread: no oracle output may depend on the thread count
(the pages' own engine had that failure, Kestrel engine write-up section 7,
pitfall 1)."""
import json
import os
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))
import make_oracle_digests  # noqa: E402

STORED = json.load(open(os.path.join(HERE, "golden", "oracle_digests.json")))


@pytest.mark.parametrize("threads", [None, 1])
def test_oracle_outputs_match_the_stored_digests(orc, threads):
    before = orc.num_threads()
    try:
        if threads:
            orc.set_num_threads(threads)
        got = make_oracle_digests.cases()
    finally:
        orc.set_num_threads(before)
    assert sorted(got) == sorted(STORED)
    bad = [k for k in STORED if got[k] != STORED[k]]
    assert not bad, "oracle outputs changed: %s" % bad
