"""The oracle against its regression fixtures (tests/golden/, written by
tests/golden/make_golden.py from the oracle itself: the pages print no worked
example).  A change to the oracle's arithmetic shows up here and has to be
justified by a passage of the pages before the fixtures are rewritten."""
import glob
import json
import os

import numpy as np
import pytest

from tests.golden import make_golden

FILES = sorted(glob.glob(os.path.join(os.path.dirname(__file__), "golden", "*.json")))


def test_every_case_has_a_fixture():
    names = {os.path.basename(f)[:-5] for f in FILES}
    assert names == set(make_golden.CASES)


@pytest.mark.parametrize("path", FILES, ids=[os.path.basename(f) for f in FILES])
def test_oracle_matches_its_fixture(path):
    rec = json.load(open(path))
    got = make_golden.compute(rec["case"])
    assert set(got) == set(rec["outputs"])
    for k, v in rec["outputs"].items():
        np.testing.assert_allclose(np.asarray(got[k]), np.asarray(v), rtol=1e-12, atol=1e-14,
                                   err_msg=k)
