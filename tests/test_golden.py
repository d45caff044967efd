"""The oracle against its own committed regression fixtures (see
tests/golden/make_golden.py): any change to the oracle's arithmetic shows up
here and must be justified and the fixtures regenerated."""
import json
import os

import numpy as np
import pytest

from tests.golden import make_golden as G

with open(G.OUT) as f:
    FIXTURES = json.load(f)


@pytest.mark.parametrize("name", sorted(FIXTURES))
def test_oracle_matches_fixture(name):
    case = {c[0]: c for c in G.cases()}[name]
    _, w, seed, extra = case
    got = G.run(w, seed, extra)
    want = FIXTURES[name]["outputs"]
    assert set(got) == set(want)
    for k in want:
        a, b = np.asarray(got[k], np.float64), np.asarray(want[k], np.float64)
        assert a.shape == b.shape, (name, k)
        assert np.allclose(a, b, rtol=1e-14, atol=1e-300), (name, k)
