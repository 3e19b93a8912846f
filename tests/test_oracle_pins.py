"""The oracle against facts that do not come from it (CPU only)."""
import pytest

import oracle
from tests import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.Oracle()


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(orc, check):
    check(orc)


def test_empty_sequence(orc):
    import numpy as np
    z = np.zeros((1, 2, 0, 4))
    assert orc.bidir_fwd(z, z, z).shape == (1, 2, 0, 4)
    o, st = orc.bidir_fwd(z, z, z, want_state=True)
    assert (st == 0).all()
    assert orc.retention_fwd(z, z, z, np.array([0.5, 0.5])).shape == (1, 2, 0, 4)
