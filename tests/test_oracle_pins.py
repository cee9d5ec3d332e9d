"""The CPU oracle against the pins that the pages and the mathematics fix
(see ``oracle_pins.py`` for what each pin compares against)."""
import pytest

from oracle import pq_oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def O():
    return pq_oracle.default()


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS,
                         ids=lambda c: c.__name__)
def test_pin(O, check):
    check(O)


def test_empty_and_bad_shapes(O):
    import numpy as np
    wq, codes, packed = O.fwd(pq_oracle.SEQ2, np.zeros((0, 8), np.float32),
                              np.zeros(0, np.float32), pack=True)
    assert wq.shape == (0, 8) and packed.shape == (0, 2)
    with pytest.raises(ValueError):  # 2-bit packing needs cols % 4 == 0
        O.fwd(pq_oracle.SEQ2, np.zeros((1, 6), np.float32),
              np.ones(1, np.float32), pack=True)
    with pytest.raises(ValueError):
        O.fwd(99, np.zeros((1, 4), np.float32), np.ones(1, np.float32))
