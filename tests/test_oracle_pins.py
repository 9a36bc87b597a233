"""The oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

import oracle
from oracle_pins import PINS


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)


def test_oracle_rejects_bad_arguments(orc):
    import numpy as np

    q = np.zeros((1, 2, 3, 4))
    k = np.zeros((1, 2, 2, 4))
    with pytest.raises(ValueError):  # Hq % Hkv != 0
        orc.attention(q, k, k)
    q = np.zeros((2, 2, 2, 4))
    k = np.zeros((2, 2, 2, 4))
    with pytest.raises(ValueError):  # block-diagonal needs B == 1
        orc.attention(q, k, k, bias=oracle.BIAS_BLOCKDIAG, seqstart_q=[0, 2])
