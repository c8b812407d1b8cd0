"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def o():
    return oracle.get()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(o, pin):
    pin(o)


def test_rejects_bad_shapes(o):
    import numpy as np
    x = np.zeros((1, 12), dtype=np.float16)
    with pytest.raises(ValueError):
        o.quantize(x, np.ones(12, np.float32), np.ones(12, np.int8), 4)
    x = np.zeros((1, 16), dtype=np.float16)
    with pytest.raises(ValueError):
        o.quantize(x, np.ones(16, np.float32), np.ones(16, np.int8), 32)
