"""The CPU oracle against facts fixed outside itself (see tests/oracle_pins.py)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_rejects_out_of_range_codes_and_bad_shapes():
    cb = np.zeros((1, 4, 2), np.float16)
    codes = np.array([[[4]]], np.uint8)      # 4 >= 2^B
    with pytest.raises(oracle.OracleError):
        oracle.dequantize(codes, cb, np.ones(1, np.float16), 1, 2, 2)
    with pytest.raises(ValueError):
        oracle.dequantize(np.zeros((1, 1, 2), np.uint8), cb, np.ones(1, np.float16), 1, 2, 2)
    with pytest.raises(TypeError):
        oracle.dequantize(codes.astype(np.uint16), cb, np.ones(1, np.float16), 1, 2, 2)
