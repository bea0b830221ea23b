"""The fp64 oracle against its pins (CPU only)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load_library(oracle.build())


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(lib, pin):
    pin(lib)


def test_oracle_rejects_bad_rows(lib):
    import numpy as np
    import torch
    q = torch.zeros(1, 1, 4, 8, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        oracle.attention_f64(q, q, q, False, 1.0, rows=np.array([4], dtype=np.int64), lib=lib)
