"""The fp64 oracle against its pins (no GPU)."""
import pytest

import oracle
from oracle_pins import ALL_PINS, BWD_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.attention_forward)


@pytest.mark.parametrize("pin", BWD_PINS, ids=lambda p: p.__name__)
def test_oracle_backward_pin(pin):
    pin(oracle.attention_forward, oracle.attention_backward)


def test_oracle_rejects_bad_arguments():
    import numpy as np
    q = np.zeros((1, 3, 4, 2))
    kv = np.zeros((1, 2, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention_forward(q, kv, kv, causal=False, scale=1.0)  # 3 % 2 != 0
    q = np.zeros((1, 2, 4, 2))
    with pytest.raises(ValueError):
        oracle.attention_forward(q, kv, kv, causal=False, scale=1.0, seqlens=np.array([5]))
    with pytest.raises(TypeError):
        oracle.attention_forward(q.astype(np.float32), kv, kv, causal=False, scale=1.0)
