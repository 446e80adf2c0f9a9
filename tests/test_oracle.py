"""The oracle against its pins (CPU only; no GPU, no CUDA library)."""
import pytest

from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(oracle, pin):
    pin(oracle)


def test_oracle_threads(oracle):
    assert oracle.num_threads() >= 1
