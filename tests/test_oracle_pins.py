"""The CPU oracle against its pins (no GPU)."""

import pytest

import oracle
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle)


def test_materialised_intermediate_size():
    """StreamIndex abstract: [B, S, H_I, S/m] FP32 at S=65,536, H_I=64, m=4 is
    256 GB -- the tensor the indexer must never build."""
    B, S, H, m, nbytes, total = oracle_pins._rows("streamindex_materialised.txt")[0]
    assert B * S * H * (S // m) * nbytes == total == 256 * 2 ** 30
