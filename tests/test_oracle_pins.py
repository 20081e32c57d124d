"""The fp64 oracle against what the pages and the mathematics fix (CPU only)."""

import pytest

from oracle import oracle as O
from oracle_pins import ALL_CHECKS


@pytest.fixture(scope="module")
def lib():
    return O.lib()


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__[len("check_"):])
def test_oracle_pin(check, lib):
    check(lib)


def test_bf16_widening_matches_torch():
    import numpy as np
    import torch

    bits = np.array([0x0000, 0x8000, 0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F, 0xFF7F, 0x3E9A], dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([O.lib().oracle_bf16_to_double(int(b)) for b in bits])
    assert np.array_equal(got, ref)
    assert np.array_equal(O.bf16_to_f64(bits), ref)
