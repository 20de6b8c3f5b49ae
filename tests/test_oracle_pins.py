"""The fp64 oracle against the values the pages and mathematics fix (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(oracle_lib, pin):
    pin(oracle_lib)


def test_oracle_threads_do_not_change_bits(oracle_lib):
    """OpenMP over tokens must not change any bit of the result."""
    import numpy as np
    wl, xb, ids, w, mats, sh = oracle_pins._tiny_forward(oracle_lib, seed=4)
    y1 = oracle_lib.moe_ffn_monolith(xb, ids, w, *mats, wl.E, shared=sh, threads=1)
    y4 = oracle_lib.moe_ffn_monolith(xb, ids, w, *mats, wl.E, shared=sh, threads=4)
    assert np.array_equal(y1, y4)
