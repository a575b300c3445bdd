"""The fp64 oracle against the pins in oracle_pins.py (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, oracle_mod):
    pin(oracle_mod.default())


def test_oracle_rejects_bad_arguments(oracle_mod):
    import numpy as np
    orc = oracle_mod.default()
    q = np.zeros((1, 8, 2, 4))
    k = np.zeros((1, 8, 1, 4))
    with pytest.raises(ValueError):
        orc.bifocal_rows(q, k, k, [0], [8], [0], w_local=1, w_pretrained=4,
                         rope_base=1e4)  # row out of range
    with pytest.raises(ValueError):
        orc.bifocal_rows(q, k, k, [0], [0], [0], w_local=-1, w_pretrained=4,
                         rope_base=1e4)
    with pytest.raises(ValueError):
        orc.bifocal_decode(q[:, 0], k, k, 8, w_local=1, w_pretrained=4,
                           rope_base=1e4)  # pos beyond the cache
