"""The CPU oracle against its pins (hand-worked examples, closed forms, brute force, invariants).

Runs on CPU only; see tests/oracle_pins.py for what each pin checks."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_capacity_formula(orc):
    # every local expert wastes fewer than block_size rows, so T*k + E_local*(bs-1) bounds N_pad
    assert orc.align_capacity(4096, 8, 128, 64) == 4096 * 8 + 128 * 63
    assert orc.align_capacity(2, 6, 40, 8) == 12 + 40 * 7
    assert orc.align_capacity(-1, 6, 40, 8) == -1


def test_invalid_arguments_rejected(orc):
    import numpy as np
    with pytest.raises(ValueError):
        orc.topk_softmax(np.zeros((2, 4), np.float32), 5, True)
    with pytest.raises(ValueError):
        orc.align_permute(np.zeros((2, 2), np.int32), 4, 2, None, 3)  # identity map needs E_local == E_global
