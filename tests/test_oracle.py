"""The fp64 oracle against closed forms, library routines, brute force and
invariants (CPU only)."""

import numpy as np
import pytest

import _oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(oracle_lib, pin):
    pin(oracle_lib)


@pytest.mark.parametrize("pin", pins.BWD_PINS, ids=lambda p: p.__name__)
def test_oracle_backward_pin(oracle_lib, pin):
    pin(oracle_lib)


def test_oracle_rejects_bad_arguments(oracle_lib):
    q = np.zeros((1, 4, 3, 8), np.uint16)
    k = np.zeros((1, 4, 2, 8), np.uint16)
    with pytest.raises(ValueError):          # Hq % Hkv != 0
        oracle_lib.attention(q, k, k, False, 1.0)
    q = np.zeros((1, 4, 2, 8), np.uint16)
    with pytest.raises(ValueError):          # row out of range
        oracle_lib.attention(q, k, k, False, 1.0, rows=[4])
    with pytest.raises(ValueError):          # bad key range
        oracle_lib.attention(q, k, k, False, 1.0, k_range=(3, 2))


def test_oracle_thread_count_does_not_change_result(oracle_lib):
    rng = np.random.default_rng(0)
    import torch
    from exact_tiled_attention_29_b200.inputs import bf16_bits
    q = bf16_bits(torch.from_numpy(rng.standard_normal((2, 37, 4, 16)).astype(np.float32)).bfloat16())
    k = bf16_bits(torch.from_numpy(rng.standard_normal((2, 41, 2, 16)).astype(np.float32)).bfloat16())
    v = bf16_bits(torch.from_numpy(rng.standard_normal((2, 41, 2, 16)).astype(np.float32)).bfloat16())
    o1, l1 = oracle_lib.attention(q, k, v, True, 0.25, nthreads=1)
    o4, l4 = oracle_lib.attention(q, k, v, True, 0.25, nthreads=5)
    assert np.array_equal(o1, o4) and np.array_equal(l1, l4)
    # the row-list path returns exactly the listed rows of the full result
    rows = [0, 5, 36]
    orr, lr = oracle_lib.attention(q, k, v, True, 0.25, rows=rows)
    assert np.array_equal(orr, o1[:, rows]) and np.array_equal(lr, l1[:, :, rows])
