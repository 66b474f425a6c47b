"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_bf16_rounding_helper_is_rne():
    # 1 + 2^-8 is a tie between bf16 neighbours 1 and 1 + 2^-7: rounds to even (1.0)
    bits = oracle_pins.f32_to_bf16_bits([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5])
    assert list(bits) == [0x3F80, 0x3F82, 0xC020]


def test_oracle_reports_thread_count(orc):
    assert orc.num_threads() >= 1


def test_invalid_shapes_rejected(orc):
    q = np.zeros((1, 3, 8), np.uint16)
    k = np.zeros((1, 2, 4, 8), np.uint16)
    with pytest.raises(Exception):
        orc.paged_attention(q, k, k, np.zeros((1, 1), np.int32), np.array([1], np.int32), 1.0)
