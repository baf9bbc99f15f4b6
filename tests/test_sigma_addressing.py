"""The 16-bit table addressing of the SwiGLU forward's sigmoid lookups
(sigma_key / sigma_pair_s in moe_gated_activation_b200/csrc/device_common.cuh),
checked on the CPU: for every bf16 pattern in either 16-bit lane and every
table address up to 16 KiB, the two lanes of c * 4 + key + sign bits (32-bit
wrap-around arithmetic) are exactly the byte addresses of the entries the
pointer form of the lookup reads.  The GPU side runs the same expression on
all 65536 inputs in the exhaustive sigmoid test."""
import numpy as np

LO, HI, NEG = 0x3300, 0x4300, 8192 * 4          # table range and negative-half byte offset


def _key(T):
    return ((T - 4 * LO) & 0xFFFF) | (((T - 4 * LO - 1) & 0xFFFF) << 16)


def _expected(T, b):
    mag = np.clip(b & 0x7FFF, LO, HI).astype(np.int64)
    return T + 4 * (mag - LO) + np.where(b & 0x8000, NEG, 0)


def test_folded_addresses_match_the_pointer_lookup():
    rng = np.random.default_rng(0)
    b = np.arange(65536, dtype=np.int64)
    partner = rng.integers(0, 65536, size=65536).astype(np.int64)
    for T in list(range(0, 16369, 16)):
        for lo_, hi_ in ((b, partner), (partner, b)):
            G = lo_ | (hi_ << 16)
            c = np.clip(lo_ & 0x7FFF, LO, HI) | (np.clip(hi_ & 0x7FFF, LO, HI) << 16)
            a = (c * 4 + _key(T) + (G & 0x80008000)) & 0xFFFFFFFF
            assert np.array_equal(a & 0xFFFF, _expected(T, lo_)), T
            assert np.array_equal(a >> 16, _expected(T, hi_)), T


def test_the_table_fits_below_64_kib():
    # highest entry: negative half, clamped magnitude HI, 4 bytes wide
    assert 16368 + NEG + 4 * (HI - LO) + 4 <= 0x10000
