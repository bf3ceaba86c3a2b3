"""Integer identities the kernels rely on, checked on the host.

The GEMV locates a 512-byte piece of the packed weights (row block b, 128-k
group g) from its index i within a CTA's share as b = i / KG with KG = K/128,
computed as (i * ceil(2^32 / KG)) >> 32. The launcher refuses shares of 2^23
pieces or more; below that the multiply-shift is exact for every KG the
library accepts (K <= 65536, so KG <= 512)."""
import numpy as np

LIMIT = 1 << 23          # pieces per CTA the launcher admits (exclusive)
MAX_KG = 65536 // 128


def magic(kg: int) -> int:
    return ((1 << 32) + kg - 1) // kg


def test_magic_error_term_bounds_the_range():
    # i * m / 2^32 = i / KG + i * e / (KG * 2^32) with e = m * KG - 2^32; the
    # quotient is exact while (i mod KG) + i * e / 2^32 < KG, which holds for
    # i < 2^23 as soon as e < 2^32 / 2^23 = 512 and e < KG
    for kg in range(1, MAX_KG + 1):
        e = magic(kg) * kg - (1 << 32)
        assert 0 <= e < kg, kg
        assert LIMIT * e < (1 << 32), kg


def test_magic_division_at_the_worst_remainders():
    # every KG, the indices just below the limit with the largest remainder
    # (where an error would show first), plus random indices in range
    rng = np.random.default_rng(5)
    for kg in range(1, MAX_KG + 1):
        m = magic(kg)
        top = (LIMIT - 1) // kg
        idx = [q * kg + kg - 1 for q in range(max(0, top - 3), top)]
        idx += [int(v) for v in rng.integers(0, LIMIT, 16)]
        for i in idx:
            if i < LIMIT:
                assert (i * m) >> 32 == i // kg, (kg, i)


def test_magic_division_fails_past_the_range_for_some_kg():
    # the limit is not vacuous: far enough past it the multiply-shift breaks
    bad = 0
    for kg in (501, 509, 511):
        m = magic(kg)
        e = m * kg - (1 << 32)
        q = ((1 << 32) // e) // kg + 2
        i = q * kg + kg - 1
        bad += ((i * m) >> 32) != i // kg
    assert bad > 0
