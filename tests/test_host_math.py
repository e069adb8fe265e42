"""Host-side arithmetic the kernels rely on (no GPU needed)."""


def test_multiply_high_division_is_exact_for_unit_rows():
    # The scoring epilogues divide row indices n (0..4096) by R (1..2048) as
    # umulhi(n, ceil(2^32 / R)); exact whenever n * R < 2^32.
    for R in list(range(2, 300)) + [511, 512, 513, 960, 1023, 1024, 1536, 2047, 2048]:
        m = ((1 << 32) + R - 1) // R
        for n in range(0, 4097):
            assert (n * m) >> 32 == n // R, (n, R)
