"""The multiply-high division the permute kernels use for their row index (kernels.h,
FastDiv): with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1, the quotient is
(mulhi(n, m) + n) >> s for every 0 <= n < 2^31.  Checked here against integer division on
the divisors the workloads use, extremes and random ones."""
import random


def fastdiv(n, d):
    s = 0
    while (1 << s) < d:
        s += 1
    m = ((((1 << 32) * ((1 << s) - d)) // d) + 1) & 0xFFFFFFFF
    t = ((n * m) >> 32) + n
    assert t < (1 << 32)
    return t >> s


def test_fastdiv_matches_integer_division():
    rng = random.Random(3)
    divisors = [1, 2, 3, 7, 24, 48, 1104, 1280, 4864, 36992, 39296, 70144, 279040,
                (1 << 30) + 1, (1 << 31) - 1] + [rng.randint(1, (1 << 31) - 1) for _ in range(300)]
    for d in divisors:
        ns = [0, 1, d - 1, d, d + 1, (1 << 31) - 1] + [rng.randrange(1 << 31) for _ in range(2000)]
        for n in ns:
            if 0 <= n < (1 << 31):
                assert fastdiv(n, d) == n // d, (n, d)
