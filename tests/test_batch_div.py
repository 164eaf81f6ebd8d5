"""The lookup kernel finds a bag's table with an unsigned division by the batch
size done as a multiply-high and two shifts (Granlund and Montgomery, "Division
by invariant integers using multiplication", PLDI 1994, Fig. 4.1). The host
computes the multiplier as libdq's make_batch_div does; this checks the method
against exact integer division for the batch sizes the workloads use and for
edge divisors."""
import random


def _make(d):
    ell = 0
    while (1 << ell) < d:
        ell += 1
    m = ((1 << 32) * ((1 << ell) - d)) // d + 1
    return m & 0xFFFFFFFF, min(ell, 1), max(ell - 1, 0)


def _div(n, v):
    m, s1, s2 = v
    t = (m * n) >> 32
    return (t + ((n - t) >> s1)) >> s2


def test_invariant_division_matches_integer_division():
    rng = random.Random(0)
    for d in [1, 2, 3, 7, 64, 97, 2048, 8192, 16384, 65536, 65537, 1 << 20, 2 ** 31 - 1, 2 ** 31]:
        v = _make(d)
        ns = [0, 1, d - 1, d, d + 1, 2 ** 31 - 1, 2 ** 32 - 1] + [rng.getrandbits(32) for _ in range(20000)]
        ns += [k * d + r for k in (1, 1000, (2 ** 31 - 1) // d) for r in (0, d - 1) if k * d + r < 2 ** 32]
        for n in ns:
            assert _div(n, v) == n // d, (d, n)
