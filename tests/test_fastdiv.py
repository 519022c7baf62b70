"""The fused token order divides positions by the length of a patch's run of frames with a multiply-high
instead of a hardware division (Granlund and Montgomery, "Division by Invariant Integers using
Multiplication", 1994, round-up method for 32-bit operands). This replays the method with the
constants make_fastdiv computes in svg_common.cuh and checks it against integer division for every
divisor a run can have and numerators up to the largest position; the GPU tests check the device code
through the fused order's bitwise equality with the permuted path."""
import numpy as np


def make_fastdiv(d):
    l = 0
    while l < 32 and (1 << l) < d:
        l += 1
    m = ((1 << 32) * ((1 << l) - d)) // d + 1
    return m & 0xFFFFFFFF, min(l, 1), max(l - 1, 0)


def fastdiv(n, f):
    m, s1, s2 = f
    n = np.asarray(n, dtype=np.uint64)
    t = (n * np.uint64(m)) >> np.uint64(32)
    return ((t + ((n - t) >> np.uint64(s1))) >> np.uint64(s2)).astype(np.int64)


def test_fastdiv_matches_integer_division():
    rng = np.random.default_rng(7)
    divisors = list(range(1, 300)) + [1000, 3599, 4096, 14399, 65537, 1 << 20, (1 << 22) - 1]
    for d in divisors:
        f = make_fastdiv(d)
        n = np.concatenate([np.arange(0, 5000), rng.integers(0, 1 << 22, 20000),
                            [(1 << 22) - 1, (1 << 31) - 1, (1 << 32) - 1]]).astype(np.uint64)
        assert np.array_equal(fastdiv(n, f), (n // np.uint64(d)).astype(np.int64)), d


def test_header_holds_the_same_constants():
    """make_fastdiv in the CUDA header computes m, s1, s2 as replayed here."""
    import os
    src = open(os.path.join(os.path.dirname(__file__), "..", "block_sparse_spatio_flash_b200", "csrc",
                            "svg_common.cuh")).read()
    assert "((1ull << 32) * ((1ull << l) - d)) / d) + 1" in src
    assert "f.s1 = l < 1 ? l : 1;" in src and "f.s2 = l > 0 ? l - 1 : 0;" in src
