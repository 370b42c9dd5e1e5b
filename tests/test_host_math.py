"""Host-side checks of arithmetic identities the kernels rely on."""
import os
import subprocess
import tempfile

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def test_division_by_grid_size_is_correctly_rounded():
    """The refit divides by qmax with one FMA correction of the product by the
    rounded reciprocal; on zero, subnormals, binade edges and 80M random
    non-negative floats it equals IEEE division."""
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "divcheck")
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-o", exe,
                               os.path.join(HERE, "support", "divcheck.c"), "-lm"])
        r = subprocess.run([exe], capture_output=True, text=True, timeout=600)
        assert r.returncode == 0 and r.stdout.strip() == "0", r.stdout


def test_multiply_high_division_by_head_dim():
    """Row -> head index uses (n * m) >> 32 with m = floor(2^32 / d) + 1,
    exact for every n < 512 d and d <= 2048 (the library caps head_dim at
    2048 and heads at 512)."""
    for d in list(range(1, 130)) + [255, 256, 1000, 1023, 1024, 2047, 2048]:
        m = (1 << 32) // d + 1
        n = np.arange(0, 512 * d, dtype=np.uint64)
        assert np.array_equal((n * np.uint64(m)) >> np.uint64(32), n // np.uint64(d)), d
