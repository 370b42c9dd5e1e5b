"""Pins for the oracle's counter-based generator (stochastic rounding,
"ssm-state-quantization" README, Findings 9).

The oracle's Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC 2011) is checked
word for word against a second implementation written by other hands:
Triton's ``tl.philox``, run on the CPU by Triton's interpreter
(``tests/support/philox_triton.py``).  The cases cover the all-zero and
all-ones counters and keys, every counter word and key word on its own, and
seeded random counters and keys.  A second pin takes the 16-bit draw of
every entry of a few rows from the independent generator, by the layout the
stochastic-rounding reading states (counter (row*N/8 + n/8, layer, slot,
step), key (seed low word, seed high word), word (n%8)/2, low half for even
n), and compares the oracle's draws with it.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SCRIPT = os.path.join(ROOT, "tests", "support", "philox_triton.py")
M32 = 0xFFFFFFFF


def _cases():
    cases = [[0, 0, 0, 0, 0, 0], [M32] * 6]
    for i in range(6):                     # one word set, the rest zero
        c = [0] * 6
        c[i] = 0x9E3779B9 ^ (0x1111 * (i + 1))
        cases.append(c)
    rng = np.random.Generator(np.random.PCG64(20111112))
    cases += rng.integers(0, 2**32, size=(40, 6), dtype=np.uint64).astype(np.int64).tolist()
    return [[int(v) & M32 for v in c] for c in cases]


# (seed, step, layer, slot) of the draw-layout pin
SR_KEYS = [(0x0123456789ABCDEF, 7, 3, 11), (12345, 1, 0, 0), (2**64 - 1, 2**32 - 1, 23, 255)]
SR_ROWS, SR_N = 3, 32


def _sr_cases():
    out = []
    for seed, step, layer, slot in SR_KEYS:
        for r in range(SR_ROWS):
            for blk in range(SR_N // 8):
                out.append([r * (SR_N // 8) + blk, layer, slot, step,
                            seed & M32, (seed >> 32) & M32])
    return out


@pytest.fixture(scope="module")
def independent():
    """Triton's Philox words for the pin cases and the draw-layout cases."""
    cases = _cases() + _sr_cases()
    r = subprocess.run([sys.executable, SCRIPT], input=json.dumps(cases),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    words = json.loads(r.stdout)
    assert len(words) == len(cases)
    n = len(_cases())
    return cases[:n], words[:n], words[n:]


def test_philox_matches_an_independent_implementation(oref, independent):
    cases, words, _ = independent
    bad = []
    for c, w in zip(cases, words):
        got = oref.philox4x32_10(c[:4], c[4:])
        if got != w:
            bad.append((c, got, w))
    assert not bad, f"{len(bad)} of {len(cases)} cases differ, first: {bad[0]}"


def test_philox_is_a_keyed_function_of_every_word(oref, independent):
    """Changing any one counter or key word changes every output word (the
    oracle has no word it ignores)."""
    cases, words, _ = independent
    base = oref.philox4x32_10([0, 0, 0, 0], [0, 0])
    for i in range(6):
        c = [0] * 6
        c[i] = 1
        w = oref.philox4x32_10(c[:4], c[4:])
        assert all(a != b for a, b in zip(w, base)), i


def test_sr_draws_take_the_stated_words(oref, independent):
    _, _, sr_words = independent
    k = 0
    for seed, step, layer, slot in SR_KEYS:
        u = oref.sr_draws(seed, step, layer, slot, SR_ROWS, SR_N)
        for r in range(SR_ROWS):
            for blk in range(SR_N // 8):
                w = sr_words[k]
                k += 1
                for e in range(8):
                    n = blk * 8 + e
                    want = (w[e // 2] >> (16 * (e % 2))) & 0xFFFF
                    assert u[r, n] == want, (seed, r, n)
