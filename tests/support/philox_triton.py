"""Philox4x32-10 by a second, independent implementation: Triton's
``tl.philox`` (its own transcription of Salmon, Moraes, Dror, Shaw, "Parallel
random numbers: as easy as 1, 2, 3", SC 2011), run on the CPU by Triton's
interpreter.  Test support only: it pins the oracle's generator and takes no
part in the library.

    python tests/support/philox_triton.py < cases.json > words.json

Input: a JSON list of [c0, c1, c2, c3, k0, k1] (uint32 each).  Output: a JSON
list of the four output words of each case.
"""
import json
import os
import sys

os.environ["TRITON_INTERPRET"] = "1"

import numpy as np  # noqa: E402
import torch  # noqa: E402
import triton  # noqa: E402
import triton.language as tl  # noqa: E402


@triton.jit
def _philox_cases(inp, out, n, BLOCK: tl.constexpr):
    i = tl.arange(0, BLOCK)
    m = i < n
    c0 = tl.load(inp + 6 * i + 0, mask=m).to(tl.uint32)
    c1 = tl.load(inp + 6 * i + 1, mask=m).to(tl.uint32)
    c2 = tl.load(inp + 6 * i + 2, mask=m).to(tl.uint32)
    c3 = tl.load(inp + 6 * i + 3, mask=m).to(tl.uint32)
    k0 = tl.load(inp + 6 * i + 4, mask=m).to(tl.uint64)
    k1 = tl.load(inp + 6 * i + 5, mask=m).to(tl.uint64)
    # tl.philox takes the key as one 64-bit seed: low word k0, high word k1
    a, b, c, d = tl.philox((k1 << 32) | k0, c0, c1, c2, c3)
    tl.store(out + 4 * i + 0, a.to(tl.int64), mask=m)
    tl.store(out + 4 * i + 1, b.to(tl.int64), mask=m)
    tl.store(out + 4 * i + 2, c.to(tl.int64), mask=m)
    tl.store(out + 4 * i + 3, d.to(tl.int64), mask=m)


def main():
    cases = np.asarray(json.load(sys.stdin), dtype=np.int64).reshape(-1, 6)
    n = cases.shape[0]
    block = triton.next_power_of_2(max(n, 1))
    inp = torch.from_numpy(cases.copy())
    out = torch.zeros((n, 4), dtype=torch.int64)
    _philox_cases[(1,)](inp, out, n, BLOCK=block)
    json.dump([[int(v) & 0xFFFFFFFF for v in row] for row in out.tolist()], sys.stdout)


if __name__ == "__main__":
    main()
