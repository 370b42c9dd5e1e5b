"""libssq: the Mamba-2 recurrent-state update with the per-request state held
in low-bit form (int8 / int4, symmetric or asymmetric grid, one scale per
(head, head_dim) row), on B200 (sm_100a).

The compute lives in ``libssq.so`` (hand-written CUDA behind a C ABI,
declared in ``include/ssq.h``).  ``quantized_recurrent_state_mamba_b200.ssq``
is the thin ctypes binding over it; importing that module loads the library
and fails loudly when it is missing.  ``workloads`` draws seeded synthetic
inputs and does no arithmetic of the method.
"""
__version__ = "0.1.0"
