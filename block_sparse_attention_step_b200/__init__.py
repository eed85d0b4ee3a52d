"""B200-native block-sparse decode attention step (SeerAttention-R).

The compute path lives in the shared library ``libseer.so`` (hand-written
sm_100a CUDA kernels behind a C ABI, declared in ``include/seer.h``); the
Python module ``seer`` is a thin ctypes binding over it.  ``workloads`` draws
the seeded synthetic inputs.  Importing the package loads nothing: the
library is opened on first use of ``seer`` and a missing build raises.
"""
__all__ = ["seer", "workloads"]
