"""Sigmoid-routed mixture-of-experts FFN (GLM-4.7-Flash / GLM-5 shapes) for B200.

The computation runs in hand-written sm_100a CUDA kernels behind a C ABI
(``libsrm_moe.so``, declared in ``include/srm_moe.h``).  ``sigmoid_routed_mixture_b200.moe``
is the thin ctypes binding; ``workloads`` holds the seeded synthetic inputs.
Submodules are imported lazily so that importing the package never needs a GPU.
"""

__all__ = ["moe", "workloads"]
