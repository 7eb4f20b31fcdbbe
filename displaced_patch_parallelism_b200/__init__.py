"""Displaced patch parallelism (DistriFusion) block step for B200: C-ABI CUDA library + binding.

The compute path is ``libdp.so`` (hand-written sm_100a kernels); ``binding``
marshals torch tensors into its C calls.  Build it with
``python -m displaced_patch_parallelism_b200.build``.
"""
from . import binding  # noqa: F401
from .binding import DPError  # noqa: F401
