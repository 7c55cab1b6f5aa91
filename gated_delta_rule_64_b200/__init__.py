"""Gated delta rule for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libgdn.so`` built from ``csrc/``;
``gdn`` exposes its entry points (``gdn_chunk_fwd``, ``gdn_decode_step``) for
torch CUDA tensors.  ``inputs`` draws seeded synthetic inputs and does not need
the library.
"""
from .inputs import Workload, make_inputs  # noqa: F401

__all__ = ["Workload", "make_inputs"]
