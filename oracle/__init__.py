"""FP64 CPU oracle for the SiLU-gated RMSNorm training path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``, never by the product path.  It shares no
code with the CUDA kernels in ``gated_norm_b200``.
"""
from .gated_norm_ref import bwd, ckpt_step, dw_rows, fwd, sigmoid, silu  # noqa: F401
