"""gated_norm_b200: SiLU-gated RMSNorm training kernels for B200 (sm_100a).

The kernels live in ``libgnorm.so`` behind the C ABI of ``include/gnorm.h``; this package
is a thin binding over it.  Importing the package loads the library and fails loudly if it
has not been built (``python gated_norm_b200/build.py``): there is no CPU fallback.
"""
from .autograd import GatedRMSNorm, GatedRMSNormFunction, gated_rmsnorm  # noqa: F401
from .gnorm import (  # noqa: F401
    GnormError,
    gnorm_build_info,
    gnorm_bwd,
    gnorm_bwd_noalloc,
    gnorm_bwd_workspace_bytes,
    gnorm_bwd_workspace_bytes_for,
    gnorm_ckpt_step,
    gnorm_ckpt_step_host,
    gnorm_ckpt_step_host_bytes,
    gnorm_device_error,
    gnorm_dw_reduce,
    gnorm_fwd,
    gnorm_fwd_bwd,
    gnorm_plan_query,
    gnorm_selftest_wait_timeout,
    gnorm_set_tuning,
    gnorm_status_string,
    workspace,
)
