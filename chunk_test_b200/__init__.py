"""B200 (sm_100a) LaCT fast-weight TTT layer forward.

The layer runs entirely in liblact_b200.so (hand-written tcgen05/TMA kernels
for the bf16 path, CUDA-core kernels for the fp32 path) behind the C ABI of
include/lact.h.  This package is the thin Python binding: `ttt_fwd` takes
torch CUDA tensors, `ttt_fwd_host` takes host tensors.
"""
from ._abi import (  # noqa: F401
    APPLY_THEN_UPDATE, UPDATE_THEN_APPLY, RULE_GD, RULE_MOMENTUM, RULE_MUON,
    LACT_OK, LACT_EINVAL, LACT_ENOSPC, LACT_ECUDA, LACT_ETIMEOUT, LACT_ENODEV, LACT_ETOOBIG,
    LACT_ECOMM, REDUCE_SUM, REDUCE_MEAN,
    NOALLOC_SCRATCH_BYTES,
    LactError, LactProblem, LactFwdOpts, LIB_PATH, lib, status_string, profile_enable, profile_read,
)
from .layer import (  # noqa: F401
    ttt_fwd, ttt_fwd_host, ttt_fwd_noalloc, ttt_bwd, workspace_bytes, bwd_workspace_bytes,
    host_workspace_bytes, launch_count, status,
    device_check, selftest_wait_timeout, make_problem, torch_distributed_allreduce, swa_fwd,
    swa_workspace_bytes,
)
