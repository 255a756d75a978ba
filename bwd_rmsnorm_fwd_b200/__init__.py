"""B200-native training RMSNorm (forward, backward with deterministic or blocked-FP32
dw, fused residual add, per-head views) behind the C-ABI library librmsnorm_train.

The library is loaded on first use and its absence is an error: there is no CPU or
eager fallback.
"""

from .api import (RMSNormTrainFunction, Workspace, bwd_path, det_plan, rmsnorm_train,
                  rmsnorm_train_bwd, rmsnorm_train_fwd, set_small_rows_limit, status)

__all__ = ["RMSNormTrainFunction", "Workspace", "bwd_path", "det_plan", "rmsnorm_train",
           "rmsnorm_train_bwd", "rmsnorm_train_fwd", "set_small_rows_limit", "status"]
