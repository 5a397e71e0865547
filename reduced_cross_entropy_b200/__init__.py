"""Reduced cross-entropy (RECE / SCE) loss on B200 (sm_100a).

The loss of "RECE: Reduced Cross-Entropy Loss for Large-Catalogue Sequential
Recommenders" (section 3, Algorithm 1) with the top-k negatives of "Scalable
Cross-Entropy Loss for Sequential Recommendations with Large Item Catalogs": every
step runs in the CUDA library ``librece_b200.so`` (C ABI: ``include/rece.h``); this
package only marshals torch tensors into it.
"""
from ._lib import ReceError
from .ops import (Plan, bucketize_sort, device_status, full_ce_bwd, full_ce_fwd,
                  full_ce_workspace_bytes, loss_bwd, loss_fwd, rece_loss)

__all__ = ["Plan", "ReceError", "bucketize_sort", "loss_fwd", "loss_bwd", "rece_loss",
           "full_ce_fwd", "full_ce_bwd", "full_ce_workspace_bytes", "device_status"]
