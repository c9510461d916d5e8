"""B200 (sm_100a) top-k sparse attention backward (SparseFlashAttentionGrad), dense
varlen FlashAttention backward and the dense lightning-indexer gradient with KL loss,
behind the C ABI of libsfa (include/sfa.h)."""
from ._native import SfaError, load  # noqa: F401
from .ops import (  # noqa: F401
    compact_indices,
    dout_absmax,
    fa_fwd,
    fa_grad,
    key_rows,
    lig_kl_grad,
    lig_kl_grad_workspace_size,
    lig_shape,
    sfa_dkv_accumulator,
    sfa_dkv_finalize,
    sfa_fwd,
    sfa_grad,
    sfa_grad_rows,
    sfa_grad_workspace_size,
    sfa_shape,
    set_wait_limit,
    softmax_grad_rowsum,
    workspace_status,
)
from .shard import balanced_row_ranges, sfa_grad_sharded  # noqa: F401
from .host import HostPipeline, sfa_grad_host  # noqa: F401

__all__ = ["sfa_grad", "sfa_fwd", "fa_grad", "fa_fwd", "compact_indices", "softmax_grad_rowsum",
           "sfa_grad_workspace_size", "sfa_shape", "SfaError", "load", "sfa_grad_rows", "sfa_dkv_accumulator",
           "sfa_dkv_finalize", "sfa_grad_sharded", "balanced_row_ranges", "sfa_grad_host", "HostPipeline",
           "workspace_status", "set_wait_limit", "lig_kl_grad", "lig_kl_grad_workspace_size", "lig_shape",
           "dout_absmax", "key_rows"]
