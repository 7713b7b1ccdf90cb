"""B200 (sm_100a) In-Kernel Broadcast Optimization: IKBO-LCB and IKBO-DCA.

Thin Python binding over the C ABI in ``include/rocs_ikbo.h`` (``librocs_ikbo.so``).
Every step of the computation runs in the library's CUDA kernels; this module only
marshals torch tensors (device memory, streams) into the C argument structs.  There is
no CPU or PyTorch fallback: if the native library is missing, importing the binding
functions raises.

Operations ("ROCS: Request-Oriented Compute Sharing ...", arXiv:2607.27744):
  * :func:`rocs_lcb_forward` -- section 3.1.2 Eq. (6) via the section 4.1 Eq. (14)
    decomposition, broadcast-add fused into the candidate GEMM epilogue (section 4.2).
  * :func:`rocs_lcb_block_forward` -- the same with each output group's bias, residual,
    group-local LayerNorm/RMSNorm and activation fused into the epilogue (section 3.1.3).
  * :func:`rocs_fm_forward` -- section 3.1.4 Eq. (10) masked FM with X^R kept on chip for all
    candidates of a request, rows written in the aligned layout of section 4.2.4
    (:func:`rocs_align_cols`, :func:`rocs_pad_cols`).
  * :func:`rocs_dca_forward` -- section 3.2 Eq. (13) candidate cross attention over K/V
    stored once per request (section 4.3).
  * :func:`rocs_dca_block_forward` -- both query groups of Eq. (13) with the K/V projections
    done once per request (section 4.1).
  * :func:`rocs_lcb_forward_host` / :func:`rocs_dca_forward_host` -- the same on batches in pinned
    host memory, copies and compute pipelined over request chunks.
  * :func:`rocs_proj_forward` -- linear query projection of the chained block (Eq. 12).
  * :func:`rocs_chain_split_forward` / :func:`chain_split_forward` -- the chain with the projection
    split over the IKBO decomposition (request term once per request, W_q folded with W_CC by
    :func:`rocs_chain_prepare_weights`), so Y^C is never written.
"""
from ._binding import (  # noqa: F401
    ROCS_BF16,
    ROCS_F32,
    RocsError,
    chain_forward,
    chain_split_forward,
    last_launch_count,
    lib_path,
    load_library,
    offsets,
    rocs_align_cols,
    rocs_chain_prepare_weights,
    rocs_chain_split_forward,
    rocs_dca_block_forward,
    rocs_dca_forward,
    rocs_dca_forward_expand,
    rocs_dca_forward_host,
    rocs_fm_forward,
    rocs_lcb_block_forward,
    rocs_lcb_block_forward_fault_injection,
    rocs_lcb_forward,
    rocs_lcb_forward_expand,
    rocs_lcb_forward_fault_injection,
    rocs_lcb_forward_host,
    rocs_lcb_forward_noalloc,
    rocs_lcb_noalloc_read_status,
    rocs_pad_cols,
    rocs_proj_forward,
    rocs_read_status,
    STATUS_NAMES,
)
