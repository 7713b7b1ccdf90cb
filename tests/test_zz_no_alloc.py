"""rocs_lcb_forward_noalloc: IKBO-LCB for callers that cannot allocate device memory.

Such callers (a plugin in a serving process whose device memory is fully reserved by the host
framework's pool, or a path on which cudaMalloc is not allowed) cannot pass a workspace; this
entry point keeps its scratch in a fixed device array declared by the library.  The test calls it
through the C ABI twice in a row with different shapes (the shared array must be reset correctly
between calls) and compares each result with rocs_lcb_forward, which uses a caller workspace, at
the bf16 tolerance used by the other parity tests.  This file is named so that pytest collects it
last; it also runs on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


def _noalloc_call(ikbo, x):
    """Call rocs_lcb_forward_noalloc through the C ABI with caller-owned outputs."""
    from attention_ikbo_b200 import _binding as b

    lib = ikbo.load_library()
    ins = [dev(t) for t in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    y_req = torch.full((x.R, x.o_r, x.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    y_cand = torch.full((x.C, x.o_c, x.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    args, keep, _, _ = b._lcb_args(*ins, x.cand_off, y_req, y_cand)
    args.workspace, args.workspace_bytes = None, 0
    rc = lib.rocs_lcb_forward_noalloc(ctypes.byref(args), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, ikbo.STATUS_NAMES.get(rc, rc)
    torch.cuda.synchronize()
    return ins, y_req, y_cand


def test_noalloc_matches_workspace_entry_point_twice():
    import attention_ikbo_b200 as ikbo

    cases = [ri.make_lcb("a", [3, 0, 150, 1, 0, 40], 256, 64, 128, 128, 128, 61, "bf16"),
             ri.make_lcb("b", ri.uniform_int(62, 1, 0, 60, 64), 256, 64, 128, 128, 128, 62, "bf16")]
    for x in cases:
        ins, y_req, y_cand = _noalloc_call(ikbo, x)
        ref_req, ref_cand = ikbo.rocs_lcb_forward(*ins, x.cand_off)
        code, detail = ikbo.rocs_read_status(ikbo.rocs_lcb_forward.last_workspace)
        assert code == 0, (code, detail)
        assert_close(host_f64(y_req), host_f64(ref_req), "bf16", "Y^R (no-alloc vs workspace)")
        assert_close(host_f64(y_cand), host_f64(ref_cand), "bf16", "Y^C (no-alloc vs workspace)")


def test_noalloc_rejects_sizes_beyond_its_array():
    import attention_ikbo_b200 as ikbo
    from attention_ikbo_b200 import _binding as b

    lib = ikbo.load_library()
    R = 200  # 200 x 64 KiB of fp32 Z exceeds the 8 MiB array
    x = ri.make_lcb("big", [1] * R, 64, 64, 128, 128, 128, 63, "bf16")
    ins = [dev(t) for t in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    args, keep, _, _ = b._lcb_args(*ins, x.cand_off, None, None)
    rc = lib.rocs_lcb_forward_noalloc(ctypes.byref(args), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 6  # ROCS_ERR_WORKSPACE
