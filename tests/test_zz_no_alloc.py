"""rocs_lcb_forward_noalloc: IKBO-LCB for callers that cannot allocate device memory.

Such callers (a plugin in a serving process whose device memory is fully reserved by the host
framework's pool, or a path on which cudaMalloc is not allowed) cannot pass a workspace; this
entry point keeps its scratch in a fixed device array declared by the library.  The test calls it
through the C ABI twice in a row with different shapes (the shared array must be reset correctly
between calls), reads its device status with rocs_lcb_noalloc_read_status after every call, and
checks each result two ways:
  * bit for bit against rocs_lcb_forward (caller workspace): it is the same kernel with the same
    launch configuration, only the scratch lives elsewhere;
  * against the fp64 oracle (every request output, sampled candidate outputs) at the bf16
    tolerance used by the other parity tests.
This file is named so that pytest collects it last; it also runs on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import assert_close, bits, dev, host_f64

pytestmark = pytest.mark.gpu


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc_call(ikbo, x):
    """Call rocs_lcb_forward_noalloc through the C ABI with caller-owned outputs; return the device
    status read through rocs_lcb_noalloc_read_status (also through the C ABI)."""
    from attention_ikbo_b200 import _binding as b

    lib = ikbo.load_library()
    ins = [dev(t) for t in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    y_req = torch.full((x.R, x.o_r, x.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    y_cand = torch.full((x.C, x.o_c, x.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    args, keep, _, _ = b._lcb_args(*ins, x.cand_off, y_req, y_cand)
    args.workspace, args.workspace_bytes = None, 0
    rc = lib.rocs_lcb_forward_noalloc(ctypes.byref(args), _stream())
    assert rc == 0, ikbo.STATUS_NAMES.get(rc, rc)
    code, detail = ctypes.c_int32(-1), ctypes.c_int32(-1)
    rc = lib.rocs_lcb_noalloc_read_status(_stream(), ctypes.byref(code), ctypes.byref(detail))
    assert rc == 0, ikbo.STATUS_NAMES.get(rc, rc)
    return ins, y_req, y_cand, (code.value, detail.value)


def test_noalloc_matches_workspace_entry_point_and_oracle_twice():
    import attention_ikbo_b200 as ikbo
    import oracle

    cases = [ri.make_lcb("a", [3, 0, 150, 1, 0, 40], 256, 64, 128, 128, 128, 61, "bf16"),
             ri.make_lcb("b", ri.uniform_int(62, 1, 0, 60, 64), 256, 64, 128, 128, 128, 62, "bf16")]
    for k, x in enumerate(cases):
        ins, y_req, y_cand, status = _noalloc_call(ikbo, x)
        assert status[0] == 0, f"case {k}: device status {status}"
        ref_req, ref_cand = ikbo.rocs_lcb_forward(*ins, x.cand_off)
        code, detail = ikbo.rocs_read_status(ikbo.rocs_lcb_forward.last_workspace)
        assert code == 0, (code, detail)
        # same kernel, same launch configuration: identical bits
        assert np.array_equal(bits(y_req), bits(ref_req)), f"case {k}: Y^R differs from rocs_lcb_forward"
        assert np.array_equal(bits(y_cand), bits(ref_cand)), f"case {k}: Y^C differs from rocs_lcb_forward"
        # and the oracle: every request, the first and last candidate of each request plus a random sample
        off = np.asarray(x.cand_off)
        rng = np.random.default_rng(100 + k)
        ends = [c for r in range(x.R) if off[r + 1] > off[r] for c in (off[r], off[r + 1] - 1)]
        sel = np.unique(np.concatenate([ends, rng.choice(x.C, size=min(x.C, 48), replace=False)])).astype(np.int64)
        o_req, o_cand = oracle.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_cand=sel)
        assert_close(host_f64(y_req), o_req, "bf16", f"case {k}: Y^R (no-alloc vs oracle)")
        assert_close(host_f64(y_cand)[sel], o_cand, "bf16", f"case {k}: Y^C (no-alloc vs oracle)")


def test_noalloc_wrapper_allocates_no_outputs():
    import attention_ikbo_b200 as ikbo

    x = ri.make_lcb("w", [2, 3], 256, 64, 128, 128, 128, 64, "bf16")
    ins = [dev(t) for t in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    with pytest.raises(ikbo.RocsError):
        ikbo.rocs_lcb_forward_noalloc(*ins, x.cand_off, None, None)
    y_req = torch.empty((x.R, x.o_r, x.d), dtype=torch.bfloat16, device="cuda")
    y_cand = torch.empty((x.C, x.o_c, x.d), dtype=torch.bfloat16, device="cuda")
    ikbo.rocs_lcb_forward_noalloc(*ins, ikbo.offsets(x.cand_off), y_req, y_cand)
    assert ikbo.rocs_lcb_noalloc_read_status() == (0, 0)
    ref_req, ref_cand = ikbo.rocs_lcb_forward(*ins, x.cand_off)
    assert np.array_equal(bits(y_req), bits(ref_req)) and np.array_equal(bits(y_cand), bits(ref_cand))


def test_noalloc_rejects_sizes_beyond_its_array():
    import attention_ikbo_b200 as ikbo
    from attention_ikbo_b200 import _binding as b

    lib = ikbo.load_library()
    R = 200  # 200 x 64 KiB of fp32 Z exceeds the 8 MiB array
    x = ri.make_lcb("big", [1] * R, 64, 64, 128, 128, 128, 63, "bf16")
    ins = [dev(t) for t in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    args, keep, _, _ = b._lcb_args(*ins, x.cand_off, None, None)
    rc = lib.rocs_lcb_forward_noalloc(ctypes.byref(args), _stream())
    assert rc == 6  # ROCS_ERR_WORKSPACE
