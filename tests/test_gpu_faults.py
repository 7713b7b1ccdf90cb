"""Failure detection without a GPU fault: every device wait in the kernels is bounded.

The LCB kernel's candidate epilogues wait (release/acquire) on a per-request ready flag written by
the request tile that computes Z (ROCS, arXiv:2607.27744, section 4.2.3).  The fault-injection entry
point makes one request tile skip that release -- a flag that nothing sets.  The kernel must end with
ROCS_ERR_TIMEOUT in the status word after the short wait limit (no trap, no hang), and the CUDA
context must stay usable: a normal call right after it is checked against the oracle.
"""
import time

import numpy as np
import pytest

import rocs_inputs as ri
from _helpers import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu

FLAG_WAIT_SITES = {311, 312, 202, 205, 103, 206}  # flag wait, or a role that gave up first in that CTA
BLOCK_WAIT_SITES = FLAG_WAIT_SITES | {313}  # + the residual wait of a staged-residual tile


def test_lcb_missing_release_times_out_and_context_survives(oracle_mod):
    import attention_ikbo_b200 as ikbo

    x = ri.make_lcb("fault", [30, 40, 50, 20], 256, 64, 128, 128, 128, 88, "bf16")
    ins = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    t0 = time.time()
    ws = ikbo.rocs_lcb_forward_fault_injection(*ins, x.cand_off, skip_release_request=2, wait_limit_ns=50_000_000)
    code, detail = ikbo.rocs_read_status(ws)
    elapsed = time.time() - t0
    assert code == 5, ikbo.STATUS_NAMES.get(code)  # ROCS_ERR_TIMEOUT
    assert detail in FLAG_WAIT_SITES, detail
    assert elapsed < 30.0
    # no fault was injected: the same call path completes normally
    ws2 = ikbo.rocs_lcb_forward_fault_injection(*ins, x.cand_off, skip_release_request=-1, wait_limit_ns=50_000_000)
    assert ikbo.rocs_read_status(ws2)[0] == 0
    # the context is still usable and correct
    y_req, y_cand = ikbo.rocs_lcb_forward(*ins, x.cand_off)
    code, detail = ikbo.rocs_read_status(ikbo.rocs_lcb_forward.last_workspace)
    assert code == 0, (code, detail)
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    assert_close(host_f64(y_req), yr, "bf16", "Y^R after the fault test")
    assert_close(host_f64(y_cand), yc, "bf16", "Y^C after the fault test")


def test_lcb_block_missing_release_times_out_and_context_survives(oracle_mod):
    """The same for the LCB block kernel (three warpgroups with a setmaxnreg split, the candidate residual
    accumulated by the tensor core): its candidate epilogues wait on the same flags."""
    import attention_ikbo_b200 as ikbo

    x = ri.make_lcb_block("fault_blk", [30, 40, 50, 20], 256, 64, 128, 128, 128, 89, "layernorm", "silu")
    L = x.lcb
    ins = [dev(a) for a in (L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc)]

    def epi(e):
        out = {"eps": e.eps, "norm": e.norm, "act": e.act}
        for k in ("bias", "gamma", "beta", "residual"):
            if getattr(e, k) is not None:
                out[k] = dev(getattr(e, k))
        return out

    er, ec = epi(x.epi_r), epi(x.epi_c)
    t0 = time.time()
    ws = ikbo.rocs_lcb_block_forward_fault_injection(*ins, L.cand_off, er, ec, skip_release_request=2,
                                                     wait_limit_ns=50_000_000)
    code, detail = ikbo.rocs_read_status(ws)
    elapsed = time.time() - t0
    assert code == 5, ikbo.STATUS_NAMES.get(code)  # ROCS_ERR_TIMEOUT
    assert detail in BLOCK_WAIT_SITES, detail
    assert elapsed < 30.0
    ws2 = ikbo.rocs_lcb_block_forward_fault_injection(*ins, L.cand_off, er, ec, skip_release_request=-1,
                                                      wait_limit_ns=50_000_000)
    assert ikbo.rocs_read_status(ws2)[0] == 0
    y_req, y_cand = ikbo.rocs_lcb_block_forward(*ins, L.cand_off, er, ec)
    code, detail = ikbo.rocs_read_status(ikbo.rocs_lcb_block_forward.last_workspace)
    assert code == 0, (code, detail)
    yr, yc = oracle_mod.lcb_block(L.cand_off, L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc, x.epi_r, x.epi_c,
                                  sel_cand=np.arange(L.C))
    assert_close(host_f64(y_req), yr, "bf16", "Y^R after the fault test")
    assert_close(host_f64(y_cand), yc, "bf16", "Y^C after the fault test")
