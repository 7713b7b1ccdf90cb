"""Edge cases across the entry points: the largest supported shapes, long key sequences, many query
tokens per candidate, no requests at all, requests without candidates, and the unfused chain at full
size.  Each against the fp64 oracle (sampled where the full output is large)."""
import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import assert_close, bits, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ikbo():
    import attention_ikbo_b200 as m

    m.load_library()
    return m


def status_ok(ikbo, ws):
    code, detail = ikbo.rocs_read_status(ws)
    assert code == 0, (ikbo.STATUS_NAMES.get(code), detail)


def test_lcb_widest_shapes(ikbo, oracle_mod):
    """n_r = 2048 (32 request K-blocks), o_r = 512 (four Y^R slices), n_c = 128."""
    x = ri.make_lcb("t", [7, 0, 150, 33], 2048, 128, 128, 512, 128, 81, "bf16")
    args = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    y_req, y_cand = ikbo.rocs_lcb_forward(*args, x.cand_off)
    status_ok(ikbo, ikbo.rocs_lcb_forward.last_workspace)
    sel = np.array([0, 6, 7, 80, 156, 157, 189])
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_cand=sel)
    assert_close(host_f64(y_req), yr, "bf16", "Y^R")
    assert_close(host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)]), yc, "bf16", "Y^C")


def _dca_check(ikbo, oracle_mod, x, sel):
    o, lse = ikbo.rocs_dca_forward(dev(x.q_t), dev(x.k_t), dev(x.v_t), x.cand_off, x.seq_off, x.q, x.scale)
    status_ok(ikbo, ikbo.rocs_dca_forward.last_workspace)
    oo, ll = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, x.v_t, x.q, x.scale, sel_cand=sel)
    rows = torch.as_tensor((np.asarray(sel)[:, None] * x.q + np.arange(x.q)).ravel(), device=o.device)
    assert_close(host_f64(o[rows]).reshape(oo.shape), oo, "bf16", "O")
    assert_close(host_f64(lse[rows]).reshape(ll.shape), ll, "bf16", "LSE")


def test_dca_long_sequence(ikbo, oracle_mod):
    """One request with 65,536 keys (512 K/V tiles) next to a short one."""
    x = ri.make_dca("t", [64, 3], [65536, 100], 2, 2, 128, 82)
    _dca_check(ikbo, oracle_mod, x, [0, 31, 63, 64, 66])


def test_dca_many_query_tokens(ikbo, oracle_mod):
    """q = 16 query tokens per candidate, 16 heads of 64: 128-row tiles hold 8 candidates."""
    x = ri.make_dca("t", [37, 0, 100], [700, 50, 1500], 16, 16, 64, 83)
    _dca_check(ikbo, oracle_mod, x, [0, 18, 36, 37, 90, 136])


def test_no_requests(ikbo):
    """R = 0: every entry point returns without launching anything and without error."""
    off = np.zeros(1, np.int32)
    e = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    lcb = ri.make_lcb("t", [], 256, 64, 128, 128, 128, 1, "bf16")
    w = [dev(a) for a in (lcb.w_rr, lcb.w_cr, lcb.w_cc)]
    y_req, y_cand = ikbo.rocs_lcb_forward(e.view(0, 256, 128), e.view(0, 64, 128), *w, off)
    assert y_req.shape == (0, 128, 128) and y_cand.shape == (0, 128, 128)
    y_req, y_cand = ikbo.rocs_fm_forward(e.view(0, 64, 128), e.view(0, 64, 128), off)
    assert y_req.shape[0] == 0 and y_cand.shape[0] == 0
    o, lse = ikbo.rocs_dca_forward(e.view(0, 2, 128), e.view(0, 2, 128), e.view(0, 2, 128), off, off, 1, 0.1)
    assert o.shape[0] == 0


def test_requests_without_candidates(ikbo, oracle_mod):
    """C = 0 with R > 0: request outputs are still produced (FM, LCB block)."""
    x = ri.make_fm("t", [0, 0, 0], 96, 64, 128, 84)
    y_req, y_cand = ikbo.rocs_fm_forward(dev(x.x_req), dev(x.x_cand), x.cand_off)
    status_ok(ikbo, ikbo.rocs_fm_forward.last_workspace)
    yr, _ = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand)
    assert y_cand.shape[0] == 0
    assert_close(host_f64(y_req)[:, :, :96], yr, "bf16", "Y^R")
    b = ri.make_lcb_block("t", [0, 0], 256, 64, 128, 128, 128, 85)
    L = b.lcb
    ep = lambda e: {"bias": dev(e.bias), "gamma": dev(e.gamma), "beta": dev(e.beta), "residual": dev(e.residual),
                    "eps": e.eps, "norm": e.norm, "act": e.act}
    y_req, y_cand = ikbo.rocs_lcb_block_forward(*[dev(a) for a in (L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc)],
                                                L.cand_off, ep(b.epi_r), None)
    status_ok(ikbo, ikbo.rocs_lcb_block_forward.last_workspace)
    b.epi_c.residual = None
    yr, _ = oracle_mod.lcb_block(L.cand_off, L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc, b.epi_r,
                                 ri.Epilogue(), sel_cand=[])
    assert_close(host_f64(y_req), yr, "bf16", "Y^R")


def test_chain_full_size_sampled(ikbo, oracle_mod):
    """The unfused chain (LCB -> projection -> DCA) on the chain workload, sampled candidates."""
    ci = ri.chain()
    x = ci.lcb
    y_req, y_cand, q, o, lse = ikbo.chain_forward(*[dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)],
                                                  x.cand_off, dev(ci.w_q), dev(ci.k_t), dev(ci.v_t), ci.seq_off,
                                                  ci.H, ci.dh, ci.scale)
    # 520 random candidates plus the first and last of every request (about 0.75 % of ~100k)
    off = np.asarray(x.cand_off).astype(np.int64)
    ends = [c for r in range(x.R) if off[r + 1] > off[r] for c in (off[r], off[r + 1] - 1)]
    sel = np.unique(np.concatenate([ri.uniform_int(23, 1, 0, x.C - 1, 520).astype(np.int64), ends]))
    assert len(sel) >= 0.005 * x.C
    yc, qo, oo, ll = oracle_mod.chain(ci, sel)
    idx = torch.as_tensor(sel, device=q.device)
    assert_close(host_f64(y_cand[idx]), yc, "bf16", "Y^C")
    assert_close(host_f64(o[idx]).reshape(oo.shape), oo, "bf16", "O")
    assert_close(host_f64(lse[idx]).reshape(ll.shape), ll, "bf16", "LSE")


def test_kernel_setup_recorded_for_the_device_used(ikbo, oracle_mod):
    """cudaFuncSetAttribute applies to the current device only: the library records its per-kernel
    set-up per device ordinal.  After launches on this device, its bit is set (and only bits of
    devices this process has used)."""
    import ctypes

    lib = ikbo.load_library()
    lib.rocs_configured_device_mask.restype = ctypes.c_uint64
    x = ri.make_lcb("m", [4, 9], 256, 64, 128, 128, 128, 82, "bf16")
    ikbo.rocs_lcb_forward(*[dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)], x.cand_off)
    status_ok(ikbo, ikbo.rocs_lcb_forward.last_workspace)
    mask = int(lib.rocs_configured_device_mask())
    d = torch.cuda.current_device()
    assert mask & (1 << d), hex(mask)
    assert mask >> torch.cuda.device_count() == 0, hex(mask)
