"""Host-resident batches: IKBO-LCB and IKBO-DCA with pinned host inputs/outputs, copies and compute
pipelined over request chunks.  Each chunk runs the device kernels on chunk-local offsets, so the
outputs must equal the device entry points' bit for bit, for any chunking (and the oracle within the
bf16 tolerance)."""
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


def pinned(a):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
        else torch.from_numpy(np.ascontiguousarray(a))
    return t.pin_memory()


@pytest.mark.parametrize("chunks", [1, 3, 64])
def test_lcb_host_matches_device_bitwise(ikbo, oracle_mod, chunks):
    x = ri.make_lcb("t", [3, 0, 170, 1, 40, 0, 9, 77], 256, 64, 128, 128, 128, 71, "bf16")
    w = [dev(a) for a in (x.w_rr, x.w_cr, x.w_cc)]
    yr_d, yc_d = ikbo.rocs_lcb_forward(dev(x.x_req), dev(x.x_cand), *w, x.cand_off)
    yr_h, yc_h = ikbo.rocs_lcb_forward_host(pinned(x.x_req), pinned(x.x_cand), *w, x.cand_off, chunks=chunks)
    torch.cuda.synchronize()
    code, detail = ikbo.rocs_read_status(ikbo.rocs_lcb_forward_host.last_staging)
    assert code == 0, (code, detail)
    assert np.array_equal(bits(yr_h), bits(yr_d)) and np.array_equal(bits(yc_h), bits(yc_d))
    sel = np.array([0, 3, 100, 172, 173, 200, 260, x.C - 1])
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_cand=sel)
    assert_close(host_f64(yc_h[torch.as_tensor(sel)]), yc, "bf16", "Y^C")
    assert_close(host_f64(yr_h), yr, "bf16", "Y^R")


def test_lcb_host_fp32(ikbo):
    x = ri.make_lcb("t", [0, 5, 1, 0, 9], 12, 7, 20, 3, 5, 21, "f32")
    w = [dev(a) for a in (x.w_rr, x.w_cr, x.w_cc)]
    yr_d, yc_d = ikbo.rocs_lcb_forward(dev(x.x_req), dev(x.x_cand), *w, x.cand_off)
    yr_h, yc_h = ikbo.rocs_lcb_forward_host(pinned(x.x_req), pinned(x.x_cand), *w, x.cand_off, chunks=2)
    torch.cuda.synchronize()
    assert torch.equal(yr_h, yr_d.cpu()) and torch.equal(yc_h, yc_d.cpu())


@pytest.mark.parametrize("chunks", [1, 2, 5])
def test_dca_host_matches_device_bitwise(ikbo, oracle_mod, chunks):
    x = ri.make_dca("t", [40, 0, 300, 7, 129], [500, 9, 0, 1300, 257], 2, 4, 128, 72)
    o_d, l_d = ikbo.rocs_dca_forward(dev(x.q_t), dev(x.k_t), dev(x.v_t), x.cand_off, x.seq_off, x.q, x.scale)
    o_h, l_h = ikbo.rocs_dca_forward_host(pinned(x.q_t), pinned(x.k_t), pinned(x.v_t), x.cand_off, x.seq_off, x.q,
                                          x.scale, chunks=chunks)
    torch.cuda.synchronize()
    code, detail = ikbo.rocs_read_status(ikbo.rocs_dca_forward_host.last_staging)
    assert code == 0, (code, detail)
    assert np.array_equal(bits(o_h), bits(o_d))
    assert torch.equal(l_h, l_d.cpu())
    sel = np.array([0, 39, 40, 200, 339, 346, x.C - 1])
    oo, ll = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, x.v_t, x.q, x.scale, sel_cand=sel)
    rows = torch.as_tensor((sel[:, None] * x.q + np.arange(x.q)).ravel())
    assert_close(host_f64(o_h[rows]).reshape(oo.shape), oo, "bf16", "O")


def test_host_calls_back_to_back_on_one_stream(ikbo):
    """Two calls share the library's staging streams: the second must not overwrite the first's slots
    before its outputs have landed."""
    a = ri.make_lcb("a", [50, 60, 70], 256, 64, 128, 128, 128, 73, "bf16")
    b = ri.make_lcb("b", [60, 50], 256, 64, 128, 128, 128, 74, "bf16")  # fits a's staging
    outs, staging = [], None
    for x in (a, b):  # the second call reuses the first call's staging slots
        w = [dev(t) for t in (x.w_rr, x.w_cr, x.w_cc)]
        outs.append((x, w, ikbo.rocs_lcb_forward_host(pinned(x.x_req), pinned(x.x_cand), *w, x.cand_off, chunks=3,
                                                      staging=staging)))
        staging = ikbo.rocs_lcb_forward_host.last_staging
    torch.cuda.synchronize()
    for x, w, (yr_h, yc_h) in outs:
        yr_d, yc_d = ikbo.rocs_lcb_forward(dev(x.x_req), dev(x.x_cand), *w, x.cand_off)
        assert np.array_equal(bits(yc_h), bits(yc_d)) and np.array_equal(bits(yr_h), bits(yr_d))
