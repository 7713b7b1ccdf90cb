"""Seeded random configurations of the LCB, DCA and FM against the fp64 oracle.

Shapes, CSR offsets (empty requests and candidate-free requests included), key lengths and token counts are
drawn from a fixed generator; each case checks every request output and a sample of candidate outputs
(the sampled rows include the first and last candidate, where tiles and requests begin and end).
Operations: ROCS (arXiv:2607.27744) section 3.1.2 Eq. (6) / section 4.1 Eq. (14) for the LCB, section 3.2
Eq. (13) for the DCA, section 3.1.4 Eq. (10) for the FM.
"""
import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ikbo():
    import attention_ikbo_b200 as m

    m.load_library()
    return m


def _status_ok(ikbo, ws):
    code, detail = ikbo.rocs_read_status(ws)
    assert code == 0, f"device status {ikbo.STATUS_NAMES.get(code)} at {detail}"


def _sample(rng, C, n):
    if C <= n:
        return np.arange(C)
    return np.unique(np.concatenate([[0, C - 1], rng.choice(C, n - 2, replace=False)]))


def _counts(rng, R, hi):
    c = rng.integers(0, hi + 1, R)
    c[rng.random(R) < 0.2] = 0
    return c


LCB_CASES = list(range(24))


@pytest.mark.parametrize("case", LCB_CASES)
def test_lcb_random(ikbo, oracle_mod, case):
    rng = np.random.default_rng(1000 + case)
    R = int(rng.integers(1, 6))
    n_r = int(rng.choice([64, 128, 192, 256]))
    n_c, d, o_r = int(rng.choice([64, 128])), int(rng.choice([64, 128])), int(rng.choice([128, 256]))
    x = ri.make_lcb("fuzz", _counts(rng, R, 40), n_r, n_c, d, o_r, 128, 50 + case, "bf16")
    args = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    y_req, y_cand = ikbo.rocs_lcb_forward(*args, x.cand_off)
    _status_ok(ikbo, ikbo.rocs_lcb_forward.last_workspace)
    sel = _sample(rng, x.C, 24)
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_req=np.arange(x.R), sel_cand=sel)
    assert_close(host_f64(y_req), yr, "bf16", "Y^R")
    if len(sel):
        assert_close(host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)]), yc, "bf16", "Y^C")


DCA_CASES = list(range(32))


@pytest.mark.parametrize("case", DCA_CASES)
def test_dca_random(ikbo, oracle_mod, case):
    rng = np.random.default_rng(2000 + case)
    R = int(rng.integers(1, 6))
    counts = _counts(rng, R, 300)
    lengths = rng.integers(0, 900, R)
    lengths[rng.random(R) < 0.15] = 0
    q, H, dh = int(rng.choice([1, 2, 3, 4])), int(rng.choice([1, 2, 4])), int(rng.choice([64, 128]))
    x = ri.make_dca("fuzz", counts, lengths, q, H, dh, 70 + case)
    o, lse = ikbo.rocs_dca_forward(dev(x.q_t), dev(x.k_t), dev(x.v_t), x.cand_off, x.seq_off, x.q, x.scale)
    _status_ok(ikbo, ikbo.rocs_dca_forward.last_workspace)
    sel = _sample(rng, x.C, 32)
    if not len(sel):
        return
    oo, ll = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, x.v_t, x.q, x.scale, sel_cand=sel)
    rows = torch.as_tensor((sel[:, None] * x.q + np.arange(x.q)[None, :]).ravel(), device=o.device)
    assert_close(host_f64(o[rows]).reshape(oo.shape), oo, "bf16", "O")
    got_l = host_f64(lse[rows]).reshape(ll.shape)
    fin = np.isfinite(ll)
    assert np.array_equal(np.isfinite(got_l), fin) and np.all(got_l[~fin] == -np.inf)
    if fin.any():
        assert_close(got_l[fin], ll[fin], "bf16", "LSE")


FM_CASES = list(range(24))


@pytest.mark.parametrize("case", FM_CASES)
def test_fm_random(ikbo, oracle_mod, case):
    rng = np.random.default_rng(3000 + case)
    R = int(rng.integers(1, 6))
    n_r = 2 * int(rng.integers(1, 129))
    n_c, d = int(rng.choice([32, 64, 128])), int(rng.choice([64, 128]))
    x = ri.make_fm("fuzz", _counts(rng, R, 50), n_r, n_c, d, 90 + case)
    y_req, y_cand = ikbo.rocs_fm_forward(dev(x.x_req), dev(x.x_cand), x.cand_off)
    _status_ok(ikbo, ikbo.rocs_fm_forward.last_workspace)
    sel = _sample(rng, x.C, 32)
    yr, yc = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand, sel_cand=sel)
    gr = host_f64(y_req)
    assert_close(gr[:, :, :n_r], yr, "bf16", "Y^R")
    assert not np.any(gr[:, :, n_r:])
    if len(sel):
        gc = host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)])
        assert_close(gc[:, :, :n_r + n_c], yc, "bf16", "Y^C")
        assert not np.any(gc[:, :, n_r + n_c:])


BLOCK_CASES = list(range(16))


def _epi_dev(e):
    out = {"eps": e.eps, "norm": e.norm, "act": e.act}
    for k in ("bias", "gamma", "beta", "residual"):
        v = getattr(e, k)
        if v is not None:
            out[k] = dev(v)
    return out


@pytest.mark.parametrize("case", BLOCK_CASES)
def test_lcb_block_random(ikbo, oracle_mod, case):
    """LCB block (section 3.1.3 Eq. (7)-(8) epilogues): each group's norm and activation drawn independently."""
    rng = np.random.default_rng(4000 + case)
    R = int(rng.integers(1, 5))
    n_r = int(rng.choice([64, 128, 256]))
    n_c, d, o_r = int(rng.choice([64, 128])), int(rng.choice([64, 128])), int(rng.choice([128, 256]))
    norms, acts = ["none", "layernorm", "rmsnorm"], ["none", "relu", "silu", "gelu"]
    x = ri.make_lcb_block("fuzz", _counts(rng, R, 30), n_r, n_c, d, o_r, 128, 110 + case,
                          str(rng.choice(norms)), str(rng.choice(acts)), residual=bool(rng.random() < 0.6),
                          norm_r=str(rng.choice(norms)), act_r=str(rng.choice(acts)))
    L = x.lcb
    args = [dev(a) for a in (L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc)]
    y_req, y_cand = ikbo.rocs_lcb_block_forward(*args, L.cand_off, _epi_dev(x.epi_r), _epi_dev(x.epi_c))
    _status_ok(ikbo, ikbo.rocs_lcb_block_forward.last_workspace)
    sel = _sample(rng, L.C, 24)
    yr, yc = oracle_mod.lcb_block(L.cand_off, L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc, x.epi_r, x.epi_c, sel_cand=sel)
    assert_close(host_f64(y_req), yr, "bf16", "Y^R")
    if len(sel):
        assert_close(host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)]), yc, "bf16", "Y^C")


def test_many_small_requests(ikbo, oracle_mod):
    """3,000 requests of 0-3 candidates (more requests than the scheduling kernels' 1,024 threads): the LCB,
    FM and DCA tile tables and request lookups across thread partitions, checked on sampled candidates."""
    rng = np.random.default_rng(5000)
    counts = rng.integers(0, 4, 3000)
    x = ri.make_lcb("many", counts, 64, 64, 64, 128, 128, 131, "bf16")
    args = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    y_req, y_cand = ikbo.rocs_lcb_forward(*args, x.cand_off)
    _status_ok(ikbo, ikbo.rocs_lcb_forward.last_workspace)
    sel = _sample(rng, x.C, 48)
    sel_req = np.unique(np.concatenate([[0, x.R - 1], rng.choice(x.R, 30, replace=False)]))
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_req=sel_req, sel_cand=sel)
    assert_close(host_f64(y_req[torch.as_tensor(sel_req, device=y_req.device)]), yr, "bf16", "Y^R")
    assert_close(host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)]), yc, "bf16", "Y^C")

    f = ri.make_fm("many", counts, 34, 32, 64, 132)
    fr, fc = ikbo.rocs_fm_forward(dev(f.x_req), dev(f.x_cand), f.cand_off)
    _status_ok(ikbo, ikbo.rocs_fm_forward.last_workspace)
    yr, yc = oracle_mod.fm(f.cand_off, f.x_req, f.x_cand, sel_cand=sel)
    assert_close(host_f64(fr)[:, :, :34], yr, "bf16", "FM Y^R")
    assert_close(host_f64(fc[torch.as_tensor(sel, device=fc.device)])[:, :, :66], yc, "bf16", "FM Y^C")

    lengths = rng.integers(0, 200, 3000)
    d = ri.make_dca("many", counts, lengths, 2, 2, 64, 133)
    o, lse = ikbo.rocs_dca_forward(dev(d.q_t), dev(d.k_t), dev(d.v_t), d.cand_off, d.seq_off, d.q, d.scale)
    _status_ok(ikbo, ikbo.rocs_dca_forward.last_workspace)
    oo, ll = oracle_mod.dca(d.cand_off, d.seq_off, d.q_t, d.k_t, d.v_t, d.q, d.scale, sel_cand=sel)
    rows = torch.as_tensor((sel[:, None] * d.q + np.arange(d.q)[None, :]).ravel(), device=o.device)
    assert_close(host_f64(o[rows]).reshape(oo.shape), oo, "bf16", "DCA O")
    got_l = host_f64(lse[rows]).reshape(ll.shape)
    fin = np.isfinite(ll)
    assert np.array_equal(np.isfinite(got_l), fin)
    if fin.any():
        assert_close(got_l[fin], ll[fin], "bf16", "DCA LSE")


def test_dca_very_many_requests(ikbo, oracle_mod):
    """More requests than the scheduling kernel ranks by key length (9,000): the unit table keeps request
    order; sampled candidates against the oracle."""
    rng = np.random.default_rng(5001)
    counts, lengths = rng.integers(0, 3, 9000), rng.integers(0, 160, 9000)
    d = ri.make_dca("vmany", counts, lengths, 1, 1, 128, 134)
    o, lse = ikbo.rocs_dca_forward(dev(d.q_t), dev(d.k_t), dev(d.v_t), d.cand_off, d.seq_off, d.q, d.scale)
    _status_ok(ikbo, ikbo.rocs_dca_forward.last_workspace)
    sel = _sample(rng, d.C, 48)
    oo, ll = oracle_mod.dca(d.cand_off, d.seq_off, d.q_t, d.k_t, d.v_t, d.q, d.scale, sel_cand=sel)
    rows = torch.as_tensor(sel, device=o.device)
    assert_close(host_f64(o[rows]).reshape(oo.shape), oo, "bf16", "O")
    got_l = host_f64(lse[rows]).reshape(ll.shape)
    fin = np.isfinite(ll)
    assert np.array_equal(np.isfinite(got_l), fin)
    if fin.any():
        assert_close(got_l[fin], ll[fin], "bf16", "LSE")
