"""DCA block on the GPU (both query groups of ROCS section 3.2, Eq. (13)): K/V projections once per
request (section 4.1), IKBO-DCA for the candidates, attention of every request's own queries;
against the block oracle, which projects a per-candidate copy of the request sequence."""
import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


def run_block(ikbo, b):
    o_c, lse_c, o_r, lse_r = ikbo.rocs_dca_block_forward(dev(b.s_seq), dev(b.w_kv), dev(b.q_c), dev(b.q_r),
                                                         b.cand_off, b.seq_off, b.q, b.q_req, b.scale)
    code, detail = ikbo.rocs_read_status(ikbo.rocs_dca_block_forward.last_workspace)
    assert code == 0, (code, detail)
    return o_c, lse_c, o_r, lse_r


def check(oracle_mod, b, outs, sel_c=None):
    o_c, lse_c, o_r, lse_r = outs
    sel_c = np.arange(b.C) if sel_c is None else np.asarray(sel_c)
    wkc, wvc, wkr, wvr = b.weights()
    oc, lc, orr, lr = oracle_mod.dca_block(b.cand_off, b.seq_off, b.s_seq, wkc, wvc, wkr, wvr, b.q_c, b.q_r, b.q,
                                           b.q_req, b.scale, sel_cand=sel_c)
    rows = (sel_c[:, None] * b.q + np.arange(b.q)[None, :]).ravel()
    if len(rows):
        assert_close(host_f64(o_c[torch.as_tensor(rows, device=o_c.device)]).reshape(oc.shape), oc, "bf16", "A^C")
    assert_close(host_f64(o_r).reshape(orr.shape), orr, "bf16", "A^R")
    fin = np.isfinite(lr)
    assert_close(host_f64(lse_r).reshape(lr.shape)[fin], lr[fin], "bf16", "LSE^R")


@pytest.mark.parametrize("counts,lengths,q,q_req,H,dh,d_s", [
    ([3, 0, 40, 7], [200, 33, 129, 0], 2, 3, 2, 128, 64),
    ([130, 2], [700, 64], 1, 5, 4, 64, 128),
])
def test_dca_block_small(oracle_mod, counts, lengths, q, q_req, H, dh, d_s):
    import attention_ikbo_b200 as ikbo

    b = ri.make_dca_block("t", counts, lengths, q, q_req, H, dh, d_s, 71 + H)
    check(oracle_mod, b, run_block(ikbo, b))


def test_dca_block_full_size_sampled(oracle_mod):
    """R=8, L_r~U{4096..8192}, d_s=256, H=4, dh=128, 2048 candidates x q=4, 64 request queries."""
    import attention_ikbo_b200 as ikbo

    b = ri.dca_block()
    rs = np.random.RandomState(5)
    sel = np.sort(rs.choice(b.C, 12, replace=False))
    check(oracle_mod, b, run_block(ikbo, b), sel_c=sel)
