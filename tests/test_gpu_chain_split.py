"""The split chain on the GPU vs the oracle: the query projection distributed over the IKBO
decomposition (ROCS, arXiv:2607.27744, section 3.2 Eq. (12) with section 4.1 Eq. (14)):
Q_i = W_q vec(Z_{m_i}) + W_fold vec(X^C_i), so Y^C is never written.  Its definition is the chain on
the exact LCB output (oracle chain with round_y=False).
"""
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


def run_split(ikbo, ci):
    x = ci.lcb
    w_fold, w_rs = ikbo.rocs_chain_prepare_weights(dev(ci.w_q), dev(x.w_rr), dev(x.w_cr), dev(x.w_cc), x.d)
    y_req, q, o, lse = ikbo.chain_split_forward(dev(x.x_req), dev(x.x_cand), w_rs, dev(ci.w_q), w_fold, x.cand_off,
                                                x.o_r, dev(ci.k_t), dev(ci.v_t), ci.seq_off, ci.H, ci.dh, ci.scale)
    code, detail = ikbo.rocs_read_status(ikbo.rocs_chain_split_forward.last_workspace)
    assert code == 0, (ikbo.STATUS_NAMES.get(code), detail)
    return w_fold, w_rs, y_req, q, o, lse


def check(oracle_mod, ci, y_req, q, o, lse, sel):
    x = ci.lcb
    yr, _ = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_cand=[])
    z, _ = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_cr, x.w_cr, x.w_cc, sel_cand=[])  # W_CR X^R
    g = host_f64(y_req)
    assert_close(g[:, :x.o_r], yr, "bf16", "Y^R")
    assert_close(g[:, x.o_r:], z, "bf16", "Z")
    _, qo, oo, ll = oracle_mod.chain(ci, sel, round_y=False)
    idx = torch.as_tensor(sel, device=q.device)
    assert_close(host_f64(q[idx]), qo, "bf16", "Q")
    assert_close(host_f64(o[idx]).reshape(oo.shape), oo, "bf16", "O")
    assert_close(host_f64(lse[idx]).reshape(ll.shape), ll, "bf16", "LSE")


def test_prepare_weights(ikbo, oracle_mod):
    ci = ri.chain(seed=57, R=2, median=4, sigma=0.5, clip=(1, 8), Llo=1, Lhi=8)
    x = ci.lcb
    w_fold, w_rs = ikbo.rocs_chain_prepare_weights(dev(ci.w_q), dev(x.w_rr), dev(x.w_cr), dev(x.w_cc), x.d)
    assert_close(host_f64(w_fold), oracle_mod.chain_fold(ci.w_q, x.w_cc, x.d), "bf16", "W_fold")
    assert np.array_equal(bits(w_rs), np.concatenate([x.w_rr, x.w_cr]))


def test_split_chain_small(ikbo, oracle_mod):
    ci = ri.chain(seed=56, R=6, median=60, sigma=1.0, clip=(1, 400), Llo=1, Lhi=600)
    ci.lcb.cand_off[2:] = ci.lcb.cand_off[2:] - (ci.lcb.cand_off[2] - ci.lcb.cand_off[1])  # request 1 empty
    ci.lcb.x_cand = ci.lcb.x_cand[:int(ci.lcb.cand_off[-1])]
    _, _, y_req, q, o, lse = run_split(ikbo, ci)
    check(oracle_mod, ci, y_req, q, o, lse, np.arange(ci.lcb.C))


def test_split_chain_full_size_sampled(ikbo, oracle_mod):
    """The chain workload at full size (C ~ 1e5 candidates) in the bench's launch configuration:
    request outputs in full, a seeded sample of candidates."""
    ci = ri.chain()
    _, _, y_req, q, o, lse = run_split(ikbo, ci)
    # 520 random candidates plus the first and last of every request (about 0.75 % of ~100k)
    off = np.asarray(ci.lcb.cand_off).astype(np.int64)
    ends = [c for r in range(ci.lcb.R) if off[r + 1] > off[r] for c in (off[r], off[r + 1] - 1)]
    sel = np.unique(np.concatenate([ri.uniform_int(19, 1, 0, ci.lcb.C - 1, 520).astype(np.int64), ends]))
    assert len(sel) >= 0.005 * ci.lcb.C
    check(oracle_mod, ci, y_req, q, o, lse, sel)
