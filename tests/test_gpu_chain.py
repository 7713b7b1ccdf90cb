"""Projection GEMM and the chained block (LCB -> projection -> DCA) on the GPU vs the oracle.

Chained block: ROCS (arXiv:2607.27744) section 3.2 Eq. (12)-(13): queries generated from
the LCB output by a linear map, then candidate cross attention.
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


@pytest.mark.parametrize("M,N,K", [(300, 256, 512), (129, 1024, 16384), (1, 512, 64)])
def test_proj(ikbo, oracle_mod, M, N, K):
    a = ri.normal(M + N, 1, (M, K))
    w = ri.normal(M + N, 2, (N, K), 1.0 / np.sqrt(K))
    out = ikbo.rocs_proj_forward(dev(a), dev(w))
    code, detail = ikbo.rocs_read_status(ikbo.rocs_proj_forward.last_workspace)
    assert code == 0, (code, detail)
    ref = oracle_mod.proj(a, w)
    assert_close(host_f64(out), ref, "bf16", "proj")


def _small_chain():
    return ri.chain(seed=55, R=5, median=60, sigma=1.0, clip=(1, 400), Llo=1, Lhi=600)


def test_chain_small(ikbo, oracle_mod):
    ci = _small_chain()
    x = ci.lcb
    outs = ikbo.chain_forward(*[dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)], x.cand_off,
                              dev(ci.w_q), dev(ci.k_t), dev(ci.v_t), ci.seq_off, ci.H, ci.dh, ci.scale)
    y_req, y_cand, q, o, lse = outs
    sel = np.arange(x.C)
    yc, qo, oo, ll = oracle_mod.chain(ci, sel)
    assert_close(host_f64(y_cand), yc, "bf16", "Y^C")
    # projection stage on the GPU's own Y^C (isolates the GEMM)
    qref = oracle_mod.proj(bits(y_cand).reshape(x.C, -1), ci.w_q)
    assert_close(host_f64(q), qref, "bf16", "Q")
    assert_close(host_f64(o).reshape(oo.shape), oo, "bf16", "O")
    assert_close(host_f64(lse).reshape(ll.shape), ll, "bf16", "LSE")
