"""LCB block on the GPU (through the C ABI) against the fp64 oracle.

Operation: ROCS (arXiv:2607.27744), section 3.1.2 Eq. (4)-(6) with the group-local epilogues of
section 3.1.3 Eq. (7)-(8): per output group a bias, a residual merge, LayerNorm/RMSNorm over d and
an activation, fused into the IKBO-LCB kernel's epilogue.
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


def _epi_dev(e):
    if e is None:
        return None
    out = {"eps": e.eps, "norm": e.norm, "act": e.act}
    for k in ("bias", "gamma", "beta", "residual"):
        v = getattr(e, k)
        if v is not None:
            out[k] = dev(v)
    return out


def run_block(ikbo, x, epi_r=True, epi_c=True):
    L = x.lcb
    args = [dev(a) for a in (L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc)]
    y_req, y_cand = ikbo.rocs_lcb_block_forward(*args, L.cand_off, _epi_dev(x.epi_r) if epi_r else None,
                                                _epi_dev(x.epi_c) if epi_c else None)
    code, detail = ikbo.rocs_read_status(ikbo.rocs_lcb_block_forward.last_workspace)
    assert code == 0, f"device status {ikbo.STATUS_NAMES.get(code)} at {detail}"
    return y_req, y_cand


def check(oracle_mod, x, y_req, y_cand, sel_cand=None):
    L = x.lcb
    sel = np.arange(L.C) if sel_cand is None else np.asarray(sel_cand)
    yr, yc = oracle_mod.lcb_block(L.cand_off, L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc, x.epi_r, x.epi_c,
                                  sel_cand=sel)
    assert_close(host_f64(y_req), yr, "bf16", "Y^R")
    got = host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)]) if len(sel) else np.zeros_like(yc)
    assert_close(got, yc, "bf16", "Y^C")


CASES = [  # (counts, n_r, n_c, d, o_r, norm, act, residual)
    ([3, 0, 17, 1, 40], 256, 64, 128, 128, "layernorm", "silu", True),
    ([1, 2, 300, 0, 5, 77], 512, 128, 128, 128, "rmsnorm", "gelu", True),
    ([9, 33, 0, 2], 64, 64, 64, 256, "layernorm", "relu", False),
    ([150, 151], 128, 128, 64, 128, "none", "gelu", True),
    ([0, 0, 4], 64, 64, 128, 128, "rmsnorm", "none", False),
    ([5, 70, 0, 3], 128, 64, 64, 128, "layernorm", "silu", True),
]


@pytest.mark.parametrize("counts,n_r,n_c,d,o_r,norm,act,res", CASES)
def test_lcb_block_small(ikbo, oracle_mod, counts, n_r, n_c, d, o_r, norm, act, res):
    x = ri.make_lcb_block("t", counts, n_r, n_c, d, o_r, 128, 40 + n_r + d, norm, act, residual=res)
    y_req, y_cand = run_block(ikbo, x)
    check(oracle_mod, x, y_req, y_cand)


def test_lcb_block_groups_differ_and_null_affine(ikbo, oracle_mod):
    x = ri.make_lcb_block("t", [5, 0, 70, 3], 128, 64, 128, 256, 128, 9, "layernorm", "relu", residual=True,
                          norm_r="rmsnorm", act_r="silu")
    x.epi_r.gamma = None  # gamma 1
    x.epi_c.beta = None  # beta 0
    x.epi_r.bias = None
    y_req, y_cand = run_block(ikbo, x)
    check(oracle_mod, x, y_req, y_cand)


def test_lcb_block_without_epilogue_equals_lcb(ikbo):
    x = ri.make_lcb_block("t", [4, 0, 90, 11], 256, 64, 128, 128, 128, 3)
    L = x.lcb
    args = [dev(a) for a in (L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc)]
    yr0, yc0 = ikbo.rocs_lcb_forward(*args, L.cand_off)
    yr1, yc1 = ikbo.rocs_lcb_block_forward(*args, L.cand_off, None, None)
    assert np.array_equal(bits(yr0), bits(yr1)) and np.array_equal(bits(yc0), bits(yc1))


def test_lcb_block_isolation_bitwise(ikbo):
    """Eq. (1)/(11): candidate inputs (X^C, the candidate residual, gamma^C) never reach Y^R."""
    x = ri.make_lcb_block("t", [6, 1, 40], 128, 64, 128, 128, 128, 8)
    yr0, _ = run_block(ikbo, x)
    x.lcb.x_cand[...] = ri.normal(123, 1, x.lcb.x_cand.shape)
    x.epi_c.residual[...] = ri.normal(123, 2, x.epi_c.residual.shape)
    x.epi_c.gamma[...] = 2.0
    yr1, _ = run_block(ikbo, x)
    assert np.array_equal(bits(yr0), bits(yr1))


def test_lcb_block_full_size_sampled(ikbo, oracle_mod):
    """The bench workload at full size (C = 43,296 candidates), in the bench's launch configuration;
    every request output and a seeded sample of candidates (first/last of each request + random)."""
    x = ri.lcb_block()
    y_req, y_cand = run_block(ikbo, x)
    off = x.lcb.cand_off
    firsts = [int(off[r]) for r in range(x.lcb.R) if off[r + 1] > off[r]]
    lasts = [int(off[r + 1]) - 1 for r in range(x.lcb.R) if off[r + 1] > off[r]]
    rnd = ri.uniform_int(17, 1, 0, x.lcb.C - 1, 64).tolist()
    sel = np.unique(np.array(firsts[::4] + lasts[::4] + rnd, dtype=np.int64))
    check(oracle_mod, x, y_req, y_cand, sel)
