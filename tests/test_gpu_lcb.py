"""IKBO-LCB on the GPU (through the C ABI) against the fp64 oracle.

Operation: ROCS (arXiv:2607.27744), section 3.1.2 Eq. (6), executed as the section 4.1
Eq. (14) decomposition with the broadcast-add fused in the candidate GEMM epilogue.
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


def run_lcb(ikbo, x, expand=False):
    args = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    y_req, y_cand = ikbo.rocs_lcb_forward(*args, x.cand_off, expand=expand)
    ws = ikbo.rocs_lcb_forward.last_workspace
    code, detail = ikbo.rocs_read_status(ws)
    assert code == 0, f"device status {ikbo.STATUS_NAMES.get(code)} at {detail}"
    return y_req, y_cand


def check_against_oracle(oracle_mod, x, y_req, y_cand, kind, sel_cand=None):
    sel_req = np.arange(x.R)
    sel = np.arange(x.C) if sel_cand is None else np.asarray(sel_cand)
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_req=sel_req, sel_cand=sel)
    assert_close(host_f64(y_req), yr, kind, "Y^R")
    got = host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)]) if len(sel) else np.zeros_like(yc)
    assert_close(got, yc, kind, "Y^C")


def test_lcb_tiny_f32(ikbo, oracle_mod):
    x = ri.lcb_tiny_f32()
    y_req, y_cand = run_lcb(ikbo, x)
    check_against_oracle(oracle_mod, x, y_req, y_cand, "f32")


def test_lcb_f32_ragged(ikbo, oracle_mod):
    x = ri.make_lcb("t", [0, 5, 1, 0, 9], 12, 7, 20, 3, 5, 21, "f32")
    y_req, y_cand = run_lcb(ikbo, x)
    check_against_oracle(oracle_mod, x, y_req, y_cand, "f32")


SHAPES = [  # (counts, n_r, n_c, d, o_r)
    ([3, 0, 17, 1, 40], 256, 64, 128, 128),
    ([1, 2, 300, 0, 5, 77], 512, 128, 128, 128),
    ([9, 33, 0, 2], 64, 64, 64, 256),
    ([150, 151], 128, 128, 64, 128),
]


@pytest.mark.parametrize("counts,n_r,n_c,d,o_r", SHAPES)
def test_lcb_bf16_small(ikbo, oracle_mod, counts, n_r, n_c, d, o_r):
    x = ri.make_lcb("t", counts, n_r, n_c, d, o_r, 128, 31 + n_r + n_c + d, "bf16")
    y_req, y_cand = run_lcb(ikbo, x)
    check_against_oracle(oracle_mod, x, y_req, y_cand, "bf16")


def test_lcb_bf16_many_ctas(ikbo, oracle_mod):
    """More candidates than CTAs: every CTA takes a range, requests straddle ranges."""
    counts = ri.uniform_int(7, 1, 0, 40, 37)
    x = ri.make_lcb("t", counts, 256, 64, 128, 128, 128, 77, "bf16")
    y_req, y_cand = run_lcb(ikbo, x)
    check_against_oracle(oracle_mod, x, y_req, y_cand, "bf16")


def test_lcb_index_probe_bit_exact(ikbo):
    """W_CC = 0, W_CR selects input row 0, X^R_r == r  ->  Y^C_i == m_i exactly (CSR handling)."""
    counts = [3, 0, 200, 1, 0, 57, 2]
    x = ri.make_lcb("t", counts, 128, 64, 128, 128, 128, 5, "bf16")
    R = x.R
    x_req = np.broadcast_to(np.arange(R, dtype=np.float32)[:, None, None], x.x_req.shape)
    x.x_req = (np.ascontiguousarray(x_req).view(np.uint32) >> 16).astype(np.uint16)
    w_cr = np.zeros((128, 128), np.float32)
    w_cr[:, 0] = 1.0
    x.w_cr = (w_cr.view(np.uint32) >> 16).astype(np.uint16)
    x.w_cc = np.zeros_like(x.w_cc)
    _, y_cand = run_lcb(ikbo, x)
    m = np.repeat(np.arange(R), counts).astype(np.float64)
    assert np.array_equal(host_f64(y_cand), np.broadcast_to(m[:, None, None], y_cand.shape))


def test_lcb_isolation_and_permutation_bitwise(ikbo):
    """Y^R does not change when every X^C changes (Eq. 1/2); permuting candidates within a
    request permutes Y^C bit for bit."""
    x = ri.make_lcb("t", [20, 35, 1], 256, 64, 128, 128, 128, 9, "bf16")
    y_req0, y_cand0 = run_lcb(ikbo, x)
    x2 = ri.make_lcb("t", [20, 35, 1], 256, 64, 128, 128, 128, 9, "bf16")
    x2.x_cand = ri.normal(1234, 2, x.x_cand.shape, 2.0)
    y_req1, _ = run_lcb(ikbo, x2)
    assert np.array_equal(bits(y_req0), bits(y_req1))
    perm = np.concatenate([np.random.RandomState(0).permutation(20), 20 + np.random.RandomState(1).permutation(35), [55]])
    x.x_cand = np.ascontiguousarray(x.x_cand[perm])
    _, y_cand1 = run_lcb(ikbo, x)
    assert np.array_equal(bits(y_cand1), bits(y_cand0)[perm])


def test_lcb_no_candidates(ikbo, oracle_mod):
    x = ri.make_lcb("t", [0, 0, 0], 128, 64, 128, 128, 128, 3, "bf16")
    y_req, y_cand = run_lcb(ikbo, x)
    assert y_cand.shape[0] == 0
    check_against_oracle(oracle_mod, x, y_req, y_cand, "bf16")


def test_lcb_expand_baseline_matches(ikbo, oracle_mod):
    x = ri.make_lcb("t", [5, 0, 12, 3], 256, 64, 128, 128, 128, 44, "bf16")
    y_req, y_cand = run_lcb(ikbo, x, expand=True)
    check_against_oracle(oracle_mod, x, y_req, y_cand, "bf16")
    y_req2, y_cand2 = run_lcb(ikbo, x)
    assert np.array_equal(bits(y_cand), bits(y_cand2)) and np.array_equal(bits(y_req), bits(y_req2))


def _sample(x, n, seed):
    rs = np.random.RandomState(seed)
    sel = set(rs.choice(x.C, size=min(n, x.C), replace=False).tolist())
    for r in range(x.R):  # first and last candidate of every request
        if x.cand_off[r + 1] > x.cand_off[r]:
            sel.update([int(x.cand_off[r]), int(x.cand_off[r + 1]) - 1])
    sel.update([0, x.C - 1])
    return np.array(sorted(sel), dtype=np.int64)


def test_lcb_bf16_full_size_sampled(ikbo, oracle_mod):
    """The full bf16 LCB workload (R=64, N_r~U{256..1024}, n_r=256, n_c=64, d=128) in the
    launch configuration the benchmark times; oracle on sampled candidates."""
    x = ri.lcb_bf16()
    y_req, y_cand = run_lcb(ikbo, x)
    check_against_oracle(oracle_mod, x, y_req, y_cand, "bf16", sel_cand=_sample(x, 256, 1))


def test_lcb_host_validation_errors(ikbo):
    x = ri.make_lcb("t", [2, 2], 128, 64, 128, 128, 128, 3, "bf16")
    args = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    with pytest.raises(ikbo.RocsError) as e:
        ikbo.rocs_lcb_forward(*args, np.array([0, 3, 2], np.int32))
    assert e.value.code == 2
    bad = ri.make_lcb("t", [2, 2], 128, 48, 128, 128, 128, 3, "bf16")  # n_c = 48 is outside the bf16 set
    with pytest.raises(ikbo.RocsError) as e:
        ikbo.rocs_lcb_forward(*[dev(a) for a in (bad.x_req, bad.x_cand, bad.w_rr, bad.w_cr, bad.w_cc)], bad.cand_off)
    assert e.value.code == 3
