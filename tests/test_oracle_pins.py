"""Pins for the fp64 oracle, each against something other than the oracle itself.

Sources (ROCS, arXiv:2607.27744, paper-archivist reading notes):
  Eq. (1)/(2)/(11)  GLM isolation and request-output identity   (section 3.1.1, 3.1.5)
  Eq. (5)/(6)       ROCSified LCB, two-group form              (section 3.1.2)
  Eq. (14)          IKBO decomposition Z = W_CR X^R, Y^C = Z_m + W_CC X^C  (section 4.1)
  Eq. (13)          group-wise cross attention                 (section 3.2)
A planted mistake in the oracle (dropped term, wrong sign/index, transposed
operand, missing max-subtraction or normalisation) fails at least one of these.
"""
import math
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

import rocs_inputs as ri

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *vals = line.split()
            out[k] = [float(v) for v in vals]
    return out


def _f32(a):
    return np.asarray(a, dtype=np.float32)


def _bf16_exact(a):
    """float values exactly representable in bf16 -> bit patterns."""
    f = np.asarray(a, dtype=np.float32)
    b = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(ri.bf16_to_f32(b), f), "value not exact in bf16"
    return b


def _w(x):
    return x if x.dtype == np.float32 else ri.bf16_to_f32(x)


def _rand_lcb(seed, counts, n_r=5, n_c=3, d=7, o_r=4, o_c=6, dtype="f32"):
    return ri.make_lcb("t", counts, n_r, n_c, d, o_r, o_c, seed, dtype)


# ------------------------------------------------------------------------------ LCB
def test_lcb_golden_two_group(oracle_mod):
    g = _read_golden("lcb_two_group.txt")
    for conv in (_f32, _bf16_exact):
        x_req = conv(np.array(g["x_req"]).reshape(1, 2, 2))
        x_cand = conv(np.array(g["x_cand"]).reshape(2, 2, 2))
        w_rr, w_cr, w_cc = (conv(np.array(g[k]).reshape(1, 2)) for k in ("w_rr", "w_cr", "w_cc"))
        yr, yc = oracle_mod.lcb([0, 2], x_req, x_cand, w_rr, w_cr, w_cc)
        assert yr.ravel().tolist() == g["y_req"]
        assert yc.ravel().tolist() == g["y_cand"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lcb_bruteforce_group_sum(oracle_mod, dtype):
    """Eq. (5): Y^(i) = sum_{j<=i} W_ij X^(j), evaluated element by element with exact
    rational arithmetic over the group loop (group 0 = request, group 1 = candidate)."""
    x = _rand_lcb(11, [2, 0, 3], dtype=dtype)
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    XR, XC = _w(x.x_req).astype(np.float64), _w(x.x_cand).astype(np.float64)
    W = {(0, 0): _w(x.w_rr), (1, 0): _w(x.w_cr), (1, 1): _w(x.w_cc)}
    m = [r for r in range(x.R) for _ in range(x.cand_off[r], x.cand_off[r + 1])]
    for r in range(x.R):
        for o in range(x.o_r):
            for c in range(x.d):
                exact = sum(Fraction(float(W[0, 0][o, k])) * Fraction(XR[r, k, c]) for k in range(x.n_r))
                assert abs(yr[r, o, c] - float(exact)) <= 1e-12 * (1 + abs(float(exact)))
    for i in range(x.C):
        groups = [XR[m[i]], XC[i]]
        for o in range(x.o_c):
            for c in range(x.d):
                exact = Fraction(0)
                for j in range(0, 2):  # j <= i for output group i = 1
                    Wij = W[1, j]
                    for k in range(Wij.shape[1]):
                        exact += Fraction(float(Wij[o, k])) * Fraction(groups[j][k, c])
                assert abs(yc[i, o, c] - float(exact)) <= 1e-12 * (1 + abs(float(exact)))


def test_lcb_decomposition_eq14(oracle_mod):
    """IKBO decomposition (Eq. 14) computed with library matmuls equals the materialised Eq. (6)."""
    x = _rand_lcb(5, [4, 1, 0, 6], n_r=9, n_c=5, d=16, o_r=8, o_c=12)
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    XR, XC = _w(x.x_req).astype(np.float64), _w(x.x_cand).astype(np.float64)
    WRR, WCR, WCC = (_w(a).astype(np.float64) for a in (x.w_rr, x.w_cr, x.w_cc))
    stacked = np.concatenate([WRR, WCR], axis=0)  # [W_RR; W_CR] . X^R in one GEMM at batch B_r
    YZ = np.einsum("on,rnd->rod", stacked, XR)
    Y_R, Z = YZ[:, : x.o_r], YZ[:, x.o_r:]
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    Y_C = Z[m] + np.einsum("on,ind->iod", WCC, XC)
    scale = np.abs(Y_C).max()
    assert np.abs(yr - Y_R).max() <= 1e-12 * np.abs(Y_R).max()
    assert np.abs(yc - Y_C).max() <= 1e-12 * scale


def test_lcb_isolation_bitwise(oracle_mod):
    """Eq. (1)/(2): request outputs do not depend on candidate inputs, bit for bit;
    and a candidate's output does not depend on other candidates."""
    x = _rand_lcb(7, [3, 5], n_r=6, n_c=4, d=8, o_r=5, o_c=5)
    yr0, yc0 = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    x2 = ri.normal(99, 1, x.x_cand.shape, 3.0, "f32")
    yr1, yc1 = oracle_mod.lcb(x.cand_off, x.x_req, x2, x.w_rr, x.w_cr, x.w_cc)
    assert np.array_equal(yr0, yr1)
    assert not np.array_equal(yc0, yc1)
    x3 = x.x_cand.copy()
    x3[4] += 1.0  # perturb candidate 4 only
    _, yc3 = oracle_mod.lcb(x.cand_off, x.x_req, x3, x.w_rr, x.w_cr, x.w_cc)
    keep = [i for i in range(x.C) if i != 4]
    assert np.array_equal(yc0[keep], yc3[keep]) and not np.array_equal(yc0[4], yc3[4])


def test_lcb_permutation_within_request(oracle_mod):
    x = _rand_lcb(8, [5, 4], n_r=4, n_c=4, d=8)
    perm = np.array([3, 0, 4, 1, 2, 8, 6, 5, 7])
    _, yc0 = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    _, yc1 = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand[perm], x.w_rr, x.w_cr, x.w_cc)
    assert np.array_equal(yc1, yc0[perm])


def test_lcb_closed_forms(oracle_mod):
    x = _rand_lcb(9, [2, 3], n_r=6, n_c=5, d=4, o_r=3, o_c=4)
    XR, XC = _w(x.x_req).astype(np.float64), _w(x.x_cand).astype(np.float64)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    WCR, WCC = _w(x.w_cr).astype(np.float64), _w(x.w_cc).astype(np.float64)
    # W_CC = 0  ->  Y^C_i = W_CR X^R_{m_i}
    _, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, np.zeros_like(x.w_cc))
    np.testing.assert_allclose(yc, (WCR @ XR)[m], rtol=1e-12, atol=1e-12)
    # W_CR = 0  ->  Y^C_i = W_CC X^C_i
    _, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, np.zeros_like(x.w_cr), x.w_cc)
    np.testing.assert_allclose(yc, WCC @ XC, rtol=1e-12, atol=1e-12)
    # one request -> a textbook GEMM [W_CR W_CC] . [X^R ; X^C_i]
    x1 = _rand_lcb(10, [4], n_r=6, n_c=5, d=4, o_r=3, o_c=4)
    _, yc = oracle_mod.lcb(x1.cand_off, x1.x_req, x1.x_cand, x1.w_rr, x1.w_cr, x1.w_cc)
    Wcat = np.concatenate([_w(x1.w_cr), _w(x1.w_cc)], axis=1).astype(np.float64)
    for i in range(4):
        Xcat = np.concatenate([_w(x1.x_req)[0], _w(x1.x_cand)[i]], axis=0).astype(np.float64)
        np.testing.assert_allclose(yc[i], Wcat @ Xcat, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lcb_index_probe_exact(oracle_mod, dtype):
    """W_CC = 0, W_CR selects input row 0, X^R_r == r  ->  Y^C_i == m_i exactly."""
    counts = [3, 0, 4, 1, 0, 2]
    x = _rand_lcb(12, counts, n_r=4, n_c=3, d=5, o_r=2, o_c=3, dtype=dtype)
    conv = _f32 if dtype == "f32" else _bf16_exact
    x_req = conv(np.broadcast_to(np.arange(x.R, dtype=np.float32)[:, None, None], x.x_req.shape))
    w_cr = np.zeros((x.o_c, x.n_r), np.float32)
    w_cr[:, 0] = 1.0
    _, yc = oracle_mod.lcb(x.cand_off, x_req, x.x_cand, x.w_rr, conv(w_cr), conv(np.zeros((x.o_c, x.n_c))))
    m = np.repeat(np.arange(x.R), counts)
    assert np.array_equal(yc, np.broadcast_to(m[:, None, None].astype(np.float64), yc.shape))


def test_lcb_selection_and_bad_offsets(oracle_mod):
    x = _rand_lcb(13, [2, 3, 1])
    yr, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    yr2, yc2 = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc, sel_req=[2, 0],
                              sel_cand=[5, 1])
    assert np.array_equal(yr2, yr[[2, 0]]) and np.array_equal(yc2, yc[[5, 1]])
    with pytest.raises(oracle_mod.OracleError) as e:
        oracle_mod.lcb(np.array([0, 3, 2, 6]), x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    assert e.value.code == oracle_mod.ORC_BAD_OFFSETS
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.lcb(np.array([1, 3, 5, 6]), x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)


# ------------------------------------------------------------------------------ DCA
def _dca_inputs(seed, counts, lengths, q=2, H=2, dh=8):
    return ri.make_dca("t", counts, lengths, q, H, dh, seed)


def test_dca_golden(oracle_mod):
    g = _read_golden("dca_softmax.txt")
    for case in ("case1", "case2"):
        k = np.array(g[f"{case}_k"])
        L = len(k)
        o, lse = oracle_mod.dca([0, 1], [0, L], _bf16_exact(np.array(g[f"{case}_q"]).reshape(1, 1, 1)),
                                _bf16_exact(k.reshape(L, 1, 1)), _bf16_exact(np.array(g[f"{case}_v"]).reshape(L, 1, 1)),
                                q=1, scale=g[f"{case}_scale"][0])
        assert abs(o.item() - g[f"{case}_o"][0]) <= 1e-12
        assert abs(lse.item() - g[f"{case}_lse"][0]) <= 1e-12


def test_dca_bruteforce_decimal(oracle_mod):
    """Naive softmax attention in 40-digit decimal arithmetic (exact inputs)."""
    getcontext().prec = 40
    x = _dca_inputs(21, [2, 1, 0], [5, 3, 2], q=2, H=2, dh=4)
    o, lse = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, x.v_t, x.q, x.scale)
    Q, K, V = (ri.bf16_to_f32(a).astype(np.float64) for a in (x.q_t, x.k_t, x.v_t))
    sc = Decimal(x.scale)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    for i in range(x.C):
        r = m[i]
        s0, s1 = x.seq_off[r], x.seq_off[r + 1]
        for t in range(x.q):
            for h in range(x.H):
                qv = [Decimal(float(v)) for v in Q[i * x.q + t, h]]
                s = [sc * sum(qv[c] * Decimal(float(K[j, h, c])) for c in range(x.dh)) for j in range(s0, s1)]
                e = [v.exp() for v in s]
                den = sum(e)
                for c in range(x.dh):
                    ref = sum(e[j] * Decimal(float(V[s0 + j, h, c])) for j in range(s1 - s0)) / den
                    assert abs(o[i, t, h, c] - float(ref)) <= 1e-12
                assert abs(lse[i, t, h] - float(den.ln())) <= 1e-12


def test_dca_matches_library_attention(oracle_mod):
    """Per request, DCA is plain non-causal attention of all its candidates' query rows over
    that request's K/V: torch's scaled_dot_product_attention in float64."""
    x = _dca_inputs(22, [3, 2, 4], [17, 9, 33], q=3, H=3, dh=16)
    o, _ = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, x.v_t, x.q, x.scale)
    Q, K, V = (torch.from_numpy(ri.bf16_to_f32(a).astype(np.float64)) for a in (x.q_t, x.k_t, x.v_t))
    for r in range(x.R):
        rows = slice(x.q * x.cand_off[r], x.q * x.cand_off[r + 1])
        keys = slice(x.seq_off[r], x.seq_off[r + 1])
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q[rows].transpose(0, 1), K[keys].transpose(0, 1), V[keys].transpose(0, 1), scale=x.scale)
        got = torch.from_numpy(o[x.cand_off[r]: x.cand_off[r + 1]].reshape(-1, x.H, x.dh)).transpose(0, 1)
        assert torch.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_dca_rows_sum_to_one(oracle_mod):
    """V = one-hot basis (L <= dh): O[:, c] is softmax weight c, so each row sums to 1 and is >= 0."""
    L, dh = 6, 8
    x = _dca_inputs(23, [3], [L], q=2, H=2, dh=dh)
    v = np.zeros((L, 2, dh), np.float32)
    for j in range(L):
        v[j, :, j] = 1.0
    o, _ = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, _bf16_exact(v), x.q, x.scale)
    assert np.all(o >= 0) and np.all(o[..., L:] == 0)
    assert np.abs(o.sum(-1) - 1.0).max() <= 1e-12


def test_dca_closed_forms(oracle_mod):
    x = _dca_inputs(24, [2, 2], [7, 1], q=1, H=1, dh=4)
    Vf = ri.bf16_to_f32(x.v_t).astype(np.float64)
    # all V rows equal -> O = v
    vconst = np.broadcast_to(np.array([1.5, -2.0, 0.25, 3.0], np.float32), x.v_t.shape)
    o, _ = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, _bf16_exact(vconst), 1, x.scale)
    assert np.abs(o - vconst[0, 0]).max() <= 1e-12
    # all K rows equal (zero) -> uniform weights -> O = mean(V_r), LSE = log L_r
    o, lse = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, np.zeros_like(x.k_t), x.v_t, 1, x.scale)
    assert np.abs(o[0, 0, 0] - Vf[0:7, 0].mean(0)).max() <= 1e-12
    assert abs(lse[0, 0, 0] - math.log(7)) <= 1e-12
    # L_r = 1 -> O = V_0 of that request
    assert np.abs(o[2, 0, 0] - Vf[7, 0]).max() <= 1e-12
    assert abs(lse[2, 0, 0] - 0.0) <= 1e-12
    # one dominant score -> O ~ that V row
    k = np.zeros((8, 1, 4), np.float32)
    k[3, 0, 0] = 64.0
    qv = np.zeros((4, 1, 4), np.float32)
    qv[:, 0, 0] = 1.0
    o, _ = oracle_mod.dca(x.cand_off, x.seq_off, _bf16_exact(qv), _bf16_exact(k), x.v_t, 1, 1.0)
    # p_3 = 1 / (1 + 7 e^-64): O equals V_3 far below double precision
    assert np.abs(o[0, 0, 0] - Vf[3, 0]).max() <= 1e-12


def test_dca_index_probe_and_empty(oracle_mod):
    counts, lengths = [2, 3, 1, 2], [4, 0, 2, 5]
    x = _dca_inputs(25, counts, lengths, q=2, H=2, dh=4)
    v = np.zeros(x.v_t.shape, np.float32)
    for r in range(x.R):
        v[x.seq_off[r]: x.seq_off[r + 1]] = r
    o, lse = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, _bf16_exact(v), x.q, x.scale)
    m = np.repeat(np.arange(x.R), counts)
    for i in range(x.C):
        if lengths[m[i]] == 0:
            assert np.all(o[i] == 0) and np.all(np.isneginf(lse[i]))
        else:
            assert np.abs(o[i] - m[i]).max() <= 1e-12


def test_dca_permutation_within_request(oracle_mod):
    x = _dca_inputs(26, [4, 3], [6, 9], q=2, H=2, dh=8)
    o0, l0 = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, x.v_t, x.q, x.scale)
    perm = np.array([2, 0, 3, 1, 6, 4, 5])
    qp = x.q_t.reshape(x.C, x.q, x.H, x.dh)[perm].reshape(x.q_t.shape)
    o1, l1 = oracle_mod.dca(x.cand_off, x.seq_off, qp, x.k_t, x.v_t, x.q, x.scale)
    assert np.array_equal(o1, o0[perm]) and np.array_equal(l1, l0[perm])


# ------------------------------------------------------------------------------ projection / chain
def test_round_bf16(oracle_mod):
    rb = oracle_mod.round_bf16
    one = 1.0
    assert rb(one + 2 ** -8) == one  # tie -> even
    assert rb(one + 3 * 2 ** -8) == one + 2 ** -6  # tie -> even (up)
    assert rb(one + 2 ** -8 + 2 ** -30) == one + 2 ** -7  # above the tie
    assert rb(-(one + 2 ** -8 + 2 ** -30)) == -(one + 2 ** -7)
    assert rb(2 ** -133 * 0.75) == 2 ** -133  # subnormal quantum
    assert rb(2.0 ** 128 * 0.999999) == math.inf
    # values exactly representable in fp32: agree with the fp32 -> bf16 RNE bit rule
    f = ri.normal(3, 9, (2000,), 10.0, "f32")
    u = f.view(np.uint32).astype(np.uint64)
    bits = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    ref = ri.bf16_to_f32(bits).astype(np.float64)
    got = np.array([rb(float(v)) for v in f])
    assert np.array_equal(got, ref)


def test_proj_matches_library_matmul(oracle_mod):
    y = ri.normal(31, 1, (5, 96))
    w = ri.normal(31, 2, (24, 96), 0.1)
    got = oracle_mod.proj(y, w)
    ref = ri.bf16_to_f32(y).astype(np.float64) @ ri.bf16_to_f32(w).astype(np.float64).T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def _small_chain(seed=41):
    return ri.chain(seed=seed, R=3, median=3, sigma=0.5, clip=(1, 6), Llo=1, Lhi=9, H=2, dh=8)


def _shrink_chain(ci):
    """shrink the LCB to n_r=8, n_c=4, d=4, o_r=4, o_c=4 so the oracle runs in milliseconds."""
    counts = np.diff(ci.lcb.cand_off)
    ci.lcb = ri.make_lcb("t", counts, 8, 4, 4, 4, 4, 41)
    ci.w_q = ri.normal(41, ri.S_WQ, (ci.H * ci.dh, 16), 0.25)
    return ci


def test_chain_composes_stages(oracle_mod):
    ci = _shrink_chain(_small_chain())
    x = ci.lcb
    sel = np.arange(x.C)
    y, qo, o, lse = oracle_mod.chain(ci, sel)
    _, yc = oracle_mod.lcb(x.cand_off, x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)
    assert np.array_equal(y, yc)
    yb = np.array([[oracle_mod.round_bf16(v) for v in row] for row in yc.reshape(x.C, -1)])
    ybits = (yb.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    qref = oracle_mod.proj(ybits, ci.w_q)
    assert np.array_equal(qo, qref)
    qb = np.array([[oracle_mod.round_bf16(v) for v in row] for row in qref])
    qbits = (qb.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16).reshape(x.C, ci.H, ci.dh)
    o2, l2 = oracle_mod.dca(x.cand_off, ci.seq_off, qbits, ci.k_t, ci.v_t, 1, ci.scale)
    assert np.array_equal(o, o2[:, 0]) and np.array_equal(lse, l2[:, 0])


def test_chain_zero_projection(oracle_mod):
    """W_q = 0 -> every query is 0 -> uniform attention -> O = mean of the request's V rows."""
    ci = _shrink_chain(_small_chain(43))
    ci.w_q = np.zeros_like(ci.w_q)
    x = ci.lcb
    _, qo, o, _ = oracle_mod.chain(ci, np.arange(x.C))
    assert np.all(qo == 0)
    V = ri.bf16_to_f32(ci.v_t).astype(np.float64)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    for i in range(x.C):
        s0, s1 = ci.seq_off[m[i]], ci.seq_off[m[i] + 1]
        assert np.abs(o[i] - V[s0:s1].mean(0)).max() <= 1e-12


def test_dca_large_scores_stable(oracle_mod):
    """Scores 800 and 796 (exp overflows double without the max shift): weights are
    sigma(4) and 1 - sigma(4) exactly as the softmax definition gives."""
    q = _bf16_exact(np.array([1.0]).reshape(1, 1, 1))
    k = _bf16_exact(np.array([800.0, 796.0]).reshape(2, 1, 1))
    v = _bf16_exact(np.array([1.0, 0.0]).reshape(2, 1, 1))
    o, lse = oracle_mod.dca([0, 1], [0, 2], q, k, v, q=1, scale=1.0)
    w0 = 1.0 / (1.0 + math.exp(-4.0))
    assert abs(o.item() - w0) <= 1e-12
    assert abs(lse.item() - (800.0 + math.log1p(math.exp(-4.0)))) <= 1e-12


# ------------------------------------------------------------------------------ DCA block (both groups)
def _block_inputs(seed, counts, lengths, q=2, q_req=3, H=2, dh=8, d_s=16):
    coff, soff = ri.counts_to_offsets(counts), ri.counts_to_offsets(lengths)
    R, C, T = len(counts), int(coff[-1]), int(soff[-1])
    g = lambda stream, shape, std=1.0: ri.normal(seed, stream, shape, std)
    return dict(cand_off=coff, seq_off=soff, s_seq=g(40, (T, d_s)), w_kc=g(41, (H * dh, d_s), 0.25),
                w_vc=g(42, (H * dh, d_s), 0.25), w_kr=g(43, (H * dh, d_s), 0.25), w_vr=g(44, (H * dh, d_s), 0.25),
                q_c=g(45, (C * q, H, dh)), q_r=g(46, (R * q_req, H, dh)), q=q, q_req=q_req, scale=1.0 / math.sqrt(dh))


def _project_bf16(oracle_mod, s_seq, w):
    """K = S W^T with a library matmul in float64, then the oracle's (separately pinned) bf16 rounding."""
    k = ri.bf16_to_f32(s_seq).astype(np.float64) @ ri.bf16_to_f32(w).astype(np.float64).T
    kb = np.vectorize(oracle_mod.round_bf16)(k).astype(np.float32)
    return (kb.view(np.uint32) >> 16).astype(np.uint16)


def test_dca_block_equals_projection_then_attention(oracle_mod):
    """Eq. (13): A^C = Attn(Q^C, S W_K^C, S W_V^C) and A^R = Attn(Q^R, S W_K^R, S W_V^R).  The block
    oracle projects a per-candidate copy of S (broadcast first); here S is projected once per request
    with a library matmul (projection first, section 4.1) and fed to the pinned attention oracle."""
    b = _block_inputs(51, [2, 0, 3], [5, 7, 4])
    H, dh = b["q_c"].shape[1], b["q_c"].shape[2]
    o_c, l_c, o_r, l_r = oracle_mod.dca_block(b["cand_off"], b["seq_off"], b["s_seq"], b["w_kc"], b["w_vc"],
                                              b["w_kr"], b["w_vr"], b["q_c"], b["q_r"], b["q"], b["q_req"], b["scale"])
    kc, vc = (_project_bf16(oracle_mod, b["s_seq"], w).reshape(-1, H, dh) for w in (b["w_kc"], b["w_vc"]))
    oo, ll = oracle_mod.dca(b["cand_off"], b["seq_off"], b["q_c"], kc, vc, b["q"], b["scale"])
    assert np.array_equal(o_c, oo) and np.array_equal(l_c, ll)
    kr, vr = (_project_bf16(oracle_mod, b["s_seq"], w).reshape(-1, H, dh) for w in (b["w_kr"], b["w_vr"]))
    R = len(b["cand_off"]) - 1
    ident = np.arange(R + 1, dtype=np.int32)  # every request attends over its own keys with its own queries
    oo, ll = oracle_mod.dca(ident, b["seq_off"], b["q_r"], kr, vr, b["q_req"], b["scale"])
    assert np.array_equal(o_r, oo) and np.array_equal(l_r, ll)


def test_dca_block_closed_forms(oracle_mod):
    """W_K = 0: uniform weights, O = mean over the request's keys of the projected V.
    A single key: O = that key's projected V exactly."""
    b = _block_inputs(52, [3, 2], [6, 1])
    H, dh = b["q_c"].shape[1], b["q_c"].shape[2]
    zero = np.zeros_like(b["w_kc"])
    o_c, _, o_r, _ = oracle_mod.dca_block(b["cand_off"], b["seq_off"], b["s_seq"], zero, b["w_vc"], zero,
                                          b["w_vr"], b["q_c"], b["q_r"], b["q"], b["q_req"], b["scale"])
    vc = ri.bf16_to_f32(_project_bf16(oracle_mod, b["s_seq"], b["w_vc"])).astype(np.float64).reshape(-1, H, dh)
    vr = ri.bf16_to_f32(_project_bf16(oracle_mod, b["s_seq"], b["w_vr"])).astype(np.float64).reshape(-1, H, dh)
    assert np.abs(o_c[:3] - vc[0:6].mean(0)).max() <= 1e-12
    assert np.abs(o_c[3:] - vc[6]).max() <= 1e-12
    assert np.abs(o_r[0] - vr[0:6].mean(0)).max() <= 1e-12 and np.abs(o_r[1] - vr[6]).max() <= 1e-12


# ------------------------------------------------------------------------------ LCB block (f4)
# Section 3.1.2 Eq. (4) (bias), section 3.1.3 Eq. (7) (group-local norm) and Eq. (8) (pointwise
# merge / activation).  Library routines (numpy matmul, torch layer_norm / rms_norm / silu / gelu
# in fp64) and closed forms pin the oracle's epilogue.
def _blk(seed, counts=(3, 0, 2, 1), n_r=5, n_c=3, d=16, o_r=4, o_c=6, norm="layernorm", act="silu", **kw):
    return ri.make_lcb_block("t", list(counts), n_r, n_c, d, o_r, o_c, seed, norm, act, **kw)


def _blk_run(oracle_mod, x, **kw):
    L = x.lcb
    return oracle_mod.lcb_block(L.cand_off, L.x_req, L.x_cand, L.w_rr, L.w_cr, L.w_cc, x.epi_r, x.epi_c, **kw)


def _library_block(x):
    """numpy matmul (Eq. 14 form) + torch fp64 norm / activation, straight from the definitions."""
    import torch.nn.functional as F
    L = x.lcb
    w = lambda a: ri.bf16_to_f32(a).astype(np.float64)
    xr, xc = w(L.x_req), w(L.x_cand)
    m = np.repeat(np.arange(L.R), np.diff(L.cand_off))
    yr = np.einsum("on,rnd->rod", w(L.w_rr), xr)
    yc = np.einsum("on,ind->iod", w(L.w_cr), xr[m]) + np.einsum("on,ind->iod", w(L.w_cc), xc)
    out = []
    for y, e in ((yr, x.epi_r), (yc, x.epi_c)):
        if e.bias is not None:
            y = y + e.bias.astype(np.float64)[None, :, None]
        if e.residual is not None:
            y = y + w(e.residual)
        t = torch.from_numpy(y)
        g = None if e.gamma is None else torch.from_numpy(e.gamma.astype(np.float64))
        b = None if e.beta is None else torch.from_numpy(e.beta.astype(np.float64))
        if e.norm == "layernorm":
            t = F.layer_norm(t, (t.shape[-1],), g, b, e.eps)
        elif e.norm == "rmsnorm":
            t = F.rms_norm(t, (t.shape[-1],), g, e.eps)
            if b is not None:
                t = t + b
        t = {"none": lambda v: v, "relu": F.relu, "silu": F.silu, "gelu": F.gelu}[e.act](t)
        out.append(t.numpy())
    return out


@pytest.mark.parametrize("norm,act", [("layernorm", "silu"), ("rmsnorm", "gelu"), ("none", "relu"),
                                      ("layernorm", "none")])
def test_lcb_block_matches_library(oracle_mod, norm, act):
    x = _blk(11, norm=norm, act=act)
    yr, yc = _blk_run(oracle_mod, x)
    lr, lc = _library_block(x)
    for a, b in ((yr, lr), (yc, lc)):
        assert np.max(np.abs(a - b)) <= 1e-12 * max(1.0, np.max(np.abs(b)))


def test_lcb_block_groups_use_their_own_parameters(oracle_mod):
    # request group RMSNorm + GELU, candidate group LayerNorm + ReLU: a swapped group fails the library check
    x = _blk(12, norm="layernorm", act="relu", norm_r="rmsnorm", act_r="gelu")
    yr, yc = _blk_run(oracle_mod, x)
    lr, lc = _library_block(x)
    assert np.max(np.abs(yr - lr)) <= 1e-12 * np.max(np.abs(lr))
    assert np.max(np.abs(yc - lc)) <= 1e-12 * np.max(np.abs(lc))


def test_lcb_block_bias_and_residual_closed_forms(oracle_mod):
    x = _blk(13, norm="none", act="none")
    L = x.lcb
    for a in (L.w_rr, L.w_cr, L.w_cc):
        a[...] = 0
    yr, yc = _blk_run(oracle_mod, x)
    # W = 0: Y = b (broadcast over d) + residual, exactly
    assert np.array_equal(yr, x.epi_r.bias.astype(np.float64)[None, :, None] + ri.bf16_to_f32(x.epi_r.residual))
    assert np.array_equal(yc, x.epi_c.bias.astype(np.float64)[None, :, None] + ri.bf16_to_f32(x.epi_c.residual))


def test_lcb_block_activation_closed_forms(oracle_mod):
    # W = 0, no residual / norm: every output entry of row o is act(b[o]), so b picks the arguments
    vals = np.array([0.0, 1.0, -1.0, math.log(3.0), -math.log(3.0), 2.5], dtype=np.float32)
    res = {}
    for act in ("relu", "silu", "gelu"):
        x = _blk(14, norm="none", act=act, residual=False, o_c=len(vals))
        for a in (x.lcb.w_rr, x.lcb.w_cr, x.lcb.w_cc):
            a[...] = 0
        x.epi_c.bias = vals.copy()
        _, yc = _blk_run(oracle_mod, x)
        res[act] = yc[0, :, 0]
        assert np.all(yc == yc[:, :, :1])  # broadcast over d and candidates
    v = vals.astype(np.float64)
    assert np.array_equal(res["relu"], np.maximum(v, 0.0))
    # odd-part identities: f(x) - f(-x) = x for SiLU and GELU (sigma(x)+sigma(-x) = Phi(x)+Phi(-x) = 1)
    for act in ("silu", "gelu"):
        assert abs(res[act][1] - res[act][2] - 1.0) <= 1e-15
        assert abs(res[act][3] - res[act][4] - v[3]) <= 1e-15
        assert res[act][0] == 0.0
    # sigma(ln 3) = 3/4, so silu(ln 3) = 0.75 ln 3; the fp32 argument is off ln 3 by dx ~ 1e-8, corrected
    # to first order with silu'(ln 3) = 3/4 + ln 3 * 3/16
    l3 = math.log(3.0)
    assert abs(res["silu"][3] - (0.75 * l3 + (0.75 + l3 * 0.1875) * (v[3] - l3))) <= 1e-14
    assert abs(res["gelu"][1] - 0.8413447460685429) <= 1e-15  # Phi(1), standard normal table


def test_lcb_block_layernorm_row_moments(oracle_mod):
    x = _blk(15, norm="layernorm", act="none", d=32)
    x.epi_r.gamma = x.epi_c.gamma = None
    x.epi_r.beta = x.epi_c.beta = None
    yr, yc = _blk_run(oracle_mod, x)
    for y in (yr, yc):
        assert np.max(np.abs(y.mean(-1))) <= 1e-13
        v = y.var(-1)
        assert np.all(v <= 1.0) and np.all(v > 0.99)  # var/(var+eps) with var = O(1), eps = 1e-5


def test_lcb_block_isolation_bitwise(oracle_mod):
    x = _blk(16)
    yr, _ = _blk_run(oracle_mod, x)
    x2 = _blk(16)
    x2.lcb.x_cand[...] = ri.normal(99, 1, x2.lcb.x_cand.shape)
    x2.epi_c.residual[...] = ri.normal(99, 2, x2.epi_c.residual.shape)
    x2.epi_c.gamma[...] = 3.0
    yr2, _ = _blk_run(oracle_mod, x2)
    assert np.array_equal(yr, yr2)


# ------------------------------------------------------------------------------ masked FM (f3)
# Section 3.1.4 Eq. (9)-(10) and the alignment transform of section 4.2.4.
def _fm_inputs(seed, counts=(2, 0, 3, 1), n_r=6, n_c=4, d=8):
    return ri.make_lcb("t", list(counts), n_r, n_c, d, 8, 8, seed, "bf16")


def test_fm_bruteforce_exact(oracle_mod):
    x = _fm_inputs(21)
    yr, yc = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand)
    xr = [[Fraction(float(v)) for v in row] for row in ri.bf16_to_f32(x.x_req).reshape(-1, x.d)]
    xc = [[Fraction(float(v)) for v in row] for row in ri.bf16_to_f32(x.x_cand).reshape(-1, x.d)]
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    dot = lambda u, v: sum(a * b for a, b in zip(u, v))
    for i in range(x.C):
        rows_r = xr[m[i] * x.n_r:(m[i] + 1) * x.n_r]
        for a in range(x.n_c):
            u = xc[i * x.n_c + a]
            want = [dot(u, v) for v in rows_r] + [dot(u, xc[i * x.n_c + b]) for b in range(x.n_c)]
            assert [Fraction(float(v)) for v in yc[i, a]] == want
    for r in range(x.R):
        rows_r = xr[r * x.n_r:(r + 1) * x.n_r]
        assert [[Fraction(float(v)) for v in row] for row in yr[r]] == [[dot(u, v) for v in rows_r] for u in rows_r]


def test_fm_matches_library_and_symmetry(oracle_mod):
    x = _fm_inputs(22, counts=(5, 3), n_r=16, n_c=8, d=32)
    yr, yc = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand)
    xr = ri.bf16_to_f32(x.x_req).astype(np.float64)
    xc = ri.bf16_to_f32(x.x_cand).astype(np.float64)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    want_c = np.concatenate([np.einsum("iac,ibc->iab", xc, xr[m]), np.einsum("iac,ibc->iab", xc, xc)], axis=2)
    assert np.max(np.abs(yc - want_c)) <= 1e-12 * np.max(np.abs(want_c))
    assert np.max(np.abs(yr - np.einsum("rac,rbc->rab", xr, xr))) <= 1e-12 * np.max(np.abs(yr))
    assert np.array_equal(yr, np.transpose(yr, (0, 2, 1)))
    self_blk = yc[:, :, x.n_r:]
    assert np.array_equal(self_blk, np.transpose(self_blk, (0, 2, 1)))


def test_fm_closed_forms(oracle_mod):
    # candidate embeddings equal to their request's: both blocks of Y^C equal Y^R of the request
    x = _fm_inputs(23, counts=(2, 1, 2), n_r=5, n_c=5, d=8)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    x.x_cand[...] = x.x_req[m]
    yr, yc = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand)
    assert np.array_equal(yc[:, :, :5], yr[m]) and np.array_equal(yc[:, :, 5:], yr[m])
    # zero candidate embeddings: Y^C = 0, Y^R unchanged
    x.x_cand[...] = 0
    yr2, yc2 = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand)
    assert np.array_equal(yr2, yr) and not np.any(yc2)


def test_fm_isolation_bitwise(oracle_mod):
    x = _fm_inputs(24)
    yr, _ = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand)
    x.x_cand[...] = ri.normal(77, 1, x.x_cand.shape)
    yr2, _ = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand)
    assert np.array_equal(yr, yr2)


def test_pad_transform_leaves_the_computation_unchanged(oracle_mod):
    # section 4.2.4: zero-pad the contiguous axis (30 -> 32 entries) and give the consumer's weight
    # matching zero columns; the consumer's result is unchanged (small integers: exact)
    rs = np.random.RandomState(5)
    y = rs.randint(-4, 5, size=(7, 3, 30)).astype(np.float64)
    w = rs.randint(-3, 4, size=(11, 3 * 30)).astype(np.float64)
    yp = oracle_mod.pad_cols(y, 32)
    assert yp.shape == (7, 3, 32) and not np.any(yp[..., 30:])
    assert np.array_equal(oracle_mod.unpad_cols(yp, 30), y)
    wp = oracle_mod.pad_cols(w.reshape(11, 3, 30), 32).reshape(11, 96)
    assert np.array_equal(yp.reshape(7, 96) @ wp.T, y.reshape(7, 90) @ w.T)


# ------------------------------------------------------------------------------ split chain (f2)
# The chain that never stores Y^C: Q_i = W_q vec(Y^C_i) with the exact LCB output, which the IKBO
# decomposition splits into W_q vec(Z_{m_i}) (once per request) + W_fold vec(X^C_i).
def _bf16_bits(a):
    return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_chain_exact_equals_rounded_chain_when_y_is_exact(oracle_mod):
    # small integers everywhere: every Y^C entry is an exact bf16 value, so rounding it changes nothing
    ci = _shrink_chain(_small_chain(44))
    x = ci.lcb
    rs = np.random.RandomState(3)
    for name in ("x_req", "x_cand"):
        setattr(x, name, _bf16_bits(rs.randint(-2, 3, size=getattr(x, name).shape)))
    for name in ("w_rr", "w_cr", "w_cc"):
        setattr(x, name, _bf16_bits(rs.randint(-1, 2, size=getattr(x, name).shape)))
    sel = np.arange(x.C)
    a = oracle_mod.chain(ci, sel, round_y=True)
    b = oracle_mod.chain(ci, sel, round_y=False)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_chain_exact_query_matches_library(oracle_mod):
    ci = _shrink_chain(_small_chain(45))
    x = ci.lcb
    y, qo, _, _ = oracle_mod.chain(ci, np.arange(x.C), round_y=False)
    w = lambda a: ri.bf16_to_f32(a).astype(np.float64)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    yc = np.einsum("on,ind->iod", w(x.w_cr), w(x.x_req)[m]) + np.einsum("on,ind->iod", w(x.w_cc), w(x.x_cand))
    assert np.max(np.abs(y - yc)) <= 1e-12 * np.max(np.abs(yc))
    q = yc.reshape(x.C, -1) @ w(ci.w_q).T
    assert np.max(np.abs(qo - q)) <= 1e-12 * np.max(np.abs(q))


def test_split_projection_identity(oracle_mod):
    # Q_i = W_q vec(Z_{m_i}) + W_fold vec(X^C_i): pins the fold's index map (a transposed fold fails)
    ci = _shrink_chain(_small_chain(46))
    x = ci.lcb
    _, qo, _, _ = oracle_mod.chain(ci, np.arange(x.C), round_y=False)
    w = lambda a: ri.bf16_to_f32(a).astype(np.float64)
    wf = oracle_mod.chain_fold(ci.w_q, x.w_cc, x.d)
    assert wf.shape == (ci.H * ci.dh, x.n_c * x.d)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off))
    z = np.einsum("on,rnd->rod", w(x.w_cr), w(x.x_req)).reshape(x.R, -1)
    q = (z @ w(ci.w_q).T)[m] + w(x.x_cand).reshape(x.C, -1) @ wf.T
    assert np.max(np.abs(qo - q)) <= 1e-12 * np.max(np.abs(q))


def test_chain_fold_closed_form(oracle_mod):
    # W_CC = identity: the folded weight is W_q itself
    n_out, o_c, d = 6, 4, 3
    wq = ri.normal(9, 1, (n_out, o_c * d))
    eye = _bf16_bits(np.eye(o_c))
    assert np.array_equal(oracle_mod.chain_fold(wq, eye, d), ri.bf16_to_f32(wq).astype(np.float64))
