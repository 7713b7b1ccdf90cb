"""Algorithmic FLOP/byte accounting used by the benchmark, checked against the amortised-cost
formula of ROCS (arXiv:2607.27744) section 5.1.1, c_amort(N) = C_C + C_R / N, and against
direct counts."""
import numpy as np

from attention_ikbo_b200 import accounting as acc


def test_lcb_amortised_cost():
    n_r, n_c, d, o_r, o_c = 256, 64, 128, 128, 128
    for N in (1, 7, 100, 1000):
        total = acc.lcb_flops(1, N, n_r, n_c, d, o_r, o_c)
        assert abs(total / N - acc.amortised_flops_per_candidate(N, n_r, n_c, d, o_r, o_c)) < 1e-6
    # C_R and C_C as GEMM counts: [W_RR; W_CR] (256 x 256) . X^R (256 x 128), and W_CC . X^C + add
    assert acc.lcb_request_flops(n_r, d, o_r, o_c) == 2 * 256 * 256 * 128
    assert acc.lcb_candidate_flops(n_c, d, o_c) == 2 * 128 * 64 * 128 + 128 * 128


def test_lcb_bytes_count_each_tensor_once():
    R, C, n_r, n_c, d, o_r, o_c = 3, 10, 64, 64, 128, 128, 128
    expect = 2 * (R * n_r * d + C * n_c * d + o_r * n_r + o_c * n_r + o_c * n_c + R * o_r * d + C * o_c * d)
    assert acc.lcb_bytes(R, C, n_r, n_c, d, o_r, o_c) == expect


def test_dca_flops_direct_count():
    cand_off, seq_off, q, H, dh = [0, 3, 3, 8], [0, 10, 30, 31], 2, 4, 64
    direct = 0
    for r in range(3):
        rows = q * (cand_off[r + 1] - cand_off[r])
        L = seq_off[r + 1] - seq_off[r]
        direct += H * (2 * rows * L * dh + 2 * rows * L * dh)  # Q K^T and P V
    assert acc.dca_flops(np.array(cand_off), np.array(seq_off), q, H, dh) == direct
