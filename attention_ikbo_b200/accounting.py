"""Algorithmic work and traffic of the IKBO kernels, counted on the non-materialised formulation.

Only what the method must do is counted: every input read once, every output written once,
request-side work once per request ("ROCS ...", arXiv:2607.27744, section 5.1.1: per-candidate
amortised cost c_amort(N) = C_C + C_R / N).  Workspace traffic (Z, flags) is on-chip / L2 and
is not counted.

LCB (section 3.1.2 Eq. (6), section 4.1 Eq. (14)):
  request part   C_R = 2 (o_r + o_c) n_r d            (one [W_RR; W_CR] GEMM per request)
  candidate part C_C = 2 o_c n_c d + o_c d             (W_CC GEMM + broadcast-add)
  bytes          X^R, X^C, the three weight blocks, Y^R, Y^C
DCA (section 3.2 Eq. (13)):
  flops  4 * sum_r q N_r L_r H dh                      (S = Q K^T and O = P V)
  bytes  Q + K + V + O (+ LSE)
Projection: flops 2 M N K, bytes in + W + out.
Masked FM (section 3.1.4 Eq. (10)):
  request part   2 n_r^2 d                             (X^R X^R^T once per request)
  candidate part 2 n_c (n_r + n_c) d                   (cross block against the shared X^R, self block)
  bytes          X^R, X^C, Y^R and Y^C at their unpadded row lengths (padding bytes are not counted)
"""
from __future__ import annotations

import numpy as np


def lcb_request_flops(n_r, d, o_r, o_c):
    return 2 * (o_r + o_c) * n_r * d


def lcb_candidate_flops(n_c, d, o_c):
    return 2 * o_c * n_c * d + o_c * d


def lcb_flops(R, C, n_r, n_c, d, o_r, o_c):
    return R * lcb_request_flops(n_r, d, o_r, o_c) + C * lcb_candidate_flops(n_c, d, o_c)


def lcb_bytes(R, C, n_r, n_c, d, o_r, o_c, elem=2):
    return elem * (R * n_r * d + C * n_c * d + o_r * n_r + o_c * n_r + o_c * n_c + R * o_r * d + C * o_c * d)


def amortised_flops_per_candidate(N, n_r, n_c, d, o_r, o_c):
    """c_amort(N) = C_C + C_R / N for one request scored against N candidates."""
    return lcb_candidate_flops(n_c, d, o_c) + lcb_request_flops(n_r, d, o_r, o_c) / N


def dca_flops(cand_off, seq_off, q, H, dh):
    n = np.diff(np.asarray(cand_off, dtype=np.int64))
    L = np.diff(np.asarray(seq_off, dtype=np.int64))
    return int(4 * q * H * dh * int(np.sum(n * L)))


def dca_bytes(C, T, q, H, dh, lse=True, elem=2):
    return elem * (2 * C * q * H * dh + 2 * T * H * dh) + (4 * C * q * H if lse else 0)


def proj_flops(M, N, K):
    return 2 * M * N * K


def proj_bytes(M, N, K, elem=2):
    return elem * (M * K + N * K + M * N)


def fm_flops(R, C, n_r, n_c, d):
    return R * 2 * n_r * n_r * d + C * 2 * n_c * (n_r + n_c) * d


def fm_bytes(R, C, n_r, n_c, d, elem=2):
    return elem * (R * n_r * d + C * n_c * d + R * n_r * n_r + C * n_c * (n_r + n_c))
