"""fp64 CPU oracle for IKBO-LCB / IKBO-DCA (ctypes wrapper over ``rocs_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The product path
(``attention_ikbo_b200``) never imports it, and it imports nothing from there.

Each function follows the ROCS paper (arXiv:2607.27744) as described in the
paper-archivist reading notes:

* :func:`lcb` -- section 3.1.2, Eq. (6), the two-group masked LCB, evaluated per
  candidate with the broadcast of ``X^R`` materialised, plus the Eq. (11) check that
  every candidate's request rows equal the request output computed once.
* :func:`dca` -- section 3.2, Eq. (13), candidate-group cross attention
  ``softmax(scale * Q K^T) V`` over the candidate's own request keys, non-causal,
  K/V copied per candidate.
* :func:`dca_block` -- section 3.2, Eq. (13) with both query groups: K/V projections of the
  request sequence (per candidate, broadcast materialised, then rounded to bf16) and the
  request-group attention A^R next to the candidate-group attention A^C.
* :func:`lcb_block` -- section 3.1.2 Eq. (4)-(6) with section 3.1.3 Eq. (7)-(8): the LCB with a
  per-row bias, a residual merge, a group-local LayerNorm/RMSNorm over d and an activation, each
  output group with its own parameters (broadcast materialised as in :func:`lcb`).
* :func:`fm` -- section 3.1.4, Eq. (9)-(10): the GLM-masked factorization machine, per candidate
  the Gram matrix of the materialised [X^R; X^C] with the block mask, plus the request output.
* :func:`pad_cols` / :func:`unpad_cols` -- the alignment transform of section 4.2.4 (zero padding of a
  contiguous dimension), written as its definition.
* :func:`chain_fold` -- the projection weight composed with W_CC (linear maps compose), used by the
  chain that splits the projection over the IKBO decomposition.
* :func:`proj` / :func:`chain` -- the chained block: LCB output -> bf16 -> linear
  query projection (section 3.2, Eq. (12), read as a plain linear map) -> bf16 -> DCA.

Pinning: every function here is checked by ``tests/test_oracle_pins.py`` against
closed forms, invariants, brute force in exact/high-precision arithmetic and
hand-derived golden cases (``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rocs_oracle.cpp")
_LIB = os.path.join(_HERE, "librocs_oracle.so")

ORC_OK, ORC_INVALID, ORC_BAD_OFFSETS, ORC_ISOLATION = 0, 1, 2, 10


class Epi(ctypes.Structure):
    """One output group's epilogue; the fields mirror ``OrcEpi`` in rocs_oracle.cpp."""
    _fields_ = [("bias", ctypes.c_void_p), ("residual", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("eps", ctypes.c_double), ("norm", ctypes.c_int32),
                ("act", ctypes.c_int32)]


NORMS = {"none": 0, "layernorm": 1, "rmsnorm": 2}
ACTS = {"none": 0, "relu": 1, "silu": 2, "gelu": 3}


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle returned {code}")
        self.code = code


def build_lib(force: bool = False) -> str:
    """Compile ``librocs_oracle.so`` (g++, OpenMP, fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        build_lib()
        lib = ctypes.CDLL(_LIB)
        i64, vp, dbl, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double, ctypes.c_int
        lib.rocs_oracle_lcb.argtypes = [i64, vp, i64, i64, i64, i64, i64, i32, vp, vp, vp, vp, vp,
                                        i64, vp, vp, i64, vp, vp, i32]
        lib.rocs_oracle_dca.argtypes = [i64, vp, vp, i64, i64, i64, dbl, vp, vp, vp, i64, vp, vp, vp, i32]
        lib.rocs_oracle_proj.argtypes = [i64, i64, i64, vp, vp, vp, i32]
        lib.rocs_oracle_chain.argtypes = [i64, vp, i64, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, vp,
                                          i64, i64, dbl, vp, vp, i64, vp, vp, vp, vp, vp, i32]
        lib.rocs_oracle_chain_exact.argtypes = lib.rocs_oracle_chain.argtypes
        lib.rocs_oracle_chain_fold.argtypes = [i64, i64, i64, i64, vp, vp, vp, i32]
        lib.rocs_oracle_dca_block.argtypes = [i64, vp, vp, i64, i64, i64, i64, i64, dbl, vp, vp, vp, vp, vp, vp, vp,
                                              i64, vp, vp, vp, i64, vp, vp, vp, i32]
        lib.rocs_oracle_lcb_block.argtypes = [i64, vp, i64, i64, i64, i64, i64, vp, vp, vp, vp, vp,
                                              ctypes.POINTER(Epi), ctypes.POINTER(Epi), i64, vp, vp, i64, vp, vp, i32]
        lib.rocs_oracle_fm.argtypes = [i64, vp, i64, i64, i64, vp, vp, i64, vp, vp, i64, vp, vp, i32]
        lib.rocs_oracle_round_bf16.restype = dbl
        lib.rocs_oracle_round_bf16.argtypes = [dbl]
        lib.rocs_oracle_max_threads.restype = i32
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def max_threads() -> int:
    return int(_L().rocs_oracle_max_threads())


def round_bf16(x: float) -> float:
    return float(_L().rocs_oracle_round_bf16(float(x)))


def _dtype_code(arr) -> int:
    if arr.dtype == np.float32:
        return 0
    if arr.dtype == np.uint16:
        return 1
    raise TypeError(f"unsupported input dtype {arr.dtype}")


def lcb(cand_off, x_req, x_cand, w_rr, w_cr, w_cc, sel_req=None, sel_cand=None, nthreads: int = 0):
    """Return ``(y_req [len(sel_req), o_r, d], y_cand [len(sel_cand), o_c, d])`` in float64.

    Inputs are fp32 arrays or bf16 bit patterns (uint16), shapes as in ``rocs_inputs``.
    ``sel_*`` default to all requests / all candidates.
    """
    cand_off = _c(cand_off, np.int32)
    R = len(cand_off) - 1
    C = int(cand_off[-1])
    dt = _dtype_code(x_req)
    _, n_r, d = x_req.shape
    n_c = x_cand.shape[1]
    o_r, o_c = w_rr.shape[0], w_cc.shape[0]
    sel_req = np.arange(R, dtype=np.int64) if sel_req is None else _c(sel_req, np.int64)
    sel_cand = np.arange(C, dtype=np.int64) if sel_cand is None else _c(sel_cand, np.int64)
    y_req = np.empty((len(sel_req), o_r, d), dtype=np.float64)
    y_cand = np.empty((len(sel_cand), o_c, d), dtype=np.float64)
    arrs = [_c(a, a.dtype) for a in (x_req, x_cand, w_rr, w_cr, w_cc)]
    rc = _L().rocs_oracle_lcb(R, _p(cand_off), n_r, n_c, d, o_r, o_c, dt, *[_p(a) for a in arrs],
                              len(sel_req), _p(sel_req), _p(y_req), len(sel_cand), _p(sel_cand), _p(y_cand),
                              nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return y_req, y_cand


def dca(cand_off, seq_off, q_t, k_t, v_t, q: int, scale: float, sel_cand=None, nthreads: int = 0):
    """Return ``(o [n_sel, q, H, dh], lse [n_sel, q, H])`` in float64 (bf16 inputs)."""
    cand_off, seq_off = _c(cand_off, np.int32), _c(seq_off, np.int32)
    R = len(cand_off) - 1
    C = int(cand_off[-1])
    H, dh = k_t.shape[1], k_t.shape[2]
    sel = np.arange(C, dtype=np.int64) if sel_cand is None else _c(sel_cand, np.int64)
    o = np.empty((len(sel), q, H, dh), dtype=np.float64)
    lse = np.empty((len(sel), q, H), dtype=np.float64)
    qa, ka, va = (_c(a, np.uint16) for a in (q_t, k_t, v_t))
    rc = _L().rocs_oracle_dca(R, _p(cand_off), _p(seq_off), q, H, dh, float(scale), _p(qa), _p(ka), _p(va),
                              len(sel), _p(sel), _p(o), _p(lse), nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return o, lse


def proj(y_bf16, w_q, nthreads: int = 0):
    """``q[k] = W_q . y[k]`` in float64; ``y_bf16 [n, n_in]`` and ``w_q [n_out, n_in]`` are bf16 bits."""
    y = _c(y_bf16, np.uint16).reshape(y_bf16.shape[0], -1)
    w = _c(w_q, np.uint16)
    out = np.empty((y.shape[0], w.shape[0]), dtype=np.float64)
    rc = _L().rocs_oracle_proj(y.shape[0], y.shape[1], w.shape[0], _p(y), _p(w), _p(out), nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return out


def chain(ci, sel_cand, nthreads: int = 0, round_y: bool = True):
    """Chained block for candidates ``sel_cand`` of a ``rocs_inputs.ChainInputs``.

    ``round_y``: Y^C is stored in bf16 between the LCB and the projection (the unfused chain); False:
    the projection consumes the exact LCB output (the chain that never stores Y^C).
    Returns ``(y_cand [n,o_c,d], q [n,H*dh], o [n,H,dh], lse [n,H])`` in float64.
    """
    x = ci.lcb
    sel = _c(sel_cand, np.int64)
    n = len(sel)
    y = np.empty((n, x.o_c, x.d), dtype=np.float64)
    qo = np.empty((n, ci.H * ci.dh), dtype=np.float64)
    o = np.empty((n, ci.H, ci.dh), dtype=np.float64)
    lse = np.empty((n, ci.H), dtype=np.float64)
    co, so = _c(x.cand_off, np.int32), _c(ci.seq_off, np.int32)
    fn = _L().rocs_oracle_chain if round_y else _L().rocs_oracle_chain_exact
    rc = fn(x.R, _p(co), x.n_r, x.n_c, x.d, x.o_r, x.o_c, _p(x.x_req), _p(x.x_cand),
                                _p(x.w_rr), _p(x.w_cr), _p(x.w_cc), _p(ci.w_q), _p(so), ci.H, ci.dh,
                                float(ci.scale), _p(ci.k_t), _p(ci.v_t), n, _p(sel), _p(y), _p(qo), _p(o),
                                _p(lse), nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return y, qo, o, lse


def dca_block(cand_off, seq_off, s_seq, w_kc, w_vc, w_kr, w_vr, q_c, q_r, q: int, q_req: int, scale: float,
              sel_cand=None, sel_req=None, nthreads: int = 0):
    """Section 3.2 Eq. (13), both groups.  Returns ``(o_c, lse_c, o_r, lse_r)`` in float64:
    o_c [n_c, q, H, dh], lse_c [n_c, q, H], o_r [n_r, q_req, H, dh], lse_r [n_r, q_req, H]."""
    cand_off, seq_off = _c(cand_off, np.int32), _c(seq_off, np.int32)
    R, C = len(cand_off) - 1, int(cand_off[-1])
    d_s = s_seq.shape[1]
    H, dh = q_c.shape[1], q_c.shape[2]
    sc = np.arange(C, dtype=np.int64) if sel_cand is None else _c(sel_cand, np.int64)
    sr = np.arange(R, dtype=np.int64) if sel_req is None else _c(sel_req, np.int64)
    o_c = np.empty((len(sc), q, H, dh)); lse_c = np.empty((len(sc), q, H))
    o_r = np.empty((len(sr), q_req, H, dh)); lse_r = np.empty((len(sr), q_req, H))
    arrs = [_c(a, np.uint16) for a in (s_seq, w_kc, w_vc, w_kr, w_vr, q_c, q_r)]
    rc = _L().rocs_oracle_dca_block(R, _p(cand_off), _p(seq_off), q, q_req, H, dh, d_s, float(scale),
                                    *[_p(a) for a in arrs], len(sc), _p(sc), _p(o_c), _p(lse_c), len(sr), _p(sr),
                                    _p(o_r), _p(lse_r), nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return o_c, lse_c, o_r, lse_r


def _epi(e, keep):
    """``e``: object with bias/residual/gamma/beta (arrays or None), eps, norm, act (names or codes)."""
    def arr(a, dt):
        if a is None:
            return None
        a = _c(a, dt)
        keep.append(a)
        return a.ctypes.data
    norm = NORMS[e.norm] if isinstance(e.norm, str) else int(e.norm)
    act = ACTS[e.act] if isinstance(e.act, str) else int(e.act)
    return Epi(arr(e.bias, np.float32), arr(e.residual, np.uint16), arr(e.gamma, np.float32),
               arr(e.beta, np.float32), float(e.eps), norm, act)


def lcb_block(cand_off, x_req, x_cand, w_rr, w_cr, w_cc, epi_r, epi_c, sel_req=None, sel_cand=None,
              nthreads: int = 0):
    """LCB block with per-group epilogues (bf16 inputs).  Returns ``(y_req, y_cand)`` in float64."""
    cand_off = _c(cand_off, np.int32)
    R, C = len(cand_off) - 1, int(cand_off[-1])
    _, n_r, d = x_req.shape
    n_c = x_cand.shape[1]
    o_r, o_c = w_rr.shape[0], w_cc.shape[0]
    sel_req = np.arange(R, dtype=np.int64) if sel_req is None else _c(sel_req, np.int64)
    sel_cand = np.arange(C, dtype=np.int64) if sel_cand is None else _c(sel_cand, np.int64)
    y_req = np.empty((len(sel_req), o_r, d), dtype=np.float64)
    y_cand = np.empty((len(sel_cand), o_c, d), dtype=np.float64)
    keep = []
    er, ec = _epi(epi_r, keep), _epi(epi_c, keep)
    arrs = [_c(a, np.uint16) for a in (x_req, x_cand, w_rr, w_cr, w_cc)]
    rc = _L().rocs_oracle_lcb_block(R, _p(cand_off), n_r, n_c, d, o_r, o_c, *[_p(a) for a in arrs],
                                    ctypes.byref(er), ctypes.byref(ec), len(sel_req), _p(sel_req), _p(y_req),
                                    len(sel_cand), _p(sel_cand), _p(y_cand), nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return y_req, y_cand


def fm(cand_off, x_req, x_cand, sel_req=None, sel_cand=None, nthreads: int = 0):
    """Eq. (10).  Returns ``(y_req [n_sel_r, n_r, n_r], y_cand [n_sel_c, n_c, n_r + n_c])`` in float64."""
    cand_off = _c(cand_off, np.int32)
    R, C = len(cand_off) - 1, int(cand_off[-1])
    _, n_r, d = x_req.shape
    n_c = x_cand.shape[1]
    sr = np.arange(R, dtype=np.int64) if sel_req is None else _c(sel_req, np.int64)
    sc = np.arange(C, dtype=np.int64) if sel_cand is None else _c(sel_cand, np.int64)
    y_req = np.empty((len(sr), n_r, n_r))
    y_cand = np.empty((len(sc), n_c, n_r + n_c))
    xr, xc = _c(x_req, np.uint16), _c(x_cand, np.uint16)
    rc = _L().rocs_oracle_fm(R, _p(cand_off), n_r, n_c, d, _p(xr), _p(xc), len(sr), _p(sr), _p(y_req), len(sc),
                             _p(sc), _p(y_cand), nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return y_req, y_cand


def pad_cols(a, cols_pad):
    """Section 4.2.4: zero-pad the last (contiguous) axis of ``a`` to ``cols_pad`` entries."""
    a = np.asarray(a)
    out = np.zeros(a.shape[:-1] + (cols_pad,), dtype=a.dtype)
    out[..., :a.shape[-1]] = a
    return out


def unpad_cols(a, cols):
    """Inverse of :func:`pad_cols`: the first ``cols`` entries of the last axis."""
    return np.ascontiguousarray(np.asarray(a)[..., :cols])


def chain_fold(w_q, w_cc, d: int, nthreads: int = 0):
    """``W_fold[k, n*d + c] = sum_o W_q[k, o*d + c] W_CC[o, n]`` in float64 (bf16 inputs)."""
    wq, wc = _c(w_q, np.uint16), _c(w_cc, np.uint16)
    n_out, o_c, n_c = wq.shape[0], wc.shape[0], wc.shape[1]
    out = np.empty((n_out, n_c * d))
    rc = _L().rocs_oracle_chain_fold(n_out, o_c, n_c, d, _p(wq), _p(wc), _p(out), nthreads)
    if rc != ORC_OK:
        raise OracleError(rc)
    return out
