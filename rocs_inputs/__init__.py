"""Seeded synthetic inputs for the IKBO workloads (LCB, DCA and the chained block).

This module is shared by the CUDA path's tests/bench and by the CPU oracle; it
holds no arithmetic of the method itself.  Every tensor is drawn from its own
counter-based SplitMix64 stream (see ``rocs_gen.c``), so the bytes depend only on
(seed, stream, element index) and never on thread count or call order.

Tensor conventions (row-major, last axis contiguous):

* LCB (ROCS paper, section 3.1.2, Eq. 5-6; section 4.1, Eq. 14):
  ``x_req [R, n_r, d]``, ``x_cand [C, n_c, d]``, ``w_rr [o_r, n_r]``,
  ``w_cr [o_c, n_r]``, ``w_cc [o_c, n_c]``; candidates of request ``r`` are rows
  ``cand_off[r] .. cand_off[r+1]-1`` (CSR; candidates of one request stored
  contiguously, section 4.2.1).
* DCA (section 3.2, Eq. 13; section 4.3.1): ``q_t [C*q, H, dh]``,
  ``k_t / v_t [sum L_r, H, dh]`` with ``seq_off`` (CSR over the key sequence).

bf16 tensors are returned as ``np.uint16`` bit patterns; fp32 as ``np.float32``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rocs_gen.c")
_LIB = os.path.join(_HERE, "librocs_gen.so")

# one stream id per tensor role
S_XREQ, S_XCAND, S_WRR, S_WCR, S_WCC, S_NCAND, S_LSEQ, S_Q, S_K, S_V, S_WQ = range(1, 12)
S_SEQ, S_WKV, S_QREQ = range(12, 15)
# epilogue parameters, one stream per (group, role): request group 20.., candidate group 30..
S_EPI_R, S_EPI_C = 20, 30
E_BIAS, E_GAMMA, E_BETA, E_RES = range(4)


def build_lib(force: bool = False) -> str:
    """Compile ``librocs_gen.so`` with gcc (OpenMP) if missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        build_lib()
        lib = ctypes.CDLL(_LIB)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.rocs_gen_u64.restype = u64
        lib.rocs_gen_u64.argtypes = [u64, u64, u64]
        lib.rocs_gen_normal_f32.argtypes = [u64, u64, u64, dbl, vp, i64]
        lib.rocs_gen_normal_bf16.argtypes = [u64, u64, u64, dbl, vp, i64]
        lib.rocs_gen_uniform_int.argtypes = [u64, u64, i64, i64, vp, i64]
        lib.rocs_gen_lognormal_int.argtypes = [u64, u64, dbl, dbl, i64, i64, vp, i64]
        _lib = lib
    return _lib


def normal(seed: int, stream: int, shape, std: float = 1.0, dtype: str = "bf16", offset: int = 0) -> np.ndarray:
    """``std * N(0,1)`` samples; ``dtype`` 'bf16' -> uint16 bit patterns, 'f32' -> float32."""
    n = int(np.prod(shape)) if len(shape) else 1
    if dtype == "bf16":
        out = np.empty(shape, dtype=np.uint16)
        _L().rocs_gen_normal_bf16(seed, stream, offset, float(std), out.ctypes.data, n)
    elif dtype == "f32":
        out = np.empty(shape, dtype=np.float32)
        _L().rocs_gen_normal_f32(seed, stream, offset, float(std), out.ctypes.data, n)
    else:
        raise ValueError(dtype)
    return out


def uniform_int(seed: int, stream: int, lo: int, hi: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    _L().rocs_gen_uniform_int(seed, stream, lo, hi, out.ctypes.data, n)
    return out


def lognormal_int(seed: int, stream: int, median: float, sigma: float, lo: int, hi: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    _L().rocs_gen_lognormal_int(seed, stream, math.log(median), sigma, lo, hi, out.ctypes.data, n)
    return out


def counts_to_offsets(counts) -> np.ndarray:
    off = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(np.asarray(counts, dtype=np.int64), out=off[1:])
    if off[-1] > np.iinfo(np.int32).max:
        raise ValueError("offsets exceed int32")
    return off.astype(np.int32)


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (a.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------------------
@dataclass
class LcbInputs:
    name: str
    dtype: str  # "f32" or "bf16"
    cand_off: np.ndarray  # int32 [R+1]
    n_r: int
    n_c: int
    d: int
    o_r: int
    o_c: int
    x_req: np.ndarray
    x_cand: np.ndarray
    w_rr: np.ndarray
    w_cr: np.ndarray
    w_cc: np.ndarray
    seed: int = 0
    recipe: str = ""

    @property
    def R(self) -> int:
        return len(self.cand_off) - 1

    @property
    def C(self) -> int:
        return int(self.cand_off[-1])


@dataclass
class DcaInputs:
    name: str
    cand_off: np.ndarray  # int32 [R+1]
    seq_off: np.ndarray  # int32 [R+1]
    q: int
    H: int
    dh: int
    scale: float
    q_t: np.ndarray  # uint16 [C*q, H, dh]
    k_t: np.ndarray  # uint16 [sumL, H, dh]
    v_t: np.ndarray  # uint16 [sumL, H, dh]
    seed: int = 0
    recipe: str = ""

    @property
    def R(self) -> int:
        return len(self.cand_off) - 1

    @property
    def C(self) -> int:
        return int(self.cand_off[-1])

    @property
    def total_L(self) -> int:
        return int(self.seq_off[-1])


@dataclass
class ChainInputs:
    name: str
    lcb: LcbInputs
    w_q: np.ndarray  # uint16 [H*dh, o_c*d]
    seq_off: np.ndarray
    H: int
    dh: int
    scale: float
    k_t: np.ndarray
    v_t: np.ndarray
    recipe: str = ""


def make_lcb(name, counts, n_r, n_c, d, o_r, o_c, seed, dtype="bf16") -> LcbInputs:
    """Embeddings ~ N(0,1); each weight block ~ N(0, 1/n_in) with n_in its own input-group size."""
    off = counts_to_offsets(counts)
    R, C = len(counts), int(off[-1])
    return LcbInputs(
        name=name, dtype=dtype, cand_off=off, n_r=n_r, n_c=n_c, d=d, o_r=o_r, o_c=o_c,
        x_req=normal(seed, S_XREQ, (R, n_r, d), 1.0, dtype),
        x_cand=normal(seed, S_XCAND, (C, n_c, d), 1.0, dtype),
        w_rr=normal(seed, S_WRR, (o_r, n_r), 1.0 / math.sqrt(n_r), dtype),
        w_cr=normal(seed, S_WCR, (o_c, n_r), 1.0 / math.sqrt(n_r), dtype),
        w_cc=normal(seed, S_WCC, (o_c, n_c), 1.0 / math.sqrt(n_c), dtype),
        seed=seed,
    )


def make_dca(name, counts, lengths, q, H, dh, seed, scale=None) -> DcaInputs:
    """Q, K, V ~ N(0,1) in bf16; K/V stored once per request (no candidate copies)."""
    coff, soff = counts_to_offsets(counts), counts_to_offsets(lengths)
    C, L = int(coff[-1]), int(soff[-1])
    return DcaInputs(
        name=name, cand_off=coff, seq_off=soff, q=q, H=H, dh=dh,
        scale=float(scale if scale is not None else 1.0 / math.sqrt(dh)),
        q_t=normal(seed, S_Q, (C * q, H, dh)),
        k_t=normal(seed, S_K, (L, H, dh)),
        v_t=normal(seed, S_V, (L, H, dh)),
        seed=seed,
    )


# ---- the five workloads (sizes as specified; the recipe strings document them) --------
def lcb_tiny_f32(seed: int = 0) -> LcbInputs:
    x = make_lcb("lcb_tiny_f32", [16, 16, 16, 16], 8, 8, 32, 4, 8, seed, "f32")
    x.recipe = "R=4, 16 candidates each; n_r=n_c=8, d=32, o_r=4, o_c=8; X~N(0,1), W~N(0,1/n_in); fp32"
    return x


def lcb_bf16(seed: int = 2, R: int = 64, lo: int = 256, hi: int = 1024) -> LcbInputs:
    counts = uniform_int(seed, S_NCAND, lo, hi, R)
    x = make_lcb("lcb_bf16", counts, 256, 64, 128, 128, 128, seed, "bf16")
    x.recipe = f"R={R}, N_r~U{{{lo}..{hi}}}; n_r=256, n_c=64, d=128, o_r=o_c=128; X~N(0,1), W~N(0,1/n_in); bf16"
    return x


def dca_bf16(seed: int = 3, R: int = 32, L: int = 2048, H: int = 8, dh: int = 128, n_cand: int = 512, q: int = 1):
    x = make_dca("dca_bf16", [n_cand] * R, [L] * R, q, H, dh, seed)
    x.recipe = f"R={R}, L={L}, H={H}, dh={dh}, N_r={n_cand}, q={q}; Q,K,V~N(0,1); scale 1/sqrt(dh)"
    return x


def dca_long(seed: int = 4, R: int = 8, lo: int = 4096, hi: int = 8192, H: int = 4, dh: int = 128,
             n_cand: int = 2048, q: int = 4):
    lengths = uniform_int(seed, S_LSEQ, lo, hi, R)
    x = make_dca("dca_long", [n_cand] * R, lengths, q, H, dh, seed)
    x.recipe = f"R={R}, L_r~U{{{lo}..{hi}}}, H={H}, dh={dh}, N_r={n_cand}, q={q}; Q,K,V~N(0,1)"
    return x


def chain(seed: int = 5, R: int = 128, median: float = 512.0, sigma: float = 1.0, clip=(32, 4096),
          Llo: int = 1024, Lhi: int = 4096, H: int = 16, dh: int = 64) -> ChainInputs:
    counts = lognormal_int(seed, S_NCAND, median, sigma, clip[0], clip[1], R)
    lcb = make_lcb("chain_lcb", counts, 512, 128, 128, 128, 128, seed, "bf16")
    lengths = uniform_int(seed, S_LSEQ, Llo, Lhi, R)
    soff = counts_to_offsets(lengths)
    L = int(soff[-1])
    n_in = lcb.o_c * lcb.d
    ci = ChainInputs(
        name="chain", lcb=lcb, w_q=normal(seed, S_WQ, (H * dh, n_in), 1.0 / math.sqrt(n_in)),
        seq_off=soff, H=H, dh=dh, scale=1.0 / math.sqrt(dh),
        k_t=normal(seed, S_K, (L, H, dh)), v_t=normal(seed, S_V, (L, H, dh)),
    )
    ci.recipe = (f"R={R}, N_r~round(lognormal(ln {median:g}, {sigma:g})) clipped {clip}; LCB n_r=512, n_c=128, d=128, "
                 f"o_r=o_c=128; W_q [{H*dh}x{n_in}] ~N(0,1/{n_in}); DCA H={H}, dh={dh}, q=1, L_r~U{{{Llo}..{Lhi}}}")
    return ci


@dataclass
class DcaBlockInputs:
    """Inputs of the DCA block (section 3.2, Eq. (13), both query groups)."""
    name: str
    cand_off: np.ndarray
    seq_off: np.ndarray
    q: int
    q_req: int
    H: int
    dh: int
    scale: float
    s_seq: np.ndarray  # uint16 [T, d_s] request sequence representation
    w_kv: np.ndarray  # uint16 [4*H*dh, d_s]: W_K^C, W_V^C, W_K^R, W_V^R stacked
    q_c: np.ndarray  # uint16 [C*q, H, dh]
    q_r: np.ndarray  # uint16 [R*q_req, H, dh]
    recipe: str = ""

    @property
    def R(self):
        return len(self.cand_off) - 1

    @property
    def C(self):
        return int(self.cand_off[-1])

    def weights(self):
        n = self.H * self.dh
        return [self.w_kv[k * n:(k + 1) * n] for k in range(4)]


def make_dca_block(name, counts, lengths, q, q_req, H, dh, d_s, seed) -> DcaBlockInputs:
    """S ~ N(0,1); projection weights ~ N(0, 1/d_s); queries ~ N(0,1)."""
    coff, soff = counts_to_offsets(counts), counts_to_offsets(lengths)
    R, C, T = len(counts), int(coff[-1]), int(soff[-1])
    return DcaBlockInputs(name=name, cand_off=coff, seq_off=soff, q=q, q_req=q_req, H=H, dh=dh,
                          scale=1.0 / math.sqrt(dh), s_seq=normal(seed, S_SEQ, (T, d_s)),
                          w_kv=normal(seed, S_WKV, (4 * H * dh, d_s), 1.0 / math.sqrt(d_s)),
                          q_c=normal(seed, S_Q, (C * q, H, dh)), q_r=normal(seed, S_QREQ, (R * q_req, H, dh)))


def dca_block(seed: int = 6, R: int = 8, lo: int = 4096, hi: int = 8192, H: int = 4, dh: int = 128, d_s: int = 256,
              n_cand: int = 2048, q: int = 4, q_req: int = 64) -> DcaBlockInputs:
    lengths = uniform_int(seed, S_LSEQ, lo, hi, R)
    x = make_dca_block("dca_block", [n_cand] * R, lengths, q, q_req, H, dh, d_s, seed)
    x.recipe = (f"R={R}, L_r~U{{{lo}..{hi}}}, d_s={d_s}, H={H}, dh={dh}, N_r={n_cand}, q={q}, request queries "
                f"q_req={q_req}; S,Q~N(0,1), W~N(0,1/d_s)")
    return x


# ---- LCB block: the LCB with per-group bias / residual / norm / activation --------------
@dataclass
class Epilogue:
    """One output group's epilogue parameters (section 3.1.2 Eq. 4 bias, section 3.1.3 Eq. 7-8).

    ``bias [o]`` fp32 per output row; ``residual`` bf16 bits with the group's output shape;
    ``gamma / beta [d]`` fp32; ``norm`` in {"none", "layernorm", "rmsnorm"}; ``act`` in
    {"none", "relu", "silu", "gelu"}.  Any array may be None (no bias / residual, gamma 1, beta 0).
    """
    bias: np.ndarray | None = None
    residual: np.ndarray | None = None
    gamma: np.ndarray | None = None
    beta: np.ndarray | None = None
    eps: float = 1e-5
    norm: str = "none"
    act: str = "none"


@dataclass
class LcbBlockInputs:
    name: str
    lcb: LcbInputs
    epi_r: Epilogue
    epi_c: Epilogue
    recipe: str = ""


def make_epilogue(seed: int, group_stream: int, o: int, d: int, rows: int, norm: str, act: str,
                  bias: bool = True, residual: bool = True, affine: bool = True, eps: float = 1e-5) -> Epilogue:
    """bias ~ N(0, 0.5^2); gamma ~ 1 + N(0, 0.1^2); beta ~ N(0, 0.1^2) (fp32); residual ~ N(0,1) bf16 [rows, o, d]."""
    g = group_stream
    return Epilogue(
        bias=normal(seed, g + E_BIAS, (o,), 0.5, "f32") if bias else None,
        residual=normal(seed, g + E_RES, (rows, o, d)) if residual else None,
        gamma=(1.0 + normal(seed, g + E_GAMMA, (d,), 0.1, "f32")).astype(np.float32) if affine else None,
        beta=normal(seed, g + E_BETA, (d,), 0.1, "f32") if affine else None,
        eps=eps, norm=norm, act=act)


def make_lcb_block(name, counts, n_r, n_c, d, o_r, o_c, seed, norm="layernorm", act="silu", residual=True,
                   norm_r=None, act_r=None) -> LcbBlockInputs:
    lcb = make_lcb(name, counts, n_r, n_c, d, o_r, o_c, seed, "bf16")
    R, C = lcb.R, lcb.C
    return LcbBlockInputs(
        name=name, lcb=lcb,
        epi_r=make_epilogue(seed, S_EPI_R, o_r, d, R, norm_r or norm, act_r or act, residual=residual),
        epi_c=make_epilogue(seed, S_EPI_C, o_c, d, C, norm, act, residual=residual))


def lcb_block(seed: int = 7, R: int = 64, lo: int = 256, hi: int = 1024, residual: bool = True) -> LcbBlockInputs:
    counts = uniform_int(seed, S_NCAND, lo, hi, R)
    x = make_lcb_block("lcb_block", counts, 256, 64, 128, 128, 128, seed, "layernorm", "silu", residual)
    x.recipe = (f"LCB as lcb_bf16 (R={R}, N_r~U{{{lo}..{hi}}}; n_r=256, n_c=64, d=128, o_r=o_c=128) with, per "
                f"group, bias~N(0,0.25), {'residual~N(0,1) bf16, ' if residual else ''}LayerNorm over d "
                f"(gamma~1+N(0,0.01), beta~N(0,0.01), eps 1e-5), SiLU; seed {seed}")
    return x


# ---- masked FM (section 3.1.4, Eq. 10) -------------------------------------------------
@dataclass
class FmInputs:
    name: str
    cand_off: np.ndarray
    n_r: int
    n_c: int
    d: int
    x_req: np.ndarray  # uint16 [R, n_r, d]
    x_cand: np.ndarray  # uint16 [C, n_c, d]
    recipe: str = ""

    @property
    def R(self):
        return len(self.cand_off) - 1

    @property
    def C(self):
        return int(self.cand_off[-1])


def make_fm(name, counts, n_r, n_c, d, seed, std=None) -> FmInputs:
    """Embeddings ~ N(0, std^2) in bf16 (std = d^-1/4 keeps the Gram entries O(1))."""
    off = counts_to_offsets(counts)
    R, C = len(counts), int(off[-1])
    s = float(std if std is not None else d ** -0.25)
    return FmInputs(name=name, cand_off=off, n_r=n_r, n_c=n_c, d=d,
                    x_req=normal(seed, S_XREQ, (R, n_r, d), s), x_cand=normal(seed, S_XCAND, (C, n_c, d), s))


def fm_bf16(seed: int = 8, R: int = 64, lo: int = 256, hi: int = 1024, n_r: int = 250, n_c: int = 64,
            d: int = 128) -> FmInputs:
    counts = uniform_int(seed, S_NCAND, lo, hi, R)
    x = make_fm("fm_bf16", counts, n_r, n_c, d, seed)
    x.recipe = (f"R={R}, N_r~U{{{lo}..{hi}}}; n_r={n_r}, n_c={n_c}, d={d}; X~N(0, d^-1/2) bf16; output rows "
                f"n_r+n_c={n_r + n_c} padded to 16-byte multiples; seed {seed}")
    return x
