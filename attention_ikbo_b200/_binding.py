"""ctypes marshalling for ``librocs_ikbo.so`` (see ``include/rocs_ikbo.h`` for the contract)."""
from __future__ import annotations

import ctypes
import functools
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "librocs_ikbo.so")

ROCS_F32, ROCS_BF16 = 0, 1
STATUS_NAMES = {0: "ROCS_OK", 1: "ROCS_ERR_INVALID_ARG", 2: "ROCS_ERR_BAD_OFFSETS", 3: "ROCS_ERR_UNSUPPORTED",
                4: "ROCS_ERR_CUDA", 5: "ROCS_ERR_TIMEOUT", 6: "ROCS_ERR_WORKSPACE", 7: "ROCS_ERR_DEVICE_INDEX"}

_i64, _i32, _vp, _f32, _sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t


class RocsError(RuntimeError):
    def __init__(self, code, what=""):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


class LcbArgs(ctypes.Structure):
    _fields_ = [("R", _i64), ("n_r", _i64), ("n_c", _i64), ("d", _i64), ("o_r", _i64), ("o_c", _i64),
                ("dtype", _i32), ("cand_off_dev", _vp), ("cand_off_host", _vp), ("x_req", _vp), ("x_cand", _vp),
                ("w_rr", _vp), ("w_cr", _vp), ("w_cc", _vp), ("y_req", _vp), ("y_cand", _vp),
                ("workspace", _vp), ("workspace_bytes", _sz)]


class LcbEpilogue(ctypes.Structure):
    _fields_ = [("bias", _vp), ("residual", _vp), ("gamma", _vp), ("beta", _vp), ("eps", _f32),
                ("norm", _i32), ("act", _i32)]


NORMS = {"none": 0, "layernorm": 1, "rmsnorm": 2}
ACTS = {"none": 0, "relu": 1, "silu": 2, "gelu": 3}


class FmArgs(ctypes.Structure):
    _fields_ = [("R", _i64), ("n_r", _i64), ("n_c", _i64), ("d", _i64), ("cand_off_dev", _vp),
                ("cand_off_host", _vp), ("x_req", _vp), ("x_cand", _vp), ("y_req", _vp), ("y_cand", _vp),
                ("ld_req", _i64), ("ld_cand", _i64), ("workspace", _vp), ("workspace_bytes", _sz)]


class ChainWeightsArgs(ctypes.Structure):
    _fields_ = [("n_out", _i64), ("o_r", _i64), ("o_c", _i64), ("n_r", _i64), ("n_c", _i64), ("d", _i64),
                ("w_q", _vp), ("w_rr", _vp), ("w_cr", _vp), ("w_cc", _vp), ("w_fold", _vp), ("w_rs", _vp)]


class ChainSplitArgs(ctypes.Structure):
    _fields_ = [("R", _i64), ("n_r", _i64), ("n_c", _i64), ("d", _i64), ("o_r", _i64), ("o_c", _i64),
                ("n_out", _i64), ("cand_off_dev", _vp), ("cand_off_host", _vp), ("x_req", _vp), ("x_cand", _vp),
                ("w_rs", _vp), ("w_q", _vp), ("w_fold", _vp), ("y_req", _vp), ("q", _vp), ("workspace", _vp),
                ("workspace_bytes", _sz)]


class DcaArgs(ctypes.Structure):
    _fields_ = [("R", _i64), ("q", _i64), ("H", _i64), ("dh", _i64), ("scale", _f32),
                ("cand_off_dev", _vp), ("cand_off_host", _vp), ("seq_off_dev", _vp), ("seq_off_host", _vp),
                ("q_ptr", _vp), ("k_ptr", _vp), ("v_ptr", _vp), ("o_ptr", _vp), ("lse_ptr", _vp),
                ("workspace", _vp), ("workspace_bytes", _sz), ("kv_ld", _i64)]


class DcaBlockArgs(ctypes.Structure):
    _fields_ = [("R", _i64), ("q", _i64), ("q_req", _i64), ("H", _i64), ("dh", _i64), ("d_s", _i64),
                ("scale", _f32), ("cand_off_dev", _vp), ("cand_off_host", _vp), ("seq_off_dev", _vp),
                ("seq_off_host", _vp), ("s_seq", _vp), ("w_kv", _vp), ("q_c", _vp), ("q_r", _vp),
                ("o_c", _vp), ("lse_c", _vp), ("o_r", _vp), ("lse_r", _vp), ("workspace", _vp),
                ("workspace_bytes", _sz)]


class ProjArgs(ctypes.Structure):
    _fields_ = [("M", _i64), ("N", _i64), ("K", _i64), ("in_", _vp), ("w", _vp), ("out", _vp),
                ("workspace", _vp), ("workspace_bytes", _sz)]


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the native library; raises if it has not been built (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m attention_ikbo_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.POINTER
        for name, argt in [("rocs_lcb_workspace_size", [P(LcbArgs)]), ("rocs_lcb_expand_workspace_size", [P(LcbArgs)]),
                           ("rocs_dca_workspace_size", [P(DcaArgs)]), ("rocs_proj_workspace_size", [P(ProjArgs)]),
                           ("rocs_dca_expand_workspace_size", [P(DcaArgs), _i64]),
                           ("rocs_dca_block_workspace_size", [P(DcaBlockArgs)]),
                           ("rocs_fm_workspace_size", [P(FmArgs)]),
                           ("rocs_chain_split_workspace_size", [P(ChainSplitArgs)])]:
            getattr(lib, name).restype = _sz
            getattr(lib, name).argtypes = argt
        for name, argt in [("rocs_lcb_forward", [P(LcbArgs), _vp]), ("rocs_lcb_forward_expand", [P(LcbArgs), _vp]),
                           ("rocs_lcb_forward_noalloc", [P(LcbArgs), _vp]),
                           ("rocs_lcb_block_forward", [P(LcbArgs), P(LcbEpilogue), P(LcbEpilogue), _vp]),
                           ("rocs_lcb_forward_fault_injection", [P(LcbArgs), _vp, _i64, _i64]),
                           ("rocs_lcb_block_forward_fault_injection",
                            [P(LcbArgs), P(LcbEpilogue), P(LcbEpilogue), _vp, _i64, _i64]),
                           ("rocs_dca_forward", [P(DcaArgs), _vp]), ("rocs_proj_forward", [P(ProjArgs), _vp]),
                           ("rocs_dca_forward_expand", [P(DcaArgs), _i64, _vp]),
                           ("rocs_dca_block_forward", [P(DcaBlockArgs), _vp]),
                           ("rocs_fm_forward", [P(FmArgs), _vp]),
                           ("rocs_chain_prepare_weights", [P(ChainWeightsArgs), _vp]),
                           ("rocs_chain_split_forward", [P(ChainSplitArgs), _vp]),
                           ("rocs_pad_cols", [_vp, _i64, _i64, _i64, _vp, _i64, _i64, _vp]),
                           ("rocs_read_status", [_vp, _vp, P(_i32), P(_i32)]),
                           ("rocs_lcb_noalloc_read_status", [_vp, P(_i32), P(_i32)])]:
            getattr(lib, name).restype = ctypes.c_int
            getattr(lib, name).argtypes = argt
        for name, argt in [("rocs_lcb_host_staging_size", [P(LcbArgs), _i64]),
                           ("rocs_dca_host_staging_size", [P(DcaArgs), _i64])]:
            getattr(lib, name).restype = _sz
            getattr(lib, name).argtypes = argt
        lib.rocs_lcb_forward_host.restype = ctypes.c_int
        lib.rocs_lcb_forward_host.argtypes = [P(LcbArgs), _i64, _vp, _sz, _vp]
        lib.rocs_dca_forward_host.restype = ctypes.c_int
        lib.rocs_dca_forward_host.argtypes = [P(DcaArgs), _i64, _vp, _sz, _vp]
        lib.rocs_align_cols.restype = _i64
        lib.rocs_align_cols.argtypes = [_i64, _i64]
        lib.rocs_status_string.restype = ctypes.c_char_p
        lib.rocs_status_string.argtypes = [ctypes.c_int]
        lib.rocs_last_launch_count.restype = ctypes.c_int
        _lib = lib
    return _lib


def last_launch_count() -> int:
    """Kernel launches enqueued by the last successful forward call on this thread."""
    return int(load_library().rocs_last_launch_count())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _on_tensor_device(fn):
    """Run ``fn`` with the device of its first CUDA tensor argument current (else the ``device``
    keyword's, else the current device), so that the library's per-device state (SM count, kernel
    attributes, the no-alloc scratch array) and the default stream belong to the device the data is on."""
    @functools.wraps(fn)
    def run(*args, **kw):
        for t in list(args) + list(kw.values()):
            if isinstance(t, torch.Tensor) and t.is_cuda:
                with torch.cuda.device(t.device):
                    return fn(*args, **kw)
        if kw.get("device") is not None and torch.device(kw["device"]).index is not None:
            with torch.cuda.device(torch.device(kw["device"])):
                return fn(*args, **kw)
        return fn(*args, **kw)
    return run


def offsets(off, device="cuda"):
    """CSR offsets as the pair the C ABI needs: (device int32 tensor, host int32 numpy array).

    Pass the returned pair back into the forward functions to avoid a host<->device copy per call.
    """
    return _offsets(off, torch.device(device))


def _offsets(off, device):
    """(device int32 tensor, host int32 numpy array) from a pair, a tensor, an array or a list."""
    if isinstance(off, tuple) and len(off) == 2:
        return off
    if isinstance(off, torch.Tensor):
        host = off.detach().to("cpu", torch.int32).contiguous().numpy()
        dev = off if (off.is_cuda and off.dtype == torch.int32 and off.is_contiguous()) else \
            torch.from_numpy(host).to(device)
    else:
        host = np.ascontiguousarray(np.asarray(off, dtype=np.int32))
        dev = torch.from_numpy(host).to(device)
    return dev, host


def _check(rc, what):
    if rc != 0:
        raise RocsError(rc, what)


def _workspace(nbytes, device, given):
    if given is not None:
        if given.numel() * given.element_size() < nbytes:
            raise RocsError(6, "workspace")
        return given
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _lcb_args(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, y_req, y_cand):
    dev = x_req.device
    dtype = {torch.float32: ROCS_F32, torch.bfloat16: ROCS_BF16}[x_req.dtype]
    off_d, off_h = _offsets(cand_off, dev)
    R, n_r, d = x_req.shape
    C = int(off_h[-1])
    n_c, o_r, o_c = x_cand.shape[1] if x_cand.dim() == 3 else w_cc.shape[1], w_rr.shape[0], w_cc.shape[0]
    if y_req is None:
        y_req = torch.empty((R, o_r, d), dtype=x_req.dtype, device=dev)
    if y_cand is None:
        y_cand = torch.empty((C, o_c, d), dtype=x_req.dtype, device=dev)
    for t in (x_req, x_cand, w_rr, w_cr, w_cc, y_req, y_cand):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == x_req.dtype):
            raise RocsError(1, "LCB tensors must be contiguous CUDA tensors of one dtype")
    a = LcbArgs(R=R, n_r=n_r, n_c=n_c, d=d, o_r=o_r, o_c=o_c, dtype=dtype,
                cand_off_dev=off_d.data_ptr(), cand_off_host=off_h.ctypes.data,
                x_req=x_req.data_ptr(), x_cand=x_cand.data_ptr() if C else None, w_rr=w_rr.data_ptr(),
                w_cr=w_cr.data_ptr(), w_cc=w_cc.data_ptr(), y_req=y_req.data_ptr(),
                y_cand=y_cand.data_ptr() if C else None)
    return a, (off_d, off_h), y_req, y_cand


@_on_tensor_device
def rocs_lcb_forward(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, y_req=None, y_cand=None, workspace=None,
                     stream=None, expand=False):
    """IKBO-LCB.  Returns ``(y_req [R,o_r,d], y_cand [C,o_c,d])``; see ``rocs_lcb_forward`` in the header.

    ``expand=True`` runs the explicit-expand ablation (``rocs_lcb_forward_expand``) instead.
    """
    lib = load_library()
    a, keep, y_req, y_cand = _lcb_args(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, y_req, y_cand)
    size_fn = lib.rocs_lcb_expand_workspace_size if expand else lib.rocs_lcb_workspace_size
    nbytes = size_fn(ctypes.byref(a))
    if nbytes == 0:
        _check(lib.rocs_lcb_forward(ctypes.byref(a), _stream(stream)), "rocs_lcb_forward")  # reports the reason
    ws = _workspace(nbytes, x_req.device, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    fn = lib.rocs_lcb_forward_expand if expand else lib.rocs_lcb_forward
    _check(fn(ctypes.byref(a), _stream(stream)), fn.__name__)
    rocs_lcb_forward.last_workspace = ws
    return y_req, y_cand


def rocs_lcb_forward_noalloc(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, y_req, y_cand, stream=None):
    """IKBO-LCB without a workspace, for callers that cannot allocate device memory.

    Uses the library's fixed device scratch array instead of a workspace (see the header for its
    size limit and for why concurrent calls on one device must be serialised).  ``y_req`` and
    ``y_cand`` must be given: this call allocates nothing.  ``cand_off`` should be the pair from
    ``offsets()`` so that no offsets tensor is created either.  The call runs with the device of
    ``x_req`` current, so the scratch array it uses is that device's.  Read its device status with
    ``rocs_lcb_noalloc_read_status``.
    """
    if y_req is None or y_cand is None:
        raise RocsError(1, "rocs_lcb_forward_noalloc: y_req and y_cand must be given (this call allocates nothing)")
    lib = load_library()
    with torch.cuda.device(x_req.device):
        a, keep, y_req, y_cand = _lcb_args(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, y_req, y_cand)
        _check(lib.rocs_lcb_forward_noalloc(ctypes.byref(a), _stream(stream)), "rocs_lcb_forward_noalloc")
    return y_req, y_cand


def rocs_lcb_noalloc_read_status(device=None, stream=None):
    """Synchronise the stream and return ``(device_code, detail)`` of the last no-alloc LCB call on
    ``device`` (default: the current device)."""
    lib = load_library()
    code, detail = ctypes.c_int32(0), ctypes.c_int32(0)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        _check(lib.rocs_lcb_noalloc_read_status(_stream(stream), ctypes.byref(code), ctypes.byref(detail)),
               "rocs_lcb_noalloc_read_status")
    return code.value, detail.value


@_on_tensor_device
def rocs_lcb_forward_fault_injection(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, skip_release_request,
                                     wait_limit_ns, stream=None):
    """Test hook: LCB whose request ``skip_release_request`` never signals its Z; the kernel must end
    with ROCS_ERR_TIMEOUT after ``wait_limit_ns``.  Returns the workspace (read it with rocs_read_status)."""
    lib = load_library()
    a, keep, y_req, y_cand = _lcb_args(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, None, None)
    ws = _workspace(lib.rocs_lcb_workspace_size(ctypes.byref(a)), x_req.device, None)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib.rocs_lcb_forward_fault_injection(ctypes.byref(a), _stream(stream), int(skip_release_request),
                                                int(wait_limit_ns)), "rocs_lcb_forward_fault_injection")
    return ws


def _epilogue(e, y_shape, dev, keep):
    """``e``: dict with optional bias [o] / gamma [d] / beta [d] (fp32), residual (bf16, output shape),
    eps, norm ("none" | "layernorm" | "rmsnorm"), act ("none" | "relu" | "silu" | "gelu"); or None."""
    if e is None:
        return None
    def t(name, dtype, shape=None):
        v = e.get(name)
        if v is None:
            return None
        if not (isinstance(v, torch.Tensor) and v.is_cuda and v.is_contiguous() and v.dtype == dtype):
            raise RocsError(1, f"epilogue {name} must be a contiguous CUDA {dtype} tensor")
        if shape is not None and tuple(v.shape) != tuple(shape):
            raise RocsError(1, f"epilogue {name} has shape {tuple(v.shape)}, expected {tuple(shape)}")
        keep.append(v)
        return v.data_ptr()
    norm, act = e.get("norm", "none"), e.get("act", "none")
    return LcbEpilogue(bias=t("bias", torch.float32, (y_shape[1],)),
                       residual=t("residual", torch.bfloat16, y_shape),
                       gamma=t("gamma", torch.float32, (y_shape[2],)), beta=t("beta", torch.float32, (y_shape[2],)),
                       eps=float(e.get("eps", 1e-5)), norm=NORMS[norm] if isinstance(norm, str) else int(norm),
                       act=ACTS[act] if isinstance(act, str) else int(act))


@_on_tensor_device
def rocs_lcb_block_forward(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, epi_req=None, epi_cand=None, y_req=None,
                           y_cand=None, workspace=None, stream=None):
    """LCB block: IKBO-LCB with each group's bias / residual / norm / activation fused into the epilogue.

    ``epi_req`` / ``epi_cand``: see :func:`_epilogue`.  Returns ``(y_req, y_cand)``.
    """
    lib = load_library()
    a, keep, y_req, y_cand = _lcb_args(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, y_req, y_cand)
    hold = []
    er = _epilogue(epi_req, tuple(y_req.shape), x_req.device, hold)
    ec = _epilogue(epi_cand, tuple(y_cand.shape), x_req.device, hold)
    nbytes = lib.rocs_lcb_workspace_size(ctypes.byref(a))
    ws = _workspace(nbytes, x_req.device, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib.rocs_lcb_block_forward(ctypes.byref(a), None if er is None else ctypes.byref(er),
                                      None if ec is None else ctypes.byref(ec), _stream(stream)),
           "rocs_lcb_block_forward")
    rocs_lcb_block_forward.last_workspace = ws
    return y_req, y_cand


@_on_tensor_device
def rocs_lcb_block_forward_fault_injection(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, epi_req, epi_cand,
                                           skip_release_request, wait_limit_ns, stream=None):
    """Test hook: LCB block whose request ``skip_release_request`` never signals its Z; the kernel must
    end with ROCS_ERR_TIMEOUT after ``wait_limit_ns``.  Returns the workspace (read it with rocs_read_status)."""
    lib = load_library()
    a, keep, y_req, y_cand = _lcb_args(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, None, None)
    hold = []
    er = _epilogue(epi_req, tuple(y_req.shape), x_req.device, hold)
    ec = _epilogue(epi_cand, tuple(y_cand.shape), x_req.device, hold)
    ws = _workspace(lib.rocs_lcb_workspace_size(ctypes.byref(a)), x_req.device, None)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib.rocs_lcb_block_forward_fault_injection(
        ctypes.byref(a), None if er is None else ctypes.byref(er), None if ec is None else ctypes.byref(ec),
        _stream(stream), int(skip_release_request), int(wait_limit_ns)), "rocs_lcb_block_forward_fault_injection")
    return ws


def rocs_lcb_forward_expand(*args, **kw):
    return rocs_lcb_forward(*args, expand=True, **kw)


def _dca_args(q_t, k_t, v_t, cand_off, seq_off, q_tokens, scale, o, lse):
    dev = q_t.device
    co_d, co_h = _offsets(cand_off, dev)
    so_d, so_h = _offsets(seq_off, dev)
    R = len(co_h) - 1
    H, dh = k_t.shape[1], k_t.shape[2]
    if o is None:
        o = torch.empty(q_t.shape, dtype=torch.bfloat16, device=dev)
    if lse is True:
        lse = torch.empty(q_t.shape[:2], dtype=torch.float32, device=dev)
    elif lse is False:
        lse = None
    for t in (q_t, k_t, v_t, o):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16):
            raise RocsError(1, "DCA tensors must be contiguous bf16 CUDA tensors")
    a = DcaArgs(R=R, q=q_tokens, H=H, dh=dh, scale=float(scale),
                cand_off_dev=co_d.data_ptr(), cand_off_host=co_h.ctypes.data,
                seq_off_dev=so_d.data_ptr(), seq_off_host=so_h.ctypes.data,
                q_ptr=q_t.data_ptr() if q_t.numel() else None, k_ptr=k_t.data_ptr() if k_t.numel() else None,
                v_ptr=v_t.data_ptr() if v_t.numel() else None, o_ptr=o.data_ptr() if o.numel() else None,
                lse_ptr=lse.data_ptr() if lse is not None else None)
    return a, (co_d, co_h, so_d, so_h), o, lse


@_on_tensor_device
def rocs_dca_forward(q_t, k_t, v_t, cand_off, seq_off, q_tokens, scale, o=None, lse=True, workspace=None,
                     stream=None, expand_chunk=None):
    """IKBO-DCA.  Returns ``(o [C*q,H,dh], lse [C*q,H] or None)``.

    ``expand_chunk=n`` runs the explicit-expand ablation with chunks of n candidates.
    """
    lib = load_library()
    a, keep, o, lse = _dca_args(q_t, k_t, v_t, cand_off, seq_off, q_tokens, scale, o, lse)
    if expand_chunk:
        nbytes = lib.rocs_dca_expand_workspace_size(ctypes.byref(a), int(expand_chunk))
    else:
        nbytes = lib.rocs_dca_workspace_size(ctypes.byref(a))
    if nbytes == 0:
        _check(lib.rocs_dca_forward(ctypes.byref(a), _stream(stream)), "rocs_dca_forward")
    ws = _workspace(nbytes, q_t.device, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    if expand_chunk:
        _check(lib.rocs_dca_forward_expand(ctypes.byref(a), int(expand_chunk), _stream(stream)),
               "rocs_dca_forward_expand")
    else:
        _check(lib.rocs_dca_forward(ctypes.byref(a), _stream(stream)), "rocs_dca_forward")
    rocs_dca_forward.last_workspace = ws
    return o, lse


def rocs_dca_forward_expand(*args, expand_chunk=1024, **kw):
    return rocs_dca_forward(*args, expand_chunk=expand_chunk, **kw)


@_on_tensor_device
def rocs_dca_block_forward(s_seq, w_kv, q_c, q_r, cand_off, seq_off, q_tokens, q_req_tokens, scale, o_c=None,
                           o_r=None, lse=True, workspace=None, stream=None):
    """DCA block (both query groups of Eq. 13): K/V projected once per request with the stacked
    weights ``w_kv = [W_K^C; W_V^C; W_K^R; W_V^R]``, then IKBO-DCA for the candidates and attention of
    every request's own ``q_req_tokens`` queries.  Returns ``(o_c, lse_c, o_r, lse_r)``."""
    lib = load_library()
    dev = q_c.device
    co_d, co_h = _offsets(cand_off, dev)
    so_d, so_h = _offsets(seq_off, dev)
    R = len(co_h) - 1
    H, dh = q_c.shape[1], q_c.shape[2]
    o_c = torch.empty(q_c.shape, dtype=torch.bfloat16, device=dev) if o_c is None else o_c
    o_r = torch.empty(q_r.shape, dtype=torch.bfloat16, device=dev) if o_r is None else o_r
    lse_c = torch.empty(q_c.shape[:2], dtype=torch.float32, device=dev) if lse else None
    lse_r = torch.empty(q_r.shape[:2], dtype=torch.float32, device=dev) if lse else None
    for t in (s_seq, w_kv, q_c, q_r, o_c, o_r):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16):
            raise RocsError(1, "DCA block tensors must be contiguous bf16 CUDA tensors")
    a = DcaBlockArgs(R=R, q=q_tokens, q_req=q_req_tokens, H=H, dh=dh, d_s=s_seq.shape[1], scale=float(scale),
                     cand_off_dev=co_d.data_ptr(), cand_off_host=co_h.ctypes.data, seq_off_dev=so_d.data_ptr(),
                     seq_off_host=so_h.ctypes.data, s_seq=s_seq.data_ptr() if s_seq.numel() else None,
                     w_kv=w_kv.data_ptr(), q_c=q_c.data_ptr() if q_c.numel() else None, q_r=q_r.data_ptr(),
                     o_c=o_c.data_ptr() if o_c.numel() else None, o_r=o_r.data_ptr(),
                     lse_c=lse_c.data_ptr() if lse_c is not None and lse_c.numel() else None,
                     lse_r=lse_r.data_ptr() if lse_r is not None else None)
    nbytes = lib.rocs_dca_block_workspace_size(ctypes.byref(a))
    if nbytes == 0:
        _check(lib.rocs_dca_block_forward(ctypes.byref(a), _stream(stream)), "rocs_dca_block_forward")
    ws = _workspace(nbytes, dev, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib.rocs_dca_block_forward(ctypes.byref(a), _stream(stream)), "rocs_dca_block_forward")
    rocs_dca_block_forward.last_workspace = ws
    return o_c, lse_c, o_r, lse_r


@_on_tensor_device
def rocs_proj_forward(inp, w, out=None, workspace=None, stream=None):
    """``out[M, N] = inp[M, K] . w[N, K]^T`` (bf16)."""
    lib = load_library()
    M, K = inp.shape[0], int(np.prod(inp.shape[1:]))
    N = w.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=inp.device)
    for t in (inp, w, out):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16):
            raise RocsError(1, "projection tensors must be contiguous bf16 CUDA tensors")
    a = ProjArgs(M=M, N=N, K=K, in_=inp.data_ptr() if M else None, w=w.data_ptr(), out=out.data_ptr() if M else None)
    ws = _workspace(lib.rocs_proj_workspace_size(ctypes.byref(a)), inp.device, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib.rocs_proj_forward(ctypes.byref(a), _stream(stream)), "rocs_proj_forward")
    rocs_proj_forward.last_workspace = ws
    return out


@_on_tensor_device
def rocs_read_status(workspace, stream=None):
    """Synchronise the stream and return ``(device_code, detail)`` of a workspace."""
    lib = load_library()
    code, detail = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(lib.rocs_read_status(_ptr(workspace), _stream(stream), ctypes.byref(code), ctypes.byref(detail)),
           "rocs_read_status")
    return code.value, detail.value


def chain_forward(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, w_q, k_t, v_t, seq_off, heads, head_dim, scale,
                  stream=None, workspaces=None):
    """Chained block: IKBO-LCB -> query projection -> IKBO-DCA (one query token per candidate).

    Returns ``(y_req, y_cand, q, o, lse)``.  Three C-ABI calls on one stream; intermediates stay bf16 in HBM.
    """
    ws = workspaces or {}
    y_req, y_cand = rocs_lcb_forward(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, workspace=ws.get("lcb"),
                                     stream=stream)
    C = y_cand.shape[0]
    q = rocs_proj_forward(y_cand.view(C, -1), w_q, workspace=ws.get("proj"), stream=stream)
    o, lse = rocs_dca_forward(q.view(C, heads, head_dim), k_t, v_t, cand_off, seq_off, 1, scale,
                              workspace=ws.get("dca"), stream=stream)
    return y_req, y_cand, q, o, lse


def rocs_align_cols(cols: int, elem_bytes: int) -> int:
    """Smallest n >= cols with n * elem_bytes a multiple of 16 (section 4.2.4 alignment)."""
    return int(load_library().rocs_align_cols(int(cols), int(elem_bytes)))


@_on_tensor_device
def rocs_pad_cols(src, ld_dst, dst=None, stream=None):
    """Copy the rows of ``src`` (last axis contiguous) into rows of ``ld_dst`` elements, zero-filling the
    tail (section 4.2.4).  With ``ld_dst`` smaller than the source's last axis the rows are cut instead."""
    lib = load_library()
    if not (src.is_cuda and src.is_contiguous()):
        raise RocsError(1, "rocs_pad_cols: src must be a contiguous CUDA tensor")
    cols = min(src.shape[-1], ld_dst)
    rows = src.numel() // src.shape[-1] if src.numel() else 0
    if dst is None:
        dst = torch.empty(tuple(src.shape[:-1]) + (ld_dst,), dtype=src.dtype, device=src.device)
    _check(lib.rocs_pad_cols(_ptr(src), rows, cols, src.shape[-1], _ptr(dst), ld_dst, src.element_size(),
                             _stream(stream)), "rocs_pad_cols")
    return dst


@_on_tensor_device
def rocs_fm_forward(x_req, x_cand, cand_off, y_req=None, y_cand=None, ld_req=0, ld_cand=0, workspace=None,
                    stream=None):
    """IKBO masked FM (Eq. 10).  Returns ``(y_req [R, n_r, ld_req], y_cand [C, n_c, ld_cand])``: the outputs
    in their first n_r / n_r + n_c columns, zeros in the padding (ld 0 = the aligned default)."""
    lib = load_library()
    dev = x_req.device
    off_d, off_h = _offsets(cand_off, dev)
    R, n_r, d = x_req.shape
    C = int(off_h[-1])
    n_c = x_cand.shape[1]
    ld_r = ld_req or rocs_align_cols(n_r, 2)
    ld_c = ld_cand or rocs_align_cols(n_r + n_c, 2)
    if y_req is None:
        y_req = torch.empty((R, n_r, ld_r), dtype=torch.bfloat16, device=dev)
    if y_cand is None:
        y_cand = torch.empty((C, n_c, ld_c), dtype=torch.bfloat16, device=dev)
    for t in (x_req, x_cand, y_req, y_cand):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16):
            raise RocsError(1, "FM tensors must be contiguous CUDA bf16 tensors")
    a = FmArgs(R=R, n_r=n_r, n_c=n_c, d=d, cand_off_dev=off_d.data_ptr(), cand_off_host=off_h.ctypes.data,
               x_req=x_req.data_ptr(), x_cand=x_cand.data_ptr() if C else None, y_req=y_req.data_ptr(),
               y_cand=y_cand.data_ptr() if C else None, ld_req=ld_r, ld_cand=ld_c)
    nbytes = lib.rocs_fm_workspace_size(ctypes.byref(a))
    if nbytes == 0:
        _check(lib.rocs_fm_forward(ctypes.byref(a), _stream(stream)), "rocs_fm_forward")
    ws = _workspace(nbytes, dev, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib.rocs_fm_forward(ctypes.byref(a), _stream(stream)), "rocs_fm_forward")
    rocs_fm_forward.last_workspace = ws
    return y_req, y_cand


@_on_tensor_device
def rocs_chain_prepare_weights(w_q, w_rr, w_cr, w_cc, d, stream=None):
    """Once per model: ``(w_fold [n_out, n_c*d], w_rs [o_r + o_c, n_r])`` for :func:`rocs_chain_split_forward`."""
    lib = load_library()
    for t in (w_q, w_rr, w_cr, w_cc):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16):
            raise RocsError(1, "chain weights must be contiguous CUDA bf16 tensors")
    n_out, (o_r, n_r), (o_c, n_c) = w_q.shape[0], w_rr.shape, w_cc.shape
    w_fold = torch.empty((n_out, n_c * d), dtype=torch.bfloat16, device=w_q.device)
    w_rs = torch.empty((o_r + o_c, n_r), dtype=torch.bfloat16, device=w_q.device)
    a = ChainWeightsArgs(n_out=n_out, o_r=o_r, o_c=o_c, n_r=n_r, n_c=n_c, d=d, w_q=w_q.data_ptr(),
                         w_rr=w_rr.data_ptr(), w_cr=w_cr.data_ptr(), w_cc=w_cc.data_ptr(), w_fold=w_fold.data_ptr(),
                         w_rs=w_rs.data_ptr())
    _check(lib.rocs_chain_prepare_weights(ctypes.byref(a), _stream(stream)), "rocs_chain_prepare_weights")
    return w_fold, w_rs


@_on_tensor_device
def rocs_chain_split_forward(x_req, x_cand, w_rs, w_q, w_fold, cand_off, o_r, y_req=None, q=None, workspace=None,
                             stream=None):
    """Split chain queries: ``(y_req [R, o_r + o_c, d] = [Y^R; Z], q [C, n_out])``; see the header."""
    lib = load_library()
    dev = x_req.device
    off_d, off_h = _offsets(cand_off, dev)
    R, n_r, d = x_req.shape
    C = int(off_h[-1])
    n_c = x_cand.shape[1]
    o_c = w_rs.shape[0] - o_r
    n_out = w_q.shape[0]
    if y_req is None:
        y_req = torch.empty((R, o_r + o_c, d), dtype=torch.bfloat16, device=dev)
    if q is None:
        q = torch.empty((C, n_out), dtype=torch.bfloat16, device=dev)
    for t in (x_req, x_cand, w_rs, w_q, w_fold, y_req, q):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16):
            raise RocsError(1, "split chain tensors must be contiguous CUDA bf16 tensors")
    a = ChainSplitArgs(R=R, n_r=n_r, n_c=n_c, d=d, o_r=o_r, o_c=o_c, n_out=n_out, cand_off_dev=off_d.data_ptr(),
                       cand_off_host=off_h.ctypes.data, x_req=x_req.data_ptr(),
                       x_cand=x_cand.data_ptr() if C else None, w_rs=w_rs.data_ptr(), w_q=w_q.data_ptr(),
                       w_fold=w_fold.data_ptr(), y_req=y_req.data_ptr(), q=q.data_ptr() if C else None)
    nbytes = lib.rocs_chain_split_workspace_size(ctypes.byref(a))
    if nbytes == 0:
        _check(lib.rocs_chain_split_forward(ctypes.byref(a), _stream(stream)), "rocs_chain_split_forward")
    ws = _workspace(nbytes, dev, workspace)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib.rocs_chain_split_forward(ctypes.byref(a), _stream(stream)), "rocs_chain_split_forward")
    rocs_chain_split_forward.last_workspace = ws
    return y_req, q


def chain_split_forward(x_req, x_cand, w_rs, w_q, w_fold, cand_off, o_r, k_t, v_t, seq_off, heads, head_dim, scale,
                        stream=None, workspaces=None):
    """Split chained block: queries from :func:`rocs_chain_split_forward` (Y^C never written), then IKBO-DCA.

    Returns ``(y_req, q, o, lse)``.
    """
    ws = workspaces or {}
    y_req, q = rocs_chain_split_forward(x_req, x_cand, w_rs, w_q, w_fold, cand_off, o_r, workspace=ws.get("split"),
                                        stream=stream)
    C = q.shape[0]
    o, lse = rocs_dca_forward(q.view(C, heads, head_dim), k_t, v_t, cand_off, seq_off, 1, scale,
                              workspace=ws.get("dca"), stream=stream)
    return y_req, q, o, lse


def _host_tensor(t, what):
    if t.is_cuda or not t.is_contiguous() or not t.is_pinned():
        raise RocsError(1, f"{what} must be a contiguous pinned host tensor")


@_on_tensor_device
def rocs_lcb_forward_host(x_req, x_cand, w_rr, w_cr, w_cc, cand_off, y_req=None, y_cand=None, chunks=8,
                          staging=None, stream=None):
    """IKBO-LCB on a host-resident batch: pinned host ``x_req``/``x_cand`` in, pinned host ``y_req``/``y_cand``
    out, device weights; copies and compute pipelined over request chunks (see the header)."""
    lib = load_library()
    dev = w_rr.device
    off_d, off_h = _offsets(cand_off, dev)
    R, n_r, d = x_req.shape
    C = int(off_h[-1])
    n_c, o_r, o_c = x_cand.shape[1], w_rr.shape[0], w_cc.shape[0]
    dt = x_req.dtype
    if y_req is None:
        y_req = torch.empty((R, o_r, d), dtype=dt, pin_memory=True)
    if y_cand is None:
        y_cand = torch.empty((C, o_c, d), dtype=dt, pin_memory=True)
    for t, n in ((x_req, "x_req"), (x_cand, "x_cand"), (y_req, "y_req"), (y_cand, "y_cand")):
        _host_tensor(t, n)
    for t in (w_rr, w_cr, w_cc):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == dt):
            raise RocsError(1, "LCB weights must be contiguous CUDA tensors of the batch dtype")
    a = LcbArgs(R=R, n_r=n_r, n_c=n_c, d=d, o_r=o_r, o_c=o_c, dtype={torch.float32: ROCS_F32, torch.bfloat16: ROCS_BF16}[dt],
                cand_off_dev=off_d.data_ptr(), cand_off_host=off_h.ctypes.data, x_req=x_req.data_ptr(),
                x_cand=x_cand.data_ptr() if C else None, w_rr=w_rr.data_ptr(), w_cr=w_cr.data_ptr(),
                w_cc=w_cc.data_ptr(), y_req=y_req.data_ptr(), y_cand=y_cand.data_ptr() if C else None)
    nbytes = lib.rocs_lcb_host_staging_size(ctypes.byref(a), int(chunks))
    if nbytes == 0:
        _check(lib.rocs_lcb_forward_host(ctypes.byref(a), int(chunks), None, 0, _stream(stream)), "rocs_lcb_forward_host")
    st = _workspace(nbytes, dev, staging)
    _check(lib.rocs_lcb_forward_host(ctypes.byref(a), int(chunks), _ptr(st), st.numel(), _stream(stream)),
           "rocs_lcb_forward_host")
    rocs_lcb_forward_host.last_staging = st
    rocs_lcb_forward_host.keep = (off_d, off_h)
    return y_req, y_cand


@_on_tensor_device
def rocs_dca_forward_host(q_t, k_t, v_t, cand_off, seq_off, q_tokens, scale, o=None, lse=True, device="cuda",
                          chunks=4, staging=None, stream=None):
    """IKBO-DCA on a host-resident batch: pinned host Q/K/V in, pinned host O (and LSE) out."""
    lib = load_library()
    dev = torch.device(device)
    co_d, co_h = _offsets(cand_off, dev)
    so_d, so_h = _offsets(seq_off, dev)
    R = len(co_h) - 1
    H, dh = k_t.shape[1], k_t.shape[2]
    if o is None:
        o = torch.empty(q_t.shape, dtype=torch.bfloat16, pin_memory=True)
    if lse is True:
        lse = torch.empty(q_t.shape[:2], dtype=torch.float32, pin_memory=True)
    elif lse is False:
        lse = None
    for t, n in ((q_t, "q"), (k_t, "k"), (v_t, "v"), (o, "o")) + (((lse, "lse"),) if lse is not None else ()):
        _host_tensor(t, n)
    a = DcaArgs(R=R, q=q_tokens, H=H, dh=dh, scale=float(scale), cand_off_dev=co_d.data_ptr(),
                cand_off_host=co_h.ctypes.data, seq_off_dev=so_d.data_ptr(), seq_off_host=so_h.ctypes.data,
                q_ptr=q_t.data_ptr() if q_t.numel() else None, k_ptr=k_t.data_ptr() if k_t.numel() else None,
                v_ptr=v_t.data_ptr() if v_t.numel() else None, o_ptr=o.data_ptr() if o.numel() else None,
                lse_ptr=lse.data_ptr() if lse is not None else None)
    nbytes = lib.rocs_dca_host_staging_size(ctypes.byref(a), int(chunks))
    if nbytes == 0:
        _check(lib.rocs_dca_forward_host(ctypes.byref(a), int(chunks), None, 0, _stream(stream)), "rocs_dca_forward_host")
    st = _workspace(nbytes, dev, staging)
    _check(lib.rocs_dca_forward_host(ctypes.byref(a), int(chunks), _ptr(st), st.numel(), _stream(stream)),
           "rocs_dca_forward_host")
    rocs_dca_forward_host.last_staging = st
    rocs_dca_forward_host.keep = (co_d, co_h, so_d, so_h)
    return o, lse
