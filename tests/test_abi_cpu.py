"""The C-ABI library without a GPU: it loads, exports every entry point the header declares,
and rejects malformed arguments on the host before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    from attention_ikbo_b200.build import build

    build()
    import attention_ikbo_b200 as m

    return m.load_library()


def declared_symbols():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        names.update(re.findall(r"ROCS_API\s+[\w\s\*]+?\b(rocs_\w+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    lib.rocs_status_string.restype = ctypes.c_char_p
    assert lib.rocs_status_string(0) == b"ROCS_OK"
    assert lib.rocs_status_string(5) == b"ROCS_ERR_TIMEOUT"


def _lcb_args(m, off, n_c=64, dtype=1, d=128, ws_bytes=0):
    off = np.asarray(off, np.int32)
    fake = 0x10000  # aligned non-null placeholders: validation fails before any dereference
    a = m._binding.LcbArgs(R=len(off) - 1, n_r=256, n_c=n_c, d=d, o_r=128, o_c=128, dtype=dtype,
                           cand_off_dev=fake, cand_off_host=off.ctypes.data, x_req=fake, x_cand=fake, w_rr=fake,
                           w_cr=fake, w_cc=fake, y_req=fake, y_cand=fake, workspace=fake if ws_bytes else None,
                           workspace_bytes=ws_bytes)
    return a, off


def test_lcb_host_validation(lib):
    import attention_ikbo_b200 as m

    a, keep = _lcb_args(m, [0, 3, 2, 6])
    assert lib.rocs_lcb_workspace_size(ctypes.byref(a)) == 0
    assert lib.rocs_lcb_forward(ctypes.byref(a), None) == 2  # ROCS_ERR_BAD_OFFSETS
    a, keep = _lcb_args(m, [1, 3])
    assert lib.rocs_lcb_forward(ctypes.byref(a), None) == 2
    a, keep = _lcb_args(m, [0, 3, 6], n_c=48)
    assert lib.rocs_lcb_forward(ctypes.byref(a), None) == 3  # ROCS_ERR_UNSUPPORTED (n_c)
    a, keep = _lcb_args(m, [0, 3, 6], d=100)
    assert lib.rocs_lcb_forward(ctypes.byref(a), None) == 3  # 200-byte rows break the 16-byte contract
    a, keep = _lcb_args(m, [0, 3, 6])
    need = lib.rocs_lcb_workspace_size(ctypes.byref(a))
    # header 256 + flags (2 ints, padded to 256) + Z 2 x 128 x 128 fp32
    assert need == 256 + 256 + 2 * 128 * 128 * 4
    a, keep = _lcb_args(m, [0, 3, 6], ws_bytes=need - 1)
    assert lib.rocs_lcb_forward(ctypes.byref(a), None) == 6  # ROCS_ERR_WORKSPACE
    a.x_req = 0x10008  # misaligned
    assert lib.rocs_lcb_forward(ctypes.byref(a), None) == 1


def test_dca_host_validation(lib):
    import attention_ikbo_b200 as m

    co = np.array([0, 2, 5], np.int32)
    so = np.array([0, 7, 6], np.int32)
    fake = 0x20000
    a = m._binding.DcaArgs(R=2, q=1, H=2, dh=128, scale=0.1, cand_off_dev=fake, cand_off_host=co.ctypes.data,
                           seq_off_dev=fake, seq_off_host=so.ctypes.data, q_ptr=fake, k_ptr=fake, v_ptr=fake,
                           o_ptr=fake, lse_ptr=None, workspace=None, workspace_bytes=0)
    assert lib.rocs_dca_forward(ctypes.byref(a), None) == 2
    so[2] = 9
    assert lib.rocs_dca_forward(ctypes.byref(a), None) == 6  # valid, but no workspace
    # 2 requests x 2 heads x ceil(rows/256) units = 4 units of 16 B after 256 + pad(3R+1 ints)
    assert lib.rocs_dca_workspace_size(ctypes.byref(a)) == 256 + 256 + 4 * 16
    a.dh = 96
    assert lib.rocs_dca_forward(ctypes.byref(a), None) == 3


def test_dca_workspace_counts_split_and_paired_units(lib):
    """Host logic of the DCA schedule, pinned through the workspace size (no GPU: the SM count falls back to
    148).  Units = H * ceil(q N_r / 256); when every request has the same number (>= 2) of K/V tiles the last
    (units mod 148) units are split in two (one more table entry each, plus 8 counters and a merge area of
    2 halves x 2 tiles x 4 warps x 32 rows x (dh + 2) fp32); at dh = 64 a request's last chunk of <= 128 rows
    is one unit per head pair."""
    import attention_ikbo_b200 as m

    fake = 0x20000
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731

    def size(counts, lengths, H, dh, q=1):
        co = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        so = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        a = m._binding.DcaArgs(R=len(counts), q=q, H=H, dh=dh, scale=0.1, cand_off_dev=fake,
                               cand_off_host=co.ctypes.data, seq_off_dev=fake, seq_off_host=so.ctypes.data,
                               q_ptr=fake, k_ptr=fake, v_ptr=fake, o_ptr=fake, lse_ptr=None, workspace=None,
                               workspace_bytes=0)
        return lib.rocs_dca_workspace_size(ctypes.byref(a))

    def expect(R, n_units, n_split, dh):
        units = a256((3 * R + 1) * 4)
        body = units + (n_units + n_split) * 16
        if n_split:
            split_buf = a256(a256(body) + n_split * 8 * 4)
            body = split_buf + n_split * 2 * 2 * 4 * 32 * (dh + 2) * 4
        return 256 + body

    # 10 requests x 8 heads x 2 chunks = 160 units, all with 3 K/V tiles: 160 mod 148 = 12 split
    assert size([512] * 10, [300] * 10, 8, 128) == expect(10, 160, 12, 128)
    # one request with a different key count: no split
    assert size([512] * 10, [300] * 9 + [420], 8, 128) == expect(10, 160, 0, 128)
    # a single K/V tile per request cannot be split
    assert size([512] * 10, [100] * 10, 8, 128) == expect(10, 160, 0, 128)
    # a multiple of 148 units leaves no partial wave
    assert size([256] * 37, [300] * 37, 4, 128) == expect(37, 148, 0, 128)
    # dh = 64: 100 rows (one chunk <= 128 rows) for 16 heads -> 8 head-pair units; dh = 128: 16 units
    assert size([100], [1000], 16, 64) == expect(1, 8, 0, 64)
    assert size([100], [1000], 16, 128) == expect(1, 16, 0, 128)
    # dh = 64, 300 rows: two chunks, the second of 44 rows paired -> 16 + 8 units; an odd head count keeps
    # its last head alone
    assert size([300], [1000], 16, 64) == expect(1, 24, 0, 64)
    assert size([300], [1000], 15, 64) == expect(1, 15 + 8, 0, 64)


def test_proj_host_validation(lib):
    import attention_ikbo_b200 as m

    a = m._binding.ProjArgs(M=10, N=200, K=64, in_=0x1000, w=0x1000, out=0x1000, workspace=None, workspace_bytes=0)
    assert lib.rocs_proj_forward(ctypes.byref(a), None) == 3
    a.N = 256
    assert lib.rocs_proj_forward(ctypes.byref(a), None) == 6


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import attention_ikbo_b200._binding as b

    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        b.load_library()


def test_fault_injection_host_validation(lib):
    import attention_ikbo_b200 as m

    a, keep = _lcb_args(m, [0, 3, 6], ws_bytes=1 << 20)
    assert lib.rocs_lcb_forward_fault_injection(ctypes.byref(a), None, 5, 10_000_000) == 1  # no request 5
    assert lib.rocs_lcb_forward_fault_injection(ctypes.byref(a), None, 0, 10) == 1  # limit below 1 ms
    f32, keep2 = _lcb_args(m, [0, 3, 6], dtype=0, ws_bytes=1 << 20)
    assert lib.rocs_lcb_forward_fault_injection(ctypes.byref(f32), None, 0, 10_000_000) == 3


def test_lcb_block_host_validation(lib):
    import attention_ikbo_b200 as m

    E = m._binding.LcbEpilogue
    a, keep = _lcb_args(m, [0, 3, 6], ws_bytes=1 << 20)
    P = ctypes.byref
    assert lib.rocs_lcb_block_forward(P(a), P(E(norm=3)), None, None) == 1  # unknown norm
    assert lib.rocs_lcb_block_forward(P(a), None, P(E(act=4)), None) == 1  # unknown activation
    assert lib.rocs_lcb_block_forward(P(a), None, P(E(eps=-1.0)), None) == 1  # negative eps
    assert lib.rocs_lcb_block_forward(P(a), None, P(E(eps=float("nan"))), None) == 1
    assert lib.rocs_lcb_block_forward(P(a), None, P(E(residual=0x10008)), None) == 1  # TMA needs 16 B
    assert lib.rocs_lcb_block_forward(P(a), P(E(bias=0x10002)), None, None) == 1  # fp32 alignment
    f32, keep2 = _lcb_args(m, [0, 3, 6], dtype=0, ws_bytes=1 << 20)
    assert lib.rocs_lcb_block_forward(P(f32), None, None, None) == 3  # bf16 kernel only
    bad, keep3 = _lcb_args(m, [0, 3, 2], ws_bytes=1 << 20)
    assert lib.rocs_lcb_block_forward(P(bad), None, None, None) == 2
    small, keep4 = _lcb_args(m, [0, 3, 6], ws_bytes=100)
    assert lib.rocs_lcb_block_forward(P(small), None, None, None) == 6
    # the block kernel's fault-injection hook validates like both of its parents
    fi = lib.rocs_lcb_block_forward_fault_injection
    assert fi(P(a), None, None, None, 5, 10_000_000) == 1  # no request 5
    assert fi(P(a), None, None, None, 0, 10) == 1  # limit below 1 ms
    assert fi(P(a), P(E(norm=3)), None, None, 0, 10_000_000) == 1  # unknown norm
    assert fi(P(f32), None, None, None, 0, 10_000_000) == 3
    assert fi(P(small), None, None, None, 0, 10_000_000) == 6


def test_fm_host_validation(lib):
    import attention_ikbo_b200 as m

    F = m._binding.FmArgs
    fake = 0x10000

    def args(off, n_r=64, n_c=64, d=128, ld_req=0, ld_cand=0, ws=1 << 20):
        off = np.asarray(off, np.int32)
        a = F(R=len(off) - 1, n_r=n_r, n_c=n_c, d=d, cand_off_dev=fake, cand_off_host=off.ctypes.data, x_req=fake,
              x_cand=fake, y_req=fake, y_cand=fake, ld_req=ld_req, ld_cand=ld_cand, workspace=fake if ws else None,
              workspace_bytes=ws)
        return a, off

    P = ctypes.byref
    for kw, code in [({"d": 96}, 3), ({"n_c": 48}, 3), ({"n_r": 63}, 3), ({"n_r": 258}, 3),
                     ({"ld_cand": 120}, 1), ({"ld_cand": 132}, 3), ({"ld_req": 60}, 1), ({"ld_cand": 392}, 3)]:
        a, keep = args([0, 3, 5], **kw)
        assert lib.rocs_fm_forward(P(a), None) == code, kw
    a, keep = args([0, 3, 2])
    assert lib.rocs_fm_forward(P(a), None) == 2
    a, keep = args([0, 3, 5], ws=0)
    assert lib.rocs_fm_forward(P(a), None) == 6
    a, keep = args([0, 3, 5])
    assert lib.rocs_fm_workspace_size(P(a)) == 256 + 256
    assert lib.rocs_align_cols(314, 2) == 320 and lib.rocs_align_cols(320, 2) == 320
    assert lib.rocs_align_cols(3, 8) == 4 and lib.rocs_align_cols(17, 1) == 32 and lib.rocs_align_cols(5, 3) == -1
    assert lib.rocs_pad_cols(fake, 4, 10, 10, fake, 16, 3, None) == 1  # element size
    assert lib.rocs_pad_cols(fake, 4, 10, 8, fake, 16, 2, None) == 1  # ld_src < cols
    assert lib.rocs_pad_cols(fake + 1, 4, 10, 10, fake, 16, 2, None) == 1  # misaligned
    assert lib.rocs_pad_cols(None, 0, 10, 10, None, 16, 2, None) == 0  # nothing to do


def test_chain_split_host_validation(lib):
    import attention_ikbo_b200 as m

    fake = 0x10000
    P = ctypes.byref
    W = m._binding.ChainWeightsArgs
    assert lib.rocs_chain_prepare_weights(P(W(n_out=256, o_r=128, o_c=128, n_r=256, n_c=64, d=128)), None) == 1
    S = m._binding.ChainSplitArgs

    def args(off, n_out=256, n_c=64, ws=1 << 22):
        off = np.asarray(off, np.int32)
        a = S(R=len(off) - 1, n_r=256, n_c=n_c, d=128, o_r=128, o_c=128, n_out=n_out, cand_off_dev=fake,
              cand_off_host=off.ctypes.data, x_req=fake, x_cand=fake, w_rs=fake, w_q=fake, w_fold=fake, y_req=fake,
              q=fake, workspace=fake if ws else None, workspace_bytes=ws)
        return a, off

    a, k = args([0, 3, 5], n_out=300)
    assert lib.rocs_chain_split_forward(P(a), None) == 3
    a, k = args([0, 3, 5], n_c=48)
    assert lib.rocs_chain_split_forward(P(a), None) == 3
    a, k = args([0, 3, 2])
    assert lib.rocs_chain_split_forward(P(a), None) == 2
    a, k = args([0, 3, 5], ws=100)
    assert lib.rocs_chain_split_forward(P(a), None) == 6
    a, k = args([0, 3, 5])
    # LCB workspace (header, flags, Z fp32 2 x 128 x 128) padded to 256, then q^R fp32 2 x 256
    assert lib.rocs_chain_split_workspace_size(P(a)) == 256 + 256 + 2 * 128 * 128 * 4 + 2 * 256 * 4


def test_host_pipeline_host_validation(lib):
    import attention_ikbo_b200 as m

    a, keep = _lcb_args(m, [0, 3, 6])
    P = ctypes.byref
    assert lib.rocs_lcb_host_staging_size(P(a), 0) == 0  # chunks >= 1
    need = lib.rocs_lcb_host_staging_size(P(a), 2)
    assert need > 256
    assert lib.rocs_lcb_forward_host(P(a), 0, 0x10000, need, None) == 1
    assert lib.rocs_lcb_forward_host(P(a), 2, 0x10000, need - 1, None) == 6
    assert lib.rocs_lcb_forward_host(P(a), 2, None, need, None) == 6
    bad, keep2 = _lcb_args(m, [0, 3, 2])
    assert lib.rocs_lcb_forward_host(P(bad), 2, 0x10000, need, None) == 2


def test_configured_device_mask_starts_empty(lib):
    """The per-device kernel set-up is recorded per device ordinal; nothing is configured before a
    launch (and nothing can be without a GPU).  Host-only query; the GPU side is in test_gpu_edges."""
    lib.rocs_configured_device_mask.restype = ctypes.c_uint64
    assert lib.rocs_configured_device_mask() == 0


def test_noalloc_status_reader_rejects_null(lib):
    lib.rocs_lcb_noalloc_read_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert lib.rocs_lcb_noalloc_read_status(None, None, None) == 1  # ROCS_ERR_INVALID_ARG, before any CUDA call
