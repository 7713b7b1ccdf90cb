"""IKBO masked FM on the GPU (through the C ABI) against the fp64 oracle, and the alignment transform.

Operation: ROCS (arXiv:2607.27744), section 3.1.4 Eq. (10), with X^R kept on chip for all candidates
of a request (section 4.1) and output rows padded to 16-byte multiples (section 4.2.4).
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


def run_fm(ikbo, x, **kw):
    y_req, y_cand = ikbo.rocs_fm_forward(dev(x.x_req), dev(x.x_cand), x.cand_off, **kw)
    code, detail = ikbo.rocs_read_status(ikbo.rocs_fm_forward.last_workspace)
    assert code == 0, f"device status {ikbo.STATUS_NAMES.get(code)} at {detail}"
    return y_req, y_cand


def check(oracle_mod, x, y_req, y_cand, sel_cand=None):
    sel = np.arange(x.C) if sel_cand is None else np.asarray(sel_cand)
    yr, yc = oracle_mod.fm(x.cand_off, x.x_req, x.x_cand, sel_cand=sel)
    gr = host_f64(y_req)
    assert_close(gr[:, :, :x.n_r], yr, "bf16", "Y^R")
    assert not np.any(gr[:, :, x.n_r:]), "Y^R padding must be zero"
    if len(sel):
        gc = host_f64(y_cand[torch.as_tensor(sel, device=y_cand.device)])
        assert_close(gc[:, :, :x.n_r + x.n_c], yc, "bf16", "Y^C")
        assert not np.any(gc[:, :, x.n_r + x.n_c:]), "Y^C padding must be zero"


CASES = [  # (counts, n_r, n_c, d)
    ([3, 0, 5, 1], 64, 64, 128),      # aligned rows
    ([2, 7, 0], 250, 64, 128),        # n_r + n_c = 314 -> rows padded to 320
    ([1, 4, 2], 256, 128, 64),        # widest rows (384)
    ([9, 0, 0, 4], 30, 32, 64),       # tiny request block, padded Y^R rows
    ([5, 3], 2, 128, 128),            # a single pair of request rows
    ([40, 1, 17], 200, 32, 128),      # several candidate tiles per request, a partial tile
]


@pytest.mark.parametrize("counts,n_r,n_c,d", CASES)
def test_fm_small(ikbo, oracle_mod, counts, n_r, n_c, d):
    x = ri.make_fm("t", counts, n_r, n_c, d, 50 + n_r + n_c + d)
    y_req, y_cand = run_fm(ikbo, x)
    assert y_req.shape[2] == ikbo.rocs_align_cols(n_r, 2) and y_cand.shape[2] == ikbo.rocs_align_cols(n_r + n_c, 2)
    check(oracle_mod, x, y_req, y_cand)


def test_fm_wider_leading_dimension(ikbo, oracle_mod):
    x = ri.make_fm("t", [4, 2], 100, 64, 128, 3)
    y_req, y_cand = run_fm(ikbo, x, ld_req=128, ld_cand=192)
    assert y_cand.shape[2] == 192
    check(oracle_mod, x, y_req, y_cand)


def test_fm_index_probe_bit_exact(ikbo):
    """X^R_r rows = r e_0, X^C rows = e_0: every cross entry of candidate i equals m_i exactly."""
    counts = [3, 0, 70, 1, 0, 9]
    x = ri.make_fm("t", counts, 48, 64, 64, 4)
    bf16 = lambda v: (np.array([v], np.float32).view(np.uint32) >> 16).astype(np.uint16)[0]  # exact for small ints
    x.x_req[...] = 0
    x.x_cand[...] = 0
    for r in range(x.R):
        x.x_req[r, :, 0] = bf16(r)
    x.x_cand[:, :, 0] = bf16(1.0)
    _, y_cand = run_fm(ikbo, x)
    m = np.repeat(np.arange(x.R), np.diff(x.cand_off)).astype(np.float64)
    g = host_f64(y_cand)
    assert np.array_equal(g[:, :, :48], np.broadcast_to(m[:, None, None], (x.C, 64, 48)))
    assert np.all(g[:, :, 48:112] == 1.0) and not np.any(g[:, :, 112:])


def test_fm_isolation_bitwise(ikbo):
    x = ri.make_fm("t", [6, 1, 40], 96, 64, 128, 8)
    yr0, _ = run_fm(ikbo, x)
    x.x_cand[...] = ri.normal(123, 1, x.x_cand.shape)
    yr1, _ = run_fm(ikbo, x)
    assert np.array_equal(bits(yr0), bits(yr1))


def test_fm_full_size_sampled(ikbo, oracle_mod):
    """The bench workload at full size, in the bench's launch configuration: every request output and
    a seeded sample of candidates (first/last of requests + random)."""
    x = ri.fm_bf16()
    y_req, y_cand = run_fm(ikbo, x)
    off = x.cand_off
    firsts = [int(off[r]) for r in range(x.R) if off[r + 1] > off[r]]
    lasts = [int(off[r + 1]) - 1 for r in range(x.R) if off[r + 1] > off[r]]
    rnd = ri.uniform_int(18, 1, 0, x.C - 1, 48).tolist()
    check(oracle_mod, x, y_req, y_cand, np.unique(np.array(firsts[::4] + lasts[::4] + rnd, dtype=np.int64)))


@pytest.mark.parametrize("dtype,cols,ld", [(torch.bfloat16, 314, 320), (torch.float32, 30, 32), (torch.uint8, 5, 16)])
def test_pad_cols_matches_definition(ikbo, oracle_mod, dtype, cols, ld):
    g = torch.Generator().manual_seed(cols)
    src = (torch.randn(37, 3, cols, generator=g) * 10).to(dtype) if dtype != torch.uint8 else \
        torch.randint(0, 255, (37, 3, cols), generator=g, dtype=torch.uint8)
    d = src.cuda()
    padded = ikbo.rocs_pad_cols(d, ld)
    want = oracle_mod.pad_cols(src.view(torch.int16 if dtype == torch.bfloat16 else dtype).numpy(), ld)
    got = padded.cpu().view(torch.int16 if dtype == torch.bfloat16 else dtype).numpy()
    assert np.array_equal(got, want)
    back = ikbo.rocs_pad_cols(padded, cols)
    assert torch.equal(back.cpu(), src)
