"""Repeated calls give bit-identical outputs: the persistent kernels claim work units dynamically, so which CTA
computes a unit changes from call to call, but every unit's arithmetic is fixed (no atomics on results, no
cross-unit reductions); a race or an ordering dependence would show up here as a differing bit."""
import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ikbo():
    import attention_ikbo_b200 as m

    m.load_library()
    return m


def test_repeated_calls_bitwise(ikbo):
    rng = np.random.default_rng(77)
    x = ri.make_lcb("det", rng.integers(0, 400, 24), 256, 64, 128, 128, 128, 301, "bf16")
    lcb_in = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    off_l = ikbo.offsets(x.cand_off)
    d = ri.make_dca("det", rng.integers(0, 600, 12), rng.integers(1, 3000, 12), 2, 4, 128, 302)
    q, k, v = dev(d.q_t), dev(d.k_t), dev(d.v_t)
    off_c, off_s = ikbo.offsets(d.cand_off), ikbo.offsets(d.seq_off)
    f = ri.make_fm("det", rng.integers(0, 400, 24), 250, 64, 128, 303)
    xr, xc = dev(f.x_req), dev(f.x_cand)
    off_f = ikbo.offsets(f.cand_off)
    ref = None
    for it in range(12):
        yr, yc = ikbo.rocs_lcb_forward(*lcb_in, off_l)
        o, lse = ikbo.rocs_dca_forward(q, k, v, off_c, off_s, d.q, d.scale)
        fr, fc = ikbo.rocs_fm_forward(xr, xc, off_f)
        out = [t.clone() for t in (yr, yc, o, lse, fr, fc)]
        if ref is None:
            ref = out
        else:
            for a, b in zip(out, ref):
                assert torch.equal(a, b), f"call {it} differs"
    for ws in (ikbo.rocs_lcb_forward.last_workspace, ikbo.rocs_dca_forward.last_workspace,
               ikbo.rocs_fm_forward.last_workspace):
        assert ikbo.rocs_read_status(ws)[0] == 0
