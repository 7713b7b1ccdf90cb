"""The LCB and DCA entry points inside a captured CUDA graph: every step of both runs in the library's kernels
on the caller's stream with caller-owned buffers, so a step (LCB then DCA) can be captured once and replayed;
replays match eager calls bit for bit, also after the inputs are rewritten in place.
"""
import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import dev

pytestmark = pytest.mark.gpu


def test_lcb_dca_graph_replay():
    import attention_ikbo_b200 as ikbo

    ikbo.load_library()
    x = ri.make_lcb("g", [3, 0, 17, 140, 9], 256, 64, 128, 128, 128, 201, "bf16")
    d = ri.make_dca("g", [5, 300, 0, 64], [900, 130, 40, 0], 2, 2, 128, 202)
    lcb_in = [dev(a) for a in (x.x_req, x.x_cand, x.w_rr, x.w_cr, x.w_cc)]
    q, k, v = dev(d.q_t), dev(d.k_t), dev(d.v_t)
    c_off, d_off, s_off = ikbo.offsets(x.cand_off), ikbo.offsets(d.cand_off), ikbo.offsets(d.seq_off)

    def step(out):
        ikbo.rocs_lcb_forward(*lcb_in, c_off, y_req=out["yr"], y_cand=out["yc"], workspace=out["ws_l"])
        ikbo.rocs_dca_forward(q, k, v, d_off, s_off, d.q, d.scale, o=out["o"], lse=out["lse"], workspace=out["ws_d"])

    yr, yc = ikbo.rocs_lcb_forward(*lcb_in, c_off)
    ws_l = ikbo.rocs_lcb_forward.last_workspace
    o, lse = ikbo.rocs_dca_forward(q, k, v, d_off, s_off, d.q, d.scale)
    ws_d = ikbo.rocs_dca_forward.last_workspace
    out = {"yr": torch.empty_like(yr), "yc": torch.empty_like(yc), "o": torch.empty_like(o),
           "lse": torch.empty_like(lse), "ws_l": torch.empty_like(ws_l), "ws_d": torch.empty_like(ws_d)}
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up off the default stream, as capture requires
        step(out)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(out)
    for t in out.values():
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for a, b in ((out["yr"], yr), (out["yc"], yc), (out["o"], o), (out["lse"], lse)):
        assert torch.equal(a, b)
    # rewrite the inputs in place; the replay must follow them
    lcb_in[1].copy_(lcb_in[1].flip(0))
    q.mul_(-0.5)
    g.replay()
    yr2, yc2 = ikbo.rocs_lcb_forward(*lcb_in, c_off)
    o2, lse2 = ikbo.rocs_dca_forward(q, k, v, d_off, s_off, d.q, d.scale)
    torch.cuda.synchronize()
    for a, b in ((out["yr"], yr2), (out["yc"], yc2), (out["o"], o2), (out["lse"], lse2)):
        assert torch.equal(a, b)
    assert not torch.equal(out["yc"], yc)
