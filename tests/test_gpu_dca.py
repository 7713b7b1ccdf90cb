"""IKBO-DCA on the GPU (through the C ABI) against the fp64 oracle.

Operation: ROCS (arXiv:2607.27744), section 3.2 Eq. (13), candidate cross attention
over K/V stored once per request, m_i resolved in the kernel (section 4.3.1).
"""
import numpy as np
import pytest
import torch

import rocs_inputs as ri
from _helpers import assert_close, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ikbo():
    import attention_ikbo_b200 as m

    m.load_library()
    return m


def run_dca(ikbo, x, expand_chunk=None):
    o, lse = ikbo.rocs_dca_forward(dev(x.q_t), dev(x.k_t), dev(x.v_t), x.cand_off, x.seq_off, x.q, x.scale,
                                   expand_chunk=expand_chunk)
    code, detail = ikbo.rocs_read_status(ikbo.rocs_dca_forward.last_workspace)
    assert code == 0, f"device status {ikbo.STATUS_NAMES.get(code)} at {detail}"
    return o, lse


def check(oracle_mod, x, o, lse, sel=None):
    sel = np.arange(x.C) if sel is None else np.asarray(sel)
    oo, ll = oracle_mod.dca(x.cand_off, x.seq_off, x.q_t, x.k_t, x.v_t, x.q, x.scale, sel_cand=sel)
    rows = (sel[:, None] * x.q + np.arange(x.q)[None, :]).ravel()
    ridx = torch.as_tensor(rows, device=o.device)
    got_o = host_f64(o[ridx]).reshape(oo.shape)
    assert_close(got_o, oo, "bf16", "O")
    got_l = host_f64(lse[ridx]).reshape(ll.shape)
    fin = np.isfinite(ll)
    assert np.array_equal(np.isfinite(got_l), fin)
    assert np.all(got_l[~fin] == -np.inf)
    if fin.any():
        assert_close(got_l[fin], ll[fin], "bf16", "LSE")


CASES = [  # (counts, lengths, q, H, dh)
    ([2, 5, 0], [5, 300, 17], 2, 2, 128),
    ([200, 1, 0, 513], [1, 129, 700, 128], 1, 3, 64),
    ([64, 70], [1000, 257], 4, 1, 128),
    ([3, 300], [128, 2049], 1, 4, 64),
]


@pytest.mark.parametrize("counts,lengths,q,H,dh", CASES)
def test_dca_small(ikbo, oracle_mod, counts, lengths, q, H, dh):
    x = ri.make_dca("t", counts, lengths, q, H, dh, 17 + q + H + dh)
    o, lse = run_dca(ikbo, x)
    check(oracle_mod, x, o, lse)


def test_dca_empty_keys(ikbo, oracle_mod):
    x = ri.make_dca("t", [3, 4, 2], [0, 50, 0], 2, 2, 64, 5)
    o, lse = run_dca(ikbo, x)
    check(oracle_mod, x, o, lse)


def test_dca_index_probe(ikbo):
    """V of request r is constant r  ->  every output of candidate i rounds to m_i."""
    counts, lengths = [3, 0, 260, 1, 7], [40, 9, 300, 1, 129]
    x = ri.make_dca("t", counts, lengths, 2, 2, 128, 8)
    v = np.zeros(x.v_t.shape, np.float32)
    for r in range(x.R):
        v[x.seq_off[r]: x.seq_off[r + 1]] = r
    x.v_t = (v.view(np.uint32) >> 16).astype(np.uint16)
    o, _ = run_dca(ikbo, x)
    m = np.repeat(np.arange(x.R), counts)
    got = np.rint(host_f64(o)).reshape(x.C, -1)
    assert np.array_equal(got, np.broadcast_to(m[:, None].astype(np.float64), got.shape))


def test_dca_permutation_within_request(ikbo, oracle_mod):
    x = ri.make_dca("t", [100, 40], [300, 77], 1, 2, 128, 12)
    o0, _ = run_dca(ikbo, x)
    perm = np.concatenate([np.random.RandomState(3).permutation(100), 100 + np.random.RandomState(4).permutation(40)])
    x.q_t = np.ascontiguousarray(x.q_t.reshape(x.C, x.q, x.H, x.dh)[perm].reshape(x.q_t.shape))
    o1, _ = run_dca(ikbo, x)
    assert_close(host_f64(o1), host_f64(o0)[perm], "bf16", "permuted O")


def test_dca_expand_baseline_matches(ikbo, oracle_mod):
    x = ri.make_dca("t", [5, 0, 9, 2], [130, 4, 64, 0], 2, 2, 128, 19)
    o, lse = run_dca(ikbo, x, expand_chunk=4)
    check(oracle_mod, x, o, lse)


def _sample(x, n, seed):
    rs = np.random.RandomState(seed)
    sel = set(rs.choice(x.C, size=min(n, x.C), replace=False).tolist())
    for r in range(x.R):
        if x.cand_off[r + 1] > x.cand_off[r]:
            sel.update([int(x.cand_off[r]), int(x.cand_off[r + 1]) - 1])
    return np.array(sorted(sel), dtype=np.int64)


def test_dca_bf16_full_size_sampled(ikbo, oracle_mod):
    """R=32, L=2048, H=8, dh=128, 512 candidates per request, q=1: 200 random candidates plus the first and
    last of every request (1.6 % of the 16,384)."""
    x = ri.dca_bf16()
    o, lse = run_dca(ikbo, x)
    sel = _sample(x, 200, 2)
    assert len(sel) >= 0.01 * x.C
    check(oracle_mod, x, o, lse, sel=sel)


def test_dca_long_full_size_sampled(ikbo, oracle_mod):
    """R=8, L_r~U{4096..8192}, H=4, dh=128, 2048 candidates per request, q=4: 168 random candidates plus the
    first and last of every request (over 1 % of the 16,384, every request represented)."""
    x = ri.dca_long()
    o, lse = run_dca(ikbo, x)
    sel = _sample(x, 168, 3)
    assert len(sel) >= 0.01 * x.C
    off = np.asarray(x.cand_off)
    assert all(((sel >= off[r]) & (sel < off[r + 1])).any() for r in range(x.R))
    check(oracle_mod, x, o, lse, sel=sel)


@pytest.mark.parametrize("dh", [64, 128])
def test_dca_split_tail_units(ikbo, oracle_mod, dh):
    """More work units than the GPU has SMs and every request with the same number (>= 2) of K/V tiles: the
    last (units mod SMs) units in claim order are split in two along the keys, each half leaves its partial
    result and the half that finishes second merges them.  Every candidate against the oracle."""
    counts = ri.uniform_int(91, 1, 1, 300, 80)
    lengths = ri.uniform_int(92, 2, 641, 768, 80)  # six K/V tiles each, ragged within the last tile
    x = ri.make_dca("split", counts, lengths, 1, 2, dh, 93)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    units = x.H * sum((x.q * int(n) + 255) // 256 for n in counts)
    assert units > sms and units % sms  # the premise: a partial last wave, so some units are split
    o, lse = run_dca(ikbo, x)
    check(oracle_mod, x, o, lse)


def test_dca_head_pairs(ikbo, oracle_mod):
    """dh = 64: a request's last chunk of at most 128 query rows is one unit for two heads (tile B holds the
    next head's rows); with H = 5 the last head of each such chunk stays alone.  Requests whose rows end in
    a short chunk, one whose rows fill whole chunks, an empty one and ragged keys; every candidate against
    the oracle."""
    x = ri.make_dca("pairs", [3, 64, 0, 129, 256, 190, 1], [300, 129, 50, 700, 1, 255, 1000], 2, 5, 64, 97)
    o, lse = run_dca(ikbo, x)
    check(oracle_mod, x, o, lse)


def _f32_to_bf16(a):
    """Round-to-nearest-even fp32 -> bf16 bits (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


@pytest.mark.parametrize("dh", [64, 128])
def test_dca_growing_max_rescale(ikbo, oracle_mod, dh):
    """Scores that grow along the key axis (non-negative queries and keys, keys scaled by a ramp): the row
    maximum rises by far more than 2^8 (in exp2 units) from one 128-key tile to the next, so every tile
    after the first takes the online softmax's rescale-and-redo path."""
    x = ri.make_dca("t", [3, 40], [700, 300], 2, 2, dh, 31)
    q = np.abs(ri.bf16_to_f32(x.q_t))
    k = np.abs(ri.bf16_to_f32(x.k_t))
    for r in range(len(x.seq_off) - 1):
        s0, s1 = int(x.seq_off[r]), int(x.seq_off[r + 1])
        k[s0:s1] *= (0.25 + 10.0 * np.arange(s1 - s0) / (s1 - s0))[:, None, None]
    x.q_t, x.k_t = _f32_to_bf16(q), _f32_to_bf16(k)
    # the premise: consecutive 128-key tiles' row maxima differ by more than 8 in log2 units
    s = np.einsum("hd,khd->hk", ri.bf16_to_f32(x.q_t)[0].astype(np.float64),
                  ri.bf16_to_f32(x.k_t)[:700].astype(np.float64)) * x.scale / np.log(2.0)
    tile_max = np.array([s[:, t * 128:(t + 1) * 128].max() for t in range(5)])  # the five full tiles
    assert np.all(np.diff(tile_max) > 8.0)
    o, lse = run_dca(ikbo, x)
    check(oracle_mod, x, o, lse)
