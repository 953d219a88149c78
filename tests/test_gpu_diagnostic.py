"""GPU parity of the distributional-stability diagnostic (histograms of the
pre-softmax scores of the unselected blocks and of their deviation from the
block-centroid score) against the fp64 oracle.

The selection both sides use is the oracle's (an input to the kernel, never
the other way round).  A score that lies within DELTA of a bin edge may fall
on either side of it in fp32, so the check brackets the kernel's cumulative
counts: for every edge e, #(x < e - DELTA) <= kernel #(x < e) <= #(x < e + DELTA),
both bounds from the oracle (its histogram with all edges shifted by -/+DELTA).
Totals are exact; the moment sums agree to fp32 rounding of the scores.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from workloads import WORKLOADS, generate_head
from tests.parity_util import to64

pytestmark = pytest.mark.gpu

DELTA = 1e-3          # |score error| bound: fp32 sums of d bf16 products, |x| < 30
MOMENT_RTOL = 1e-5


@pytest.fixture(scope="module")
def P():
    from block_sparse_attention_stats_b200.build import build
    build()
    import block_sparse_attention_stats_b200 as P
    return P


def _oracle_selection(q, k, v, wl, rows):
    st = O.block_stats(q, k, v, wl.block_size)
    N = st["kbar"].shape[0]
    cov = None
    if wl.cov_weight != 0.0:
        cov = O.covariance_norms(k, v, wl.block_size, st["kbar"], st["hbar"])
    k_sel = O.num_selected(N, wl.density)
    sc = O.selection_scores(st["qbar"], st["kbar"], wl.scale, cov, wl.cov_weight, rows)
    sel = np.tile(np.arange(k_sel), (N, 1))          # rows the kernel does not read
    sel[rows] = O.select_blocks(sc, k_sel, wl.sink_idx)
    return sel


def _cum(h, nbins):
    """#(values < edge_m) for m = 0 .. nbins from an under/overflow histogram."""
    return np.cumsum(np.asarray(h, dtype=np.int64))[:nbins + 1]


def _check(P, wl, heads, lo, hi, nbins, stride):
    N = -(-wl.L // wl.block_size)
    rows = list(range(0, N, stride))
    tot = None
    for (b, h) in heads:
        Q, K, V = generate_head(wl, b, h, "cpu")
        q64, k64, v64 = to64(Q), to64(K), to64(V)
        sel = _oracle_selection(q64, k64, v64, wl, rows)
        idx = torch.from_numpy(sel.astype(np.int32)).view(1, 1, N, -1).cuda()
        g = P.pisa_tail_score_histogram(Q.view(1, 1, wl.L, wl.d).cuda(),
                                        K.view(1, 1, wl.L, wl.d).cuda(), idx, lo, hi, nbins,
                                        wl.block_size, wl.scale, stride)
        P.pisa_device_status()
        r = {dl: O.tail_score_histogram(q64, k64, wl.block_size, sel, wl.scale, lo + dl,
                                        hi + dl, nbins, rows)
             for dl in (-DELTA, 0.0, DELTA)}
        ref = r[0.0]
        assert g["n"] == ref["n"] > 0
        for key in ("hist_x", "hist_y"):
            gh = g[key].cpu().numpy()
            assert gh.sum() == ref["n"]
            cg = _cum(gh, nbins)
            lo_b, hi_b = _cum(r[-DELTA][key], nbins), _cum(r[DELTA][key], nbins)
            bad = np.nonzero((cg < lo_b) | (cg > hi_b))[0]
            assert bad.size == 0, f"{key} head {(b, h)}: edges {bad[:8]} out of bracket"
            # the bracket is narrow (few values sit within DELTA of any one edge),
            # or else the values sit exactly on edges (y = 0 for a one-key block)
            # and the counts must agree exactly
            if (hi_b - lo_b).max() > 1e-2 * ref["n"] + 2:
                assert (gh == ref[key]).all(), f"{key} head {(b, h)}: values on edges"
        for s, s2 in (("sum_x", "sum_x2"), ("sum_y", "sum_y2")):
            scale = math.sqrt(ref["n"] * ref[s2])
            assert abs(g[s] - ref[s]) <= MOMENT_RTOL * scale + 1e-9, (s, g[s], ref[s])
            assert abs(g[s2] - ref[s2]) <= MOMENT_RTOL * 2 * ref[s2] + 1e-9, (s2, g[s2], ref[s2])
        if tot is None:
            tot = ref
    return tot


def test_flux_shape_all_query_blocks(P):
    """L=4608, d=128, covariance-aware selection at density 0.15, sink -1."""
    wl = WORKLOADS["flux"].with_(H=2)
    ref = _check(P, wl, [(0, 0), (0, 1)], -8.0, 8.0, 64, 1)
    # the centred deviations have mean ~0 over each block: their total is tiny
    assert abs(ref["sum_y"]) <= 1e-9 * math.sqrt(ref["n"] * ref["sum_y2"])


@pytest.mark.parametrize("L,d,stride,nbins,lo,hi", [
    (1000, 64, 3, 40, -6.0, 6.0),       # ragged last block, strided query blocks
    (777, 64, 1, 1, -0.5, 0.5),         # one bin: most values under/overflow
    (65, 128, 1, 4096, -64.0, 64.0),    # two blocks (one key in the last), max bins
])
def test_ragged_and_bins(P, L, d, stride, nbins, lo, hi):
    wl = WORKLOADS["flux"].with_(H=1, L=L, d=d, density=0.25, sink_idx=0, cov_weight=0.0,
                                 cluster_kind="block")
    _check(P, wl, [(0, 0)], lo, hi, nbins, stride)


def test_wan_full_size_sampled_query_blocks(P):
    """Full Wan 2.1 sequence (L=75600, d=128), one head, every 197th query block."""
    wl = WORKLOADS["wan"]
    _check(P, wl, [(0, 7)], -8.0, 8.0, 64, 197)


def test_rejects_bad_arguments(P):
    q = torch.zeros(1, 1, 640, 128, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(1, 1, 10, 1, dtype=torch.int32, device="cuda")
    for kw in (dict(lo=1.0, hi=1.0), dict(nbins=0), dict(nbins=4097), dict(query_stride=0)):
        with pytest.raises(RuntimeError):
            P.pisa_tail_score_histogram(q, q, idx, **{**dict(lo=-1.0, hi=1.0), **kw})
    with pytest.raises(RuntimeError):
        P.pisa_tail_score_histogram(q.float(), q.float(), idx)
