"""Pins of the fp64 oracle against things other than itself.

Each test ties one part of the oracle to a hand-worked example, a library
routine, a closed form, an invariant or a brute-force search, chosen so that a
dropped term, a wrong sign or index, or a transposed operand fails at least
one of them.  CPU only.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from workloads import WORKLOADS, generate_head

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _sdpa(q, k, v, scale):
    """Dense softmax attention from torch's library routine, fp64 on the CPU."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)
    return out[0, 0].numpy()


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _ev(x):
    if isinstance(x, str):
        return eval(x, {"__builtins__": {}}, {"e": math.e})
    return float(x)


def _arr(rows):
    return np.array([[_ev(c) for c in r] for r in rows], dtype=np.float64)


# ----------------------------------------------------------------------------
# hand-worked examples (tests/golden/worked_examples.json)
# ----------------------------------------------------------------------------

with open(GOLDEN) as f:
    _EXAMPLES = json.load(f)["examples"]


@pytest.mark.parametrize("ex", _EXAMPLES, ids=[e["name"] for e in _EXAMPLES])
def test_worked_example(ex):
    q, k, v = (np.array(ex[n], dtype=np.float64) for n in ("q", "k", "v"))
    b, s = ex["block_size"], ex["scale"]
    st = O.block_stats(q, k, v, b, keep_blockwise=True)
    for key in ("qbar", "kbar", "vsum", "hbar"):
        if key in ex:
            np.testing.assert_allclose(st[key], _arr(ex[key]), rtol=0, atol=1e-14)
    if "cov" in ex:
        cov = O.covariance_norms(k, v, b, st["kbar"], st["hbar"])
        np.testing.assert_allclose(cov, [_ev(c) for c in ex["cov"]], rtol=1e-14, atol=1e-14)
    N = st["kbar"].shape[0]
    ksel = O.num_selected(N, ex["density"])
    lam = ex["cov_weight"]
    cov = O.covariance_norms(k, v, b, st["kbar"], st["hbar"]) if lam else None
    sc = O.selection_scores(st["qbar"], st["kbar"], s, cov, lam)
    idx = O.select_blocks(sc, ksel, ex["sink_idx"])
    assert idx.tolist() == ex["idx"]
    for mode in ("hyd", "0th", "1st"):
        key = "o_" + mode
        if key not in ex:
            continue
        o = O.piecewise_attention(q, k, v, b, idx, st, s, mode)
        np.testing.assert_allclose(o, _arr(ex[key]), rtol=1e-13, atol=1e-13)
        r = O.pisa_attention_head(q, k, v, b, ex["density"], ex["sink_idx"], mode, scale=s,
                                  cov_weight=lam)
        np.testing.assert_allclose(r["out"], _arr(ex[key]), rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------------------
# special cases that reduce to dense softmax attention (torch SDPA, fp64)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("L,b,d", [(200, 16, 8), (64, 64, 16), (130, 32, 4)])
def test_density_one_is_dense_attention(L, b, d):
    q, k, v = _rand((L, d), 1), _rand((L, d), 2), _rand((L, d), 3)
    s = 1 / math.sqrt(d)
    ref = _sdpa(q, k, v, s)
    for mode in ("hyd", "0th"):
        for sink in (None, 0, -1):
            r = O.pisa_attention_head(q, k, v, b, 1.0, sink, mode)
            np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-12)
    # also via the dense oracle routine
    np.testing.assert_allclose(O.dense_attention(q, k, v, s), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("density", [0.05, 0.2, 0.5])
def test_block_size_one_is_exact(density):
    """block_size 1: kbar_j = k_j, H_j = 0, so the tail is exact for any density."""
    L, d = 97, 8
    q, k, v = _rand((L, d), 4), _rand((L, d), 5), _rand((L, d), 6)
    ref = _sdpa(q, k, v, 1 / math.sqrt(d))
    for mode in ("hyd", "0th"):
        r = O.pisa_attention_head(q, k, v, 1, density, None, mode)
        np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("sink", [None, 0, -1])
@pytest.mark.parametrize("b,L", [(8, 60), (128, 300)])
def test_identical_keys_per_block_is_exact(sink, b, L):
    """All keys of a block equal: exp(s q k_n) = alpha for every n, so the
    zeroth-order tail (alpha vsum, n_j alpha) is exact and H_j = 0; the ragged
    last block (4, or 44, tokens) checks n_j in the denominator."""
    d = 6
    N = -(-L // b)
    centres = _rand((N, d), 7)
    k = np.repeat(centres, b, axis=0)[:L]
    q, v = _rand((L, d), 8) * 1.5, _rand((L, d), 9)
    ref = _sdpa(q, k, v, 1 / math.sqrt(d))
    for density in (0.15, 0.3, 0.6):
        for mode in ("hyd", "0th"):
            r = O.pisa_attention_head(q, k, v, b, density, sink, mode)
            np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-12)


def test_zero_queries_give_mean_value():
    """q = 0: every exponent is 0 and the first-order term vanishes, so
    o_t = (sum of all values) / L for any selection."""
    L, b, d = 150, 16, 5
    q = np.zeros((L, d))
    k, v = _rand((L, d), 10), _rand((L, d), 11)
    for mode in ("hyd", "0th"):
        r = O.pisa_attention_head(q, k, v, b, 0.25, -1, mode)
        np.testing.assert_allclose(r["out"], np.broadcast_to(v.mean(0), (L, d)),
                                   rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------------------
# block statistics
# ----------------------------------------------------------------------------

def test_hbar_closed_form():
    """Hbar = (K^T V - sum_j kbar_j^T vsum_j) / N, from a different grouping of
    the same sums (ragged last block included)."""
    L, b, d = 203, 32, 7
    q, k, v = _rand((L, d), 12), _rand((L, d), 13), _rand((L, d), 14)
    st = O.block_stats(q, k, v, b)
    N = st["kbar"].shape[0]
    closed = (k.T @ v - st["kbar"].T @ st["vsum"]) / N
    np.testing.assert_allclose(st["hbar"], closed, rtol=1e-12, atol=1e-12)


def test_block_first_order_matrix_is_scaled_cross_covariance():
    """H_j = n_j * cross-covariance(k, v) of block j, from numpy.cov."""
    L, b, d = 70, 16, 3
    q, k, v = _rand((L, d), 15), _rand((L, d), 16), _rand((L, d), 17)
    st = O.block_stats(q, k, v, b, keep_blockwise=True)
    _, starts, counts = O.block_partition(L, b)
    for j in range(len(starts)):
        kb = k[starts[j]:starts[j] + counts[j]]
        vb = v[starts[j]:starts[j] + counts[j]]
        c = np.cov(kb.T, vb.T, bias=True)[:d, d:]
        np.testing.assert_allclose(st["H"][j], counts[j] * c, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(st["qbar"][j], q[starts[j]:starts[j] + counts[j]].mean(0),
                                   rtol=1e-13, atol=1e-13)


def test_covariance_norm_matches_numpy_norm():
    L, b, d = 96, 16, 4
    q, k, v = _rand((L, d), 18), _rand((L, d), 19), _rand((L, d), 20)
    st = O.block_stats(q, k, v, b, keep_blockwise=True)
    M = O.covariance_norms(k, v, b, st["kbar"], st["hbar"])
    ref = np.array([np.linalg.norm(Hj - st["hbar"], "fro") for Hj in st["H"]])
    np.testing.assert_allclose(M, ref, rtol=1e-12)


def test_first_order_term_adds_nothing_to_denominator():
    """Per-token first-order expansion summed over a block: the deviation terms
    cancel, leaving n_j alpha."""
    L, b, d = 64, 16, 8
    q, k, v = _rand((L, d), 21), _rand((L, d), 22), _rand((L, d), 23)
    st = O.block_stats(q, k, v, b)
    s = 1 / math.sqrt(d)
    for j in range(4):
        kb = k[j * b:(j + 1) * b]
        for t in range(0, L, 7):
            a = math.exp(s * q[t] @ st["kbar"][j])
            per_token = sum(a * (1 + s * q[t] @ (kn - st["kbar"][j])) for kn in kb)
            assert abs(per_token - b * a) <= 1e-12 * b * a


# ----------------------------------------------------------------------------
# first-order accuracy: Taylor order of the approximation
# ----------------------------------------------------------------------------

def test_taylor_order_of_hybrid_and_zeroth():
    """Keys k_{j,n} = kbar_j + eps delta_n with the same deviations delta and
    values w_n in every block, so H_j = Hbar for all j.  Then the hybrid tail is
    the exact first-order Taylor expansion (error O(eps^2)) and the zeroth-order
    tail drops a first-order term (error O(eps)).  A wrong sign, scale or
    orientation of the first-order term makes the hybrid error O(eps)."""
    b, N, d = 4, 8, 4
    L = b * N
    rng = np.random.default_rng(24)
    kbar = rng.standard_normal((N, d))
    delta = rng.standard_normal((b, d))
    delta -= delta.mean(0)
    w = rng.standard_normal((b, d))
    q = rng.standard_normal((L, d))
    v = np.tile(w, (N, 1))

    def errs(eps):
        k = np.repeat(kbar, b, axis=0) + eps * np.tile(delta, (N, 1))
        ref = _sdpa(q, k, v, 1 / math.sqrt(d))
        e = {}
        for mode in ("hyd", "0th"):
            r = O.pisa_attention_head(q, k, v, b, 0.25, None, mode)
            e[mode] = np.abs(r["out"] - ref).max()
        return e

    e1, e2, e3 = errs(0.02), errs(0.01), errs(0.005)
    for a, c in ((e1, e2), (e2, e3)):
        assert 3.4 < a["hyd"] / c["hyd"] < 4.6
        assert 1.7 < a["0th"] / c["0th"] < 2.3
    assert e3["hyd"] < 0.05 * e3["0th"]


def test_blockwise_first_order_is_second_order_accurate():
    """Keys k_{j,n} = kbar_j + eps delta_{j,n} with DIFFERENT deviations and
    values per block (H_j all differ): the block-wise first-order tail is the
    exact first-order expansion of every unselected block (error O(eps^2)),
    while the hybrid (shared Hbar) and zeroth-order tails are O(eps)."""
    b, N, d = 4, 8, 4
    L = b * N
    rng = np.random.default_rng(38)
    kbar = rng.standard_normal((N, d))
    delta = rng.standard_normal((N, b, d))
    delta -= delta.mean(axis=1, keepdims=True)
    q = rng.standard_normal((L, d))
    v = rng.standard_normal((L, d))

    def errs(eps):
        k = (kbar[:, None, :] + eps * delta).reshape(L, d)
        ref = _sdpa(q, k, v, 1 / math.sqrt(d))
        return {m: np.abs(O.pisa_attention_head(q, k, v, b, 0.25, None, m)["out"] - ref).max()
                for m in ("1st", "hyd", "0th")}

    e1, e2, e3 = errs(0.02), errs(0.01), errs(0.005)
    for a, c in ((e1, e2), (e2, e3)):
        assert 3.4 < a["1st"] / c["1st"] < 4.6
        assert 1.7 < a["hyd"] / c["hyd"] < 2.3
    assert e3["1st"] < 0.05 * e3["hyd"]


def test_blockwise_first_order_equals_hybrid_when_blocks_share_H():
    """Same deviations and values in every block: H_j = Hbar, so the two
    first-order variants coincide."""
    b, N, d = 4, 6, 3
    L = b * N
    rng = np.random.default_rng(39)
    delta = rng.standard_normal((b, d))
    delta -= delta.mean(0)
    k = (rng.standard_normal((N, 1, d)) + 0.3 * delta[None]).reshape(L, d)
    v = np.tile(rng.standard_normal((b, d)), (N, 1))
    q = rng.standard_normal((L, d))
    h = O.pisa_attention_head(q, k, v, b, 0.34, -1, "hyd")["out"]
    f = O.pisa_attention_head(q, k, v, b, 0.34, -1, "1st")["out"]
    np.testing.assert_allclose(f, h, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------

def _bruteforce_select(scores_row, k_sel, sink):
    """Rank counting: block j is kept iff fewer than k_sel blocks beat it,
    where j' beats j if its score is higher or equal with a lower index."""
    N = len(scores_row)
    cand = [j for j in range(N) if j != sink]
    need = k_sel - (0 if sink is None else 1)
    keep = []
    for j in cand:
        beaten = sum(1 for jj in cand if scores_row[jj] > scores_row[j]
                     or (scores_row[jj] == scores_row[j] and jj < j))
        if beaten < need:
            keep.append(j)
    if sink is not None:
        keep.append(sink)
    return sorted(keep)


@pytest.mark.parametrize("sink_idx", [None, 0, -1])
def test_selection_matches_bruteforce(sink_idx):
    rng = np.random.default_rng(25)
    for N in (1, 2, 5, 9, 16):
        # integer-valued scores force exact ties
        scores = rng.integers(-3, 4, size=(6, N)).astype(np.float64)
        for k_sel in range(1, N + 1):
            idx = O.select_blocks(scores, k_sel, sink_idx)
            sink = None if sink_idx is None else (0 if sink_idx == 0 else N - 1)
            for r in range(scores.shape[0]):
                assert idx[r].tolist() == _bruteforce_select(scores[r], k_sel, sink)


def test_selection_exhaustive_subsets():
    """Without ties, the selected set is the k-subset with the largest score sum."""
    rng = np.random.default_rng(26)
    N, k_sel = 7, 3
    scores = rng.standard_normal((5, N))
    idx = O.select_blocks(scores, k_sel, None)
    for r in range(5):
        best = max(itertools.combinations(range(N), k_sel),
                   key=lambda c: sum(scores[r, list(c)]))
        assert idx[r].tolist() == list(best)


def test_selection_invariants_on_workload():
    wl = WORKLOADS["tiny"]
    q, k, v = generate_head(wl, 0, 1)
    for sink in (None, 0, -1):
        r = O.pisa_attention_head(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                  64, 0.25, sink, "hyd")
        N = 16
        assert r["k_sel"] == 4
        for row in r["idx"]:
            assert len(set(row.tolist())) == 4
            assert list(row) == sorted(row)
            assert 0 <= row.min() and row.max() < N
            if sink is not None:
                assert (0 if sink == 0 else N - 1) in row


def test_num_selected_values():
    """k_sel for the workloads' block counts and densities."""
    cases = [(16, 0.25, 4), (72, 0.15, 10), (72, 0.05, 3), (72, 0.10, 7), (72, 0.25, 18),
             (72, 1.0, 72), (1182, 0.125, 147), (1861, 0.10, 186), (5, 0.01, 1), (3, 1.0, 3)]
    for N, dens, want in cases:
        assert O.num_selected(N, dens) == want
    with pytest.raises(ValueError):
        O.num_selected(10, 0.0)
    with pytest.raises(ValueError):
        O.num_selected(10, 1.5)


# ----------------------------------------------------------------------------
# invariants of the output
# ----------------------------------------------------------------------------

def test_constant_values_reproduce_the_value():
    L, b, d = 90, 16, 6
    q, k = _rand((L, d), 27), _rand((L, d), 28)
    row = _rand((d,), 29)
    v = np.broadcast_to(row, (L, d)).copy()
    for mode in ("hyd", "0th"):
        r = O.pisa_attention_head(q, k, v, b, 0.3, 0, mode)
        np.testing.assert_allclose(r["out"], v, rtol=1e-12, atol=1e-12)


def test_linear_in_values():
    L, b, d = 80, 16, 6
    q, k = _rand((L, d), 30), _rand((L, d), 31)
    v1, v2 = _rand((L, d), 32), _rand((L, d), 33)
    for mode in ("hyd", "0th"):
        f = lambda vv: O.pisa_attention_head(q, k, vv, b, 0.4, None, mode)["out"]
        np.testing.assert_allclose(f(2 * v1 - 3 * v2), 2 * f(v1) - 3 * f(v2),
                                   rtol=1e-10, atol=1e-11)


def test_permuting_tokens_inside_kv_blocks():
    """Block statistics and the exact part are sums over a block's tokens."""
    L, b, d = 96, 16, 5
    q, k, v = _rand((L, d), 34), _rand((L, d), 35), _rand((L, d), 36)
    perm = np.arange(L)
    rng = np.random.default_rng(37)
    for j in range(L // b):
        perm[j * b:(j + 1) * b] = rng.permutation(np.arange(j * b, (j + 1) * b))
    for mode in ("hyd", "0th"):
        a = O.pisa_attention_head(q, k, v, b, 0.34, -1, mode, cov_weight=0.1)
        c = O.pisa_attention_head(q, k[perm], v[perm], b, 0.34, -1, mode, cov_weight=0.1)
        assert (a["idx"] == c["idx"]).all()
        np.testing.assert_allclose(a["out"], c["out"], rtol=1e-12, atol=1e-12)


def test_hybrid_differs_from_zeroth_only_through_hbar():
    """With linearly dependent values Hbar is far from zero and hyd != 0th;
    with Hbar forced to zero they coincide."""
    wl = WORKLOADS["tiny"].with_(L=256, H=1)
    q, k, v = (x.double().numpy() for x in generate_head(wl, 0, 0, value_mode="linear"))
    st = O.block_stats(q, k, v, 64)
    assert np.abs(st["hbar"]).max() > 0.1
    sc = O.selection_scores(st["qbar"], st["kbar"], wl.scale)
    idx = O.select_blocks(sc, 1, None)
    oh = O.piecewise_attention(q, k, v, 64, idx, st, wl.scale, "hyd")
    o0 = O.piecewise_attention(q, k, v, 64, idx, st, wl.scale, "0th")
    assert np.abs(oh - o0).max() > 1e-3
    st0 = dict(st, hbar=np.zeros_like(st["hbar"]))
    np.testing.assert_allclose(O.piecewise_attention(q, k, v, 64, idx, st0, wl.scale, "hyd"),
                               o0, rtol=0, atol=0)


def test_error_to_dense_falls_with_density():
    """Sanity (not a pin): on a clustered workload the error against dense
    attention shrinks as density grows, and vanishes at density 1."""
    wl = WORKLOADS["flux"].with_(L=640, H=1, cluster_kind="block", dtype="f32")
    q, k, v = (x.double().numpy() for x in generate_head(wl, 0, 0))
    ref = _sdpa(q, k, v, wl.scale)
    errs = []
    for dens in (0.1, 0.3, 0.6, 1.0):
        r = O.pisa_attention_head(q, k, v, 64, dens, None, "hyd")
        errs.append(np.abs(r["out"] - ref).max())
    assert errs[0] >= errs[1] >= errs[2] and errs[3] < 1e-12


# ----------------------------------------------------------------------------
# input generator
# ----------------------------------------------------------------------------

def test_generator_is_deterministic_and_per_head():
    wl = WORKLOADS["tiny"]
    a = generate_head(wl, 0, 1)
    b = generate_head(wl, 0, 1)
    c = generate_head(wl, 0, 0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])
    assert a[0].dtype == torch.float32 and a[0].shape == (1024, 64)


# ----------------------------------------------------------------------------
# distributional-stability diagnostic
# ----------------------------------------------------------------------------

def test_tail_histogram_bruteforce_and_identities():
    """Counts against a per-element loop with explicit bin arithmetic; the
    deviations y sum to zero over each block (so their mean is 0); the total
    count is (tokens) x (keys of unselected blocks)."""
    L, b, d = 40, 8, 3
    rng = np.random.default_rng(40)
    q, k = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    s, lo, hi, nb = 0.7, -2.0, 2.0, 8
    N = 5
    sel = np.array([[0, 2], [1, 3], [2, 4], [0, 1], [3, 4]])
    r = O.tail_score_histogram(q, k, b, sel, s, lo, hi, nb)
    hx = np.zeros(nb + 2, dtype=np.int64)
    hy = np.zeros(nb + 2, dtype=np.int64)
    width = (hi - lo) / nb
    n_tot = 0
    for i in range(N):
        for j in range(N):
            if j in sel[i]:
                continue
            kb = k[j * b:(j + 1) * b]
            cen = kb.mean(axis=0)
            for t in range(i * b, (i + 1) * b):
                for kn in kb:
                    n_tot += 1
                    for h, val in ((hx, s * q[t] @ kn), (hy, s * q[t] @ (kn - cen))):
                        if val < lo:
                            h[0] += 1
                        elif val >= hi:
                            h[-1] += 1
                        else:
                            h[1 + min(nb - 1, int((val - lo) // width))] += 1
    assert (r["hist_x"] == hx).all() and (r["hist_y"] == hy).all()
    assert r["n"] == n_tot == N * b * (N - 2) * b
    assert abs(r["sum_y"]) < 1e-9


def test_tail_histogram_values_on_bin_edges():
    """Hand-worked: d = 1, s = 1, every query 1, so x is the key itself.  Bins of
    [-2, 2) are 0.5 wide and half-open; a value on an inner edge starts the next
    bin, 2 goes to the overflow bin.  Query block 0 (8 tokens) sees block 1's keys
    -2, -1.5, -1, -0.5, 0, 0.5, 1, 2 -> bins 1..7 and overflow, 8 each; query
    block 1 sees block 0's keys -3, 3, -2.25, 1.75, 0.25, -0.75, 1.5, -1.25 ->
    underflow, overflow, underflow, bin 8, bin 5, bin 3, bin 8, bin 2, 8 each."""
    k = np.array([-3, 3, -2.25, 1.75, 0.25, -0.75, 1.5, -1.25,
                  -2, -1.5, -1, -0.5, 0, 0.5, 1, 2], dtype=np.float64)[:, None]
    q = np.ones((16, 1))
    r = O.tail_score_histogram(q, k, 8, np.array([[0], [1]]), 1.0, -2.0, 2.0, 8)
    want = 8 * np.array([2, 1, 2, 2, 1, 2, 1, 1, 2, 2])
    assert r["hist_x"].tolist() == want.tolist()
