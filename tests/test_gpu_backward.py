"""GPU parity of the zeroth-order backward (and of the forward's lse) against
the fp64 gradient oracle.

The selection both sides use is the oracle's (passed to the kernels as idx);
the block statistics are the library's own (their parity is tested with the
forward).  Tolerances per gradient tensor, as for the forward output:
relative Frobenius error <= 1e-2 and max-abs error <= 2e-2 * max |reference|.
Error budget: bf16 operands of the P.dout, dz.q and dz.k products (relative
2^-9 per element, averaged over the contraction) and bf16 rounding of the
results (2^-9).  Delta_t has two routes, both tested: formed in f32 from
the kernel's own P and dP (an extra sweep; sum_m dz_tm then cancels to f32
rounding), or as dout_t . o_t from the forward's float32 output.  For the
second the forward normalises o_t by the sum of the same bf16-rounded weights
its numerator uses, so Delta_t differs from the backward's sum_m P_tm dP_tm
only through each weight's deviation from their common rounding factor; when
one key holds nearly all the weight (the L=65 and L=129 cases below) that
deviation vanishes.  Forming Delta_t from the bf16 output instead would add
2^-9 |dout_t| |o_t| to every dz_tm: 12% of dq in the L=65 case.
"""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import WORKLOADS, generate_head
from tests.parity_util import to64

pytestmark = pytest.mark.gpu

REL_FRO = 1e-2
MAX_ABS_REL = 2e-2


@pytest.fixture(scope="module")
def P():
    from block_sparse_attention_stats_b200.build import build
    build()
    import block_sparse_attention_stats_b200 as P
    return P


def _oracle_selection(q, k, v, wl, rows=None):
    st = O.block_stats(q, k, v, wl.block_size)
    N = st["kbar"].shape[0]
    k_sel = O.num_selected(N, wl.density)
    rows = list(range(N)) if rows is None else rows
    sc = O.selection_scores(st["qbar"], st["kbar"], wl.scale, None, 0.0, rows)
    sel = np.tile(np.arange(k_sel), (N, 1))
    sel[rows] = O.select_blocks(sc, k_sel, wl.sink_idx)
    return sel


def _errs(a, e):
    a, e = np.asarray(a, np.float64), np.asarray(e, np.float64)
    den = max(np.linalg.norm(e), 1e-30)
    return np.linalg.norm(a - e) / den, np.abs(a - e).max() / max(np.abs(e).max(), 1e-30)


def _gpu_head(P, wl, Q, K, V, G, sel, o32=True):
    """Forward (mode 0th, with lse) and backward of one head through the C ABI;
    with o32 the backward's Delta comes from the forward's float32 output."""
    q, k, v, g = (x.view(1, 1, wl.L, wl.d).cuda() for x in (Q, K, V, G))
    st = P.pisa_block_stats(q, k, v, wl.block_size)
    idx = torch.from_numpy(sel.astype(np.int32)).view(1, 1, sel.shape[0], -1).cuda()
    of = torch.empty(q.shape, dtype=torch.float32, device="cuda") if o32 else None
    out, lse = P.pisa_sparse_attention_fwd(q, k, v, st["kbar"], st["vsum"], st["hbar"], idx,
                                           "0th", wl.block_size, wl.scale, out_f32=of)
    if o32:
        # the float32 copy is the output before its rounding to bf16
        assert torch.equal(of.to(torch.bfloat16), out)
    dq, dk, dv = P.pisa_sparse_attention_bwd(q, k, v, g, lse, st["kbar"], st["vsum"], idx,
                                             wl.block_size, wl.scale, out_f32=of)
    P.pisa_device_status()
    return [to64(x[0, 0]) for x in (out, dq, dk, dv)] + [lse[0, 0].double().cpu().numpy()]


def _lse_bound(q64, k64, v64, wl, tok, rounded_sum=False):
    """|lse error| <= max over the row's keys of the logit error (d lse / d z_m
    = P_m sums to 1).  Exact logits: f32 sums of exact bf16 products (~1e-6
    relative); centroid logits: kbar_j enters the tensor cores rounded to bf16,
    so |dz| <= 2^-9 s sum_c |q_c kbar_jc|.  Per token: that bound over all j,
    plus 1e-5 for the f32 sums and the log.  When the forward sums the
    bf16-rounded weights (it keeps a float32 output), each weight is off by at
    most 2^-9 relative, so D_t is too and ln D_t moves by at most 2^-9 more."""
    kbar = O.block_stats(q64, k64, v64, wl.block_size)["kbar"]
    return (2.0 ** -9 * wl.scale * (np.abs(q64[tok]) @ np.abs(kbar).T).max(axis=1) + 1e-5
            + (2.0 ** -9 if rounded_sum else 0.0))


def _dout(wl, b, h):
    return generate_head(wl.with_(seed=wl.seed + 7919), b, h, "cpu")[2]


def _check_head(P, wl, b, h, o32=True):
    Q, K, V = generate_head(wl, b, h, "cpu")
    G = _dout(wl, b, h)
    q64, k64, v64, g64 = to64(Q), to64(K), to64(V), to64(G)
    sel = _oracle_selection(q64, k64, v64, wl)
    out, dq, dk, dv, lse = _gpu_head(P, wl, Q, K, V, G, sel, o32)
    r = O.zeroth_order_backward(q64, k64, v64, g64, wl.block_size, sel, wl.scale)
    rep = {}
    for name, a, e in (("out", out, r["out"]), ("dq", dq, r["dq"]), ("dk", dk, r["dk"]),
                       ("dv", dv, r["dv"])):
        rf, ma = _errs(a, e)
        rep[name] = (rf, ma)
        assert rf <= REL_FRO and ma <= MAX_ABS_REL, f"{name} head {(b, h)}: rel-fro {rf:.3g}, max {ma:.3g}"
    tok = np.arange(wl.L)
    bad = np.abs(lse - r["lse"]) > _lse_bound(q64, k64, v64, wl, tok, o32)
    assert not bad.any(), f"lse off at tokens {np.nonzero(bad)[0][:8]}"
    return rep


@pytest.mark.parametrize("L,d,density,sink", [
    (1000, 128, 0.2, -1),      # ragged last block (40 tokens), sink = last block
    (777, 64, 0.25, 0),        # d = 64, sink = first block
    (4673, 128, 0.125, None),  # one-token last block, no sink
    (65, 64, 0.5, -1),         # N = 2, the sink is a one-token block
    (64, 128, 0.2, None),      # N = 1: no tail at all
    (640, 128, 1.0, None),     # every block exact: dense attention's gradient
])
@pytest.mark.parametrize("o32", [True, False], ids=["delta_from_out_f32", "delta_sweep"])
def test_backward_matches_oracle(P, L, d, density, sink, o32):
    wl = WORKLOADS["flux"].with_(B=1, H=1, L=L, d=d, density=density, sink_idx=sink,
                                 cov_weight=0.0, mode="0th", cluster_kind="block")
    _check_head(P, wl, 0, 0, o32)


@pytest.mark.parametrize("L,d,density,sink", [
    (4608, 128, 0.15, -1),     # FLUX-like shape, 36 blocks of 128 tokens
    (1000, 128, 0.25, None),   # last block 104 tokens: its second tile is partial
    (777, 64, 0.25, 0),        # d = 64; last block 9 tokens in one tile, odd tile count
    (129, 128, 0.5, -1),       # N = 2 with a one-token sink block
])
@pytest.mark.parametrize("o32", [True, False], ids=["delta_from_out_f32", "delta_sweep"])
def test_backward_block_size_128(P, L, d, density, sink, o32):
    """128-token blocks: dq per query block (both halves share S_i), dk/dv per key
    block over the query tiles of the blocks that selected it, centroid gradients
    with n_j = 128."""
    wl = WORKLOADS["flux"].with_(B=1, H=1, L=L, d=d, block_size=128, density=density,
                                 sink_idx=sink, cov_weight=0.0, mode="0th",
                                 cluster_kind="image" if L == 4608 else "block")
    _check_head(P, wl, 0, 0, o32)


def test_single_token(P):
    """L = 1: the output is v_0 whatever q and k are, so the exact gradient is
    dq = 0, dk = 0, dv = dout (a relative comparison is meaningless at 0)."""
    wl = WORKLOADS["flux"].with_(B=1, H=1, L=1, d=128, density=0.2, sink_idx=0,
                                 cov_weight=0.0, mode="0th", cluster_kind="block")
    Q, K, V = generate_head(wl, 0, 0, "cpu")
    G = _dout(wl, 0, 0)
    out, dq, dk, dv, lse = _gpu_head(P, wl, Q, K, V, G, np.zeros((1, 1), dtype=np.int64))
    # |dz| = P dP (1 - P) with 1 - P at f32 rounding of exp(z - lse)
    bound = 1e-5 * wl.scale * np.abs(to64(G)).sum() * np.abs(to64(V)).max() * np.abs(to64(K)).max()
    assert np.abs(dq).max() <= bound and np.abs(dk).max() <= bound
    np.testing.assert_array_equal(dv, to64(G))
    np.testing.assert_array_equal(out, to64(V))
    q64 = to64(Q)[0]
    assert abs(lse[0] - wl.scale * q64 @ to64(K)[0]) <= 1e-5 * (1 + abs(lse[0]))


def test_backward_flux_shape_two_heads(P):
    """FLUX-like shape (L=4608, d=128, density 0.15, sink -1), two heads."""
    wl = WORKLOADS["flux"].with_(H=2, cov_weight=0.0, mode="0th")
    for h in range(2):
        _check_head(P, wl, 0, h)


def test_autograd_entry_point_and_reproducibility(P):
    """piecewise_sparse_attention_0th (the trainable API) gives the gradients of
    the low-level calls bit for bit, and a second run repeats them exactly."""
    wl = WORKLOADS["flux"].with_(B=2, H=2, L=1500, d=128, density=0.2, sink_idx=-1,
                                 cov_weight=0.0, mode="0th", cluster_kind="block")
    from workloads import generate_qkv
    Q, K, V = (x.cuda() for x in generate_qkv(wl, "cpu"))
    G = torch.randn(Q.shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).cuda()
    grads = []
    for _ in range(2):
        q, k, v = (x.clone().requires_grad_(True) for x in (Q, K, V))
        out = P.piecewise_sparse_attention_0th(q, k, v, density=wl.density, block_size=64,
                                               sink_idx=-1)
        out.backward(G)
        grads.append((out.detach(), q.grad, k.grad, v.grad))
    for a, b in zip(grads[0], grads[1]):
        assert torch.equal(a, b)
    st = P.pisa_block_stats(Q, K, V, 64)
    idx = P.pisa_select(st["qbar"], st["kbar"], wl.density, -1)
    of = torch.empty(Q.shape, dtype=torch.float32, device="cuda")
    out, lse = P.pisa_sparse_attention_fwd(Q, K, V, st["kbar"], st["vsum"], st["hbar"], idx, "0th",
                                           out_f32=of)
    ref = P.pisa_sparse_attention_bwd(Q, K, V, G, lse, st["kbar"], st["vsum"], idx, out_f32=of)
    assert torch.equal(out, grads[0][0])
    for a, b in zip(ref, grads[0][1:]):
        assert torch.equal(a, b)
    # without the float32 copy the forward is the whole-path entry point's
    out_plain, _ = P.pisa_sparse_attention_fwd(Q, K, V, st["kbar"], st["vsum"], st["hbar"], idx,
                                               "0th")
    assert torch.equal(P.pisa_attention(Q, K, V, wl.density, 64, -1, "0th"), out_plain)


def test_lse_of_hyd_equals_zeroth_order(P):
    """D_t has no first-order term: the hyd forward writes the same lse."""
    wl = WORKLOADS["flux"].with_(H=1, L=2000)
    Q, K, V = (x.view(1, 1, wl.L, wl.d).cuda() for x in generate_head(wl, 0, 0, "cpu"))
    st = P.pisa_block_stats(Q, K, V, 64)
    idx = P.pisa_select(st["qbar"], st["kbar"], wl.density, -1)
    _, l0 = P.pisa_sparse_attention_fwd(Q, K, V, st["kbar"], st["vsum"], st["hbar"], idx, "0th")
    _, l1 = P.pisa_sparse_attention_fwd(Q, K, V, st["kbar"], st["vsum"], st["hbar"], idx, "hyd")
    assert torch.equal(l0, l1)


def test_wan_full_size_sampled(P):
    """Full Wan 2.1 sequence (L=75600, d=128), one head, with dout zero outside
    every 197th query block.  Rows with dout_t = 0 contribute nothing to any
    gradient (dP_t = 0, Delta_t = 0), so the full-size dq, dk and dv equal the
    oracle's gradients of the sum over the sampled query blocks alone, and are
    compared over all 75600 rows."""
    wl = WORKLOADS["wan"].with_(mode="0th")
    b, h = 0, 11
    Q, K, V = generate_head(wl, b, h, "cpu")
    N = -(-wl.L // 64)
    rows = list(range(0, N, 197))
    G = torch.zeros_like(Q)
    G_full = _dout(wl, b, h)
    for i in rows:
        G[64 * i:64 * (i + 1)] = G_full[64 * i:64 * (i + 1)]
    q64, k64, v64, g64 = to64(Q), to64(K), to64(V), to64(G)
    sel = _oracle_selection(q64, k64, v64, wl, rows)
    # the other rows keep the fixed selection {0 .. k_sel-1}; with dout = 0 there
    # they enter no gradient
    out, dq, dk, dv, lse = _gpu_head(P, wl, Q, K, V, G, sel)
    r = O.zeroth_order_backward(q64, k64, v64, g64, 64, sel, wl.scale, query_blocks=rows)
    tok = r["rows"]
    for name, a, e in (("out", out[tok], r["out"][tok]), ("dq", dq, r["dq"]), ("dk", dk, r["dk"]),
                       ("dv", dv, r["dv"])):
        rf, ma = _errs(a, e)
        assert rf <= REL_FRO and ma <= MAX_ABS_REL, f"{name}: rel-fro {rf:.3g}, max {ma:.3g}"
    assert not (np.abs(lse[tok] - r["lse"][tok]) > _lse_bound(q64, k64, v64, wl, tok, True)).any()
    other = np.setdiff1d(np.arange(wl.L), tok)
    assert not dq[other].any()
