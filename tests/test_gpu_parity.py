"""GPU parity: libpisa (through the C ABI) against the fp64 oracle.

Inputs come from the seeded generator on the CPU and are copied to the GPU;
nothing the oracle sees comes from the CUDA path.  Selection must match the
oracle exactly except for certified rounding ties (reported, never hidden);
outputs must match within max-abs 2e-2 and relative Frobenius 1e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from workloads import WORKLOADS, generate_qkv, generate_head
from tests.parity_util import (MAX_ABS_TOL, REL_FRO_TOL, compare_selection, output_errors,
                               to64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from block_sparse_attention_stats_b200.build import build
    build()
    import block_sparse_attention_stats_b200 as P
    return P


def _run_case(P, wl, value_mode="normal", check_stats=True, heads=None):
    """Full path on the GPU vs the oracle for every head of `wl`."""
    Q, K, V = generate_qkv(wl, "cpu", value_mode=value_mode)
    q, k, v = (x.cuda() for x in (Q, K, V))
    out = P.pisa_attention_ex(q, k, v, wl.density, wl.block_size, wl.sink_idx, wl.mode,
                              cov_weight=wl.cov_weight)
    st = P.pisa_block_stats(q, k, v, wl.block_size, want_cov=wl.cov_weight != 0.0)
    idx = P.pisa_select(st["qbar"], st["kbar"], wl.density, wl.sink_idx, cov=st["cov"],
                        cov_weight=wl.cov_weight)
    P.pisa_device_status()
    out64, idx_np = to64(out), idx.cpu().numpy()
    ties = 0
    for b in range(wl.B):
        for h in range(wl.H):
            if heads is not None and (b, h) not in heads:
                continue
            r = O.pisa_attention_head(to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]),
                                      wl.block_size, wl.density, wl.sink_idx, wl.mode,
                                      cov_weight=wl.cov_weight)
            if check_stats:
                for key in ("qbar", "kbar", "vsum"):
                    np.testing.assert_allclose(to64(st[key][b, h]), r[key], rtol=1e-4,
                                               atol=1e-4 * max(1.0, np.abs(r[key]).max()))
                hb = r["hbar"]
                np.testing.assert_allclose(to64(st["hbar"][b, h]), hb, rtol=0,
                                           atol=1e-4 * max(1.0, np.abs(hb).max()))
                if wl.cov_weight != 0.0:
                    np.testing.assert_allclose(to64(st["cov"][b, h]), r["cov"], rtol=1e-4)
            rep = compare_selection(idx_np[b, h], r, wl.scale, wl.cov_weight, wl.sink_idx)
            assert not rep.bad_rows, f"head {(b, h)}: selection differs in rows {rep.bad_rows[:8]}"
            ties += len(rep.tie_rows)
            rows = np.ones(wl.L, dtype=bool)
            for i in rep.tie_rows:
                rows[i * wl.block_size:(i + 1) * wl.block_size] = False
            ma, rf = output_errors(out64[b, h][rows], r["out"][rows])
            assert ma <= MAX_ABS_TOL and rf <= REL_FRO_TOL, \
                f"head {(b, h)}: max-abs {ma:.3g}, rel-fro {rf:.3g}"
    return ties


def test_tiny_f32(P):
    """The small f32 workload of the benchmark (d=64, 16 blocks, density 0.25)."""
    assert _run_case(P, WORKLOADS["tiny"]) == 0


def test_flux_covariance_two_heads(P):
    """FLUX-like shape (L=4608, d=128, covariance-aware scoring, sink=-1), 2 heads."""
    assert _run_case(P, WORKLOADS["flux"].with_(H=2)) == 0


@pytest.mark.parametrize("density", [0.05, 0.10, 0.25, 1.0])
def test_flux_zeroth_order_density_sweep(P, density):
    assert _run_case(P, WORKLOADS["flux_0th"].with_(H=2, density=density)) == 0


@pytest.mark.parametrize("L,sink,mode,d", [
    (1000, None, "hyd", 128),   # ragged last block of 40 tokens
    (4673, -1, "hyd", 128),     # sink is a 1-token block
    (777, 0, "0th", 64),
    (65, -1, "hyd", 64),        # N = 2
    (64, None, "hyd", 128),     # N = 1
    (1, 0, "0th", 128),         # a single token
    (3000, None, "hyd", 64),
])
def test_ragged_and_degenerate(P, L, sink, mode, d):
    wl = WORKLOADS["flux"].with_(B=2, H=2, L=L, d=d, sink_idx=sink, mode=mode, cov_weight=0.1,
                                 cluster_kind="block", density=0.2)
    assert _run_case(P, wl) == 0


@pytest.mark.parametrize("L,d,sink,mode,cov", [
    (4608, 128, -1, "hyd", 0.1),    # FLUX-like shape, 36 blocks of 128 tokens
    (1000, 128, None, "hyd", 0.0),  # last block 104 tokens: its second tile is partial
    (4673, 128, -1, "0th", 0.1),    # last block 65 tokens: its second tile holds 1 token
    (900, 64, 0, "hyd", 0.1),       # last block 4 tokens in one tile; odd tile count
    (129, 128, -1, "hyd", 0.0),     # N = 2 with a one-token sink block
    (100, 64, None, "0th", 0.0),    # N = 1
])
def test_block_size_128(P, L, d, sink, mode, cov):
    """128-token blocks: statistics, selection and attention at block level,
    exact tiles of 64 tokens, centroids with n_j = 128."""
    wl = WORKLOADS["flux"].with_(B=2, H=2, L=L, d=d, block_size=128, sink_idx=sink, mode=mode,
                                 cov_weight=cov, cluster_kind="block", density=0.2)
    assert _run_case(P, wl) == 0


@pytest.mark.parametrize("L,d,sink,mode,cov", [
    (4608, 128, -1, "hyd", 0.1),    # FLUX-like shape, 36 blocks of 128 tokens
    (1000, 128, None, "hyd", 0.0),  # last block 104 tokens
    (4673, 128, -1, "0th", 0.1),    # last block 65 tokens
    (900, 64, 0, "hyd", 0.1),       # odd tile count, d = 64
    (129, 128, -1, "hyd", 0.0),     # N = 2
    (100, 64, None, "0th", 0.0),    # N = 1
    (70000, 128, None, "hyd", 0.0), # 547 blocks: the separate step takes its two-pass path
])
def test_block_size_128_selection_in_fused_kernel(P, L, d, sink, mode, cov):
    """With 128-token blocks the fused kernel can select inside (each CTA is
    one query block).  Up to 512 blocks the separate step scores with the same
    float32 FMA chain, so the sets and the outputs are equal bit for bit.  On
    longer rows the separate step's scores come from the tensor cores: a row
    may differ only where the oracle certifies a rounding tie, and rows that
    agree give the same output rows bit for bit.  The fused sets match the
    oracle."""
    wl = WORKLOADS["flux"].with_(B=1, H=2, L=L, d=d, block_size=128, sink_idx=sink, mode=mode,
                                 cov_weight=cov, cluster_kind="block", density=0.2)
    Q, K, V = generate_qkv(wl, "cpu")
    q, k, v = (x.cuda() for x in (Q, K, V))
    N = -(-L // 128)
    k_sel = O.num_selected(N, wl.density)
    idx_f = torch.full((1, 2, N, k_sel), -1, dtype=torch.int32, device="cuda")
    idx_s = torch.full_like(idx_f, -1)
    out_f = P.pisa_attention_ex(q, k, v, wl.density, 128, sink, mode, cov_weight=cov,
                                fuse_select=True, idx_out=idx_f)
    out_s = P.pisa_attention_ex(q, k, v, wl.density, 128, sink, mode, cov_weight=cov,
                                idx_out=idx_s)
    P.pisa_device_status()
    if N <= 512:
        assert torch.equal(idx_f, idx_s)
        assert torch.equal(out_f, out_s)
    else:
        for h in range(2):
            diff = (idx_f[0, h] != idx_s[0, h]).any(-1).cpu().numpy()
            if diff.any():
                st = O.block_stats(to64(Q[0, h]), to64(K[0, h]), to64(V[0, h]), 128)
                rows = list(range(N))
                sc = O.selection_scores(st["qbar"], st["kbar"], wl.scale, None, 0.0, rows)
                orc = dict(qbar=st["qbar"], kbar=st["kbar"], cov=None, rows=np.asarray(rows),
                           idx=O.select_blocks(sc, k_sel, sink), scores=sc)
                rep = compare_selection(idx_s[0, h].cpu().numpy(), orc, wl.scale, 0.0, sink)
                assert not rep.bad_rows, rep.bad_rows
                assert set(np.nonzero(diff)[0]) <= set(rep.tie_rows)
            same = np.repeat(~diff, 128)[:L]
            assert torch.equal(out_f[0, h][torch.from_numpy(same).cuda()],
                               out_s[0, h][torch.from_numpy(same).cuda()])
    heads = [(0, 0), (0, 1)] if L < 20000 else [(0, 1)]
    for (b, h) in heads:
        r = O.pisa_attention_head(to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]), 128, wl.density,
                                  sink, mode, cov_weight=cov)
        rep = compare_selection(idx_f[b, h].cpu().numpy(), r, wl.scale, cov, sink)
        assert not rep.bad_rows and not rep.tie_rows, (rep.bad_rows, rep.tie_rows)
        ma, rf = output_errors(to64(out_f[b, h]), r["out"])
        assert ma <= MAX_ABS_TOL and rf <= REL_FRO_TOL, (h, ma, rf)


def test_selection_in_fused_kernel_needs_128_token_blocks(P):
    wl = WORKLOADS["flux"].with_(H=1, L=1000, cluster_kind="block")
    Q, K, V = (x.cuda() for x in generate_qkv(wl, "cpu"))
    with pytest.raises(RuntimeError):
        P.pisa_attention_ex(Q, K, V, wl.density, 64, wl.sink_idx, "hyd", fuse_select=True)


def test_block_size_128_f32(P):
    """f32 inputs with 128-token blocks (the f32 statistics kernels)."""
    assert _run_case(P, WORKLOADS["tiny"].with_(block_size=128, cov_weight=0.1)) == 0


@pytest.mark.parametrize("L,d,sink,cov", [(4608, 128, -1, 0.1), (1000, 128, None, 0.0),
                                          (777, 64, 0, 0.0)])
def test_blockwise_first_order(P, L, d, sink, cov):
    """Mode 1st: every unselected block through its own first-order expansion
    (linear values make the H_j large and distinct)."""
    wl = WORKLOADS["flux"].with_(H=2, L=L, d=d, sink_idx=sink, cov_weight=cov, mode="1st",
                                 cluster_kind="image" if L == 4608 else "block")
    assert _run_case(P, wl, value_mode="linear") == 0


def test_linear_values_first_order_visible(P):
    """V = K W + noise makes Hbar large, so the hyd term is exercised."""
    wl = WORKLOADS["flux"].with_(H=2, L=2048, cluster_kind="block", cov_weight=0.0,
                                 sink_idx=None, density=0.125)
    assert _run_case(P, wl, value_mode="linear") == 0


def test_exact_score_ties_go_to_lower_index(P):
    """Blocks 8..15 repeat blocks 0..7, so their scores are bit-identical on both
    sides.  With k_sel = 3 the k-th place falls inside a pair of equal scores
    and the lower index must win."""
    wl = WORKLOADS["flux"].with_(H=1, L=1024, cov_weight=0.0, sink_idx=None, density=3 / 16,
                                 cluster_kind="block")
    Q, K, V = generate_qkv(wl, "cpu")
    for X in (Q, K, V):
        X[:, :, 512:] = X[:, :, :512]
    q, k, v = (x.cuda() for x in (Q, K, V))
    st = P.pisa_block_stats(q, k, v)
    idx = P.pisa_select(st["qbar"], st["kbar"], wl.density).cpu().numpy()[0, 0]
    P.pisa_device_status()
    r = O.pisa_attention_head(to64(Q[0, 0]), to64(K[0, 0]), to64(V[0, 0]), 64, wl.density,
                              None, "hyd")
    assert idx.shape[1] == 3
    assert (idx == r["idx"]).all()
    for row in idx:
        s = set(int(x) for x in row)
        # a selected duplicate implies its lower twin is selected too
        assert all((j - 8) in s for j in s if j >= 8)


def test_sparse_attention_step_alone(P):
    """pisa_sparse_attention given the oracle's own statistics and selection."""
    wl = WORKLOADS["flux"].with_(H=2, L=2000, cluster_kind="block", sink_idx=-1)
    Q, K, V = generate_qkv(wl, "cpu", value_mode="linear")
    outs = []
    for h in range(2):
        r = O.pisa_attention_head(to64(Q[0, h]), to64(K[0, h]), to64(V[0, h]), 64, wl.density,
                                  -1, "hyd")
        outs.append(r)
    f = lambda key: torch.tensor(np.stack([o[key] for o in outs])[None], dtype=torch.float32,
                                 device="cuda")
    idx = torch.tensor(np.stack([o["idx"] for o in outs])[None], dtype=torch.int32, device="cuda")
    for mode in ("hyd", "0th"):
        out = P.pisa_sparse_attention(Q.cuda(), K.cuda(), V.cuda(), f("kbar"), f("vsum"),
                                      f("hbar"), idx, mode=mode)
        P.pisa_device_status()
        for h in range(2):
            ref = outs[h]["out"] if mode == "hyd" else O.piecewise_attention(
                to64(Q[0, h]), to64(K[0, h]), to64(V[0, h]), 64, outs[h]["idx"],
                dict(kbar=outs[h]["kbar"], vsum=outs[h]["vsum"], hbar=outs[h]["hbar"]),
                wl.scale, "0th")
            ma, rf = output_errors(to64(out[0, h]), ref)
            assert ma <= MAX_ABS_TOL and rf <= REL_FRO_TOL, (mode, h, ma, rf)


@pytest.mark.parametrize("L,d,dtype", [(1024, 64, torch.float32), (2000, 128, torch.bfloat16)])
def test_dense_attention(P, L, d, dtype):
    wl = WORKLOADS["flux"].with_(H=2, L=L, d=d, cluster_kind="block",
                                 dtype="f32" if dtype == torch.float32 else "bf16")
    Q, K, V = generate_qkv(wl, "cpu")
    out = P.pisa_dense_attention(Q.cuda(), K.cuda(), V.cuda())
    P.pisa_device_status()
    for h in range(2):
        ref = O.dense_attention(to64(Q[0, h]), to64(K[0, h]), to64(V[0, h]), wl.scale)
        ma, rf = output_errors(to64(out[0, h]), ref)
        assert ma <= MAX_ABS_TOL and rf <= REL_FRO_TOL


def test_pisa_attention_default_entry_point(P):
    """The allocation-inside entry point equals the caller-workspace one bitwise."""
    wl = WORKLOADS["flux"].with_(H=3, L=3000, cluster_kind="block", cov_weight=0.0)
    Q, K, V = (x.cuda() for x in generate_qkv(wl, "cpu"))
    a = P.pisa_attention(Q, K, V, wl.density, 64, wl.sink_idx, "hyd")
    nbytes = P.pisa_workspace_bytes(1, 3, 3000, 128, 64, wl.density)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    b = P.pisa_attention_ex(Q, K, V, wl.density, 64, wl.sink_idx, "hyd", workspace=ws)
    P.pisa_device_status()
    assert torch.equal(a, b)


@pytest.mark.parametrize("block_size,mode", [(64, "hyd"), (64, "0th"), (128, "hyd")])
def test_identical_keys_per_block_give_dense_attention(P, block_size, mode):
    """When every key of a block is the same vector, each block's centroid is its
    keys and H_j = 0, so the zeroth-order tail is exact and the method equals dense
    softmax attention at any density (including the partial last block, whose
    weight n_j must be its true size).  Compared with the oracle's dense
    attention, which shares no arithmetic with the tail path."""
    L, d = 1000, 128
    wl = WORKLOADS["flux"].with_(H=2, L=L, d=d, block_size=block_size, density=0.15,
                                 sink_idx=-1, mode=mode, cov_weight=0.0, cluster_kind="block")
    Q, K, V = generate_qkv(wl, "cpu")
    for s0 in range(0, L, block_size):
        K[:, :, s0:s0 + block_size] = K[:, :, s0:s0 + 1]
    q, k, v = (x.cuda() for x in (Q, K, V))
    out = P.pisa_attention_ex(q, k, v, wl.density, block_size, wl.sink_idx, mode)
    P.pisa_device_status()
    for h in range(wl.H):
        ref = O.dense_attention(to64(Q[0, h]), to64(K[0, h]), to64(V[0, h]), wl.scale)
        ma, rf = output_errors(to64(out[0, h]), ref)
        assert ma <= MAX_ABS_TOL and rf <= REL_FRO_TOL, (h, ma, rf)
