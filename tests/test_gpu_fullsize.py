"""GPU parity at the full video-scale workloads, on sampled heads and query blocks.

The whole problem (all heads) runs on the GPU exactly as the benchmark runs
it; the oracle recomputes two heads' statistics in full and a seeded sample
of query blocks (always the first and the last, partial, block).  The inputs
are generated on the GPU; the sampled heads are regenerated on the CPU and
must agree bitwise, so the oracle sees the same bytes.
"""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import WORKLOADS, generate_head, generate_qkv
from tests.parity_util import (MAX_ABS_TOL, REL_FRO_TOL, block_rows, compare_selection,
                               output_errors, to64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from block_sparse_attention_stats_b200.build import build
    build()
    import block_sparse_attention_stats_b200 as P
    return P


def sample_blocks(N: int, n: int, seed: int):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, N - 1), size=min(n - 2, N - 2), replace=False)
    return sorted(set([0, N - 1] + [int(x) for x in mid]))


@pytest.mark.parametrize("name", ["wan", "hunyuan", "flux", "wan_b128"])
def test_fullsize_sampled(P, name):
    wl = WORKLOADS[name]
    Q, K, V = generate_qkv(wl, "cuda")
    out = P.pisa_attention_ex(Q, K, V, wl.density, wl.block_size, wl.sink_idx, wl.mode,
                              cov_weight=wl.cov_weight)
    st = P.pisa_block_stats(Q, K, V, wl.block_size, want_cov=wl.cov_weight != 0.0)
    idx = P.pisa_select(st["qbar"], st["kbar"], wl.density, wl.sink_idx, cov=st["cov"],
                        cov_weight=wl.cov_weight)
    P.pisa_device_status()
    N = O.block_partition(wl.L, wl.block_size)[0]
    for (b, h) in [(0, 0), (0, wl.H - 1)]:
        q, k, v = generate_head(wl, b, h, "cpu")
        assert torch.equal(q, Q[b, h].cpu()) and torch.equal(k, K[b, h].cpu()) \
            and torch.equal(v, V[b, h].cpu()), "CPU and GPU generators disagree"
        blocks = sample_blocks(N, 16, 1000 + h)
        r = O.pisa_attention_head(to64(q), to64(k), to64(v), wl.block_size, wl.density,
                                  wl.sink_idx, wl.mode, cov_weight=wl.cov_weight,
                                  query_blocks=blocks)
        rep = compare_selection(idx[b, h].cpu().numpy()[blocks], r, wl.scale, wl.cov_weight,
                                wl.sink_idx)
        assert not rep.bad_rows, f"{name} head {h}: selection differs in blocks {rep.bad_rows}"
        keep = [i for i in blocks if i not in rep.tie_rows]
        rows = block_rows(wl.L, wl.block_size, keep)
        ma, rf = output_errors(to64(out[b, h])[rows], r["out"][rows])
        assert ma <= MAX_ABS_TOL and rf <= REL_FRO_TOL, (name, h, ma, rf)
        np.testing.assert_allclose(to64(st["hbar"][b, h]), r["hbar"], rtol=0,
                                   atol=1e-4 * max(1.0, np.abs(r["hbar"]).max()))
