"""pisa_block_stats_noalloc: block statistics without any device allocation.

Some callers cannot allocate device memory: hosts that hand a library only
the buffers of one call and forbid cudaMalloc, or loops that cannot take the
device synchronisation an allocation may cause.  For them the library keeps
the statistics pass's scratch in a static device array.  This file checks,
through the C ABI, that two calls in a row give the same statistics as the
workspace entry point pisa_block_stats, and that a shape too large for the
static array is refused.  It is collected last so that a failure here cannot
stop the other GPU tests from running.
"""
import ctypes

import numpy as np
import pytest
import torch

from workloads import WORKLOADS, generate_qkv

pytestmark = pytest.mark.gpu


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    np.testing.assert_allclose(a, b, rtol=1e-4, atol=1e-4 * max(1.0, np.abs(b).max()))


def test_noalloc_block_stats_matches_workspace_entry_point():
    from block_sparse_attention_stats_b200.build import build
    build()
    import block_sparse_attention_stats_b200 as P
    from block_sparse_attention_stats_b200 import _lib

    lib = _lib.load()
    cases = [
        # first call: Wan2.1-like rows with 2 heads, bf16, no covariance
        (WORKLOADS["wan"].with_(H=2), False),
        # second call in a row: different shape, f32, covariance on; the static
        # array still holds the first call's partial sums
        (WORKLOADS["tiny"].with_(L=1000, B=2), True),
    ]
    for wl, cov in cases:
        Q, K, V = (x.cuda() for x in generate_qkv(wl, "cpu"))
        got = P.pisa_block_stats_noalloc(Q, K, V, wl.block_size, want_cov=cov)
        ref = P.pisa_block_stats(Q, K, V, wl.block_size, want_cov=cov)
        P.pisa_device_status()
        for key in ("qbar", "kbar", "vsum", "hbar") + (("cov",) if cov else ()):
            _close(got[key], ref[key])

    # a shape whose scratch exceeds the static array is refused up front
    B, H, L, d = 1, 600, 128, 128
    need = lib.pisa_block_stats_workspace_bytes(B, H, L, d, 64)
    assert need > (32 << 20)
    q = torch.zeros((B, H, L, d), dtype=torch.bfloat16, device="cuda")
    f = torch.zeros((B, H, 2, d), dtype=torch.float32, device="cuda")
    hb = torch.zeros((B, H, d, d), dtype=torch.float32, device="cuda")
    st = lib.pisa_block_stats_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), _lib.PISA_BF16,
                                      B, H, L, d, 64, 0, f.data_ptr(), f.data_ptr(),
                                      f.data_ptr(), hb.data_ptr(), None,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == _lib.PISA_ERR_WORKSPACE
    assert b"scratch" in lib.pisa_last_error()
