"""pisa_block_stats_noalloc: block statistics without any device allocation.

Some callers cannot allocate device memory: hosts that hand a library only
the buffers of one call and forbid cudaMalloc, or loops that cannot take the
device synchronisation an allocation may cause.  For them the library keeps
the statistics pass's scratch in a static device array.  This file checks,
through the C ABI, that calls in a row give bit for bit the statistics of the
workspace entry point pisa_block_stats (same kernels, same reduction order),
that repeated calls leave the device's free memory unchanged, and that a shape
too large for the static array is refused.  It is collected last so that a
failure here cannot stop the other GPU tests from running.
"""
import pytest
import torch

from workloads import WORKLOADS, generate_qkv

pytestmark = pytest.mark.gpu

KEYS = ("qbar", "kbar", "vsum", "hbar", "cov")


def _outputs(ref):
    # preallocated outputs of the same shapes, filled with NaN so that an
    # element the call fails to write cannot match
    return {k: (None if ref[k] is None else torch.full_like(ref[k], float("nan"))) for k in KEYS}


def _assert_equal(got, ref, what):
    for k in KEYS:
        if ref[k] is None:
            assert got[k] is None
            continue
        assert torch.equal(got[k], ref[k]), f"{what}: {k} differs from pisa_block_stats"


def test_noalloc_block_stats_matches_workspace_entry_point():
    from block_sparse_attention_stats_b200.build import build
    build()
    import block_sparse_attention_stats_b200 as P
    from block_sparse_attention_stats_b200 import _lib

    lib = _lib.load()
    cases = [
        # Wan2.1-like rows with 2 heads, bf16, no covariance
        ("wan h2", WORKLOADS["wan"].with_(H=2), False),
        # a different shape, f32 inputs, covariance on, ragged last block; the
        # static array still holds the previous call's partial sums
        ("tiny L1000 B2", WORKLOADS["tiny"].with_(L=1000, B=2), True),
    ]
    runs = []
    for name, wl, cov in cases:
        Q, K, V = (x.cuda() for x in generate_qkv(wl, "cpu"))
        ref = P.pisa_block_stats(Q, K, V, wl.block_size, want_cov=cov)
        out = _outputs(ref)
        got = P.pisa_block_stats_noalloc(Q, K, V, wl.block_size, want_cov=cov, out=out)
        P.pisa_device_status()
        _assert_equal(got, ref, name)
        runs.append((name, wl, cov, (Q, K, V), ref, out))

    # two more calls in a row, into fresh NaN-filled outputs, with the device's
    # free memory measured around them: nothing may be allocated
    for _, _, _, _, _, out in runs:
        for k in KEYS:
            if out[k] is not None:
                out[k].fill_(float("nan"))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch_alloc0 = torch.cuda.memory_allocated()
    for name, wl, cov, (Q, K, V), ref, out in runs:
        P.pisa_block_stats_noalloc(Q, K, V, wl.block_size, want_cov=cov, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    assert torch.cuda.memory_allocated() == torch_alloc0
    P.pisa_device_status()
    for name, wl, cov, _, ref, out in runs:
        _assert_equal(out, ref, name + " (second call)")

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
