"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The self-test kernel waits on an mbarrier that nothing completes, with the
library's own bounded wait and a 10 ms limit.  The host must read
PISA_ERR_TIMEOUT from the device status word, the status must clear, and the
context must stay usable for a normal call afterwards.
"""
import pytest
import torch

from workloads import WORKLOADS, generate_qkv

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from block_sparse_attention_stats_b200.build import build
    build()
    import block_sparse_attention_stats_b200 as P
    from block_sparse_attention_stats_b200 import _lib

    P.pisa_device_status()                       # clean before
    P.pisa_selftest_timeout(10_000_000)
    with pytest.raises(P.PisaError) as ei:
        P.pisa_device_status()
    assert ei.value.status == _lib.PISA_ERR_TIMEOUT
    P.pisa_device_status()                       # the word was cleared
    wl = WORKLOADS["flux"].with_(H=1, L=512, cluster_kind="block", cov_weight=0.0)
    Q, K, V = (x.cuda() for x in generate_qkv(wl, "cpu"))
    out = P.pisa_attention(Q, K, V, 0.25)
    P.pisa_device_status()
    assert torch.isfinite(out.float()).all()
    with pytest.raises(P.PisaError):
        P.pisa_selftest_timeout(0)
