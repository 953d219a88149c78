"""The FLOP counts behind the bench's roofline numbers, checked on the CPU
against brute-force loops over (head, query block, key block).

Algorithmic work of the fused kernel per query token of block i (the method's
per-token work, a definition in the bench's docstrings): 4d FLOPs per exact
key of S_i, 4d per centroid of U_i, and in mode hyd 2d^2 per token for q H.
The zeroth-order backward does five products of 2d FLOPs per (token, key)
pair of the augmented softmax.  Blocks hold b tokens except the last.
"""
import numpy as np
import pytest
import torch

import bench
from workloads import WORKLOADS


def _idx(B, H, N, k_sel, seed, force_last=False):
    rng = np.random.default_rng(seed)
    rows = []
    for _ in range(B * H * N):
        pick = rng.choice(N, size=k_sel, replace=False)
        if force_last and N - 1 not in pick:
            pick[0] = N - 1
        rows.append(np.sort(pick))
    return torch.from_numpy(np.asarray(rows, dtype=np.int32)).view(B, H, N, k_sel)


def _brute(wl, idx, per_exact, per_tail, per_token):
    B, H, N, k_sel = idx.shape
    n = [min(wl.block_size, wl.L - wl.block_size * j) for j in range(N)]
    tot = 0.0
    for b in range(B):
        for h in range(H):
            for i in range(N):
                sel = set(int(x) for x in idx[b, h, i])
                for j in range(N):
                    tot += n[i] * (per_exact * n[j] if j in sel else per_tail)
                tot += n[i] * per_token
    return tot


@pytest.mark.parametrize("L,b,d,k_sel,mode,last", [
    (1000, 64, 128, 3, "hyd", True),     # ragged last block, selected by every row
    (1000, 64, 64, 5, "0th", False),
    (4608, 128, 128, 7, "hyd", False),   # 128-token blocks
    (129, 128, 128, 1, "0th", True),     # one-token last block
])
def test_fused_kernel_flops(L, b, d, k_sel, mode, last):
    wl = WORKLOADS["flux"].with_(B=1, H=2, L=L, d=d, block_size=b, mode=mode)
    N = -(-L // b)
    idx = _idx(1, 2, N, k_sel, 1, last)
    want = _brute(wl, idx, 4 * d, 4 * d, 2 * d * d if mode == "hyd" else 0)
    assert bench.k3_algorithmic_flops(wl, idx) == pytest.approx(want, rel=1e-12)


@pytest.mark.parametrize("L,b,k_sel,last", [(1000, 64, 3, True), (777, 64, 4, False),
                                            (1000, 128, 2, True)])
def test_backward_flops(L, b, k_sel, last):
    wl = WORKLOADS["flux"].with_(B=1, H=2, L=L, d=128, block_size=b, mode="0th")
    N = -(-L // b)
    idx = _idx(1, 2, N, k_sel, 2, last)
    want = _brute(wl, idx, 10 * 128, 10 * 128, 0)
    assert bench.bwd_flops(wl, idx)[0] == pytest.approx(want, rel=1e-12)


def test_block_wise_first_order_reads_every_key():
    wl = WORKLOADS["flux"].with_(B=1, H=3, L=1000, d=64, mode="1st")
    idx = _idx(1, 3, 16, 4, 3)
    assert bench.k3_algorithmic_flops(wl, idx) == 4.0 * 64 * 1000 * 1000 * 3


class _FakeNvml:
    """Stands in for pynvml: one GPU whose local CPUs are given as 64-bit words."""

    def __init__(self, words):
        self.words = words
        self.bus_ids = []

    def nvmlInit(self):
        pass

    def nvmlShutdown(self):
        pass

    def nvmlDeviceGetHandleByPciBusId(self, bus_id):
        self.bus_ids.append(bus_id)
        return object()

    def nvmlDeviceGetCpuAffinity(self, handle, n):
        return self.words[:n] + [0] * max(0, n - len(self.words))


class _Props:
    pci_domain_id, pci_bus_id, pci_device_id = 0, 0x1B, 0


def _local_cpus(monkeypatch, words, allowed, ncpu=128):
    import sys
    fake = _FakeNvml(words)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda dev: _Props())
    monkeypatch.setattr(bench.os, "cpu_count", lambda: ncpu)
    monkeypatch.setattr(bench.os, "sched_getaffinity", lambda pid: set(allowed))
    return bench.gpu_local_cpus(0), fake


def test_gpu_local_cpus_decodes_the_mask_and_keeps_allowed_cpus(monkeypatch):
    # CPUs 0-15 and 64-79 are local to the GPU; the process may run on 8-71
    words = [0xFFFF, 0xFFFF]
    got, fake = _local_cpus(monkeypatch, words, range(8, 72))
    assert got == set(range(8, 16)) | set(range(64, 72))
    assert fake.bus_ids == ["00000000:1B:00.0"]


def test_gpu_local_cpus_none_when_the_sets_do_not_meet(monkeypatch):
    got, _ = _local_cpus(monkeypatch, [0xFF], range(32, 48))
    assert got is None


def test_gpu_local_cpus_none_without_nvml(monkeypatch):
    import sys
    monkeypatch.setitem(sys.modules, "pynvml", None)    # import fails
    assert bench.gpu_local_cpus(0) is None
