"""Python binding of libpisa: argument marshalling only.

Each function has the name of the C entry point it calls (include/pisa.h),
takes CUDA torch tensors, passes their device pointers and the current CUDA
stream, and raises PisaError on a non-OK status.  Every step of the path runs
in libpisa's CUDA kernels; torch only provides device memory and streams.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional, Tuple

import torch

from . import _lib as L

_DT = {torch.bfloat16: L.PISA_BF16, torch.float32: L.PISA_F32}
_MODE = {"hyd": L.PISA_MODE_HYD, "0th": L.PISA_MODE_0TH, "1st": L.PISA_MODE_1ST}


class PisaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = L.load()
        msg = lib.pisa_status_string(status).decode()
        last = lib.pisa_last_error().decode()
        super().__init__(f"{fn}: {msg} (status {status}){' - ' + last if last else ''}")
        self.status = status


def _check(fn: str, status: int):
    if status != L.PISA_OK:
        raise PisaError(fn, status)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _sink(sink_idx: Optional[int]) -> int:
    if sink_idx is None:
        return L.PISA_SINK_NONE
    if sink_idx not in (0, -1):
        raise ValueError("sink_idx must be None, 0 or -1")
    return sink_idx


def _qkv_dims(q, k, v):
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must be [B, H, L, d] with equal shapes")
    if q.dtype != k.dtype or q.dtype != v.dtype or q.dtype not in _DT:
        raise ValueError("q, k, v must share dtype bf16 or float32")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous [B, H, L, d] (the library reads rows of d)")
    return q.shape


def _require(t, shape, dtype, name):
    """A tensor argument the library reads or writes as a dense array."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---- sizes ------------------------------------------------------------------

def pisa_num_blocks(L_: int, block_size: int = 64) -> int:
    return L.load().pisa_num_blocks(L_, block_size)


def pisa_num_selected(N: int, density: float) -> int:
    return L.load().pisa_num_selected(N, float(density))


def pisa_workspace_bytes(B, H, L_, d, block_size, density, dtype=torch.bfloat16,
                         want_cov=False) -> int:
    return L.load().pisa_workspace_bytes(B, H, L_, d, block_size, float(density), _DT[dtype],
                                         int(bool(want_cov)))


# ---- the three steps ----------------------------------------------------------

def pisa_block_stats(q, k, v, block_size: int = 64, want_cov: bool = False,
                     workspace: Optional[torch.Tensor] = None, out: Optional[dict] = None,
                     stream=None):
    """Returns dict(qbar, kbar, vsum [B,H,N,d], hbar [B,H,d,d], cov [B,H,N] or None).
    `out` may pass a dict of preallocated outputs of those shapes."""
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    N = lib.pisa_num_blocks(Ln, block_size)
    f = dict(dtype=torch.float32, device=q.device)
    if out is not None:
        qbar, kbar, vsum, hbar, cov = (out[n] for n in ("qbar", "kbar", "vsum", "hbar", "cov"))
    else:
        qbar, kbar, vsum = (torch.empty((B, H, N, d), **f) for _ in range(3))
        hbar = torch.empty((B, H, d, d), **f)
        cov = torch.empty((B, H, N), **f) if want_cov else None
    need = lib.pisa_block_stats_workspace_bytes(B, H, Ln, d, block_size)
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check("pisa_block_stats", lib.pisa_block_stats(
        _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], B, H, Ln, d, block_size, int(want_cov),
        _ptr(qbar), _ptr(kbar), _ptr(vsum), _ptr(hbar), _ptr(cov), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    return dict(qbar=qbar, kbar=kbar, vsum=vsum, hbar=hbar, cov=cov)


def pisa_block_stats_noalloc(q, k, v, block_size: int = 64, want_cov: bool = False,
                             out: Optional[dict] = None, stream=None):
    """pisa_block_stats for callers that must not allocate device memory: the
    library keeps the scratch partial sums in its own static device array
    (shapes needing more than PISA_NOALLOC_SCRATCH_BYTES are refused).  Calls
    on one device share that array, so order them on one stream."""
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    N = lib.pisa_num_blocks(Ln, block_size)
    f = dict(dtype=torch.float32, device=q.device)
    if out is not None:
        qbar, kbar, vsum, hbar, cov = (out[n] for n in ("qbar", "kbar", "vsum", "hbar", "cov"))
    else:
        qbar, kbar, vsum = (torch.empty((B, H, N, d), **f) for _ in range(3))
        hbar = torch.empty((B, H, d, d), **f)
        cov = torch.empty((B, H, N), **f) if want_cov else None
    _check("pisa_block_stats_noalloc", lib.pisa_block_stats_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], B, H, Ln, d, block_size, int(want_cov),
        _ptr(qbar), _ptr(kbar), _ptr(vsum), _ptr(hbar), _ptr(cov), _stream(stream)))
    return dict(qbar=qbar, kbar=kbar, vsum=vsum, hbar=hbar, cov=cov)


def pisa_select(qbar, kbar, density: float, sink_idx: Optional[int] = None,
                cov: Optional[torch.Tensor] = None, cov_weight: float = 0.0,
                scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Returns idx [B, H, N, k_sel] int32, ascending per row."""
    lib = L.load()
    B, H, N, d = qbar.shape
    s = 1.0 / math.sqrt(d) if scale is None else float(scale)
    k_sel = lib.pisa_num_selected(N, float(density))
    if k_sel < 1:
        raise ValueError("density must be in (0, 1]")
    idx = torch.empty((B, H, N, k_sel), dtype=torch.int32, device=qbar.device) \
        if out is None else out
    need = lib.pisa_select_workspace_bytes(B, H, N)
    ws = workspace if workspace is not None else _workspace(need, qbar.device)
    _check("pisa_select", lib.pisa_select(
        _ptr(qbar), _ptr(kbar), _ptr(cov), float(cov_weight), s, B, H, N, d, float(density),
        _sink(sink_idx), _ptr(idx), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return idx


def pisa_sparse_attention(q, k, v, kbar, vsum, hbar, idx, mode: str = "hyd",
                          block_size: int = 64, scale: Optional[float] = None,
                          out: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream=None):
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    k_sel = idx.shape[-1]
    out = torch.empty_like(q) if out is None else out
    need = lib.pisa_sparse_attention_workspace_bytes(B, H, Ln, d, block_size, _DT[q.dtype])
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check("pisa_sparse_attention", lib.pisa_sparse_attention(
        _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(kbar), _ptr(vsum), _ptr(hbar), _ptr(idx),
        k_sel, B, H, Ln, d, block_size, 0.0 if scale is None else float(scale), _MODE[mode],
        _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return out


def pisa_sparse_attention_fwd(q, k, v, kbar, vsum, hbar, idx, mode: str = "0th",
                              block_size: int = 64, scale: Optional[float] = None,
                              out: Optional[torch.Tensor] = None,
                              lse: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None, stream=None,
                              out_f32: Optional[torch.Tensor] = None):
    """pisa_sparse_attention that also returns lse [B, H, L] float32 (ln D_t).
    `out_f32` (float32 [B, H, L, d]), if given, receives the output before its
    rounding to the input dtype; the backward forms its row term from it."""
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    k_sel = idx.shape[-1]
    _require(out_f32, q.shape, torch.float32, "out_f32")
    _require(lse, (B, H, Ln), torch.float32, "lse")
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, H, Ln, dtype=torch.float32, device=q.device) if lse is None else lse
    need = lib.pisa_sparse_attention_workspace_bytes(B, H, Ln, d, block_size, _DT[q.dtype])
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check("pisa_sparse_attention_fwd", lib.pisa_sparse_attention_fwd(
        _ptr(q), _ptr(k), _ptr(v), _DT[q.dtype], _ptr(kbar), _ptr(vsum), _ptr(hbar), _ptr(idx),
        k_sel, B, H, Ln, d, block_size, 0.0 if scale is None else float(scale), _MODE[mode],
        _ptr(out), _ptr(lse), _ptr(out_f32), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out, lse


def pisa_sparse_attention_bwd(q, k, v, dout, lse, kbar, vsum, idx, block_size: int = 64,
                              scale: Optional[float] = None,
                              grads: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None,
                              workspace: Optional[torch.Tensor] = None, stream=None,
                              out_f32: Optional[torch.Tensor] = None):
    """Gradients (dq, dk, dv) of the zeroth-order forward, bf16 [B, H, L, d].
    With `out_f32` (the forward's float32 output) the row term
    Delta_t = dout_t . out_t comes from it and dq takes one sweep, else two."""
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    if q.dtype != torch.bfloat16:
        raise ValueError("the backward takes bf16 q, k, v, dout")
    _require(dout, q.shape, torch.bfloat16, "dout")
    _require(lse, (B, H, Ln), torch.float32, "lse")
    _require(out_f32, q.shape, torch.float32, "out_f32")
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k),
                                                  torch.empty_like(v))
    for g_, n_ in zip((dq, dk, dv), ("dq", "dk", "dv")):
        _require(g_, q.shape, torch.bfloat16, n_)
    need = lib.pisa_sparse_attention_bwd_workspace_bytes(B, H, Ln, d, block_size, idx.shape[-1])
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check("pisa_sparse_attention_bwd", lib.pisa_sparse_attention_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse), _ptr(out_f32), _ptr(kbar), _ptr(vsum),
        _ptr(idx), idx.shape[-1], B, H, Ln, d, block_size,
        0.0 if scale is None else float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    return dq, dk, dv


class _PiecewiseAttention0th(torch.autograd.Function):
    """Zeroth-order piecewise attention with its backward (every step in libpisa)."""

    @staticmethod
    def forward(ctx, q, k, v, density, block_size, sink_idx, scale):
        if q.dtype != torch.bfloat16:
            raise ValueError("piecewise_sparse_attention_0th trains on bf16 q, k, v")
        q, k, v = (x.contiguous() for x in (q, k, v))
        st = pisa_block_stats(q, k, v, block_size)
        idx = pisa_select(st["qbar"], st["kbar"], density, sink_idx, scale=scale)
        o32 = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        out, lse = pisa_sparse_attention_fwd(q, k, v, st["kbar"], st["vsum"], st["hbar"], idx,
                                             "0th", block_size, scale, out_f32=o32)
        ctx.save_for_backward(q, k, v, lse, o32, st["kbar"], st["vsum"], idx)
        ctx.block_size, ctx.scale = block_size, scale
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, lse, o32, kbar, vsum, idx = ctx.saved_tensors
        dq, dk, dv = pisa_sparse_attention_bwd(q, k, v, dout.contiguous(), lse, kbar, vsum, idx,
                                               ctx.block_size, ctx.scale, out_f32=o32)
        return dq, dk, dv, None, None, None, None


def piecewise_sparse_attention_0th(q, k, v, density: float = 0.15, block_size: int = 64,
                                   sink_idx: Optional[int] = None,
                                   scale: Optional[float] = None) -> torch.Tensor:
    """The authors' trainable zeroth-order variant: bf16 [B, H, L, d] in and out,
    differentiable with respect to q, k and v (selection held fixed)."""
    return _PiecewiseAttention0th.apply(q, k, v, density, block_size, sink_idx, scale)


def piecewise_sparse_attention_hyd(q, k, v, density: float = 0.15, block_size: int = 64,
                                   sink_idx: Optional[int] = None) -> torch.Tensor:
    """The paper version (zeroth-order tail + global first-order term), forward only."""
    return pisa_attention(q, k, v, density, block_size, sink_idx, "hyd")


piecewise_sparse_attention = piecewise_sparse_attention_hyd


# ---- the whole path --------------------------------------------------------------

def pisa_attention(q, k, v, density: float, block_size: int = 64,
                   sink_idx: Optional[int] = None, mode: str = "hyd",
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bf16 piecewise sparse attention with default options (scratch memory is
    allocated stream-ordered inside the library)."""
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    out = torch.empty_like(q) if out is None else out
    _check("pisa_attention", lib.pisa_attention(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Ln, d, block_size, float(density),
        _sink(sink_idx), _MODE[mode], _stream(stream)))
    return out


def pisa_attention_ex(q, k, v, density: float, block_size: int = 64,
                      sink_idx: Optional[int] = None, mode: str = "hyd",
                      scale: Optional[float] = None, cov_weight: float = 0.0,
                      workspace: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, stream=None,
                      fuse_select: bool = False,
                      idx_out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """pisa_attention with options; the workspace (if given) is caller-owned scratch
    of pisa_workspace_bytes(...) bytes and nothing is allocated by the library.
    fuse_select (block_size 128): each CTA of the fused kernel selects its own
    exact blocks.  idx_out: int32 [B, H, N, k_sel] receiving the selection used."""
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    out = torch.empty_like(q) if out is None else out
    opts = L.PisaOptions()
    opts.scale = 0.0 if scale is None else float(scale)
    opts.cov_weight = float(cov_weight)
    opts.dtype = _DT[q.dtype]
    opts.fuse_select = int(bool(fuse_select))
    if idx_out is not None:
        N = lib.pisa_num_blocks(Ln, block_size)
        shape = (B, H, N, lib.pisa_num_selected(N, float(density)))
        if idx_out.dtype != torch.int32 or tuple(idx_out.shape) != shape \
                or not idx_out.is_contiguous() or idx_out.device != q.device:
            raise ValueError(f"idx_out must be a contiguous int32 tensor of shape {shape} "
                             "on the inputs' device")
        opts.idx_out = _ptr(idx_out)
    if workspace is not None:
        opts.workspace = _ptr(workspace)
        opts.ws_bytes = workspace.numel() * workspace.element_size()
    _check("pisa_attention_ex", lib.pisa_attention_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Ln, d, block_size, float(density),
        _sink(sink_idx), _MODE[mode], ctypes.byref(opts), _stream(stream)))
    return out


def pisa_dense_attention(q, k, v, scale: Optional[float] = None,
                         out: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    lib = L.load()
    B, H, Ln, d = _qkv_dims(q, k, v)
    out = torch.empty_like(q) if out is None else out
    need = lib.pisa_dense_attention_workspace_bytes(B, H, Ln, d, _DT[q.dtype])
    ws = workspace if workspace is not None else _workspace(need, q.device)
    _check("pisa_dense_attention", lib.pisa_dense_attention(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _DT[q.dtype], B, H, Ln, d,
        0.0 if scale is None else float(scale), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def pisa_tail_score_histogram(q, k, idx, lo: float = -8.0, hi: float = 8.0, nbins: int = 64,
                              block_size: int = 64, scale: Optional[float] = None,
                              query_stride: int = 1, stream=None):
    """Histograms of the pre-softmax scores x = s q k of the unselected blocks and
    of their deviation y = s q (k - kbar_j) from the block-centroid score; returns
    dict(hist_x, hist_y [nbins + 2] int64 with under/overflow bins, n, mean_x,
    var_x, mean_y, var_y, edges)."""
    lib = L.load()
    B, H, Ln, d = q.shape
    hx = torch.empty(nbins + 2, dtype=torch.int64, device=q.device)
    hy = torch.empty(nbins + 2, dtype=torch.int64, device=q.device)
    mom = torch.empty(5, dtype=torch.float64, device=q.device)
    _check("pisa_tail_score_histogram", lib.pisa_tail_score_histogram(
        _ptr(q), _ptr(k), _DT[q.dtype], _ptr(idx), idx.shape[-1], B, H, Ln, d, block_size,
        0.0 if scale is None else float(scale), float(lo), float(hi), int(nbins),
        int(query_stride), _ptr(hx), _ptr(hy), _ptr(mom), _stream(stream)))
    m = mom.cpu().tolist()
    n = max(m[0], 1.0)
    return dict(hist_x=hx, hist_y=hy, n=m[0], sum_x=m[1], sum_x2=m[2], sum_y=m[3], sum_y2=m[4],
                mean_x=m[1] / n, var_x=m[2] / n - (m[1] / n) ** 2,
                mean_y=m[3] / n, var_y=m[4] / n - (m[3] / n) ** 2,
                edges=torch.linspace(lo, hi, nbins + 1))


def pisa_selftest_timeout(limit_ns: int = 10_000_000, stream=None) -> None:
    """Run the bounded-wait self-test kernel (see include/pisa.h); the following
    pisa_device_status call raises PisaError with status PISA_ERR_TIMEOUT."""
    _check("pisa_selftest_timeout", L.load().pisa_selftest_timeout(int(limit_ns), _stream(stream)))


def pisa_device_status(stream=None) -> None:
    """Synchronise the stream and raise if a kernel flagged a device-side error."""
    _check("pisa_device_status", L.load().pisa_device_status(_stream(stream)))
