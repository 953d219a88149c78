"""Counter-based seeded generator for synthetic Q/K/V shaped like DiT attention.

Random numbers
--------------
Every value is a pure function of (seed, tensor tag, batch b, head h, element
counter), so any single head can be regenerated on its own, on the CPU or on a
GPU, without producing the others:

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; the 64-bit finaliser with Stafford's "Mix13"
  constants) keyed per (seed, tag, b, h): draw number c of a stream is
  ``mix64(key + (c + 1) * GAMMA)`` with GAMMA = 0x9E3779B97F4A7C15.
* Standard normals by the Box-Muller transform (Box and Muller, 1958) in
  float64: normal number c uses draws 2c and 2c+1.
* The float64 values are rounded to float32 (round to nearest even) and, for
  bf16 workloads, then to bfloat16 (round to nearest even).

All integer arithmetic is done in torch int64, whose multiplication wraps
modulo 2**64 on both the CPU and CUDA devices, so both devices give the same
64-bit draws.  The transcendental functions of Box-Muller may differ by an ulp
between devices; after rounding to bf16/fp32 this almost never shows, and the
full-size parity test checks the heads it samples for bitwise agreement.

Workload structure
------------------
Clustered queries and keys, as in the image/video DiT workloads of the PISA
pages (FLUX.1-dev image attention with text tokens last; Wan2.1 and
HunyuanVideo video attention over a frames x height x width latent grid):
per (b, h) draw cluster centres c ~ N(0, 1)^d, then
``K_t = c_cl(t) + 0.5 eps``, ``Q_t = c_cl(t) + 0.5 eps'`` and ``V ~ N(0, 1)``.
``cl(t)`` groups tokens into spatial (or spatio-temporal) tiles of the token
grid; text tokens form clusters of 64 consecutive tokens at the end.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX_C1 = 0xBF58476D1CE4E5B9
MIX_C2 = 0x94D049BB133111EB

# tensor tags of the independent streams
TAG_CENTRES = 1
TAG_Q = 2
TAG_K = 3
TAG_V = 4
TAG_W = 5      # linear-value variant: mixing matrix
TAG_E = 6      # linear-value variant: noise

DEFAULT_SEED = 20260202


def _signed(x: int) -> int:
    x &= MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


def _mix64_int(z: int) -> int:
    """SplitMix64 finaliser on a Python int (exact modulo 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX_C1) & MASK64
    z = ((z ^ (z >> 27)) * MIX_C2) & MASK64
    return z ^ (z >> 31)


def _srl(x: torch.Tensor, k: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (x >> k) & ((1 << (64 - k)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _signed(MIX_C1)
    z = (z ^ _srl(z, 27)) * _signed(MIX_C2)
    return z ^ _srl(z, 31)


def stream_key(seed: int, tag: int, b: int, h: int) -> int:
    """64-bit key of the stream for (seed, tensor tag, batch, head)."""
    k = _mix64_int(seed * GAMMA + 1)
    k = _mix64_int(k + tag * GAMMA)
    k = _mix64_int(k + ((b << 20) + h) * GAMMA)
    return k


def stream_uniform_u64(key: int, start: int, count: int,
                       device="cpu") -> torch.Tensor:
    """Draws start .. start+count-1 of the SplitMix64 stream `key` (int64 bit patterns)."""
    c = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = c * _signed(GAMMA) + _signed(key)
    return _mix64(z)


def stream_normal(key: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Standard normals start .. start+count-1 of stream `key`, float64, by Box-Muller."""
    out = torch.empty(count, dtype=torch.float64, device=device)
    chunk = 1 << 22
    two53 = 2.0 ** -53
    for o in range(0, count, chunk):
        n = min(chunk, count - o)
        r = stream_uniform_u64(key, 2 * (start + o), 2 * n, device).view(n, 2)
        u1 = (_srl(r[:, 0], 11) + 1).to(torch.float64) * two53   # (0, 1]
        u2 = _srl(r[:, 1], 11).to(torch.float64) * two53         # [0, 1)
        out[o:o + n] = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
    return out


# ----------------------------------------------------------------------------
# token -> cluster maps
# ----------------------------------------------------------------------------

def cluster_map(kind: str, L: int, grid: Optional[Tuple[int, int, int]] = None,
                tile: Tuple[int, int, int] = (3, 8, 8), image_side: int = 64,
                image_tile: int = 8, text_cluster: int = 64,
                device="cpu") -> Tuple[torch.Tensor, int]:
    """Cluster id of every token and the number of clusters.

    kind = "block": cluster = t div 64.
    kind = "image": the first image_side**2 tokens are a raster image grid cut
      into image_tile x image_tile tiles; the remaining (text) tokens form
      clusters of `text_cluster` consecutive tokens.
    kind = "video": the first F*Y*X tokens are a (frame, y, x) raster grid cut
      into `tile` = (tf, ty, tx) tiles; the remaining (text) tokens form clusters
      of `text_cluster` consecutive tokens.
    """
    t = torch.arange(L, dtype=torch.int64, device=device)
    if kind == "block":
        cl = t // 64
        return cl, int((L + 63) // 64)
    if kind == "image":
        n_img = image_side * image_side
        per_row = (image_side + image_tile - 1) // image_tile
        r, c = t // image_side, t % image_side
        cl = (r // image_tile) * per_row + c // image_tile
        n_img_cl = per_row * per_row
        txt = n_img_cl + (t - n_img) // text_cluster
        cl = torch.where(t < n_img, cl, txt)
        n_txt = max(0, L - n_img)
        return cl, n_img_cl + (n_txt + text_cluster - 1) // text_cluster
    if kind == "video":
        F, Y, X = grid
        tf, ty, tx = tile
        nf, ny, nx = -(-F // tf), -(-Y // ty), -(-X // tx)
        n_vid = F * Y * X
        f, y, x = t // (Y * X), (t // X) % Y, t % X
        cl = ((f // tf) * ny + y // ty) * nx + x // tx
        n_vid_cl = nf * ny * nx
        txt = n_vid_cl + (t - n_vid) // text_cluster
        cl = torch.where(t < n_vid, cl, txt)
        n_txt = max(0, L - n_vid)
        return cl, n_vid_cl + (n_txt + text_cluster - 1) // text_cluster
    raise ValueError(f"unknown cluster map {kind!r}")


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, method parameters and input recipe."""
    name: str
    B: int
    H: int
    L: int
    d: int
    block_size: int
    density: float
    mode: str                      # "hyd", "0th" or "1st" (block-wise first order)
    sink_idx: Optional[int]        # None, 0 or -1
    dtype: str                     # "bf16" or "f32"
    cov_weight: float              # lambda of covariance-aware scoring (0 = off)
    cluster_kind: str
    grid: Optional[Tuple[int, int, int]] = None
    seed: int = DEFAULT_SEED
    noise: float = 0.5
    densities: Tuple[float, ...] = field(default=())

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    # small case the oracle finishes in seconds; clusters = blocks
    "tiny": Workload("tiny", B=1, H=2, L=1024, d=64, block_size=64, density=0.25,
                     mode="hyd", sink_idx=None, dtype="f32", cov_weight=0.0,
                     cluster_kind="block", seed=DEFAULT_SEED + 1),
    # FLUX.1-dev 1024x1024: 64x64 latent image tokens + 512 text tokens last
    "flux": Workload("flux", B=1, H=24, L=4608, d=128, block_size=64, density=0.15,
                     mode="hyd", sink_idx=-1, dtype="bf16", cov_weight=0.1,
                     cluster_kind="image", seed=DEFAULT_SEED + 2),
    "flux_0th": Workload("flux_0th", B=1, H=24, L=4608, d=128, block_size=64,
                         density=0.15, mode="0th", sink_idx=-1, dtype="bf16",
                         cov_weight=0.1, cluster_kind="image", seed=DEFAULT_SEED + 3,
                         densities=(0.05, 0.10, 0.15, 0.25, 1.0)),
    # the same FLUX shape with the block-wise first-order tail ("first-order-only")
    "flux_1st": Workload("flux_1st", B=1, H=24, L=4608, d=128, block_size=64, density=0.15,
                         mode="1st", sink_idx=-1, dtype="bf16", cov_weight=0.1,
                         cluster_kind="image", seed=DEFAULT_SEED + 2),
    # Wan2.1-14B 720p-ish latent video: 21 frames x 45 x 80
    "wan": Workload("wan", B=1, H=40, L=75600, d=128, block_size=64, density=0.125,
                    mode="hyd", sink_idx=None, dtype="bf16", cov_weight=0.0,
                    cluster_kind="video", grid=(21, 45, 80), seed=DEFAULT_SEED + 4),
    # the FLUX and Wan shapes with 128-token blocks (the upper end of the block
    # range the pages give)
    "flux_b128": Workload("flux_b128", B=1, H=24, L=4608, d=128, block_size=128,
                          density=0.15, mode="hyd", sink_idx=-1, dtype="bf16", cov_weight=0.1,
                          cluster_kind="image", seed=DEFAULT_SEED + 2),
    "wan_b128": Workload("wan_b128", B=1, H=40, L=75600, d=128, block_size=128,
                         density=0.125, mode="hyd", sink_idx=None, dtype="bf16",
                         cov_weight=0.0, cluster_kind="video", grid=(21, 45, 80),
                         seed=DEFAULT_SEED + 4),
    # HunyuanVideo-13B 720p: 33 x 45 x 80 video tokens + 256 text tokens last
    "hunyuan": Workload("hunyuan", B=1, H=24, L=33 * 45 * 80 + 256, d=128,
                        block_size=64, density=0.10, mode="hyd", sink_idx=-1,
                        dtype="bf16", cov_weight=0.0, cluster_kind="video",
                        grid=(33, 45, 80), seed=DEFAULT_SEED + 5),
}


def _round_io(x64: torch.Tensor, dtype) -> torch.Tensor:
    x32 = x64.to(torch.float32)
    return x32 if dtype == torch.float32 else x32.to(dtype)


def generate_head(wl: Workload, b: int, h: int, device="cpu",
                  value_mode: str = "normal") -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q, K, V of one (b, h) as [L, d] tensors in the workload's I/O dtype.

    value_mode = "normal": V ~ N(0, 1) (the workloads' recipe).
    value_mode = "linear": V = K W + 0.5 eps with W ~ N(0, 1/d); a test-only
      recipe under which the block first-order matrices are far from zero.
    """
    L, d = wl.L, wl.d
    cl, ncl = cluster_map(wl.cluster_kind, L, grid=wl.grid, device=device)
    centres = stream_normal(stream_key(wl.seed, TAG_CENTRES, b, h), 0, ncl * d,
                            device).view(ncl, d)
    base = centres[cl]
    k64 = base + wl.noise * stream_normal(stream_key(wl.seed, TAG_K, b, h), 0, L * d,
                                          device).view(L, d)
    q64 = base + wl.noise * stream_normal(stream_key(wl.seed, TAG_Q, b, h), 0, L * d,
                                          device).view(L, d)
    del base
    if value_mode == "normal":
        v64 = stream_normal(stream_key(wl.seed, TAG_V, b, h), 0, L * d, device).view(L, d)
    elif value_mode == "linear":
        w = stream_normal(stream_key(wl.seed, TAG_W, b, h), 0, d * d,
                          device).view(d, d) / math.sqrt(d)
        e = stream_normal(stream_key(wl.seed, TAG_E, b, h), 0, L * d, device).view(L, d)
        v64 = k64 @ w + 0.5 * e
    else:
        raise ValueError(value_mode)
    dt = wl.torch_dtype
    return _round_io(q64, dt), _round_io(k64, dt), _round_io(v64, dt)


def generate_qkv(wl: Workload, device="cpu", heads: Optional[Sequence[Tuple[int, int]]] = None,
                 value_mode: str = "normal", pin_memory: bool = False):
    """Q, K, V as [B, H, L, d] tensors (all heads), or a dict {(b, h): (q, k, v)}."""
    if heads is not None:
        return {(b, h): generate_head(wl, b, h, device, value_mode) for (b, h) in heads}
    shape = (wl.B, wl.H, wl.L, wl.d)
    kw = dict(dtype=wl.torch_dtype, device=device)
    if pin_memory and str(device) == "cpu":
        kw["pin_memory"] = True
    Q, K, V = torch.empty(shape, **kw), torch.empty(shape, **kw), torch.empty(shape, **kw)
    for b in range(wl.B):
        for h in range(wl.H):
            q, k, v = generate_head(wl, b, h, device, value_mode)
            Q[b, h].copy_(q)
            K[b, h].copy_(k)
            V[b, h].copy_(v)
    return Q, K, V
