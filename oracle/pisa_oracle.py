"""Plain fp64 CPU oracle of PISA piecewise sparse attention (forward).

TEST INFRASTRUCTURE ONLY -- the CUDA library never calls this module and this
module never imports the CUDA library.  Only the tests, the smoke check and the
CPU-baseline legs of the benchmark use it.

Everything is float64 numpy on one (batch, head) at a time, with arrays shaped
[L, d] (tokens x head dim).  Library primitives used as single steps: matrix
products, ``numpy.lexsort``.  There is no blocking, fusion or reordering beyond
what the definitions below state.

Sources (cited by page title and section):

* [GS] "Technical Summary: PISA - Piecewise Sparse Attention for Efficient
  Diffusion Transformers" (gist.science), section 2 "Methodology":
  - "Core Algorithm": S_i / U_i split, o_t = N_t / D_t, the numerator N_t
    equation and alpha_{t,j} = exp(q_t kbar_j^T);
  - "Global First-Order Correction": Hbar is the mean of the block-wise
    first-order matrices across all blocks;
  - "Covariance-Aware Routing": M_j = || H_j - Hbar ||;
  - "Key Insights" 2, "Normalization Consistency": both approximations enter
    the softmax numerator and denominator;
  - "Hardware Implementation": pre-computation of block centroids, value sums
    and Hbar.
* [GH] "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
  Transformers" (authors' README mirror): "Kernel variants" (_hyd = paper
  version, _0th = zeroth-order only) and "Attention sink for MMDiT" (sink_idx
  None / 0 / -1 forces the first / last K/V block into the exact top-k branch of
  every query block; density, block_size arguments).
* [SK] "Pisa Sparse Attention" (skillmd.com agent skill), "Implementation":
  the covariance weight 0.1 and the Frobenius norm of the covariance term.
* [AT] atlas.scime.ai summary, "Surprising findings": the "first-order-only"
  variant, and [GS] "Global First-Order Correction": a distinct first-order
  term for every unselected block (memory-bound) -- mode "1st" below.

Readings where the pages are silent:

* softmax scale s = 1/sqrt(d) multiplies every q.k product (exact logits, the
  centroid logits, the selection scores and the first-order term s q Hbar);
* the block first-order matrix is the SUM H_j = sum_n (k_{j,n} - kbar_j)^T
  v_{j,n}: expanding exp(s q k_n) to first order about kbar_j gives
  alpha (1 + s q (k_n - kbar_j)^T), whose sum over the block weighted by v_n is
  alpha SigmaV_j + alpha s q H_j, and whose plain sum is alpha n_j (the
  deviations sum to zero); replacing H_j by Hbar gives the three terms of the
  N_t equation, and D_t has no first-order term;
* D_t = sum_{S_i} sum_n exp(s q k) + sum_{U_i} n_j alpha_{t,j};
* Hbar = (1/N) sum over all N blocks (selected or not, partial last included);
* M_j is the Frobenius norm; the selection score is
  s qbar_i . kbar_j + lambda M_j (lambda = cov_weight, 0 disables);
* qbar_i is the arithmetic mean of the queries of block i;
* k_sel = clamp(floor(density N + 1e-6), 1, N); the sink counts inside k_sel;
* ties in the selection go to the lower block index; S_i is output ascending;
* the last block may be partial (n_j < block_size).
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Optional, Sequence

import numpy as np


# ----------------------------------------------------------------------------
# block partition
# ----------------------------------------------------------------------------

def block_partition(L: int, block_size: int):
    """Regular blocks of `block_size` tokens ([SK] "Architecture Overview":
    block partitioning; [GH] ``block_size`` argument).

    Returns (N, starts, counts): block j holds tokens starts[j] ..
    starts[j] + counts[j] - 1; only the last block may be shorter.
    """
    if L < 1 or block_size < 1:
        raise ValueError("L and block_size must be >= 1")
    N = -(-L // block_size)
    starts = np.arange(N, dtype=np.int64) * block_size
    counts = np.minimum(starts + block_size, L) - starts
    return N, starts, counts


def num_selected(N: int, density: float) -> int:
    """Number of exactly computed blocks per query block: density is the
    fraction of K/V blocks kept exact ([GH] ``density``; FLUX at density 0.15
    is the "85% sparsity" setting).  Reading: floor with a 1e-6 guard, clamped
    to [1, N]."""
    if not (0.0 < density <= 1.0):
        raise ValueError("density must be in (0, 1]")
    return int(min(N, max(1, math.floor(density * N + 1e-6))))


# ----------------------------------------------------------------------------
# pre-computation ([GS] "Hardware Implementation", step 1)
# ----------------------------------------------------------------------------

def block_stats(q: np.ndarray, k: np.ndarray, v: np.ndarray, block_size: int,
                keep_blockwise: bool = False) -> Dict[str, np.ndarray]:
    """Block statistics of one head.

    qbar_i  mean query of block i (pooled query for relevance scoring)
    kbar_j  block centroid: mean key of block j ([GS] "Core Algorithm")
    vsum_j  sum of the values of block j ([GS] "Core Algorithm")
    H_j     block first-order matrix sum_n (k_{j,n} - kbar_j)^T v_{j,n}, d x d
    hbar    mean of H_j over all N blocks ([GS] "Global First-Order Correction")
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, d = k.shape
    N, starts, counts = block_partition(L, block_size)
    qbar = np.empty((N, d))
    kbar = np.empty((N, d))
    vsum = np.empty((N, d))
    H = np.empty((N, d, d))
    for j in range(N):
        sl = slice(starts[j], starts[j] + counts[j])
        qbar[j] = q[sl].sum(axis=0) / counts[j]
        kbar[j] = k[sl].sum(axis=0) / counts[j]
        vsum[j] = v[sl].sum(axis=0)
        delta = k[sl] - kbar[j]
        H[j] = delta.T @ v[sl]
    hbar = H.sum(axis=0) / N
    out = dict(qbar=qbar, kbar=kbar, vsum=vsum, hbar=hbar, counts=counts.astype(np.float64))
    if keep_blockwise:
        out["H"] = H
    return out


def covariance_norms(k: np.ndarray, v: np.ndarray, block_size: int,
                     kbar: np.ndarray, hbar: np.ndarray) -> np.ndarray:
    """M_j = || H_j - Hbar ||_F ([GS] "Covariance-Aware Routing"; Frobenius
    norm as in [SK] "Implementation")."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, d = k.shape
    N, starts, counts = block_partition(L, block_size)
    M = np.empty(N)
    for j in range(N):
        sl = slice(starts[j], starts[j] + counts[j])
        Hj = (k[sl] - kbar[j]).T @ v[sl]
        M[j] = math.sqrt(float(((Hj - hbar) ** 2).sum()))
    return M


# ----------------------------------------------------------------------------
# covariance-aware top-k routing ([GS] "Covariance-Aware Routing";
# [GH] "Attention sink for MMDiT")
# ----------------------------------------------------------------------------

def selection_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float,
                     cov: Optional[np.ndarray] = None, cov_weight: float = 0.0,
                     rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """score_ij = s qbar_i . kbar_j + lambda M_j for the requested query blocks."""
    qb = qbar if rows is None else qbar[np.asarray(rows, dtype=np.int64)]
    sc = scale * (qb @ kbar.T)
    if cov_weight != 0.0:
        sc = sc + cov_weight * cov[None, :]
    return sc


def _sink_block(sink_idx: Optional[int], N: int) -> Optional[int]:
    if sink_idx is None:
        return None
    if sink_idx == 0:
        return 0
    if sink_idx == -1:
        return N - 1
    raise ValueError("sink_idx must be None, 0 or -1")


def select_blocks(scores: np.ndarray, k_sel: int, sink_idx: Optional[int]) -> np.ndarray:
    """Per query block: the k_sel highest-scoring K/V blocks (ties to the lower
    block index), with the sink block forced in when sink_idx is 0 or -1.
    Returns an int64 array [rows, k_sel], each row ascending."""
    R, N = scores.shape
    sink = _sink_block(sink_idx, N)
    out = np.empty((R, k_sel), dtype=np.int64)
    j = np.arange(N)
    for r in range(R):
        order = np.lexsort((j, -scores[r]))  # score descending, then j ascending
        if sink is None:
            chosen = order[:k_sel]
        else:
            others = order[order != sink][:k_sel - 1]
            chosen = np.concatenate([[sink], others])
        out[r] = np.sort(chosen)
    return out


# ----------------------------------------------------------------------------
# exact-or-approximate attention ([GS] "Core Algorithm")
# ----------------------------------------------------------------------------

def piecewise_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, block_size: int,
                        selected: np.ndarray, stats: Dict[str, np.ndarray],
                        scale: float, mode: str,
                        query_blocks: Optional[Iterable[int]] = None) -> np.ndarray:
    """o_t = N_t / D_t for every token t of the requested query blocks.

    For token t of query block i (S_i = selected[i], U_i = the other blocks):
      D_t = sum_{j in S_i} sum_n exp(s q_t k_{j,n}) + sum_{j in U_i} n_j alpha_{t,j}
      N_t = sum_{j in S_i} sum_n exp(s q_t k_{j,n}) v_{j,n}
            + sum_{j in U_i} alpha_{t,j} vsum_j
            + [mode hyd] (s q_t Hbar) sum_{j in U_i} alpha_{t,j}
            + [mode 1st] sum_{j in U_i} alpha_{t,j} (s q_t H_j)
      alpha_{t,j} = exp(s q_t kbar_j)
    Mode "1st" (block-wise first order) needs stats["H"], the per-block H_j.
    One per-row constant (the row maximum of all exponents) is factored out of
    N_t and D_t to keep exp() in range; it cancels in the quotient.

    Returns an array [L, d] with rows of the requested blocks filled (NaN elsewhere).
    """
    if mode not in ("hyd", "0th", "1st"):
        raise ValueError("mode must be 'hyd', '0th' or '1st'")
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L, d = q.shape
    N, starts, counts = block_partition(L, block_size)
    kbar, vsum, hbar = stats["kbar"], stats["vsum"], stats["hbar"]
    out = np.full((L, d), np.nan)
    blocks = range(N) if query_blocks is None else query_blocks
    for i in blocks:
        rows = slice(starts[i], starts[i] + counts[i])
        qi = q[rows]
        S = selected[i] if selected.shape[0] == N else None
        if S is None:
            raise ValueError("selected must have one row per query block")
        in_S = np.zeros(N, dtype=bool)
        in_S[S] = True
        U = np.nonzero(~in_S)[0]
        ex = np.concatenate([np.arange(starts[j], starts[j] + counts[j]) for j in S])
        lg_exact = scale * (qi @ k[ex].T)              # [n_i, |exact keys|]
        lg_tail = scale * (qi @ kbar[U].T)             # [n_i, |U|]
        m = lg_exact.max(axis=1)
        if U.size:
            m = np.maximum(m, lg_tail.max(axis=1))
        p_exact = np.exp(lg_exact - m[:, None])
        alpha = np.exp(lg_tail - m[:, None])
        D = p_exact.sum(axis=1) + alpha @ counts[U].astype(np.float64)
        Nt = p_exact @ v[ex] + alpha @ vsum[U]
        if mode == "hyd":
            Nt = Nt + (scale * (qi @ hbar)) * alpha.sum(axis=1)[:, None]
        elif mode == "1st" and U.size:
            # sum_j alpha_tj H_j as one product, then contract with s q_t
            W = (alpha @ stats["H"][U].reshape(U.size, d * d)).reshape(-1, d, d)
            Nt = Nt + scale * np.einsum("ta,tab->tb", qi, W)
        out[rows] = Nt / D[:, None]
    return out


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                    rows: Optional[slice] = None) -> np.ndarray:
    """Full softmax attention softmax(s q k^T) v in fp64 (the dense baseline)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    qq = q if rows is None else q[rows]
    lg = scale * (qq @ k.T)
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    return (p @ v) / p.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------
# whole path for one head / for [B, H, L, d] arrays
# ----------------------------------------------------------------------------

def pisa_attention_head(q, k, v, block_size: int, density: float,
                        sink_idx: Optional[int], mode: str,
                        scale: Optional[float] = None, cov_weight: float = 0.0,
                        query_blocks: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Statistics -> selection -> piecewise attention for one head.

    With `query_blocks` given, only those query blocks are selected and
    attended (the statistics always cover the whole head).  Returns a dict with
    qbar, kbar, vsum, hbar, cov (or None), k_sel, idx [rows, k_sel] and out [L, d].
    """
    q = np.asarray(q, dtype=np.float64)
    L, d = q.shape
    s = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = block_stats(q, k, v, block_size, keep_blockwise=(mode == "1st"))
    N = st["kbar"].shape[0]
    cov = None
    if cov_weight != 0.0:
        cov = covariance_norms(k, v, block_size, st["kbar"], st["hbar"])
    k_sel = num_selected(N, density)
    rows = list(range(N)) if query_blocks is None else list(query_blocks)
    sc = selection_scores(st["qbar"], st["kbar"], s, cov, cov_weight, rows)
    idx_rows = select_blocks(sc, k_sel, sink_idx)
    sel = np.zeros((N, k_sel), dtype=np.int64)
    sel[rows] = idx_rows
    out = piecewise_attention(q, k, v, block_size, sel, st, s, mode, query_blocks=rows)
    return dict(qbar=st["qbar"], kbar=st["kbar"], vsum=st["vsum"], hbar=st["hbar"],
                cov=cov, k_sel=k_sel, rows=np.asarray(rows), idx=idx_rows,
                scores=sc, out=out)


def pisa_attention(Q, K, V, block_size: int, density: float, sink_idx: Optional[int],
                   mode: str, scale: Optional[float] = None,
                   cov_weight: float = 0.0) -> np.ndarray:
    """Whole path over [B, H, L, d] arrays; returns the output [B, H, L, d] in fp64."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, H, L, d = Q.shape
    out = np.empty((B, H, L, d))
    for b in range(B):
        for h in range(H):
            r = pisa_attention_head(Q[b, h], K[b, h], V[b, h], block_size, density,
                                    sink_idx, mode, scale, cov_weight)
            out[b, h] = r["out"]
    return out


# ----------------------------------------------------------------------------
# distributional-stability diagnostic ([GS] "Key Insights" 1)
# ----------------------------------------------------------------------------

def tail_score_histogram(q, k, block_size: int, selected: np.ndarray, scale: float,
                         lo: float, hi: float, nbins: int,
                         query_blocks: Optional[Iterable[int]] = None) -> Dict[str, np.ndarray]:
    """Distribution of the pre-softmax scores of the unselected (non-critical)
    blocks, and of their deviation from the block-centroid score.

    For every token t of the requested query blocks i, every unselected block
    j in U_i and every key n of block j:
        x = s q_t k_n                     (pre-softmax score)
        y = s q_t (k_n - kbar_j)          (the variable of the block's Taylor
                                           expansion about its centroid)
    Histograms over nbins equal bins of [lo, hi), with one underflow bin in
    front and one overflow bin at the end (nbins + 2 counts each), plus the
    count and the sums of x, x^2, y, y^2.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    L, d = q.shape
    N, starts, counts = block_partition(L, block_size)
    edges = np.linspace(lo, hi, nbins + 1)
    hx = np.zeros(nbins + 2, dtype=np.int64)
    hy = np.zeros(nbins + 2, dtype=np.int64)
    mom = np.zeros(5)
    blocks = range(N) if query_blocks is None else query_blocks

    def add(h, vals):
        h[0] += int((vals < lo).sum())
        h[-1] += int((vals >= hi).sum())
        inside = vals[(vals >= lo) & (vals < hi)]
        h[1:-1] += np.histogram(inside, bins=edges)[0]

    for i in blocks:
        qi = q[starts[i]:starts[i] + counts[i]]
        in_S = np.zeros(N, dtype=bool)
        in_S[selected[i]] = True
        for j in np.nonzero(~in_S)[0]:
            kb = k[starts[j]:starts[j] + counts[j]]
            x = scale * (qi @ kb.T)
            y = scale * (qi @ (kb - kb.mean(axis=0)).T)
            add(hx, x.ravel())
            add(hy, y.ravel())
            mom += [x.size, x.sum(), (x * x).sum(), y.sum(), (y * y).sum()]
    return dict(hist_x=hx, hist_y=hy, n=mom[0], sum_x=mom[1], sum_x2=mom[2],
                sum_y=mom[3], sum_y2=mom[4], edges=edges)
