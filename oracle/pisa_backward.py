"""Plain fp64 CPU oracle of the gradients of the zeroth-order ("_0th") PISA
forward.

TEST INFRASTRUCTURE ONLY -- the CUDA library never calls this module and this
module never imports the CUDA library.  Only the tests use it.

The forward is restated here in plain PyTorch float64 CPU operations, from the
same definitions as ``pisa_oracle.piecewise_attention`` (mode "0th"), so that
autograd (a library primitive used as one step) gives the gradients with
respect to q, k and v.  The selection is a discrete step: it is held fixed and
passed in.  The statistics are part of the differentiated function: the
centroid kbar_j is the mean key of block j and SigmaV_j the sum of its values,
so the gradient of every tail term reaches the keys and values of block j
through them.

Sources (cited by page title and section):

* [GS] "Technical Summary: PISA - Piecewise Sparse Attention for Efficient
  Diffusion Transformers" (gist.science), section 2 "Methodology", "Core
  Algorithm": the S_i / U_i split and o_t = N_t / D_t with
  alpha_{t,j} = exp(s q_t kbar_j);
* [GH] "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
  Transformers" (authors' README mirror), "Kernel variants": the _0th variant
  (zeroth-order tail only) is the one that supports backward for training.

Readings: the gradient is that of the function the _0th
forward computes, selection held constant; lse_t = ln D_t (natural log, D_t
as written, without any factored-out constant).
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import numpy as np
import torch

from .pisa_oracle import block_partition


def _as64(x) -> torch.Tensor:
    return torch.as_tensor(np.asarray(x, dtype=np.float64)).clone()


def zeroth_order_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_size: int,
                         selected: np.ndarray, scale: float,
                         query_blocks: Optional[Iterable[int]] = None):
    """Differentiable fp64 restatement of the _0th forward for one head.

    For token t of query block i (S_i = selected[i], U_i = the other blocks):
      D_t = sum_{j in S_i} sum_n exp(s q_t k_{j,n}) + sum_{j in U_i} n_j alpha_{t,j}
      N_t = sum_{j in S_i} sum_n exp(s q_t k_{j,n}) v_{j,n} + sum_{j in U_i} alpha_{t,j} SigmaV_j
      o_t = N_t / D_t,  lse_t = ln D_t,  alpha_{t,j} = exp(s q_t kbar_j)
    Returns (rows, out [rows, d], lse [rows]) for the requested query blocks
    (all by default), rows being the token indices in order.
    """
    L, d = q.shape
    N, starts, counts = block_partition(L, block_size)
    kbar = torch.stack([k[starts[j]:starts[j] + counts[j]].mean(dim=0) for j in range(N)])
    vsum = torch.stack([v[starts[j]:starts[j] + counts[j]].sum(dim=0) for j in range(N)])
    n_j = torch.as_tensor(counts, dtype=torch.float64)
    blocks = range(N) if query_blocks is None else list(query_blocks)
    outs, lses, rows = [], [], []
    for i in blocks:
        r = slice(starts[i], starts[i] + counts[i])
        qi = q[r]
        in_S = np.zeros(N, dtype=bool)
        in_S[np.asarray(selected[i])] = True
        U = torch.as_tensor(np.nonzero(~in_S)[0])
        ex = torch.as_tensor(np.concatenate(
            [np.arange(starts[j], starts[j] + counts[j]) for j in np.nonzero(in_S)[0]]))
        lg_exact = scale * (qi @ k[ex].T)
        lg_tail = scale * (qi @ kbar[U].T)
        m = lg_exact.max(dim=1).values
        if U.numel():
            m = torch.maximum(m, lg_tail.max(dim=1).values)
        m = m.detach()                       # a constant factor of N_t and D_t
        p_exact = torch.exp(lg_exact - m[:, None])
        alpha = torch.exp(lg_tail - m[:, None])
        D = p_exact.sum(dim=1) + alpha @ n_j[U]
        Nt = p_exact @ v[ex] + alpha @ vsum[U]
        outs.append(Nt / D[:, None])
        lses.append(m + torch.log(D))
        rows.append(np.arange(starts[i], starts[i] + counts[i]))
    return np.concatenate(rows), torch.cat(outs), torch.cat(lses)


def zeroth_order_backward(q, k, v, dout, block_size: int, selected: np.ndarray, scale: float,
                          query_blocks: Optional[Iterable[int]] = None) -> Dict[str, np.ndarray]:
    """Gradients of sum_t dout_t . o_t with respect to q, k, v (fp64, one head).

    With `query_blocks` given only those blocks' outputs enter the sum: dq is
    then exact on their rows (zero elsewhere) and dk, dv hold only their
    contribution.  Returns out, lse (NaN outside the requested rows), dq, dk,
    dv as numpy float64 arrays.
    """
    q, k, v = (_as64(x).requires_grad_(True) for x in (q, k, v))
    g = _as64(dout)
    rows, out, lse = zeroth_order_forward(q, k, v, block_size, selected, scale, query_blocks)
    (out * g[torch.as_tensor(rows)]).sum().backward()
    L, d = q.shape
    o_full = np.full((L, d), np.nan)
    l_full = np.full(L, np.nan)
    o_full[rows] = out.detach().numpy()
    l_full[rows] = lse.detach().numpy()
    return dict(out=o_full, lse=l_full, dq=q.grad.numpy(), dk=k.grad.numpy(),
                dv=v.grad.numpy(), rows=rows)
