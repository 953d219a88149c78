"""Pins of the fp64 gradient oracle of the zeroth-order forward.

* its forward equals the (separately pinned) numpy oracle's mode "0th";
* every gradient element against central finite differences of the numpy
  forward oracle, whose statistics are recomputed from the perturbed inputs
  (so the chain rule through the centroids and value sums is checked);
* special cases that reduce to dense attention, whose gradient and
  log-sum-exp come from torch's own scaled_dot_product_attention / logsumexp;
* invariants: sum_n dv_n = sum_t dout_t; sum_n dk_n = 0 (shifting every key
  by one vector shifts each row's logits by a constant).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O


def _f(q, k, v, dout, b, sel, s):
    st = O.block_stats(q, k, v, b)
    o = O.piecewise_attention(q, k, v, b, sel, st, s, "0th")
    return float((o * dout).sum())


def _case(L, b, d, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((L, d)), rng.standard_normal((L, d)),
            rng.standard_normal((L, d)), rng.standard_normal((L, d)))


def test_forward_matches_numpy_oracle():
    q, k, v, _ = _case(50, 8, 5, 1)
    N = 7
    sel = np.array([[0, 3], [1, 6], [0, 2], [3, 4], [0, 6], [5, 6], [2, 6]])
    r = O.zeroth_order_backward(q, k, v, np.zeros_like(q), 8, sel, 0.6)
    st = O.block_stats(q, k, v, 8)
    ref = O.piecewise_attention(q, k, v, 8, sel, st, 0.6, "0th")
    np.testing.assert_allclose(r["out"], ref, rtol=1e-12, atol=1e-12)
    assert N == sel.shape[0]


def test_every_gradient_element_against_finite_differences():
    """L=10, block 4 (last block 2 tokens), one exact block per query block."""
    L, b, d, s = 10, 4, 3, 0.8
    q, k, v, g = _case(L, b, d, 2)
    sel = np.array([[2], [0], [1]])
    r = O.zeroth_order_backward(q, k, v, g, b, sel, s)
    eps = 1e-6
    for name, x, grad in (("q", q, r["dq"]), ("k", k, r["dk"]), ("v", v, r["dv"])):
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            fp = _f(*(xp if n == name else args[n] for n in "qkv"), g, b, sel, s)
            fm = _f(*(xm if n == name else args[n] for n in "qkv"), g, b, sel, s)
            fd[idx] = (fp - fm) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8, err_msg=name)


def test_directional_derivative_larger_case():
    """L=70 (ragged), block 8, two exact blocks with a forced first block."""
    L, b, d, s = 70, 8, 6, 0.5
    q, k, v, g = _case(L, b, d, 3)
    N = 9
    rng = np.random.default_rng(4)
    sel = np.array([np.sort(np.r_[0, rng.choice(np.arange(1, N), 1)]) for _ in range(N)])
    r = O.zeroth_order_backward(q, k, v, g, b, sel, s)
    dq_, dk_, dv_ = (rng.standard_normal((L, d)) for _ in range(3))
    eps = 1e-5
    fp = _f(q + eps * dq_, k + eps * dk_, v + eps * dv_, g, b, sel, s)
    fm = _f(q - eps * dq_, k - eps * dk_, v - eps * dv_, g, b, sel, s)
    pred = (r["dq"] * dq_).sum() + (r["dk"] * dk_).sum() + (r["dv"] * dv_).sum()
    assert abs((fp - fm) / (2 * eps) - pred) <= 1e-7 * max(1.0, abs(pred))


def _sdpa_grads(q, k, v, g, s):
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None],
                                                         scale=s)[0]
    (o * torch.tensor(g)).sum().backward()
    lse = torch.logsumexp(s * torch.tensor(q) @ torch.tensor(k).T, dim=1).numpy()
    return o.detach().numpy(), lse, qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("b,every_block", [(8, True), (1, False)])
def test_reduces_to_dense_attention(b, every_block):
    """Every block exact (density 1), or block_size 1 (each centroid is its own
    key, n_j = 1): the method is dense attention, gradients included."""
    L, d, s = 40, 4, 0.7
    q, k, v, g = _case(L, b, d, 5)
    N = -(-L // b)
    if every_block:
        sel = np.tile(np.arange(N), (N, 1))
    else:
        sel = np.array([[i] for i in range(N)])
    r = O.zeroth_order_backward(q, k, v, g, b, sel, s)
    o, lse, dq, dk, dv = _sdpa_grads(q, k, v, g, s)
    for a, e in ((r["out"], o), (r["lse"], lse), (r["dq"], dq), (r["dk"], dk), (r["dv"], dv)):
        np.testing.assert_allclose(a, e, rtol=1e-10, atol=1e-12)


def test_invariants():
    L, b, d, s = 100, 16, 8, 1 / math.sqrt(8)
    q, k, v, g = _case(L, b, d, 6)
    N = 7
    sel = np.array([[0, (i + 3) % N] if (i + 3) % N else [0, 1] for i in range(N)])
    sel.sort(axis=1)
    r = O.zeroth_order_backward(q, k, v, g, b, sel, s)
    np.testing.assert_allclose(r["dv"].sum(axis=0), g.sum(axis=0), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(r["dk"].sum(axis=0), 0.0, atol=1e-11)
    assert np.abs(r["dk"]).max() > 1e-3      # not trivially zero


def test_query_block_subset_rows():
    """Restricting to some query blocks leaves dq of those rows unchanged."""
    L, b, d, s = 64, 8, 4, 0.5
    q, k, v, g = _case(L, b, d, 7)
    sel = np.array([[0, i] if i else [0, 1] for i in range(8)])
    full = O.zeroth_order_backward(q, k, v, g, b, sel, s)
    part = O.zeroth_order_backward(q, k, v, g, b, sel, s, query_blocks=[2, 5])
    rows = np.r_[16:24, 40:48]
    np.testing.assert_allclose(part["dq"][rows], full["dq"][rows], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(part["lse"][rows], full["lse"][rows], rtol=1e-13)
    assert np.isnan(part["lse"][0])
