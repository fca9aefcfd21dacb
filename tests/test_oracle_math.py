"""Pins of the oracle's arithmetic (forward and backward) against fixed mathematics.

* Special cases whose allowed set is the full causal set must equal textbook dense causal
  attention, computed here by PyTorch's own CPU fp64 scaled_dot_product_attention(is_causal=True)
  and its autograd (an independent library routine).
* Q = 0 gives uniform weights: lse_i = ln |A(i)| and O_i = mean of the allowed v_j, exactly.
* Masked-V perturbation ("长序列为何不必让每个 token 看见全部历史？…" §10): adding 1e4 to the value
  of a key outside A(i) leaves O_i unchanged.
* Central finite differences of L = sum(O * dO) match the oracle gradients (all six set kinds).
* The sampled-row and sampled-key entry points equal the full evaluation.
* Every pin above is repeated with query-key rows of width d and value rows of width e != d (the
  head widths of the pages' models), where the dense special cases also fix the 1/sqrt(d) scale.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import FA1, FA2, FU, SA1, SA2, SU

ALL = (SA1, SA2, SU, FA1, FA2, FU)


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def dense_causal(q, k, v, do):
    """Textbook dense causal attention and its gradients (PyTorch CPU fp64)."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    o.backward(torch.tensor(do, dtype=torch.float64))
    s = torch.matmul(tq, tk.transpose(-1, -2)) / math.sqrt(q.shape[-1])
    n = q.shape[-2]
    s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return (o.detach().numpy(), lse.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(),
            tv.grad.numpy())


# (kind, l, c, o) choices whose set is the full causal set {0..i} for n = 40
FULL_CASES = [(SA1, 39, 0, 0), (SA1, 100, 0, 0), (SA2, 1, 0, 0), (SU, 1, 0, 0), (FA1, 40, 0, 0),
              (FA1, 64, 0, 0), (FA2, 8, 8, 0), (FU, 8, 8, 0), (FU, 64, 3, 0)]


@pytest.mark.parametrize("kind,l,c,o", FULL_CASES)
def test_special_cases_equal_dense_causal(kind, l, c, o):
    B, H, n, d = 2, 1, 40, 16
    q, k, v, do = (rand((B, H, n, d), s) for s in range(4))
    p = oracle.Problem.from_kinds([kind], [o], l, c)
    O, lse = p.fwd(q, k, v)
    dq, dk, dv = p.bwd(q, k, v, do)
    Ot, lset, dqt, dkt, dvt = dense_causal(q, k, v, do)
    for a, b in ((O, Ot), (lse, lset), (dq, dqt), (dk, dkt), (dv, dvt)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("kind,l,c", [(SA1, 5, 0), (SA2, 5, 0), (SU, 5, 0), (FA1, 8, 0),
                                      (FA2, 8, 3), (FU, 8, 3)])
def test_zero_query_closed_form(kind, l, c):
    n, d = 50, 8
    q = np.zeros((1, 1, n, d))
    k, v = rand((1, 1, n, d), 1), rand((1, 1, n, d), 2)
    O, lse = oracle.Problem.from_kinds([kind], [1 if kind == FA2 else 0], l, c).fwd(q, k, v)
    for i in range(n):
        s = oracle.row_set(kind, i, l, c, 1 if kind == FA2 else 0)
        if len(s) == 0:
            assert lse[0, 0, i] == -np.inf and np.all(O[0, 0, i] == 0)
            continue
        assert abs(lse[0, 0, i] - math.log(len(s))) < 1e-12
        np.testing.assert_allclose(O[0, 0, i], v[0, 0, s].mean(axis=0), rtol=0, atol=1e-12)


def test_masked_value_perturbation():
    n, d, l, c = 64, 8, 8, 2
    q, k, v = (rand((1, 6, n, d), s) for s in range(3))
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 2, 2], l, c)
    O, _ = p.fwd(q, k, v)
    for h, kind in enumerate(ALL):
        for i in (5, 17, 40, 63):
            s = set(oracle.row_set(kind, i, l, c, p.off[h]).tolist())
            outside = [j for j in range(n) if j not in s]
            v2 = v.copy()
            v2[0, h, outside] += 1e4
            O2, _ = p.fwd(q, k, v2)
            np.testing.assert_allclose(O2[0, h, i], O[0, h, i], rtol=0, atol=1e-9)
            inside = sorted(s)[0] if s else None
            if inside is not None:  # control: perturbing an allowed key does move the row
                v3 = v.copy()
                v3[0, h, inside] += 1e4
                O3, _ = p.fwd(q, k, v3)
                assert np.abs(O3[0, h, i] - O[0, h, i]).max() > 1e-3


def test_finite_differences_all_kinds():
    n, d, l, c = 24, 6, 5, 2
    q, k, v, do = (rand((1, 6, n, d), 10 + s) for s in range(4))
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 1, 1], l, c)
    dq, dk, dv = p.bwd(q, k, v, do)
    eps = 1e-6

    def loss(qq, kk, vv):
        O, _ = p.fwd(qq, kk, vv)
        return float((O * do).sum())

    rng = np.random.default_rng(7)
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(40):
            h, i, t = rng.integers(6), rng.integers(n), rng.integers(d)
            args = [q.copy(), k.copy(), v.copy()]
            args[which][0, h, i, t] += eps
            lp = loss(*args)
            args[which][0, h, i, t] -= 2 * eps
            lm = loss(*args)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[0, h, i, t]) <= 1e-6 * max(1.0, abs(fd)), (which, h, i, t)


def test_row_sums_and_convex_hull():
    n, d, l, c = 80, 4, 8, 2
    q, k = rand((1, 6, n, d), 3), rand((1, 6, n, d), 4)
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 0, 0], l, c)
    O, _ = p.fwd(q, k, np.ones((1, 6, n, d)))
    cnt = np.stack([oracle.set_counts(kd, n, l, c, 0) for kd in ALL])
    np.testing.assert_allclose(O[0][cnt > 0], 1.0, rtol=0, atol=1e-13)
    v = rand((1, 6, n, d), 5)
    O, _ = p.fwd(q, k, v)
    for h, kind in enumerate(ALL):
        for i in range(n):
            s = oracle.row_set(kind, i, l, c, 0)
            if len(s):
                assert np.all(O[0, h, i] <= v[0, h, s].max(0) + 1e-12)
                assert np.all(O[0, h, i] >= v[0, h, s].min(0) - 1e-12)


def test_sampled_entry_points_match_full():
    B, H, n, d, l, c = 2, 6, 70, 8, 8, 2
    q, k, v, do = (rand((B, H, n, d), 20 + s) for s in range(4))
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 2, 2], l, c)
    O, lse = p.fwd(q, k, v)
    dq, dk, dv = p.bwd(q, k, v, do)
    rows = np.array([0, 5, 69, 70 + 33, 3 * 70 + 1, B * H * n - 1])
    Or, lr = p.fwd_rows(q, k, v, rows)
    np.testing.assert_array_equal(Or, O.reshape(-1, d)[rows])
    np.testing.assert_array_equal(lr, lse.reshape(-1)[rows])
    dqr, lr2, Dr = p.bwd_rows(q, k, v, do, rows)
    np.testing.assert_allclose(dqr, dq.reshape(-1, d)[rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lr2, lr, rtol=0, atol=1e-13)
    # D_i equals dO_i . O_i
    np.testing.assert_allclose(Dr, (do.reshape(-1, d)[rows] * Or).sum(-1), rtol=0, atol=1e-12)
    dkr, dvr = p.bwd_keys(q, k, v, do, rows)
    np.testing.assert_allclose(dkr, dk.reshape(-1, d)[rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dvr, dv.reshape(-1, d)[rows], rtol=0, atol=1e-13)


def test_empty_rows_have_no_gradient_flow():
    n, d, l, c = 32, 4, 16, 4
    q, k, v, do = (rand((1, 1, n, d), 30 + s) for s in range(4))
    p = oracle.Problem.from_kinds([FA2], [0], l, c)
    O, lse = p.fwd(q, k, v)
    dq, dk, dv = p.bwd(q, k, v, do)
    empty = np.arange(l - c)
    assert np.all(np.isneginf(lse[0, 0, empty])) and np.all(O[0, 0, empty] == 0)
    assert np.all(dq[0, 0, empty] == 0)
    # keys that are not summary positions are read by nobody
    nonsum = [j for j in range(n) if j % l < l - c]
    assert np.all(dk[0, 0, nonsum] == 0) and np.all(dv[0, 0, nonsum] == 0)


# ---- head widths: query/key rows of width d, value rows of width e ------------------------------
# "Sparse Transformers 深度解读报告" §4.5: the models use per-head widths 512/16 = 32 (ImageNet 64),
# 512/8 = 64 (Enwik8) and 256/2 = 128 (CIFAR-10, whose query-key projection is half-size, d = 64
# against e = 128).  The score scale is 1/sqrt(d), the width of the dot product ([G] §01); PyTorch's
# SDPA takes the same convention (scale 1/sqrt of the query width, output of the value width), so
# the dense special cases pin it independently.
WIDTHS = [(32, 32), (128, 128), (64, 128), (8, 24)]


@pytest.mark.parametrize("d,e", WIDTHS)
@pytest.mark.parametrize("kind,l,c,o", [(SA1, 39, 0, 0), (SA2, 1, 0, 0), (FA1, 40, 0, 0), (FU, 8, 8, 0)])
def test_widths_special_cases_equal_dense_causal(d, e, kind, l, c, o):
    B, H, n = 1, 2, 40
    q, k = rand((B, H, n, d), 40), rand((B, H, n, d), 41)
    v, do = rand((B, H, n, e), 42), rand((B, H, n, e), 43)
    p = oracle.Problem.from_kinds([kind, kind], [o, o], l, c)
    O, lse = p.fwd(q, k, v)
    dq, dk, dv = p.bwd(q, k, v, do)
    assert O.shape == (B, H, n, e) and dq.shape == (B, H, n, d) and dv.shape == (B, H, n, e)
    Ot, lset, dqt, dkt, dvt = dense_causal(q, k, v, do)
    for a, b in ((O, Ot), (lse, lset), (dq, dqt), (dk, dkt), (dv, dvt)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("d,e", [(16, 32), (32, 8)])
def test_widths_zero_query_closed_form(d, e):
    n, l, c = 48, 8, 3
    q = np.zeros((1, 6, n, d))
    k, v = rand((1, 6, n, d), 44), rand((1, 6, n, e), 45)
    offs = [0, 0, 0, 0, 1, 1]
    O, lse = oracle.Problem.from_kinds(list(ALL), offs, l, c).fwd(q, k, v)
    for h, kind in enumerate(ALL):
        for i in range(n):
            s = oracle.row_set(kind, i, l, c, offs[h])
            if len(s) == 0:
                assert lse[0, h, i] == -np.inf and np.all(O[0, h, i] == 0)
                continue
            assert abs(lse[0, h, i] - math.log(len(s))) < 1e-12
            np.testing.assert_allclose(O[0, h, i], v[0, h, s].mean(axis=0), rtol=0, atol=1e-12)


def test_widths_finite_differences():
    n, d, e, l, c = 20, 4, 10, 5, 2
    q, k = rand((1, 6, n, d), 50), rand((1, 6, n, d), 51)
    v, do = rand((1, 6, n, e), 52), rand((1, 6, n, e), 53)
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 1, 1], l, c)
    grads = p.bwd(q, k, v, do)
    eps = 1e-6

    def loss(qq, kk, vv):
        return float((p.fwd(qq, kk, vv)[0] * do).sum())

    rng = np.random.default_rng(54)
    for which, grad in enumerate(grads):
        width = grad.shape[-1]
        for _ in range(40):
            h, i, t = rng.integers(6), rng.integers(n), rng.integers(width)
            args = [q.copy(), k.copy(), v.copy()]
            args[which][0, h, i, t] += eps
            lp = loss(*args)
            args[which][0, h, i, t] -= 2 * eps
            fd = (lp - loss(*args)) / (2 * eps)
            assert abs(fd - grad[0, h, i, t]) <= 1e-6 * max(1.0, abs(fd)), (which, h, i, t)


def test_widths_sampled_entry_points_match_full():
    B, H, n, d, e, l, c = 2, 6, 40, 8, 16, 8, 2
    q, k = rand((B, H, n, d), 60), rand((B, H, n, d), 61)
    v, do = rand((B, H, n, e), 62), rand((B, H, n, e), 63)
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 2, 2], l, c)
    O, lse = p.fwd(q, k, v)
    dq, dk, dv = p.bwd(q, k, v, do)
    rows = np.array([0, 7, 39, 40 + 21, 5 * 40 + 3, B * H * n - 1])
    Or, lr = p.fwd_rows(q, k, v, rows)
    np.testing.assert_array_equal(Or, O.reshape(-1, e)[rows])
    np.testing.assert_array_equal(lr, lse.reshape(-1)[rows])
    dqr, _, Dr = p.bwd_rows(q, k, v, do, rows)
    np.testing.assert_allclose(dqr, dq.reshape(-1, d)[rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(Dr, (do.reshape(-1, e)[rows] * Or).sum(-1), rtol=0, atol=1e-12)
    dkr, dvr = p.bwd_keys(q, k, v, do, rows)
    np.testing.assert_allclose(dkr, dk.reshape(-1, d)[rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dvr, dv.reshape(-1, e)[rows], rtol=0, atol=1e-13)


def test_widths_shape_errors():
    p = oracle.Problem.from_kinds([SA1], [0], 4)
    q = np.zeros((1, 1, 8, 4))
    with pytest.raises(ValueError):
        p.fwd(q, np.zeros((1, 1, 8, 6)), np.zeros((1, 1, 8, 6)))  # k narrower/wider than q
    with pytest.raises(ValueError):
        p.bwd(q, q, np.zeros((1, 1, 8, 6)), np.zeros((1, 1, 8, 4)))  # dO not as wide as v
