"""Pins of the oracle's decode step (one new query row per batch-head at position pos, against the
key/value cache rows 0..pos).

* Row pos of the pattern only reads keys j <= pos ("Sparse Transformers 深度解读报告" §2.1: every
  allowed set is a subset of {j <= i}), so the decode result must equal row pos of the full
  forward pass when the forward's query row pos is the decode query -- checked against the
  oracle's forward, which has its own pins (test_oracle_math, test_oracle_sets).
* Changing any cache row after pos leaves the result unchanged.
* Closed forms: at pos = 0 the local-band head sees key 0 alone (O = v_0, lse = q.k_0 / sqrt(d)),
  and the fixed summary head sees no key (O = 0, lse = -inf).
* With q = 0 the weights are uniform: lse = ln |A(pos)| and O is the mean of the allowed v_j.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import FA1, FA2, FU, SA1, SA2, SU

ALL = (SA1, SA2, SU, FA1, FA2, FU)


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("pos", [0, 1, 7, 8, 9, 31, 33, 63])
def test_decode_equals_forward_row(pos):
    B, H, n, d, l, c = 2, 6, 64, 8, 8, 3
    k, v = rand((B, H, n, d), 1), rand((B, H, n, d), 2)
    qrow = rand((B, H, d), 3)
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 2, 2], l, c)
    q = rand((B, H, n, d), 4)
    q[:, :, pos] = qrow
    O, lse = p.fwd(q, k, v)
    o, l_ = p.decode(qrow, k, v, pos)
    np.testing.assert_array_equal(o, O[:, :, pos])
    np.testing.assert_array_equal(l_, lse[:, :, pos])


def test_decode_ignores_rows_after_pos():
    B, H, n, d, l, c, pos = 1, 6, 48, 8, 8, 2, 29
    k, v, qrow = rand((B, H, n, d), 5), rand((B, H, n, d), 6), rand((B, H, d), 7)
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 1, 1], l, c)
    o1, l1 = p.decode(qrow, k, v, pos)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, pos + 1:] += 1e3
    v2[:, :, pos + 1:] -= 1e3
    o2, l2 = p.decode(qrow, k2, v2, pos)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_decode_closed_forms_at_position_zero():
    B, H, n, d, l, c = 1, 2, 16, 8, 8, 2
    k, v, qrow = rand((B, H, n, d), 8), rand((B, H, n, d), 9), rand((B, H, d), 10)
    p = oracle.Problem.from_kinds([SA1, FA2], [0, 0], l, c)
    o, lse = p.decode(qrow, k, v, 0)
    np.testing.assert_allclose(o[0, 0], v[0, 0, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], qrow[0, 0] @ k[0, 0, 0] / math.sqrt(d), rtol=1e-15, atol=0)
    assert np.all(o[0, 1] == 0) and lse[0, 1] == -np.inf


@pytest.mark.parametrize("kind", ALL)
def test_decode_zero_query_is_uniform(kind):
    B, H, n, d, l, c, pos = 1, 1, 40, 4, 8, 3, 37
    k, v = rand((B, H, n, d), 11), rand((B, H, n, d), 12)
    p = oracle.Problem.from_kinds([kind], [1 if kind in (FA2, FU) else 0], l, c)
    o, lse = p.decode(np.zeros((B, H, d)), k, v, pos)
    keys = oracle.row_set(kind, pos, l, c, 1 if kind in (FA2, FU) else 0)
    np.testing.assert_allclose(lse[0, 0], math.log(len(keys)), rtol=0, atol=1e-14)
    np.testing.assert_allclose(o[0, 0], v[0, 0, keys].mean(0), rtol=0, atol=1e-14)


@pytest.mark.parametrize("d,e", [(32, 32), (64, 128), (128, 128)])
def test_decode_equals_forward_row_widths(d, e):
    """Query-key rows of width d, value rows of width e: the decode row is still row pos of the
    forward (whose widths are pinned in test_oracle_math)."""
    B, H, n, l, c, pos = 1, 6, 40, 8, 3, 37
    k, v = rand((B, H, n, d), 13), rand((B, H, n, e), 14)
    q = rand((B, H, n, d), 15)
    p = oracle.Problem.from_kinds(list(ALL), [0, 0, 0, 0, 2, 2], l, c)
    O, lse = p.fwd(q, k, v)
    o, l_ = p.decode(q[:, :, pos].copy(), k, v, pos)
    assert o.shape == (B, H, e)
    np.testing.assert_array_equal(o, O[:, :, pos])
    np.testing.assert_array_equal(l_, lse[:, :, pos])
