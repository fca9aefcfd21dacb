"""Pins of the oracle's allowed sets against what the pages and plain counting fix.

Each check is independent of the oracle's predicate code: closed-form counts derived by hand,
the shape each set must have, the worked example printed on the fixed-pattern page, two-hop
connectivity of the union graph (brute force), causality, and the empty-row census.
Sources: "Sparse Transformers（稀疏 Transformer）深度解读报告" §2.1 (sparsity and connectivity
properties), §2.2 (strided and fixed sets, worked example); "长序列为何不必让每个 token 看见全部
历史？滑动窗口、块稀疏与全局 token" §02 (every row needs an allowed key), §12 (all allowed edges
satisfy j <= i).
"""
import os

import numpy as np
import pytest

import oracle
from oracle import FA1, FA2, FU, SA1, SA2, SU

HERE = os.path.dirname(os.path.abspath(__file__))

PARAMS = [  # (n, l, c)
    (64, 8, 2), (100, 7, 3), (256, 16, 4), (300, 32, 8), (512, 64, 16), (257, 1, 1),
    (96, 96, 32), (130, 128, 8),
]


def closed_count(kind, i, l, c, o):
    """|A(i)| written out by hand from the set definitions (0-based positions)."""
    if kind == SA1:
        return min(i, l) + 1
    if kind == SA2:
        return i // l + 1
    if kind == SU:  # band plus stride positions; i itself and i-l (if any) are in both
        return (min(i, l) + 1) + (i // l + 1) - 1 - (1 if i >= l else 0)
    if kind == FA1:
        return i % l + 1
    if kind == FA2:  # full summary runs of earlier blocks, plus the part of this block's run <= i
        return (i // l) * c + min(max(i % l - (l - c - o) + 1, 0), c)
    if kind == FU:
        return (i % l + 1) + (i // l) * c
    raise ValueError(kind)


def offsets(l, c):
    return sorted({(k * c) % l for k in range(max(1, l // max(c, 1)))}) if c else [0]


@pytest.mark.parametrize("n,l,c", PARAMS)
def test_counts_match_closed_forms(n, l, c):
    for kind in (SA1, SA2, SU, FA1, FA2, FU):
        offs = offsets(l, c) if kind in (FA2, FU) else [0]
        cc = c if kind in (FA2, FU) else 0
        if kind in (FA2, FU) and c == 0:
            continue
        for o in offs:
            got = oracle.set_counts(kind, n, l, cc, o)
            want = np.array([closed_count(kind, i, l, cc, o) for i in range(n)])
            np.testing.assert_array_equal(got, want, err_msg=f"kind={kind} o={o}")


@pytest.mark.parametrize("n,l,c", [(200, 16, 4), (130, 7, 3), (256, 64, 16)])
def test_set_shapes(n, l, c):
    """The shape each set must have, independent of how membership is tested."""
    for i in range(n):
        s = oracle.row_set(SA1, i, l)
        np.testing.assert_array_equal(s, np.arange(max(0, i - l), i + 1))   # contiguous band
        s = oracle.row_set(SA2, i, l)
        np.testing.assert_array_equal(s, np.arange(i % l, i + 1, l))        # stride-l ladder to i
        s = oracle.row_set(FA1, i, l)
        np.testing.assert_array_equal(s, np.arange((i // l) * l, i + 1))    # own block up to i
        for o in offsets(l, c):
            s = oracle.row_set(FA2, i, l, c, o)
            runs = [np.arange(u * l + l - c - o, u * l + l - o) for u in range(i // l + 1)]
            want = np.concatenate(runs)
            np.testing.assert_array_equal(s, want[want <= i])                # c-wide runs
        u = oracle.row_set(SU, i, l)
        np.testing.assert_array_equal(u, np.union1d(oracle.row_set(SA1, i, l),
                                                     oracle.row_set(SA2, i, l)))


def test_worked_example_fixed_pattern():
    """Golden: the fixed-pattern worked example (l = 128, c = 8)."""
    names = {"sA1": SA1, "sA2": SA2, "sU": SU, "fA1": FA1, "fA2": FA2, "fU": FU}
    rows = []
    with open(os.path.join(HERE, "golden", "fixed_worked_example.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    assert len(rows) >= 5
    for kind, l, c, o, i0, i1, j0, j1, expect in rows:
        kind, l, c, o = names[kind], int(l), int(c), int(o)
        for i in range(int(i0), int(i1) + 1):
            s = set(oracle.row_set(kind, i, l, c, o).tolist())
            for j in range(int(j0), int(j1) + 1):
                assert (j in s) == bool(int(expect)), (kind, i, j)


@pytest.mark.parametrize("family,n,l,c", [("strided", 256, 16, 0), ("strided", 200, 14, 0),
                                          ("strided", 512, 23, 0), ("fixed", 256, 16, 4),
                                          ("fixed", 240, 16, 1), ("fixed", 512, 32, 8)])
def test_two_hop_connectivity(family, n, l, c):
    """Union graph reaches every j <= i in at most two steps; each head alone does not."""
    if family == "strided":
        k1, k2 = SA1, SA2
    else:
        k1, k2 = FA1, FA2
    A1 = np.zeros((n, n), dtype=np.int64)
    A2 = np.zeros((n, n), dtype=np.int64)
    for i in range(n):
        A1[i, oracle.row_set(k1, i, l, c, 0)] = 1
        A2[i, oracle.row_set(k2, i, l, c, 0)] = 1
    U = ((A1 + A2) > 0).astype(np.int64)
    two = ((U @ U) > 0) | (U > 0)
    lower = np.tril(np.ones((n, n), dtype=bool))
    assert np.array_equal(two, lower), "union graph is not two-hop connected"
    for A in (A1, A2):  # negative control: a single factorized head is not enough
        t = ((A @ A) > 0) | (A > 0)
        assert not np.array_equal(t, lower)


@pytest.mark.parametrize("n,l,c", [(300, 32, 8), (512, 128, 32), (97, 10, 5)])
def test_causal_and_nonempty_rows(n, l, c):
    for kind in (SA1, SA2, SU, FA1, FU):
        for i in range(n):
            s = oracle.row_set(kind, i, l, c, 0)
            assert len(s) >= 1 and s.max() <= i and s.min() >= 0
    for o in offsets(l, c):
        counts = oracle.set_counts(FA2, n, l, c, o)
        empty = np.nonzero(counts == 0)[0]
        # Exactly the first l-c-o rows (before the first summary run) have no allowed key.
        np.testing.assert_array_equal(empty, np.arange(min(n, l - c - o)))


def test_head_assignment():
    kind, off = oracle.head_kinds(oracle.FIXED, oracle.ALTERNATING, 8, 128, 32)
    assert kind.tolist() == [FA1, FA2] * 4
    assert off[1::2].tolist() == [0, 32, 64, 96]
    kind, off = oracle.head_kinds(oracle.STRIDED, oracle.ALTERNATING, 2, 16)
    assert kind.tolist() == [SA1, SA2]
    kind, off = oracle.head_kinds(oracle.STRIDED, oracle.MERGED, 3, 16)
    assert kind.tolist() == [SU] * 3
    kind, off = oracle.head_kinds(oracle.FIXED, oracle.MERGED, 4, 128, 32)
    assert kind.tolist() == [FU] * 4 and off.tolist() == [0, 32, 64, 96]
    with pytest.raises(ValueError):
        oracle.head_kinds(3, 1, 2, 16)


def test_complexity_counts():
    """O(n sqrt n) per head when l ~ sqrt n; fixed head 2 ~ c times strided head 2."""
    n, l = 12288, 128
    tot = int(oracle.set_counts(SA1, n, l).sum())
    assert tot == 1576896
    assert abs(tot / (n * l) - 1) < 0.01
    n, l, c = 16384, 128, 8
    r = oracle.set_counts(FA2, n, l, c, 0).sum() / oracle.set_counts(SA2, n, l).sum()
    assert abs(r / c - 1) < 0.1
