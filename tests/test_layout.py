"""Host-side checks of the C ABI library (no GPU): exports, argument errors, and the block layout.

* The library loads and exports every function include/st_attn.h declares.
* Invalid arguments give the documented status codes, with no crash.
* Natural-frame CSR + element masks expand, row by row, to exactly the oracle's allowed sets
  (bit-exact), for every head of every workload and for small sweeps; FULL blocks are exactly the
  blocks whose every pair is allowed; no empty block is listed.
* The execution frames (natural, grid-column, compacted summary) enumerate, per row, exactly the
  oracle's allowed set, using the same interval and frame rules as the kernels.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from workloads import ALTERNATING, FIXED, MERGED, STRIDED, WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

bsf = pytest.importorskip("block_sparse_factorized_b200")
from block_sparse_factorized_b200 import _abi  # noqa: E402


def header_functions():
    src = open(os.path.join(ROOT, "include", "st_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(st_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = _abi.load()
    names = header_functions()
    assert len(names) >= 14
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(_abi.EXPORTED)
    assert b"sm_100a" in lib.st_version()
    assert lib.st_status_string(0) == b"ok"


def _build(family, mode, H, n, l, c=0, block=128, step=0):
    lib = _abi.load()
    h = ctypes.c_void_p()
    pat = _abi.st_pattern_t(family, mode, H, step)
    st = lib.st_layout_build(ctypes.byref(pat), n, l, c, block, ctypes.byref(h))
    if st == 0:
        lib.st_layout_destroy(h)
    return st


def test_argument_errors():
    S, F, A = bsf.ST_STRIDED, bsf.ST_FIXED, bsf.ST_PER_HEAD_ALTERNATING
    assert _build(S, A, 2, 256, 16) == 0
    assert _build(3, A, 2, 256, 16) == 1          # bad family
    assert _build(S, 9, 2, 256, 16) == 1          # bad head mode
    assert _build(S, A, 0, 256, 16) == 1          # no heads
    assert _build(S, A, 2, 0, 16) == 1            # n
    assert _build(S, A, 2, 256, 0) == 1           # l
    assert _build(S, A, 2, 256, 16, block=96) == 1
    assert _build(F, A, 2, 256, 16, c=0) == 1     # fixed needs 1 <= c <= l
    assert _build(F, A, 2, 256, 16, c=17) == 1
    lib = _abi.load()
    assert lib.st_layout_build(None, 256, 16, 0, 128, None) == 1
    # a layout the kernels cannot run (n % 128 != 0) still builds and exports, but cannot upload
    lay = bsf.Layout(S, A, 2, 200, 10)
    rp, ci, mi, mk = lay.export(0)
    assert rp[-1] == len(ci)
    assert lib.st_layout_upload(lay.handle, None) == 2
    with pytest.raises(bsf.StError):
        lay.info()
    # calls on a layout that was never uploaded: argument errors first, then NOT_UPLOADED
    lay = bsf.Layout(S, A, 2, 256, 16)
    fake = ctypes.c_void_p(1 << 20)
    d = _abi.st_desc_t(1, 2, 256, 64, 1, 0)
    assert lib.st_attn_fwd(fake, fake, fake, lay.handle, fake, fake, None, 0, ctypes.byref(d), None) == 4
    # row widths (query-key d, value dv; dv = 0 means d): the bf16 forward takes (32, 32),
    # (64, 64), (128, 128) and (64, 128), the bf16 backward (32, 32), (64, 64) and (64, 128) --
    # those pass the width check and meet NOT_UPLOADED -- fp32 I/O only (64, 64); other widths
    # are valid but unsupported, a negative value width is invalid
    for dqk, dv, dt, fwd_want, bwd_want in ((32, 0, 1, 4, 4), (128, 0, 1, 4, 2), (64, 128, 1, 4, 4),
                                            (64, 64, 1, 4, 4), (64, 0, 2, 4, 4), (32, 0, 2, 2, 2),
                                            (48, 0, 1, 2, 2), (64, 32, 1, 2, 2), (256, 0, 1, 2, 2),
                                            (64, -1, 1, 1, 1)):
        d = _abi.st_desc_t(1, 2, 256, dqk, dt, dv)
        assert lib.st_attn_fwd(fake, fake, fake, lay.handle, fake, fake, None, 0, ctypes.byref(d),
                               None) == fwd_want, (dqk, dv, dt)
        assert lib.st_attn_bwd(fake, fake, fake, fake, fake, fake, lay.handle, fake, fake, fake, None, 0,
                               ctypes.byref(d), None) == bwd_want, (dqk, dv, dt)
    d = _abi.st_desc_t(1, 3, 256, 64, 1, 0)      # heads mismatch
    assert lib.st_attn_fwd(fake, fake, fake, lay.handle, fake, fake, None, 0, ctypes.byref(d), None) == 1
    d = _abi.st_desc_t(1, 2, 256, 64, 7, 0)      # bad dtype
    assert lib.st_attn_fwd(fake, fake, fake, lay.handle, fake, fake, None, 0, ctypes.byref(d), None) == 1
    d = _abi.st_desc_t(1, 2, 256, 64, 1, 0)
    assert lib.st_attn_fwd(None, fake, fake, lay.handle, fake, fake, None, 0, ctypes.byref(d), None) == 1
    assert lib.st_attn_bwd(fake, fake, fake, fake, fake, fake, lay.handle, fake, fake, fake, None, 0,
                           ctypes.byref(d), None) == 4
    assert lib.st_layout_check(lay.handle, None) == 4
    assert lib.st_selftest_wait_timeout(None, None) == 1
    assert lib.st_selftest_wait_timeout(lay.handle, None) == 4
    # sizes that are not positive, or so many rows that byte counts could wrap, are invalid
    # arguments; the workspace queries answer 0 for them
    for bad in ((0, 2, 256, 64), (1, 2, 256, 0), (1 << 31, 2, 256, 64), (1 << 20, 2, 1 << 30, 64)):
        d = _abi.st_desc_t(*bad, 1, 0)
        assert lib.st_attn_fwd(fake, fake, fake, lay.handle, fake, fake, None, 0, ctypes.byref(d), None) == 1
        assert lib.st_attn_fwd_workspace_bytes(ctypes.byref(d), lay.handle) == 0
        assert lib.st_attn_bwd_workspace_bytes(ctypes.byref(d), lay.handle) == 0
        assert lib.st_attn_decode_workspace_bytes(ctypes.byref(d), lay.handle) == 0
    # the forward always takes a workspace: the persistent kernel's unit counters come first
    d = _abi.st_desc_t(1, 2, 256, 64, 1, 0)
    assert lib.st_attn_fwd_workspace_bytes(ctypes.byref(d), lay.handle) == 256
    d = _abi.st_desc_t(1, 2, 256, 64, 2, 0)
    assert lib.st_attn_fwd_workspace_bytes(ctypes.byref(d), lay.handle) == 256 + 5 * 2 * 256 * 64 * 2
    # the split backward's main phase takes dq too (dQ of single-contributor heads is stored there)
    d = _abi.st_desc_t(1, 2, 256, 64, 1, 0)
    assert lib.st_attn_bwd_main(fake, fake, fake, fake, fake, lay.handle, None, fake, fake, fake, 0,
                                ctypes.byref(d), None) == 1


def test_decode_argument_errors():
    """The decode step checks its arguments before anything is launched (and needs no upload)."""
    S, A = bsf.ST_STRIDED, bsf.ST_PER_HEAD_ALTERNATING
    lib = _abi.load()
    lay = bsf.Layout(S, A, 2, 256, 16)
    fake, odd = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    d = _abi.st_desc_t(1, 2, 256, 64, 1, 0)
    # a chunk counter per (batch, head) (256 B after rounding), then 256 rows of cache -> 4 chunks of
    # 64 keys, 68 floats each, per (batch, head), rounded to 256 B
    need = lib.st_attn_decode_workspace_bytes(ctypes.byref(d), lay.handle)
    assert need == 256 + 2304
    ws = ctypes.c_void_p(1 << 24)

    def call(q=fake, pos=100, desc=d, w=ws, wb=need):
        return lib.st_attn_decode(q, fake, fake, lay.handle, pos, fake, fake, w, wb, ctypes.byref(desc), None)

    assert call(q=None) == 1                      # NULL pointer
    assert call(pos=-1) == 1 and call(pos=256) == 1   # position outside [0, n)
    assert call(desc=_abi.st_desc_t(1, 3, 256, 64, 1, 0)) == 1   # heads are not the layout's
    assert call(desc=_abi.st_desc_t(1, 2, 512, 64, 1, 0)) == 1   # n is not the layout's
    assert call(desc=_abi.st_desc_t(1, 2, 256, 64, 1, 32)) == 2   # no kernel for (64, 32)
    assert call(desc=_abi.st_desc_t(1, 2, 256, 48, 1, 0)) == 2    # nor for 48-wide rows
    assert call(desc=_abi.st_desc_t(1, 2, 256, 64, 1, -1)) == 1   # negative value width
    # the chunk record is dv + 4 floats: 2 x 4 x 132 x 4 bytes at dv = 128
    wide = _abi.st_desc_t(1, 2, 256, 64, 1, 128)
    assert lib.st_attn_decode_workspace_bytes(ctypes.byref(wide), lay.handle) == 256 + 4352
    assert call(desc=wide) == 8                                  # the 64-wide workspace is too small
    assert call(q=odd) == 3                       # misaligned
    assert call(w=None) == 8 and call(wb=need - 1) == 8          # workspace missing / too small
    keys = np.empty(256, dtype=np.int64)
    cnt = ctypes.c_int64()
    kp = keys.ctypes.data_as(ctypes.c_void_p)
    assert lib.st_decode_row_keys(lay.handle, 2, 0, kp, ctypes.byref(cnt)) == 1   # no head 2
    assert lib.st_decode_row_keys(lay.handle, 0, 256, kp, ctypes.byref(cnt)) == 1
    assert lib.st_decode_row_keys(lay.handle, 1, 40, kp, ctypes.byref(cnt)) == 0
    assert list(keys[:cnt.value]) == [8, 24, 40]  # strided head 2 at i = 40, l = 16


def expand_block_row(row_ptr, col_idx, mask_id, masks, qb, B, n):
    """Dense [B, n] allowed matrix of query block qb from the exported CSR."""
    out = np.zeros((B, n), dtype=bool)
    for e in range(row_ptr[qb], row_ptr[qb + 1]):
        kb, m = col_idx[e], mask_id[e]
        if m < 0:
            blk = np.ones((B, B), dtype=bool)
        else:
            bits = np.unpackbits(masks[m].view(np.uint8), bitorder="little")
            blk = bits.reshape(B, B).astype(bool)
        assert blk.any(), "an empty block is listed"
        cols = slice(kb * B, min(n, kb * B + B))
        out[:, cols] |= blk[:, : cols.stop - cols.start]
        if m >= 0:
            assert not blk.all(), "a FULL block is stored with a mask"
    return out


def oracle_block_row(kind, o, qb, B, n, l, c):
    out = np.zeros((B, n), dtype=bool)
    for r in range(B):
        i = qb * B + r
        if i < n:
            out[r, oracle.row_set(kind, i, l, c, o)] = True
    return out


def check_layout_bitexact(lay, n, l, c, qblocks=None):
    B = lay.block
    seen = set()
    for h in range(lay.num_heads):
        kind, o = lay.head_kind(h)
        if (kind, o) in seen:
            continue
        seen.add((kind, o))
        row_ptr, col_idx, mask_id, masks = lay.export(h)
        nqb = (n + B - 1) // B
        assert len(row_ptr) == nqb + 1
        blocks = range(nqb) if qblocks is None else qblocks
        for qb in blocks:
            got = expand_block_row(row_ptr, col_idx, mask_id, masks, qb, B, n)
            want = oracle_block_row(kind, o, qb, B, n, l, c)
            assert np.array_equal(got, want), (kind, o, qb)
            # a block is listed iff it holds an allowed pair
            listed = set(col_idx[row_ptr[qb]:row_ptr[qb + 1]].tolist())
            active = {j // B for j in np.nonzero(want.any(axis=0))[0]}
            assert listed == active
        assert len(set(map(bytes, masks))) == len(masks), "masks are not deduplicated"


SWEEP = [  # (family, mode, H, n, l, c, block)
    (1, 1, 2, 256, 16, 0, 64), (1, 1, 2, 256, 16, 0, 128), (1, 2, 3, 384, 24, 0, 64),
    (1, 3, 1, 200, 7, 0, 64), (1, 4, 1, 200, 7, 0, 128), (2, 1, 8, 512, 64, 16, 64),
    (2, 2, 4, 384, 32, 8, 128), (2, 4, 3, 300, 20, 5, 64), (2, 1, 4, 256, 256, 32, 128),
]


@pytest.mark.parametrize("cfg", SWEEP)
def test_natural_csr_bitexact_sweep(cfg):
    fam, mode, H, n, l, c, B = cfg
    lay = bsf.Layout(fam, mode, H, n, l, c, block=B)
    check_layout_bitexact(lay, n, l, c)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_natural_csr_bitexact_workloads(name):
    w = WORKLOADS[name]
    B = 64 if w.dtype == "fp32" else 128
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c, block=B)
    nqb = w.n // B
    qbl = None if nqb <= 96 else sorted(set(np.linspace(0, nqb - 1, 24).astype(int).tolist()))
    check_layout_bitexact(lay, w.n, w.l, w.c, qbl)


EXEC_SWEEP = [  # (family, mode, H, n, l, c) -- kernel-runnable layouts, every row checked
    (1, 1, 2, 256, 16, 0), (1, 2, 2, 256, 16, 0), (1, 1, 2, 384, 3, 0), (1, 2, 2, 384, 3, 0),
    (1, 1, 2, 512, 2, 0), (1, 2, 2, 256, 1, 0), (1, 1, 2, 256, 256, 0), (1, 2, 2, 768, 4, 0),
    (2, 1, 8, 512, 128, 32), (2, 2, 4, 512, 128, 32), (2, 1, 4, 1024, 256, 8),
    (2, 2, 4, 768, 64, 16), (2, 4, 4, 384, 128, 128), (1, 1, 2, 3072, 64, 0),
    (1, 2, 2, 3072, 64, 0), (1, 1, 2, 32768, 256, 0), (2, 1, 2, 512, 128, 128),
    (2, 1, 6, 1024, 256, 128), (2, 3, 2, 512, 64, 16), (1, 1, 3, 384, 12, 0),
    # edges: one tile (n = l = 128), l = 1 over one tile, summary runs of 1, 2 and 64 keys
    # (128, 64 and 2 runs per compacted tile), merged fixed heads with c = 1, the 64-head maximum
    (1, 1, 2, 128, 128, 0), (1, 2, 2, 128, 1, 0), (2, 1, 2, 128, 128, 1), (2, 1, 4, 512, 64, 1),
    (2, 2, 2, 256, 128, 2), (2, 1, 2, 512, 128, 64), (2, 2, 2, 512, 64, 1), (2, 1, 64, 256, 128, 2),
]


@pytest.mark.parametrize("cfg", EXEC_SWEEP)
def test_exec_frames_match_sets(cfg):
    fam, mode, H, n, l, c = cfg
    lay = bsf.Layout(fam, mode, H, n, l, c)
    rows = range(n) if n <= 1024 else sorted(set(np.linspace(0, n - 1, 160).astype(int).tolist()))
    for h in range(H):
        kind, o = lay.head_kind(h)
        for i in rows:
            got = lay.exec_row(h, i)
            want = oracle.row_set(kind, i, l, c, o)
            assert np.array_equal(got, want), (cfg, h, i)


def test_exec_tile_counts():
    """Active 128 x 128 tile pairs the kernels compute, per batch element."""
    w = WORKLOADS["fixed_n12288_l128_c32"]
    info = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).info()
    assert info["exec_tiles"] == 5184          # 4 x 96 (same block) + 4 x 1200 (summary)
    assert info["allowed_pairs"] == 78673920   # sum of |A(h, i)| over heads and rows
    assert info["passes"] == 1
    w = WORKLOADS["strided_n12288_l128"]
    info = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).info()
    assert info["exec_tiles"] == 2552
    w = WORKLOADS["strided_merged_n12288_l128"]
    info = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).info()
    assert info["exec_tiles"] == 5104 and info["passes"] == 2
    w = WORKLOADS["strided_n65536_l256"]
    info = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).info()
    assert info["exec_tiles"] == 9204
    for name, wl in WORKLOADS.items():
        info = bsf.Layout(wl.family, wl.head_mode, wl.heads, wl.n, wl.l, wl.c).info()
        kinds = [oracle.head_kinds(wl.family, wl.head_mode, wl.heads, wl.l, wl.c)]
        total = 0
        for kd, off in zip(*kinds[0]):
            total += int(oracle.set_counts(int(kd), wl.n, wl.l, wl.c, int(off)).sum())
        assert info["allowed_pairs"] == total, name


def test_dq_direct_heads():
    """Heads whose every query tile is read by exactly one backward item (summed over passes)
    have their dQ written by the main kernel instead of accumulated."""
    w = WORKLOADS["fixed_n12288_l128_c32"]
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c)
    assert lay.info()["dq_direct_heads"] == 4   # the four same-block heads (l = 128 = one tile)
    for name in ("strided_n12288_l128", "strided_merged_n12288_l128", "strided_n65536_l256",
                 "strided_merged_n3072_l64"):
        wl = WORKLOADS[name]
        assert bsf.Layout(wl.family, wl.head_mode, wl.heads, wl.n, wl.l, wl.c).info()["dq_direct_heads"] == 0
    # n = 512, l = 128, c = 32: the summary keys of all four blocks fill one compacted tile, so the
    # summary head is direct too
    assert bsf.Layout(FIXED, ALTERNATING, 2, 512, 128, 32).info()["dq_direct_heads"] == 2
    # l = 256: odd query tiles read two key tiles of their block; in the summary head, query tile 0
    # (rows 0-127 of block 0, all before the block's summary run) is read by no item, so its dQ
    # rows are left to the accumulator's zeros
    assert bsf.Layout(FIXED, ALTERNATING, 2, 1024, 256, 32).info()["dq_direct_heads"] == 0
    # merged fixed heads: same-block pass plus the earlier blocks' summaries (two items per tile)
    assert bsf.Layout(FIXED, MERGED, 2, 1024, 128, 32).info()["dq_direct_heads"] == 0


@pytest.mark.parametrize("family,mode,H,n,l,c", [
    (STRIDED, ALTERNATING, 2, 512, 16, 0), (STRIDED, MERGED, 2, 512, 16, 0), (STRIDED, MERGED, 1, 384, 128, 0),
    (FIXED, ALTERNATING, 6, 512, 16, 4), (FIXED, MERGED, 4, 512, 16, 4), (FIXED, ALTERNATING, 4, 1024, 128, 32),
    (FIXED, MERGED, 2, 1024, 128, 32)])
def test_decode_row_keys_match_sets(family, mode, H, n, l, c):
    """The cache rows the decode step reads are exactly the oracle's A(h, pos), in order."""
    lay = bsf.Layout(family, mode, H, n, l, c)
    # every position for the short sequences, a sample (both block ends, both sides of 2l) otherwise
    rows = range(n) if n <= 512 else sorted(set(list(range(0, 2 * l + 3)) +
                                                np.linspace(0, n - 1, 40).astype(int).tolist()))
    for h in range(H):
        kind, o = lay.head_kind(h)
        for pos in rows:
            got = lay.decode_row_keys(h, pos)
            want = oracle.row_set(kind, pos, l, c, o)
            assert np.array_equal(got, want), (h, kind, o, pos)
