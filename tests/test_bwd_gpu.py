"""Backward parity of the CUDA path (recomputing backward, through the C ABI binding) against the
fp64 oracle's plain-calculus gradients.

Small cases compare every element of dQ, dK and dV; the long sequences (2^18 and 2^20 keys)
compare dQ on sampled query rows and dK, dV on sampled keys, each evaluated one by one by the
oracle (the benchmark workloads are compared on every element in test_full_size_gpu.py).  Keys that no
query reads must get exactly zero gradient, rows with no allowed key exactly zero dQ.
"""
import numpy as np
import pytest
import torch

import ctypes

import oracle
from parity import check_grads, cuda_inputs, problem_of, rel_l2, sample_rows, to64
from test_fwd_gpu import FP32, SMALL
from workloads import ALTERNATING, FIXED, MERGED, STRIDED, WORKLOADS, Workload

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")


def run(w, qd, kd, vd, dod):
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c,
                     a2_offset_step=w.offset_step).upload()
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    dq, dk, dv = bsf.st_attn_bwd(qd, kd, vd, o, lse, dod, lay)
    torch.cuda.synchronize()
    lay.check()
    return lay, o, lse, dq, dk, dv


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_bwd_small_all_elements(w):
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    _, _, _, dq, dk, dv = run(w, qd, kd, vd, dod)
    ref = problem_of(w).bwd(to64(q), to64(k), to64(v), to64(do))
    check_grads((to64(dq), to64(dk), to64(dv)), ref, w.name)
    # structural zeros: keys read by nobody, rows that read nobody
    kinds, offs = oracle.head_kinds(w.family, w.head_mode, w.heads, w.l, w.c, w.offset_step)
    for h in range(w.heads):
        cnt = oracle.set_counts(int(kinds[h]), w.n, w.l, w.c, int(offs[h]))
        empty = np.nonzero(cnt == 0)[0]
        assert torch.all(dq[:, h, empty] == 0)
        unread = np.nonzero(np.all(ref[1][:, h] == 0, axis=(0, 2)) & np.all(ref[2][:, h] == 0, axis=(0, 2)))[0]
        assert torch.all(dk[:, h, unread] == 0) and torch.all(dv[:, h, unread] == 0)


# longer sequences (l about sqrt(n)), sampled rows and keys: frames and work lists at 2^18 and 2^20
# keys (the benchmark workloads are compared on every element in test_full_size_gpu.py)
BIG = [Workload("s_n262144_l512_long", STRIDED, ALTERNATING, 262144, 512, 0, 1, 4),
       Workload("s_merged_n262144_l512_long", STRIDED, MERGED, 262144, 512, 0, 1, 2),
       Workload("s_n1048576_l1024_long", STRIDED, ALTERNATING, 1048576, 1024, 0, 1, 2),
       Workload("f_n262144_l512_c128_long", FIXED, ALTERNATING, 262144, 512, 128, 1, 2)]


@pytest.mark.parametrize("w", FP32, ids=lambda w: w.name)
def test_bwd_fp32_all_elements(w):
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    _, _, _, dq, dk, dv = run(w, qd, kd, vd, dod)
    assert dq.dtype == dk.dtype == dv.dtype == torch.float32
    ref = problem_of(w).bwd(to64(q), to64(k), to64(v), to64(do))
    check_grads((to64(dq), to64(dk), to64(dv)), ref, w.name)


def sample_keys(w, count, seed=1):
    """Flat key indices (b*H + h)*n + j: block and tile edges of every head plus random keys.  A
    summary key of the fixed pattern's second head (or of a merged fixed head) is read by every
    later row, and the oracle evaluates each reading row in full; at 2^18 keys those heads are
    sampled in their last two blocks only, where the reading rows are few.  Same-block and strided
    heads are sampled anywhere."""
    rng = np.random.default_rng(seed)
    kinds, _ = oracle.head_kinds(w.family, w.head_mode, w.heads, w.l, w.c, w.offset_step)
    keys = set()
    for b in range(w.batch):
        for h in range(w.heads):
            base = (b * w.heads + h) * w.n
            late = w.n >= (1 << 18) and int(kinds[h]) in (oracle.FA2, oracle.FU)
            lo = w.n - 2 * w.l if late else 0
            edges = (0, w.l - 1, w.l - w.c - 1 if w.c else 1, 127, 128, w.n // 2 - 1, w.n - 1)
            for j in edges:
                if lo <= j < w.n:
                    keys.add(base + j)
            per_head = max(1, count // (w.batch * w.heads))
            keys.update((base + rng.integers(lo, w.n, size=per_head)).tolist())
    return np.array(sorted(keys), dtype=np.int64)


@pytest.mark.parametrize("w", BIG, ids=lambda w: w.name)
def test_bwd_full_size_sampled(w):
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    _, _, _, dq, dk, dv = run(w, qd, kd, vd, dod)
    prob = problem_of(w)
    f64 = [to64(t) for t in (q, k, v, do)]
    rows = sample_rows(w, 200)
    dq_ref, _, _ = prob.bwd_rows(*f64, rows)
    keys = sample_keys(w, 120 if w.n < (1 << 20) else 24)  # the oracle's key pass grows with n
    dk_ref, dv_ref = prob.bwd_keys(*f64, keys)
    got = (to64(dq).reshape(-1, 64)[rows], to64(dk).reshape(-1, 64)[keys],
           to64(dv).reshape(-1, 64)[keys])
    check_grads(got, (dq_ref, dk_ref, dv_ref), w.name)
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()


def test_bwd_repeatable():
    """dK and dV accumulate in a fixed order (bitwise repeatable); dQ uses atomics."""
    w = SMALL[9]
    (qd, kd, vd, dod), _ = cuda_inputs(w)
    _, o, lse, dq1, dk1, dv1 = run(w, qd, kd, vd, dod)
    _, _, _, dq2, dk2, dv2 = run(w, qd, kd, vd, dod)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    assert rel_l2(to64(dq1), to64(dq2)) < 1e-3


def test_autograd_wrapper():
    w = SMALL[1]
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (qd, kd, vd))
    out = bsf.SparseAttention.apply(qg, kg, vg, lay)
    out.backward(dod)
    ref = problem_of(w).bwd(to64(q), to64(k), to64(v), to64(do))
    check_grads((to64(qg.grad), to64(kg.grad), to64(vg.grad)), ref, "autograd")


@pytest.mark.parametrize("w", [Workload("f_n512_l128_c32_b2", FIXED, ALTERNATING, 512, 128, 32, 2, 2),
                               Workload("f_n1024_l128_c32_H4", FIXED, ALTERNATING, 1024, 128, 32, 1, 4)],
                         ids=lambda w: w.name)
def test_bwd_phases_and_direct_dq(w):
    """st_attn_bwd_prepare / _main / _finish called one by one give st_attn_bwd's results, and
    the dQ of heads whose query tiles are each read by a single backward item (written by the main
    kernel, no accumulation) is bitwise repeatable."""
    from block_sparse_factorized_b200 import _abi
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    lay, o, lse, dq1, dk1, dv1 = run(w, qd, kd, vd, dod)
    lib = _abi.load()
    desc = bsf._desc(qd)
    nbytes = int(lib.st_attn_bwd_workspace_bytes(ctypes.byref(desc), lay.handle))
    ws = torch.empty(nbytes, dtype=torch.uint8, device=qd.device)
    dq2, dk2, dv2 = (torch.full_like(qd, float("nan")) for _ in range(3))
    P = ctypes.c_void_p
    ptr = lambda t: P(t.data_ptr())  # noqa: E731
    sp = P(torch.cuda.current_stream().cuda_stream)
    _abi.check(lib.st_attn_bwd_prepare(ptr(o), ptr(dod), lay.handle, ptr(dk2), ptr(dv2), ptr(ws), nbytes,
                                       ctypes.byref(desc), sp), "st_attn_bwd_prepare")
    _abi.check(lib.st_attn_bwd_main(ptr(qd), ptr(kd), ptr(vd), ptr(lse), ptr(dod), lay.handle, ptr(dq2),
                                    ptr(dk2), ptr(dv2), ptr(ws), nbytes, ctypes.byref(desc), sp),
               "st_attn_bwd_main")
    _abi.check(lib.st_attn_bwd_finish(lay.handle, ptr(dq2), ptr(ws), nbytes, ctypes.byref(desc), sp),
               "st_attn_bwd_finish")
    torch.cuda.synchronize()
    lay.check()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
    info = lay.info()
    kinds, _ = oracle.head_kinds(w.family, w.head_mode, w.heads, w.l, w.c, w.offset_step)
    # which heads are direct: the same-block heads (one key tile per query tile at l = 128), and
    # the summary heads when every summary key fits one compacted tile (n / l * c <= 128)
    direct = [h for h in range(w.heads)
              if int(kinds[h]) == oracle.FA1 or (w.n // w.l) * w.c <= 128]
    assert info["dq_direct_heads"] == len(direct)
    for h in range(w.heads):
        if h in direct:
            assert torch.equal(dq1[:, h], dq2[:, h]), h
        else:
            assert rel_l2(to64(dq1[:, h]), to64(dq2[:, h])) < 1e-3, h
    ref = problem_of(w).bwd(to64(q), to64(k), to64(v), to64(do))
    check_grads((to64(dq2), to64(dk2), to64(dv2)), ref, w.name)


@pytest.mark.parametrize("w", [SMALL[2], SMALL[7], SMALL[15]], ids=lambda w: w.name)
def test_bwd_guard_zones(w):
    """dQ, dK and dV written into views with guard zones on both sides: the backward pass (TMA
    stores clipped at the frame edges, the dK/dV partials of split key tiles, merge passes) writes
    nothing outside its outputs, and the gradients still match the oracle."""
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    numel, guard = qd.numel(), 8192
    bufs = [torch.full((numel + 2 * guard,), 7.0, dtype=qd.dtype, device=qd.device) for _ in range(3)]
    dq, dk, dv = (b[guard:guard + numel].view_as(qd) for b in bufs)
    bsf.st_attn_bwd(qd, kd, vd, o, lse, dod, lay, dq=dq, dk=dk, dv=dv, check=True)
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.all(b[:guard] == 7.0) and torch.all(b[-guard:] == 7.0)
    ref = problem_of(w).bwd(to64(q), to64(k), to64(v), to64(do))
    check_grads((to64(dq), to64(dk), to64(dv)), ref, w.name)
