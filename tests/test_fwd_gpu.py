"""Forward parity of the CUDA path (through the C ABI binding) against the fp64 oracle.

Small cases compare every element; the long sequences (2^18 and 2^20 keys) compare sampled rows
evaluated one by one by the oracle (the benchmark workloads are compared on every element in
test_full_size_gpu.py).  Invariants that hold at
any size (Q = 0 closed form, masked-V perturbation, determinism, guard zones) run on the GPU too.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import check_o_lse, cuda_inputs, problem_of, sample_rows, to64
from workloads import (ALTERNATING, FIXED, MERGED, SINGLE_A1, SINGLE_A2, STRIDED, WORKLOADS,
                       Workload)

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")

SMALL = [
    Workload("s_n256_l16", STRIDED, ALTERNATING, 256, 16, 0, 1, 2),
    Workload("s_n768_l24", STRIDED, ALTERNATING, 768, 24, 0, 2, 4),
    Workload("s_n384_l3_R128", STRIDED, ALTERNATING, 384, 3, 0, 1, 2),
    Workload("s_n512_l1", STRIDED, SINGLE_A2, 512, 1, 0, 1, 2),
    Workload("s_n1024_l4_R256", STRIDED, ALTERNATING, 1024, 4, 0, 1, 2),
    Workload("s_n256_l256", STRIDED, ALTERNATING, 256, 256, 0, 1, 2),
    Workload("s_single_a1_n640_l40", STRIDED, SINGLE_A1, 640, 40, 0, 1, 2),
    Workload("s_merged_n768_l24", STRIDED, MERGED, 768, 24, 0, 2, 2),
    Workload("s_merged_n3072_l64", STRIDED, MERGED, 3072, 64, 0, 1, 2),
    Workload("f_n1024_l128_c32", FIXED, ALTERNATING, 1024, 128, 32, 2, 8),
    Workload("f_n1024_l64_c16", FIXED, ALTERNATING, 1024, 64, 16, 1, 4),
    Workload("f_n1024_l256_c8", FIXED, ALTERNATING, 1024, 256, 8, 1, 4),
    Workload("f_single_a2_n512_l32_c4", FIXED, SINGLE_A2, 512, 32, 4, 1, 8),
    Workload("f_merged_n1024_l128_c32", FIXED, MERGED, 1024, 128, 32, 1, 4),
    # long backward items: summary key tile 0 is read by 96 query tiles, more than one backward
    # chunk (48), so its dK/dV are the sum of two chunks' partials -- also in a merge pass
    Workload("f_n12288_l128_c32_long", FIXED, ALTERNATING, 12288, 128, 32, 1, 2),
    Workload("f_merged_n12288_l128_c32_long", FIXED, MERGED, 12288, 128, 32, 1, 1),
    # degenerate sets: c = l (pattern 2 reads every earlier key), c = 128 with three head-2
    # offsets, fixed head 1 alone, odd batch and head counts
    Workload("f_n512_l128_c128", FIXED, ALTERNATING, 512, 128, 128, 1, 2),
    Workload("f_n1024_l256_c128_H6", FIXED, ALTERNATING, 1024, 256, 128, 1, 6),
    Workload("f_single_a1_n512_l64", FIXED, SINGLE_A1, 512, 64, 16, 1, 2),
    Workload("s_n384_l12_b3_H3", STRIDED, ALTERNATING, 384, 12, 0, 3, 3),
]


def run_fwd(w, qd, kd, vd):
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c,
                     a2_offset_step=w.offset_step).upload()
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    torch.cuda.synchronize()
    lay.check()
    return lay, o, lse


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fwd_small_all_elements(w):
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    _, o, lse = run_fwd(w, qd, kd, vd)
    o_ref, lse_ref = problem_of(w).fwd(to64(q), to64(k), to64(v))
    check_o_lse(to64(o), lse.cpu().numpy(), o_ref, lse_ref, w.name)


# longer sequences (l about sqrt(n)), sampled rows: frames and work lists at 2^18 and 2^20 keys
# (the benchmark workloads themselves are compared on every element in test_full_size_gpu.py)
BIG = [Workload("s_n262144_l512_long", STRIDED, ALTERNATING, 262144, 512, 0, 1, 4),
        Workload("s_merged_n262144_l512_long", STRIDED, MERGED, 262144, 512, 0, 1, 2),
        Workload("s_n1048576_l1024_long", STRIDED, ALTERNATING, 1048576, 1024, 0, 1, 2),
        Workload("f_n262144_l512_c128_long", FIXED, ALTERNATING, 262144, 512, 128, 1, 2)]

# fp32 I/O: the n = 256 fp32 workload plus fixed and merged variants, every element compared
FP32 = [WORKLOADS["strided_n256_l16_fp32"],
        Workload("f32_fixed_n512_l128_c32", FIXED, ALTERNATING, 512, 128, 32, 1, 4, dtype="fp32"),
        Workload("f32_s_merged_n768_l24", STRIDED, MERGED, 768, 24, 0, 1, 2, dtype="fp32"),
        Workload("f32_f_merged_n512_l128_c32", FIXED, MERGED, 512, 128, 32, 1, 2, dtype="fp32"),
        Workload("f32_fixed_n12288_l128_c32_long", FIXED, SINGLE_A2, 12288, 128, 32, 1, 1, dtype="fp32")]


@pytest.mark.parametrize("w", FP32, ids=lambda w: w.name)
def test_fwd_fp32_all_elements(w):
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    assert qd.dtype == torch.float32
    _, o, lse = run_fwd(w, qd, kd, vd)
    assert o.dtype == torch.float32
    o_ref, lse_ref = problem_of(w).fwd(to64(q), to64(k), to64(v))
    check_o_lse(to64(o), lse.cpu().numpy(), o_ref, lse_ref, w.name)


@pytest.mark.parametrize("w", BIG, ids=lambda w: w.name)
def test_fwd_full_size_sampled_rows(w):
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    _, o, lse = run_fwd(w, qd, kd, vd)
    rows = sample_rows(w, 400)
    o_ref, lse_ref = problem_of(w).fwd_rows(to64(q), to64(k), to64(v), rows)
    o_got = to64(o).reshape(-1, w.d)[rows]
    lse_got = lse.cpu().numpy().reshape(-1)[rows].astype(np.float64)
    check_o_lse(o_got, lse_got, o_ref, lse_ref, w.name)
    assert torch.isfinite(o).all()


@pytest.mark.parametrize("w", [SMALL[1], SMALL[7], SMALL[9], SMALL[11], SMALL[13]],
                         ids=lambda w: w.name)
def test_fwd_zero_query_closed_form(w):
    """Q = 0: lse_i = ln |A(i)| and O_i = mean of the allowed v_j (uniform weights)."""
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    qd = torch.zeros_like(qd)
    _, o, lse = run_fwd(w, qd, kd, vd)
    kinds, offs = oracle.head_kinds(w.family, w.head_mode, w.heads, w.l, w.c, w.offset_step)
    lse = lse.cpu().numpy()
    o = to64(o)
    v64 = to64(v)
    for h in range(w.heads):
        cnt = oracle.set_counts(int(kinds[h]), w.n, w.l, w.c, int(offs[h]))
        for b in range(w.batch):
            want = np.where(cnt > 0, np.log(np.maximum(cnt, 1)), -np.inf)
            got = lse[b, h]
            assert np.array_equal(np.isneginf(got), np.isneginf(want))
            fin = cnt > 0
            assert np.abs(got[fin] - want[fin]).max() <= 1e-3
            for i in np.linspace(0, w.n - 1, 17).astype(int):
                s = oracle.row_set(int(kinds[h]), int(i), w.l, w.c, int(offs[h]))
                if len(s):
                    mean = v64[b, h, s].mean(axis=0)
                    assert np.abs(o[b, h, i] - mean).max() <= 2e-2


def test_fwd_masked_value_perturbation():
    w = SMALL[9]
    (qd, kd, vd, _), _ = cuda_inputs(w)
    _, o1, _ = run_fwd(w, qd, kd, vd)
    kinds, offs = oracle.head_kinds(w.family, w.head_mode, w.heads, w.l, w.c)
    # for head 1 (fixed pattern-2) no query in [200, 1023] reads key 5 (not a summary position)
    vd2 = vd.clone()
    vd2[:, 1, 5] += 10000.0
    _, o2, _ = run_fwd(w, qd, kd, vd2)
    assert torch.equal(o1[:, 1], o2[:, 1])
    # control: a summary key does move the output of later rows
    vd3 = vd.clone()
    vd3[:, 1, 100] += 10000.0
    _, o3, _ = run_fwd(w, qd, kd, vd3)
    assert not torch.equal(o1[:, 1, 200:], o3[:, 1, 200:])


def test_fwd_masked_value_inside_active_tiles():
    """Perturbed keys that share a tile with allowed keys but are masked for the checked rows."""
    w = SMALL[1]  # strided, l = 24: head 0 band {i-24..i}, head 1 stride-24 ladder
    (qd, kd, vd, _), _ = cuda_inputs(w)
    _, o1, _ = run_fwd(w, qd, kd, vd)
    vd2 = vd.clone()
    vd2[:, 0, 60] += 10000.0   # band: rows 85.. and rows < 60 do not read key 60
    vd2[:, 1, 61] += 10000.0   # stride: only rows 61 + 24 m read key 61
    _, o2, _ = run_fwd(w, qd, kd, vd2)
    assert torch.equal(o1[:, 0, :60], o2[:, 0, :60])
    assert torch.equal(o1[:, 0, 85:], o2[:, 0, 85:])
    assert not torch.equal(o1[:, 0, 60:85], o2[:, 0, 60:85])
    readers = torch.arange(61, w.n, 24)
    others = torch.ones(w.n, dtype=torch.bool)
    others[readers] = False
    assert torch.equal(o1[:, 1, others], o2[:, 1, others])
    assert not torch.equal(o1[:, 1, readers], o2[:, 1, readers])


def test_fwd_deterministic_and_guarded():
    w = SMALL[13]
    (qd, kd, vd, _), _ = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    numel = qd.numel()
    guard = 4096
    obuf = torch.full((numel + 2 * guard,), 7.0, dtype=qd.dtype, device=qd.device)
    lbuf = torch.full((numel // 64 + 2 * guard,), 7.0, dtype=torch.float32, device=qd.device)
    o = obuf[guard:guard + numel].view_as(qd)
    lse = lbuf[guard:guard + numel // 64].view(qd.shape[:3])
    bsf.st_attn_fwd(qd, kd, vd, lay, o=o, lse=lse)
    first = (o.clone(), lse.clone())
    bsf.st_attn_fwd(qd, kd, vd, lay, o=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(first[0], o) and torch.equal(first[1], lse)
    assert torch.all(obuf[:guard] == 7.0) and torch.all(obuf[-guard:] == 7.0)
    assert torch.all(lbuf[:guard] == 7.0) and torch.all(lbuf[-guard:] == 7.0)
    lay.check()


def test_fwd_workspace_too_small_is_refused():
    """A caller's workspace smaller than st_attn_fwd_workspace_bytes is refused with
    ST_ERR_WORKSPACE before anything runs, whatever the workspace tensor's dtype (the binding
    sends its size in bytes)."""
    w = FP32[1]  # fp32 I/O: the forward's workspace holds the bf16 high/low copies of q, k, v
    (qd, kd, vd, _), _ = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    need = bsf.st_attn_fwd_workspace_bytes(qd, lay)
    assert need > 1 << 16
    small = torch.empty(need // 8, dtype=torch.float32, device=qd.device)  # need / 2 bytes
    with pytest.raises(bsf.StError) as e:
        bsf.st_attn_fwd(qd, kd, vd, lay, workspace=small)
    assert e.value.status == 8  # ST_ERR_WORKSPACE
    ok = torch.empty(need // 4 + 1, dtype=torch.float32, device=qd.device)
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay, workspace=ok, check=True)
    assert torch.isfinite(o).all()
