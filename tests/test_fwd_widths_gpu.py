"""Forward parity at the other head widths: query-key rows of width d and value rows of width dv
("Sparse Transformers 深度解读报告" §4.5: per-head widths 32 for ImageNet 64 (512 / 16 heads),
64 for Enwik8 (512 / 8), 128 for CIFAR-10 (256 / 2) whose query-key projection is half-size,
d = 64 against dv = 128).

Every element of small cases (each frame: natural, grid column, summary; merged heads, whose
second pass folds O of width dv into the first pass's) and sampled rows of the n = 12288 fixed
workload against the fp64 oracle at the forward tolerances (O max-abs 2e-2 and relative L2 5e-3,
lse max-abs 1e-3, -inf exactly on empty rows).  Scores are scaled by 1/sqrt(d).
"""
import numpy as np
import pytest
import torch

from parity import check_o_lse, cuda_inputs, problem_of, sample_rows, to64
from workloads import ALTERNATING, FIXED, MERGED, STRIDED, WORKLOADS, Workload

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")

WIDTHS = [(32, 32), (128, 128), (64, 128)]

SMALL = [
    Workload("s_n768_l24", STRIDED, ALTERNATING, 768, 24, 0, 2, 4),
    Workload("s_n384_l3_R128", STRIDED, ALTERNATING, 384, 3, 0, 1, 2),
    Workload("s_merged_n768_l24", STRIDED, MERGED, 768, 24, 0, 2, 2),
    Workload("f_n1024_l128_c32", FIXED, ALTERNATING, 1024, 128, 32, 2, 8),
    Workload("f_n1024_l256_c8", FIXED, ALTERNATING, 1024, 256, 8, 1, 4),
    Workload("f_merged_n1024_l128_c32", FIXED, MERGED, 1024, 128, 32, 1, 4),
]


def layout_of(w):
    return bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c, a2_offset_step=w.offset_step).upload()


@pytest.mark.parametrize("d,dv", WIDTHS, ids=lambda x: str(x))
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_fwd_widths_all_elements(w, d, dv):
    w = w.with_(d=d, dv=dv)
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    lay = layout_of(w)
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    torch.cuda.synchronize()
    lay.check()
    assert o.shape == (w.batch, w.heads, w.n, dv)
    o_ref, lse_ref = problem_of(w).fwd(to64(q), to64(k), to64(v))
    check_o_lse(to64(o), to64(lse), o_ref, lse_ref, f"{w.name} d={d} dv={dv}")


@pytest.mark.parametrize("d,dv", WIDTHS, ids=lambda x: str(x))
def test_fwd_widths_full_size_sampled_rows(d, dv):
    w = WORKLOADS["fixed_n12288_l128_c32"].with_(d=d, dv=dv)
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    lay = layout_of(w)
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    torch.cuda.synchronize()
    lay.check()
    rows = sample_rows(w, 256)
    o_ref, lse_ref = problem_of(w).fwd_rows(to64(q), to64(k), to64(v), rows)
    check_o_lse(to64(o).reshape(-1, dv)[rows], to64(lse).reshape(-1)[rows], o_ref, lse_ref,
                f"{w.name} d={d} dv={dv}")


@pytest.mark.parametrize("d,dv", WIDTHS, ids=lambda x: str(x))
def test_fwd_widths_zero_query_closed_form(d, dv):
    """Q = 0: lse_i = ln |A(i)| and O_i is the mean of the allowed value rows (any width)."""
    w = Workload("f_n1024_l128_c32", FIXED, ALTERNATING, 1024, 128, 32, 1, 4, d=d, dv=dv)
    (qd, kd, vd, _), (_, _, v, _) = cuda_inputs(w)
    qd.zero_()
    lay = layout_of(w)
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    torch.cuda.synchronize()
    o_ref, lse_ref = problem_of(w).fwd(np.zeros(w.shape()), to64(kd.cpu()), to64(v))
    check_o_lse(to64(o), to64(lse), o_ref, lse_ref, f"zero query d={d} dv={dv}")


def test_widths_without_kernels_are_rejected():
    """The fp32 forward takes 64-wide rows only."""
    w = Workload("f_n512_l128_c32", FIXED, ALTERNATING, 512, 128, 32, 1, 2, d=32, dv=32)
    (qd, kd, vd, dod), _ = cuda_inputs(w)
    lay = layout_of(w)
    with pytest.raises(bsf.StError):
        bsf.st_attn_fwd(qd.float(), kd.float(), vd.float(), lay)
