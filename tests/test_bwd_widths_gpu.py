"""Backward parity at the other head widths: query-key rows of width d, value rows of width dv
("Sparse Transformers 深度解读报告" §4.5: per-head widths 32 for ImageNet 64 (512 / 16 heads)
and, for CIFAR-10 (256 / 2 heads), value rows of 128 with a half-size query-key projection, d = 64).

Every element of dQ (width d), dK (width d) and dV (width dv) of small cases -- each frame, merged
heads, key tiles long enough to be split into chunks -- and of a whole workload, against the
fp64 oracle at the gradient tolerance (relative L2 <= 1e-2 over each whole tensor; scores scaled
by 1/sqrt(d)).  Rows of 128 for both widths have no backward kernel: TMEM holds S, dP, dV, dK
and dQ of one key tile in 512 columns only up to d + dv + d = 256, so that call is refused.
"""
import numpy as np
import pytest
import torch

from parity import check_grads, cuda_inputs, problem_of, to64
from workloads import ALTERNATING, FIXED, MERGED, STRIDED, Workload

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")

WIDTHS = [(32, 32), (64, 128)]

SMALL = [
    Workload("s_n768_l24", STRIDED, ALTERNATING, 768, 24, 0, 2, 4),
    Workload("s_n384_l3_R128", STRIDED, ALTERNATING, 384, 3, 0, 1, 2),
    Workload("s_merged_n768_l24", STRIDED, MERGED, 768, 24, 0, 2, 2),
    Workload("f_n1024_l128_c32", FIXED, ALTERNATING, 1024, 128, 32, 2, 8),
    Workload("f_n1024_l256_c8", FIXED, ALTERNATING, 1024, 256, 8, 1, 4),
    Workload("f_merged_n1024_l128_c32", FIXED, MERGED, 1024, 128, 32, 1, 4),
    # summary key tile 0 read by 96 query tiles: split into chunks whose partials are summed
    Workload("f_n12288_l128_c32_long", FIXED, ALTERNATING, 12288, 128, 32, 1, 2),
    Workload("f_merged_n6144_l128_c32_long", FIXED, MERGED, 6144, 128, 32, 1, 1),
]

# (the d = 32 benchmark workload, strided n = 12288, is compared whole in test_full_size_gpu.py)
FULL = [Workload("strided_merged_n3072_l64_dv128", STRIDED, MERGED, 3072, 64, 0, 4, 2, d=64, dv=128)]


def run(w):
    (qd, kd, vd, dod), host = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c, a2_offset_step=w.offset_step).upload()
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    dq, dk, dv = bsf.st_attn_bwd(qd, kd, vd, o, lse, dod, lay, check=True)
    assert dq.shape == qd.shape and dk.shape == kd.shape and dv.shape == vd.shape
    ref = problem_of(w).bwd(*(to64(t) for t in host))
    return check_grads((to64(dq), to64(dk), to64(dv)), ref, f"{w.name} d={w.d} dv={w.dv or w.d}")


@pytest.mark.parametrize("d,dv", WIDTHS, ids=lambda x: str(x))
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_bwd_widths_all_elements(w, d, dv):
    run(w.with_(d=d, dv=dv))


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_bwd_widths_whole_workload(w):
    m = run(w)
    print(f"\n[widths parity] {w.name}: dQ/dK/dV rel-L2 {m['dq']:.2e}/{m['dk']:.2e}/{m['dv']:.2e}")


def test_bwd_rows_of_128_are_refused():
    w = Workload("f_n512_l128_c32", FIXED, ALTERNATING, 512, 128, 32, 1, 2, d=128, dv=128)
    (qd, kd, vd, dod), _ = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)  # the forward has a kernel for them
    with pytest.raises(bsf.StError) as e:
        bsf.st_attn_bwd(qd, kd, vd, o, lse, dod, lay)
    assert e.value.status == 2  # ST_ERR_UNSUPPORTED
