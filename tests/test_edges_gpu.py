"""Parity at the edge shapes of the execution frames, every element against the fp64 oracle:
one 128-row tile (n = l = 128, and l = 1 over one tile), fixed-pattern summary runs of 1, 2 and
64 keys (128, 64 and 2 runs per compacted tile), merged fixed heads with c = 1, the 64-head
maximum, and a large batch x heads count.  The same shapes' frames are checked against the
oracle's sets on the CPU (test_layout's execution-frame sweep)."""
import pytest
import torch

from parity import check_grads, check_o_lse, cuda_inputs, problem_of, to64
from workloads import ALTERNATING, FIXED, MERGED, SINGLE_A2, STRIDED, Workload

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")

EDGES = [
    Workload("s_n128_l128", STRIDED, ALTERNATING, 128, 128, 0, 2, 2),
    Workload("s_n128_l1", STRIDED, ALTERNATING, 128, 1, 0, 1, 2),
    Workload("f_n128_l128_c1", FIXED, ALTERNATING, 128, 128, 1, 1, 2),
    Workload("f_n512_l64_c1", FIXED, ALTERNATING, 512, 64, 1, 1, 4),
    Workload("f_merged_n256_l128_c2", FIXED, MERGED, 256, 128, 2, 2, 2),
    Workload("f_n512_l128_c64", FIXED, ALTERNATING, 512, 128, 64, 1, 2),
    Workload("f_merged_n512_l64_c1", FIXED, MERGED, 512, 64, 1, 1, 2),
    Workload("f_n256_l128_c2_H64", FIXED, ALTERNATING, 256, 128, 2, 1, 64),
    Workload("f_single_a2_n256_l128_c4_b32_H16", FIXED, SINGLE_A2, 256, 128, 4, 32, 16),
]


def run(w):
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c, a2_offset_step=w.offset_step).upload()
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    dq, dk, dv = bsf.st_attn_bwd(qd, kd, vd, o, lse, dod, lay)
    torch.cuda.synchronize()
    lay.check()
    return (o, lse, dq, dk, dv), (q, k, v, do)


@pytest.mark.parametrize("w", EDGES, ids=lambda w: w.name)
def test_edges_fwd_bwd_all_elements(w):
    (o, lse, dq, dk, dv), (q, k, v, do) = run(w)
    prob = problem_of(w)
    o_ref, lse_ref = prob.fwd(to64(q), to64(k), to64(v))
    check_o_lse(to64(o), to64(lse), o_ref, lse_ref, w.name)
    ref = prob.bwd(to64(q), to64(k), to64(v), to64(do))
    check_grads((to64(dq), to64(dk), to64(dv)), ref, w.name)
