"""Whole-tensor parity at the benchmark workloads: the CUDA path (through the C ABI binding, in
the launch configuration the benchmark times) against the fp64 oracle's full evaluation.

Every element of O, lse, dQ, dK and dV is compared, and rel-L2 is taken over each whole tensor:
  O:          max-abs <= 2e-2 and rel-L2 <= 5e-3
  lse:        max-abs <= 1e-3, -inf exactly on the rows with no allowed key
  dQ, dK, dV: rel-L2 <= 1e-2 each
The workloads are the strided, fixed and merged shapes that stand in for the pages' image, text
and audio data ("Sparse Transformers（稀疏 Transformer）深度解读报告" §4.1-4.5) -- n from 256 to 65,536.
The longer sequences (n = 2^18, 2^20) stay with sampled rows and keys in the forward and
backward test files, where the oracle's full evaluation would take too long.
"""
import numpy as np
import pytest
import torch

from parity import check_grads, check_o_lse, cuda_inputs, problem_of, to64
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")


@pytest.mark.parametrize("w", list(WORKLOADS.values()), ids=lambda w: w.name)
def test_full_size_all_elements(w):
    (qd, kd, vd, dod), (q, k, v, do) = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c,
                     a2_offset_step=w.offset_step).upload()
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    dq, dk, dv = bsf.st_attn_bwd(qd, kd, vd, o, lse, dod, lay)
    torch.cuda.synchronize()
    lay.check()
    got_o, got_lse = to64(o), lse.cpu().numpy().astype(np.float64)
    got_g = [to64(t) for t in (dq, dk, dv)]
    del qd, kd, vd, dod, o, lse, dq, dk, dv
    prob = problem_of(w)
    f64 = [to64(t) for t in (q, k, v, do)]
    o_ref, lse_ref = prob.fwd(*f64[:3])
    fm = check_o_lse(got_o, got_lse, o_ref, lse_ref, w.name)
    del o_ref, lse_ref, got_o
    g_ref = prob.bwd(*f64)
    gm = check_grads(got_g, g_ref, w.name)
    print(f"\n[full-size parity] {w.name}: O max-abs {fm['o_max_abs']:.2e} rel-L2 {fm['o_rel_l2']:.2e}, "
          f"lse max-abs {fm['lse_max_abs']:.2e}, dQ/dK/dV rel-L2 {gm['dq']:.2e}/{gm['dk']:.2e}/{gm['dv']:.2e}")
