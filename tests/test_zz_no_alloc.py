"""st_attn_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers (a plug-in whose host application owns every device allocation, or code that cannot
afford cudaMalloc's implicit synchronisation) get their scratch from a fixed array inside the
library.  These tests call the entry point through the C ABI and check that two calls in a row
give the same gradients as the ordinary st_attn_bwd with a caller-provided workspace, within the
gradient tolerance the other tests use, that both calls also meet that tolerance against the fp64
oracle, and that a problem too large for the fixed array is refused before anything runs.  The
file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import GRAD_REL_L2, check_grads, cuda_inputs, problem_of, rel_l2, to64
from workloads import ALTERNATING, FIXED, MERGED, STRIDED, WORKLOADS, Workload

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")
from block_sparse_factorized_b200 import _abi  # noqa: E402

CASES = [
    Workload("noalloc_fixed_n1024_l128_c32", FIXED, ALTERNATING, 1024, 128, 32, 2, 4),
    Workload("noalloc_strided_merged_n768_l24", STRIDED, MERGED, 768, 24, 0, 1, 2),
    Workload("noalloc_fp32_strided_n256_l16", STRIDED, ALTERNATING, 256, 16, 0, 1, 2, dtype="fp32"),
]


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point_twice(w):
    lib = _abi.load()
    (q, k, v, do), host = cuda_inputs(w)
    oracle_grads = problem_of(w).bwd(*(to64(t) for t in host))
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    o, lse = bsf.st_attn_fwd(q, k, v, lay)
    ref = bsf.st_attn_bwd(q, k, v, o, lse, do, lay)
    torch.cuda.synchronize()
    desc = bsf._desc(q)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        st = lib.st_attn_bwd_noalloc(_p(q), _p(k), _p(v), _p(o), _p(lse), _p(do), lay.handle,
                                     _p(dq), _p(dk), _p(dv), ctypes.byref(desc), stream)
        assert st == 0, _abi.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        lay.check()
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            assert torch.isfinite(got).all(), (call, name)
            err = rel_l2(to64(got), to64(want))
            assert err <= GRAD_REL_L2, (call, name, err)
        check_grads((to64(dq), to64(dk), to64(dv)), oracle_grads, f"{w.name} call {call}")


def test_noalloc_refuses_problems_beyond_the_fixed_scratch():
    lib = _abi.load()
    w = WORKLOADS["fixed_n12288_l128_c32"]  # needs about 51 MB of scratch
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    desc = _abi.st_desc_t(w.batch, w.heads, w.n, 64, 1, 0)
    assert lib.st_attn_bwd_workspace_bytes(ctypes.byref(desc), lay.handle) > 32 << 20
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    st = lib.st_attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, lay.handle, fake, fake, fake,
                                 ctypes.byref(desc), None)
    assert st == 8  # ST_ERR_WORKSPACE
