"""The failure path of the kernels, exercised without a real failure.

Every wait in the kernels is bounded (1 s): a wait that runs out records a timeout in the
layout's device error word and its kernel ends, so the GPU is never left hanging and the host
learns of it from st_layout_check.  st_selftest_wait_timeout launches one warp whose only wait is
on an mbarrier that nothing completes; the test checks that the timeout is reported once
(ST_ERR_DEVICE_TIMEOUT, then cleared) and that the context stays usable: a forward pass right
after it matches the oracle.
"""
import pytest
import torch

from parity import check_o_lse, cuda_inputs, problem_of, to64
from workloads import ALTERNATING, FIXED, Workload

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")


def test_device_timeout_is_reported_and_context_stays_usable():
    w = Workload("f_n512_l128_c32", FIXED, ALTERNATING, 512, 128, 32, 1, 2)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c).upload()
    lay.check()  # nothing recorded yet
    lay.selftest_wait_timeout()
    with pytest.raises(bsf.StError) as exc:
        lay.check()  # waits for the warp, which gives up after the wait limit
    assert exc.value.status == bsf.ST_ERR_DEVICE_TIMEOUT
    lay.check()  # the error word was cleared
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    o, lse = bsf.st_attn_fwd(qd, kd, vd, lay)
    torch.cuda.synchronize()
    lay.check()
    o_ref, lse_ref = problem_of(w).fwd(to64(q), to64(k), to64(v))
    check_o_lse(to64(o), to64(lse), o_ref, lse_ref, "forward after a device timeout")
