"""Decode-step parity of the CUDA path (st_attn_decode, through the C ABI binding) against the fp64
oracle's decode, which is pinned to the forward's row pos (test_oracle_decode).

For each workload and position: the query row is the workload's Q[:, :, pos], the caches its K and
V; the decode output must match the oracle at the forward tolerances (O max-abs 2e-2 and
relative L2 5e-3, lse max-abs 1e-3, -inf exactly where the oracle's set is empty), and the CUDA
forward's row pos within the same bar.  Cache rows after pos are overwritten with large values
first: the decode step must not read them.
"""
import numpy as np
import pytest
import torch

from parity import check_o_lse, cuda_inputs, problem_of, to64
from test_fwd_gpu import FP32
from workloads import ALTERNATING, FIXED, MERGED, SINGLE_A2, STRIDED, WORKLOADS, Workload

pytestmark = pytest.mark.gpu

bsf = pytest.importorskip("block_sparse_factorized_b200")

CASES = [WORKLOADS["fixed_n12288_l128_c32"], WORKLOADS["strided_n12288_l128"],
         WORKLOADS["strided_merged_n3072_l64"], WORKLOADS["strided_n65536_l256"],
         Workload("f_merged_n4096_l128_c32", FIXED, MERGED, 4096, 128, 32, 2, 2),
         Workload("f_alt_n2048_l64_c16_H6", FIXED, ALTERNATING, 2048, 64, 16, 1, 6),
         Workload("s_merged_n1536_l48", STRIDED, MERGED, 1536, 48, 0, 2, 3),
         Workload("f_single_a2_n1024_l128_c128", FIXED, SINGLE_A2, 1024, 128, 128, 1, 2)]


def positions(w, count=4, seed=0):
    rng = np.random.default_rng(seed)
    base = {0, 1, w.l - 1, w.l, w.l + 1, 2 * w.l + 5, w.n // 2, w.n - 1}
    base.update(rng.integers(0, w.n, size=count).tolist())
    return sorted(p for p in base if 0 <= p < w.n)


def run_case(w, with_fwd=True):
    (qd, kd, vd, _), (q, k, v, _) = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c, a2_offset_step=w.offset_step).upload()
    if with_fwd:
        o_fwd, lse_fwd = bsf.st_attn_fwd(qd, kd, vd, lay)
    prob = problem_of(w)
    k64, v64 = to64(k), to64(v)
    for pos in positions(w):
        kc, vc = kd.clone(), vd.clone()
        kc[:, :, pos + 1:] = 1e3  # rows the step must not read
        vc[:, :, pos + 1:] = -1e3
        qrow = qd[:, :, pos].contiguous()
        o, lse = bsf.st_attn_decode(qrow, kc, vc, lay, pos)
        torch.cuda.synchronize()
        o_ref, lse_ref = prob.decode(to64(q[:, :, pos]), k64, v64, pos)
        check_o_lse(to64(o), to64(lse), o_ref, lse_ref, f"{w.name} pos {pos}")
        if with_fwd:
            check_o_lse(to64(o), to64(lse), to64(o_fwd[:, :, pos]), to64(lse_fwd[:, :, pos]),
                        f"{w.name} pos {pos} vs forward row")


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_decode_matches_oracle(w):
    run_case(w)


@pytest.mark.parametrize("w", FP32[:4], ids=lambda w: w.name)
def test_decode_fp32(w):
    run_case(w)


def test_decode_empty_set_and_errors():
    """The fixed summary head at pos 0 (offset 0, c < l) has no allowed key: O = 0, lse = -inf;
    positions outside [0, n) are rejected before anything is launched."""
    w = Workload("f_alt_n512_l128_c32", FIXED, ALTERNATING, 512, 128, 32, 1, 2)
    (qd, kd, vd, _), _ = cuda_inputs(w)
    lay = bsf.Layout(w.family, w.head_mode, w.heads, w.n, w.l, w.c)  # not uploaded: not needed
    o, lse = bsf.st_attn_decode(qd[:, :, 0].contiguous(), kd, vd, lay, 0)
    torch.cuda.synchronize()
    assert torch.all(o[:, 1] == 0) and torch.all(torch.isneginf(lse[:, 1]))
    assert torch.all(torch.isfinite(lse[:, 0]))
    for bad in (-1, w.n):
        with pytest.raises(bsf.StError):
            bsf.st_attn_decode(qd[:, :, 0].contiguous(), kd, vd, lay, bad)


@pytest.mark.parametrize("d,dv", [(32, 32), (128, 128), (64, 128)], ids=lambda x: str(x))
@pytest.mark.parametrize("w", [WORKLOADS["fixed_n12288_l128_c32"], WORKLOADS["strided_merged_n3072_l64"],
                               Workload("f_merged_n4096_l128_c32", FIXED, MERGED, 4096, 128, 32, 2, 2)],
                         ids=lambda w: w.name)
def test_decode_widths(w, d, dv):
    """Query-key rows of width d, value rows of width dv ("Sparse Transformers 深度解读报告" §4.5's
    per-head widths): the decode step against the oracle's decode and the forward's row pos."""
    run_case(w.with_(d=d, dv=dv))


@pytest.mark.parametrize("d,dv", [(32, 32), (64, 128)], ids=lambda x: str(x))
def test_decode_widths_fp32(d, dv):
    """fp32 I/O at the other widths (the forward has no fp32 kernel there: oracle only)."""
    run_case(FP32[0].with_(d=d, dv=dv), with_fwd=False)


def test_decode_long_rows():
    """Long rows: a fixed summary head at n = 2^18 has up to 65,664 allowed keys, over a thousand
    64-key chunks of one row, combined through the workspace by the row's last chunk."""
    run_case(Workload("f_alt_n262144_l128_c32", FIXED, ALTERNATING, 1 << 18, 128, 32, 1, 2))
