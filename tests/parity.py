"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI binding and compare
with the fp64 oracle on the same (rounded) inputs.

Tolerances (bf16 I/O, fp32 accumulation; fp32 I/O uses the same bar):
  O:          max |x - y| <= 2e-2  and  ||x - y|| / ||y|| <= 5e-3
  lse:        max |x - y| <= 1e-3, and -inf exactly where the oracle has -inf (empty rows)
  dQ, dK, dV: ||x - y|| / ||y|| <= 1e-2 each
  no NaN or Inf anywhere except lse = -inf on empty rows.
"""
import numpy as np
import torch

import oracle

O_MAX_ABS, O_REL_L2, LSE_MAX_ABS, GRAD_REL_L2 = 2e-2, 5e-3, 1e-3, 1e-2


def rel_l2(x, y):
    x, y = np.asarray(x, np.float64), np.asarray(y, np.float64)
    den = np.linalg.norm(y)
    return float(np.linalg.norm(x - y) / den) if den > 0 else float(np.linalg.norm(x - y))


def problem_of(w):
    return oracle.Problem(w.family, w.head_mode, w.heads, w.l, w.c, w.offset_step)


def to64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_o_lse(o, lse, o_ref, lse_ref, what=""):
    o = np.asarray(o, np.float64)
    lse = np.asarray(lse, np.float64)
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf_ref), f"{what}: -inf rows differ"
    assert not np.any(np.isnan(lse)) and not np.any(np.isposinf(lse)), f"{what}: bad lse"
    fin = ~ninf_ref
    err_lse = float(np.abs(lse[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    err_o = float(np.abs(o - o_ref).max())
    rl = rel_l2(o, o_ref)
    assert err_lse <= LSE_MAX_ABS, f"{what}: lse max-abs {err_lse:.3e}"
    assert err_o <= O_MAX_ABS, f"{what}: O max-abs {err_o:.3e}"
    assert rl <= O_REL_L2, f"{what}: O rel-L2 {rl:.3e}"
    return {"o_max_abs": err_o, "o_rel_l2": rl, "lse_max_abs": err_lse}


def check_grads(got, want, what=""):
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, want):
        g = np.asarray(g, np.float64)
        assert np.all(np.isfinite(g)), f"{what}: non-finite {name}"
        e = rel_l2(g, r)
        assert e <= GRAD_REL_L2, f"{what}: {name} rel-L2 {e:.3e}"
        out[name] = e
    return out


def sample_rows(w, count, seed=0):
    """Flat row indices (b*H + h)*n + i: every head, both ends of the sequence, tile and block
    boundaries, plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(w.batch):
        for h in range(w.heads):
            base = (b * w.heads + h) * w.n
            for i in (0, 1, w.l - 1, w.l, 127, 128, w.n // 2, w.n - 129, w.n - 128, w.n - 1):
                if 0 <= i < w.n:
                    rows.add(base + i)
    total = w.batch * w.heads * w.n
    rows.update(rng.integers(0, total, size=count).tolist())
    return np.array(sorted(rows), dtype=np.int64)


def cuda_inputs(w):
    from workloads import make_inputs
    q, k, v, do = make_inputs(w)
    dev = torch.device("cuda")
    return [t.to(dev) for t in (q, k, v, do)], (q, k, v, do)
