"""Seeded synthetic workloads shared by the tests, the smoke check and the benchmark.

This module holds shapes and random draws only -- none of the attention arithmetic.  Both the
CUDA path and the CPU oracle receive the very same tensors produced here.

Recipe: one CPU ``torch.Generator`` seeded with ``seed`` (0 by default) draws Q, K, V and dO, in
that order, as iid N(0, 1) fp32 of shape [batch, heads, n, d]; each is then rounded to the
workload's I/O dtype.  The oracle gets those rounded values widened to fp64.

The workloads stand in for the pages' data (no dataset is needed or present): a 32x32x3 image
raster (n = 3072), Enwik8-length text (n = 12288, l = 128, c = 32; per-head alternating, and
merged heads as the text model uses them), a 64x64x3 raster (n = 12288, stride 128) and a
65,536-sample audio clip (l = 256), plus a small fp32 case.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

STRIDED, FIXED = 1, 2
ALTERNATING, MERGED, SINGLE_A1, SINGLE_A2 = 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    name: str
    family: int          # STRIDED or FIXED
    head_mode: int       # ALTERNATING, MERGED, SINGLE_A1, SINGLE_A2
    n: int
    l: int
    c: int
    batch: int
    heads: int
    d: int = 64           # width of the query and key rows
    dtype: str = "bf16"  # "bf16" or "fp32"
    offset_step: int = 0  # fixed-pattern head-2 sub-block step (0: c)
    seed: int = 0
    dv: int = 0           # width of the value (and output-gradient) rows; 0: d

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def shape(self):
        return (self.batch, self.heads, self.n, self.d)

    def value_shape(self):
        return (self.batch, self.heads, self.n, self.dv or self.d)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "strided_n256_l16_fp32": Workload("strided_n256_l16_fp32", STRIDED, ALTERNATING, 256, 16, 0,
                                      1, 2, dtype="fp32"),
    "strided_merged_n3072_l64": Workload("strided_merged_n3072_l64", STRIDED, MERGED, 3072, 64,
                                         0, 4, 8),
    "fixed_n12288_l128_c32": Workload("fixed_n12288_l128_c32", FIXED, ALTERNATING, 12288, 128,
                                      32, 2, 8),
    "strided_n12288_l128": Workload("strided_n12288_l128", STRIDED, ALTERNATING, 12288, 128, 0,
                                    2, 16),
    "strided_merged_n12288_l128": Workload("strided_merged_n12288_l128", STRIDED, MERGED, 12288,
                                           128, 0, 2, 16),
    "strided_n65536_l256": Workload("strided_n65536_l256", STRIDED, ALTERNATING, 65536, 256, 0,
                                    1, 8),
    # the 64x64x3 raster at the image model's own head width: 16 heads of 512 / 16 = 32
    "strided_n12288_l128_d32": Workload("strided_n12288_l128_d32", STRIDED, ALTERNATING, 12288, 128, 0,
                                        2, 16, d=32),
    # the text model's own setting: fixed pattern with merged heads (each head reads its block and
    # every earlier block's summary run), n = 12288, l = 128, c = 32, 8 heads
    "fixed_merged_n12288_l128_c32": Workload("fixed_merged_n12288_l128_c32", FIXED, MERGED, 12288,
                                             128, 32, 2, 8),
}

# The headline workload: fixed pattern, text-shaped, n = 12288.
HEADLINE = "fixed_n12288_l128_c32"


def make_inputs(w: Workload, with_grad_out: bool = True):
    """Return (q, k, v, do) CPU tensors in the workload's dtype, drawn as described above."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shp, vshp = w.shape(), w.value_shape()
    q = torch.randn(shp, generator=g, dtype=torch.float32)
    k = torch.randn(shp, generator=g, dtype=torch.float32)
    v = torch.randn(vshp, generator=g, dtype=torch.float32)
    do = torch.randn(vshp, generator=g, dtype=torch.float32) if with_grad_out else None
    dt = w.torch_dtype
    out = [q.to(dt), k.to(dt), v.to(dt)]
    out.append(do.to(dt) if do is not None else None)
    return tuple(out)
