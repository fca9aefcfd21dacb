"""Host logic of the Python binding, without a GPU: the shape groups that _check_tensors accepts
(query-key width for q, k; value width for v, o, dO) and the descriptor _desc builds (the value
width is sent as 0 when it equals the query-key width)."""
import pytest
import torch

import block_sparse_factorized_b200 as bsf


class FakeCuda:
    """Stands in for a contiguous CUDA tensor: only the attributes the checks read."""

    def __init__(self, shape, dtype=torch.bfloat16, device="cuda:0"):
        self.shape, self.dtype, self.device, self.is_cuda = torch.Size(shape), dtype, device, True

    def is_contiguous(self):
        return True

    def dim(self):
        return len(self.shape)


Q = FakeCuda((2, 8, 256, 64))
V64, V128 = FakeCuda((2, 8, 256, 64)), FakeCuda((2, 8, 256, 128))


@pytest.mark.parametrize("qk,vo", [((Q, Q), (V64,)), ((Q, Q), (V64, V64, V64)), ((Q,), (V128, V128)),
                                   ((Q, Q), ())])
def test_accepted_shape_groups(qk, vo):
    bsf._check_tensors(qk, vo)


@pytest.mark.parametrize("qk,vo", [
    ((Q, FakeCuda((2, 8, 256, 32))), (V64,)),          # k narrower than q
    ((Q, Q), (V128, V64)),                             # o not as wide as v
    ((Q, Q), (FakeCuda((2, 8, 128, 64)),)),            # v shorter than q
    ((Q, Q), (FakeCuda((2, 8, 256, 64), torch.float32),)),  # mixed dtypes
    ((Q, Q), (FakeCuda((2, 8, 256, 64), device="cuda:1"),)),  # mixed devices
    ((Q, Q), (torch.zeros(2, 8, 256, 64, dtype=torch.bfloat16),)),  # a CPU tensor: no CPU path
])
def test_rejected_shape_groups(qk, vo):
    with pytest.raises(ValueError):
        bsf._check_tensors(qk, vo)


def test_descriptor_widths():
    q = torch.zeros(2, 8, 256, 64, dtype=torch.bfloat16)
    d = bsf._desc(q)
    assert (d.batch, d.heads, d.n, d.d, d.dtype, d.dv) == (2, 8, 256, 64, bsf.ST_BF16, 0)
    assert bsf._desc(q, q).dv == 0
    assert bsf._desc(q, torch.zeros(2, 8, 256, 128, dtype=torch.bfloat16)).dv == 128
    assert bsf._desc(q.float()).dtype == bsf.ST_FP32
    with pytest.raises(TypeError):
        bsf._desc(q.half())
    with pytest.raises(ValueError):
        bsf._desc(q[0])


class FakeWorkspace(FakeCuda):
    """A workspace tensor stand-in with a dtype of its own: the binding must send its real size."""

    def __init__(self, numel, dtype, device="cuda:0", contiguous=True, is_cuda=True):
        super().__init__((numel,), dtype, device)
        self._n, self._contig, self.is_cuda = numel, contiguous, is_cuda

    def numel(self):
        return self._n

    def element_size(self):
        return torch.tensor([], dtype=self.dtype).element_size()

    def is_contiguous(self):
        return self._contig


def test_workspace_size_is_the_buffer_size_in_bytes():
    """The C side compares the byte count the binding sends with what the call needs, so the
    binding sends the caller's buffer size (numel x element size), never the size the library
    asked for."""
    assert bsf._workspace_bytes(None, "cuda:0") == 0
    assert bsf._workspace_bytes(FakeWorkspace(1000, torch.uint8), "cuda:0") == 1000
    assert bsf._workspace_bytes(FakeWorkspace(1000, torch.float32), "cuda:0") == 4000
    assert bsf._workspace_bytes(FakeWorkspace(10, torch.bfloat16), "cuda:0") == 20
    with pytest.raises(ValueError):
        bsf._workspace_bytes(FakeWorkspace(1000, torch.uint8, device="cuda:1"), "cuda:0")
    with pytest.raises(ValueError):
        bsf._workspace_bytes(FakeWorkspace(1000, torch.uint8, contiguous=False), "cuda:0")
    with pytest.raises(ValueError):
        bsf._workspace_bytes(torch.zeros(1000, dtype=torch.uint8), "cuda:0")  # a CPU tensor
