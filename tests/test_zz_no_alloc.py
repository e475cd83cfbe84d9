"""gptl_colsum_noalloc: the column sums of gptl_colsum without any temporary
device memory from the caller.

Some callers cannot give the library scratch memory: a custom operator
inside a framework that plans every device allocation itself, or a
deployment that allows no device allocation once it has started.  For them
the library keeps the partial sums in a fixed 4 MiB array of its own.  This
file checks, through the C ABI, that calls in a row give the same sums as
gptl_colsum (which uses caller scratch) bit for bit, since both pick the same
split and run the same kernels, and that they agree with numpy's sums within
the tolerance of the column-sum kernel test.  The cases cover the array's
full width (n * groups = 16384), the deepest split (64 partial rows), a row
pitch wider than n with a matrix pitch wider than rows * ld, and sizes beyond
the array, which are refused before anything is launched.  The file is named
so that pytest collects it last."""
import numpy as np
import pytest
import torch

from transformer_layer_step_b200 import gptlayer as G
from gpu_util import need_gpu, dev_tensor, rounded, stream, check_device_error

pytestmark = pytest.mark.gpu

# (dtype, rows, n, groups, ld, gstride); ld = gstride = None means dense
CASES = [
    ("bf16", 4096, 2304, 2, None, None),
    ("fp16", 777, 1024, 3, None, None),
    ("bf16", 2048, 8192, 2, None, None),        # n * groups = 16384, the array's full width
    ("fp16", 4096, 256, 1, None, None),         # one 256-column strip: 64 partial rows
    ("bf16", 600, 1024, 3, 1088, 600 * 1088 + 512),   # strided rows and matrices
]


def _layout(rows, n, groups, ld, gstride):
    ld = n if ld is None else ld
    gstride = rows * ld if gstride is None else gstride
    return ld, gstride


def _device_matrix(a, ld, gstride, dtype):
    """Places a [groups][rows][n] array in a flat buffer with the given pitches
    (the padding holds large values, which a wrong pitch would add in)."""
    groups, rows, n = a.shape
    flat = np.full(groups * gstride, 1e4)
    for g in range(groups):
        view = flat[g * gstride:g * gstride + rows * ld].reshape(rows, ld)
        view[:, :n] = a[g]
    return dev_tensor(flat, dtype)


def _colsum_with_scratch(at, rows, n, groups, ld, gstride, dtype):
    out = torch.empty(groups * n, dtype=torch.float32, device="cuda")
    scratch = torch.empty(G.colsum_scratch_bytes(n, groups), dtype=torch.uint8, device="cuda")
    G.colsum(rows, n, groups, ld, gstride, dtype, at, out, scratch, stream())
    return out


def test_colsum_noalloc_matches_colsum_in_a_row():
    need_gpu()
    # different shapes back to back: no call may see an earlier call's partials
    for call, (dtype, rows, n, groups, ld, gstride) in enumerate(CASES):
        ld, gstride = _layout(rows, n, groups, ld, gstride)
        rng = np.random.default_rng(100 + call)
        a = rounded(rng.standard_normal((groups, rows, n)), dtype)
        at = _device_matrix(a, ld, gstride, dtype)
        ref = _colsum_with_scratch(at, rows, n, groups, ld, gstride, dtype)
        for _ in range(2):
            out = torch.full((groups * n,), float("nan"), dtype=torch.float32, device="cuda")
            G.colsum_noalloc(rows, n, groups, ld, gstride, dtype, at, out, stream())
            check_device_error()
            got, want = out.cpu().numpy(), ref.cpu().numpy()
            np.testing.assert_array_equal(got, want)
            np.testing.assert_allclose(got, a.sum(axis=1).reshape(-1), rtol=0, atol=1e-3)


def test_colsum_noalloc_refuses_oversized():
    need_gpu()
    a = torch.zeros((2, 16, 8256), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(2 * 8256, dtype=torch.float32, device="cuda")
    before = G.launch_count()
    with pytest.raises(G.GptlError) as e:
        G.colsum_noalloc(16, 8256, 2, 8256, 16 * 8256, "bf16", a, out, stream())
    assert e.value.code == G.E_TOO_LARGE
    assert G.launch_count() == before
