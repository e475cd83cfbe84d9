"""gptl_colsum_noalloc: the column sums of gptl_colsum without any temporary
device memory from the caller.

Some callers cannot give the library scratch memory: a custom operator
inside a framework that plans every device allocation itself, or a
deployment that allows no device allocation once it has started.  For them
the library keeps the partial sums in a fixed 4 MiB array of its own.  This
file checks, through the C ABI, that two calls in a row give the same sums
as gptl_colsum (which uses caller scratch), within the tolerance of the
column-sum kernel test, and that sizes beyond the array are refused before
anything is launched.  It is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

from transformer_layer_step_b200 import gptlayer as G
from gpu_util import need_gpu, dev_tensor, rounded, stream, check_device_error

pytestmark = pytest.mark.gpu


def _colsum_with_scratch(at, rows, n, groups, dtype):
    out = torch.empty(groups * n, dtype=torch.float32, device="cuda")
    scratch = torch.empty(G.colsum_scratch_bytes(n, groups), dtype=torch.uint8, device="cuda")
    G.colsum(rows, n, groups, n, rows * n, dtype, at, out, scratch, stream())
    return out


def test_colsum_noalloc_matches_colsum_twice():
    need_gpu()
    # two different shapes back to back: the second call must not see the first's partials
    for call, (dtype, rows, n, groups) in enumerate([("bf16", 4096, 2304, 2), ("fp16", 777, 1024, 3)]):
        rng = np.random.default_rng(100 + call)
        a = rounded(rng.standard_normal((groups, rows, n)), dtype)
        at = dev_tensor(a, dtype)
        ref = _colsum_with_scratch(at, rows, n, groups, dtype)
        out = torch.full((groups * n,), float("nan"), dtype=torch.float32, device="cuda")
        G.colsum_noalloc(rows, n, groups, n, rows * n, dtype, at, out, stream())
        check_device_error()
        got, want = out.cpu().numpy(), ref.cpu().numpy()
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-3)
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
