"""Pin: the oracle's backward pass equals central finite differences of its
forward pass, for every parameter, bias, gamma, beta and the input.

Tiny shapes (h 8, 2 heads, ffn 32, seq 5, batch 2) with t = 1 and t = 2
shards, loss L = sum(Out * R) so that dOut = R exercises every column."""
import numpy as np
import pytest

import oracle

DIMS = dict(b=2, s=5, h=8, a=2, f=32)


def _rand_params(rng, h, f, t, std=0.3):
    return {
        "ln1_g": 1.0 + 0.2 * rng.standard_normal(h), "ln1_b": 0.2 * rng.standard_normal(h),
        "w_qkv": std * rng.standard_normal((t, 3 * h // t, h)),
        "b_qkv": 0.2 * rng.standard_normal((t, 3 * h // t)),
        "w_o": std * rng.standard_normal((t, h, h // t)), "b_o": 0.2 * rng.standard_normal(h),
        "ln2_g": 1.0 + 0.2 * rng.standard_normal(h), "ln2_b": 0.2 * rng.standard_normal(h),
        "w_1": std * rng.standard_normal((t, f // t, h)),
        "b_1": 0.2 * rng.standard_normal((t, f // t)),
        "w_2": std * rng.standard_normal((t, h, f // t)), "b_2": 0.2 * rng.standard_normal(h),
    }


@pytest.mark.parametrize("t", [1, 2])
def test_backward_matches_finite_differences(t):
    rng = np.random.default_rng(1234 + t)
    dims = dict(DIMS, t=t)
    T, h, f = dims["b"] * dims["s"], dims["h"], dims["f"]
    x = rng.standard_normal((T, h))
    params = _rand_params(rng, h, f, t)
    r = rng.standard_normal((T, h))

    def loss(xx, pp):
        out, _ = oracle.layer_fwd(xx, pp, dims)
        return float((out * r).sum())

    _, cache = oracle.layer_fwd(x, params, dims)
    dx, grads = oracle.layer_bwd(cache, params, dims, r)

    eps = 1e-6

    def fd(get_arr):
        arr = get_arr()
        g = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = arr[idx]
            arr[idx] = old + eps
            lp = loss(x, params)
            arr[idx] = old - eps
            lm = loss(x, params)
            arr[idx] = old
            g[idx] = (lp - lm) / (2 * eps)
        return g

    checks = {"x": (fd(lambda: x), dx)}
    for name in params:
        checks[name] = (fd(lambda n=name: params[n]), grads[name])
    for name, (num, ana) in checks.items():
        assert num.shape == ana.shape, name
        err = np.abs(num - ana).max() / max(np.abs(num).max(), 1e-12)
        assert err < 1e-6, (name, err)
