"""The seeded input recipe: shapes, value sets, distributions, prefix rule."""
import math

import numpy as np
import pytest

import workloads as W


def test_named_workloads_match_their_sizes():
    assert W.WORKLOADS["tiny_f32"].d == 64 and W.WORKLOADS["tiny_f32"].dtype == "f32"
    h = W.WORKLOADS[W.HEADLINE]
    assert (h.d, h.n_experts, h.k, h.tokens, h.dtype) == (512, 256, 2, 16384, "bf16")
    assert W.WORKLOADS["d2048_n1024"].k == 4


@pytest.mark.parametrize("name", ["tiny_f32", "d512_n64"])
def test_recipe_distributions(name):
    wl = W.WORKLOADS[name]
    inp = W.generate(wl, seed=0, tokens=min(wl.tokens, 1024))
    d = wl.d
    assert inp.w_base.dtype == np.int8 and set(np.unique(inp.w_base)) <= {-1, 0, 1}
    p0 = (inp.w_base == 0).mean()
    assert abs(p0 - wl.p0) < 0.03
    assert abs((inp.w_base == 1).mean() - (inp.w_base == -1).mean()) < 0.03
    assert inp.theta.shape == (wl.n_experts, wl.stages, d // 2)
    assert inp.theta.dtype == np.float32
    assert inp.theta.min() >= -np.pi and inp.theta.max() <= np.pi
    assert abs(inp.w_gate.std() - 1 / math.sqrt(d)) < 0.1 / math.sqrt(d)
    assert inp.alpha == np.float32(1 / math.sqrt(d))
    assert len(inp.outliers) == int(round(wl.outlier_frac * d))
    x = inp.x_f64()
    if len(inp.outliers):
        assert x[:, inp.outliers].std() > 10 * np.delete(x, inp.outliers, axis=1).std()
    assert str(inp.x.dtype) == ("torch.float32" if wl.dtype == "f32" else "torch.bfloat16")


def test_token_prefix_rule():
    wl = W.WORKLOADS["d512_n64"]
    a = W.generate(wl, seed=0, tokens=64)
    b = W.generate(wl, seed=0, tokens=16)
    assert np.array_equal(a.x_f64()[:16], b.x_f64())
    assert np.array_equal(a.theta, b.theta)


def test_bias_variance():
    wl = W.custom("b", d=64, n_experts=4096, k=2, tokens=2, bias_var=0.5)
    inp = W.generate(wl)
    assert abs(inp.bias.var() - 0.5) < 0.05
