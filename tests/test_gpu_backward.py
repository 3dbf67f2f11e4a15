"""Backward pass through the C ABI against the oracle's float64 chain rule
(itself pinned by finite differences in test_oracle_backward.py)."""
import numpy as np
import pytest

import workloads as W
from oracle import bfmoe_oracle as O

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_butterfly_experts_b200.build as b
    b.build()


def _rel(a, b):
    """max |a - b| relative to max |b| (whole tensor)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


# float32 arithmetic throughout: sums of up to R*d products for the base and
# router weights, L-stage walks for the angles
TOL = 2e-4


@pytest.mark.parametrize("d,N,k,T,dt", [(4, 3, 1, 9, "f32"), (8, 5, 2, 37, "f32"), (64, 8, 2, 256, "f32"),
                                        (128, 16, 3, 70, "bf16"), (512, 16, 2, 301, "bf16"),
                                        (32, 4, 4, 50, "bf16")])
def test_backward_matches_oracle(d, N, k, T, dt):
    import ternary_butterfly_experts_b200 as B
    wl = W.custom("bw", d=d, n_experts=N, k=k, tokens=T, dtype=dt, bias_var=0.5, outlier_frac=0.02,
                  outlier_scale=5.0)
    inp = W.generate(wl, seed=d + N + T)
    rng = np.random.default_rng(7)
    gy = rng.normal(size=(T, d)).astype(np.float32)
    layer = B.Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    x = inp.x.cuda().contiguous()
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = torch.from_numpy(inp.bias).cuda()
    code = B.BFMOE_BF16 if dt == "bf16" else B.BFMOE_F32
    ws = B.workspace(d, N, T, k, code)
    routing = B.bfmoe_router_topk(x, wg, bias, k, ws)
    g = B.bfmoe_backward(layer, x, k, wg, routing, torch.from_numpy(gy).cuda())
    B.bfmoe_check_device_error()
    ref = O.backward(inp.x_f64(), inp.w_base, float(inp.alpha), inp.theta, inp.phi, inp.w_gate, inp.bias, k,
                     gy.astype(np.float64))
    assert np.array_equal(routing[0].cpu().numpy(), ref["idx"])
    for key in ("dx", "dtheta", "dphi", "dw_base", "dw_gate", "dbias"):
        err = _rel(g[key].cpu().numpy(), ref[key])
        assert err <= TOL, (key, err)
    assert abs(float(g["dalpha"].item()) - ref["dalpha"]) <= TOL * max(1.0, abs(ref["dalpha"]))


def test_backward_pages_example_sample():
    """The pages' example layer (d=512, N=64, k=2, 1% outlier channels) on
    1024 tokens: the same comparison for every gradient."""
    import ternary_butterfly_experts_b200 as B
    wl = W.WORKLOADS["d512_n64"].with_tokens(1024)
    inp = W.generate(wl, seed=0)
    rng = np.random.default_rng(3)
    gy = rng.normal(size=(wl.tokens, wl.d)).astype(np.float32)
    layer = B.Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    x = inp.x.cuda().contiguous()
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = None
    ws = B.workspace(wl.d, wl.n_experts, wl.tokens, wl.k, B.BFMOE_BF16)
    routing = B.bfmoe_router_topk(x, wg, bias, wl.k, ws)
    g = B.bfmoe_backward(layer, x, wl.k, wg, routing, torch.from_numpy(gy).cuda(), bias_grad=False)
    B.bfmoe_check_device_error()
    ref = O.backward(inp.x_f64(), inp.w_base, float(inp.alpha), inp.theta, inp.phi, inp.w_gate, None, wl.k,
                     gy.astype(np.float64))
    for key in ("dx", "dtheta", "dphi", "dw_base", "dw_gate"):
        err = _rel(g[key].cpu().numpy(), ref[key])
        print(f"backward {key}: rel err {err:.2e}")
        assert err <= TOL, (key, err)
