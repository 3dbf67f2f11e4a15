"""Add-only decode forward (bfmoe_decode_forward) vs the float64 oracle.

The decode kernel keeps every intermediate in float32 and rounds y once, so
its bound is tighter than the tensor-core path's: 1e-5 per-token relative L2
on float32 inputs, and on bfloat16 inputs the rounding of y to bfloat16
(relative error at most 2^-9 per element) plus float32 noise: 2.5e-3.
"""
import numpy as np
import pytest

import workloads as W
from oracle import bfmoe_oracle as O
from tests.parity_util import check_routing, gate_tol

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

TOL = {"f32": 1e-5, "bf16": 2.5e-3}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_butterfly_experts_b200.build as b
    b.build()


def B():
    import ternary_butterfly_experts_b200 as m
    return m


def run_decode(inp):
    wl = inp.wl
    layer = B().Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    x = inp.x.cuda().contiguous()
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = None if inp.bias is None else torch.from_numpy(inp.bias).cuda()
    code = B().BFMOE_BF16 if wl.dtype == "bf16" else B().BFMOE_F32
    ws = B().workspace(wl.d, wl.n_experts, x.shape[0], wl.k, code)
    idx, gates, _, offsets, rows = B().bfmoe_router_topk(x, wg, bias, wl.k, ws)
    y = B().bfmoe_decode_forward(layer, x, wl.k, idx, gates)
    B().bfmoe_check_device_error()
    return layer, x, idx, gates, offsets, rows, ws, y


def check_against_oracle(inp, idx, gates, y):
    wl = inp.wl
    x = inp.x_f64()
    logits = O.router_logits(x, inp.w_gate, inp.bias)
    idx_g = idx.cpu().numpy().astype(np.int64)
    check_routing(logits, idx_g, wl.k)
    g_ref = O.gates_for(logits, idx_g)
    assert np.abs(gates.cpu().numpy() - g_ref).max() < gate_tol(wl.d)
    y_ref = O.forward_tokens(x, inp.w_base, inp.alpha, inp.theta, inp.phi, idx_g, g_ref)
    rel = O.rel_l2_per_token(y.float().cpu().numpy().astype(np.float64), y_ref)
    assert rel.max() <= TOL[wl.dtype], f"max per-token relative L2 {rel.max():.3e}"
    return float(rel.max())


CASES = [
    # name, d, N, k, T, dtype
    ("d4_n2_k1", 4, 2, 1, 5, "f32"),      # one packed word, four codes used
    ("d8_n4_k2", 8, 4, 2, 3, "bf16"),
    ("d16_n3_k3", 16, 3, 3, 7, "f32"),
    ("d64_n8_k2", 64, 8, 2, 64, "f32"),  # the float32 headline family
    ("d256_n16_k2", 256, 16, 2, 33, "bf16"),
    ("d2048_n16_k4", 2048, 16, 4, 9, "bf16"),
    ("d4096_n8_k8", 4096, 8, 8, 3, "f32"),  # slots in two passes of four (shared-memory bound)
]


@pytest.mark.parametrize("name,d,N,k,T,dt", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(name, d, N, k, T, dt):
    inp = W.generate(W.custom(name, d=d, n_experts=N, k=k, tokens=T, dtype=dt), seed=d + T)
    _, _, idx, gates, _, _, _, y = run_decode(inp)
    err = check_against_oracle(inp, idx, gates, y)
    print(f"{name}: max rel L2 {err:.2e}")


@pytest.mark.parametrize("T", [1, 64])
def test_decode_headline_shape(T):
    """d = 512, N = 256, k = 2 (the headline layer) at decode batch sizes."""
    inp = W.generate(W.WORKLOADS["d512_n256"], seed=0, tokens=T)
    layer, x, idx, gates, offsets, rows, ws, y = run_decode(inp)
    err = check_against_oracle(inp, idx, gates, y)
    # the tensor-core forward on the same routing agrees within its own bound
    y_tc = B().bfmoe_forward(layer, x, 2, idx, gates, offsets, rows, ws)
    torch.cuda.synchronize()
    rel = O.rel_l2_per_token(y.float().cpu().numpy().astype(np.float64), y_tc.float().cpu().numpy().astype(np.float64))
    assert rel.max() <= 1e-2
    print(f"T={T}: max rel L2 {err:.2e}, vs tensor-core path {rel.max():.2e}")


def test_decode_empty_batch():
    inp = W.generate(W.custom("e", d=64, n_experts=4, k=2, tokens=2, dtype="f32"), seed=1)
    layer = B().Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    x = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    idx = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    g = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    y = B().bfmoe_decode_forward(layer, x, 2, idx, g)
    assert y.shape == (0, 64)


def test_decode_out_of_range_expert_is_reported():
    """An expert id outside [0, N) is skipped by the kernel's own check and
    recorded in the device error word (no out-of-bounds access)."""
    inp = W.generate(W.custom("bad", d=64, n_experts=4, k=2, tokens=3, dtype="f32"), seed=2)
    layer = B().Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    x = inp.x.cuda().contiguous()
    idx = torch.tensor([[0, 1], [2, 9], [3, 0]], dtype=torch.int32, device="cuda")
    g = torch.full((3, 2), 0.5, dtype=torch.float32, device="cuda")
    B().bfmoe_decode_forward(layer, x, 2, idx, g)
    with pytest.raises(B().BfmoeError):
        B().bfmoe_check_device_error()
    B().bfmoe_check_device_error()  # the word is cleared by the read


def test_router_without_buckets_matches_with_buckets():
    """counts / offsets / rows all NULL: the same idx and gates, no buckets."""
    inp = W.generate(W.WORKLOADS["d512_n256"], seed=3, tokens=64)
    x = inp.x.cuda().contiguous()
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = torch.from_numpy(inp.bias).cuda()
    ws = B().workspace(512, 256, 64, 2, B().BFMOE_BF16)
    i1, g1, c1, _, _ = B().bfmoe_router_topk(x, wg, bias, 2, ws)
    i2, g2, c2, o2, r2 = B().bfmoe_router_topk(x, wg, bias, 2, ws, buckets=False)
    assert c2 is None and o2 is None and r2 is None
    assert torch.equal(i1, i2) and torch.equal(g1, g2)
