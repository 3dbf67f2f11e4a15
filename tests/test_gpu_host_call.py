"""bfmoe_moe_forward_host: host buffers in and out, copies overlapped with the
work in token chunks (needs a B200)."""
import numpy as np
import pytest

import workloads as W
from oracle import bfmoe_oracle as O
from tests.parity_util import TOL

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_butterfly_experts_b200.build as b
    b.build()


def _model(inp):
    import ternary_butterfly_experts_b200 as B
    wl = inp.wl
    layer = B.Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    bias = None if inp.bias is None else torch.from_numpy(inp.bias).cuda()
    return B.ButterflyMoE(layer, torch.from_numpy(inp.w_gate).cuda(), bias, wl.k, inp.x.shape[0], dt)


def _oracle_check(inp, y, tol):
    """Per-token relative L2 against the oracle with its own routing; tokens
    whose k-th and (k+1)-th logits are within 1e-5 (several routings correct)
    are left out."""
    x = inp.x_f64()
    logits = O.router_logits(x, inp.w_gate, inp.bias)
    idx, near = O.topk(logits, inp.wl.k)
    ref = O.forward_tokens(x, inp.w_base, inp.alpha, inp.theta, inp.phi, idx, O.gates_for(logits, idx))
    rel = O.rel_l2_per_token(y, ref)[~near]
    assert rel.max() <= tol, f"max per-token relative L2 {rel.max():.3e}"


@pytest.mark.parametrize("d,N,k,T,dt", [(512, 32, 2, 1000, "bf16"), (64, 8, 2, 700, "f32"), (256, 16, 3, 513, "bf16")])
def test_host_call_matches_oracle_for_every_chunking(d, N, k, T, dt):
    inp = W.generate(W.custom("h", d=d, n_experts=N, k=k, tokens=T, dtype=dt, bias_var=0.5), seed=d + T)
    model = _model(inp)
    x_host = inp.x.contiguous().pin_memory()
    y_host = torch.empty_like(x_host).pin_memory()
    y_dev = model(inp.x.cuda())
    torch.cuda.synchronize()
    for chunk in (0, 256, 384, T):
        y_host.zero_()
        model.forward_host(x_host, y_host, chunk=chunk)
        torch.cuda.synchronize()
        import ternary_butterfly_experts_b200 as B
        B.bfmoe_check_device_error()
        y = y_host.float().numpy().astype(np.float64)
        _oracle_check(inp, y, TOL[dt])
        if chunk >= T:  # one chunk: the very same kernels as the device call
            assert np.array_equal(y, y_dev.float().cpu().numpy().astype(np.float64))


def test_host_call_in_a_cuda_graph():
    inp = W.generate(W.custom("hg", d=512, n_experts=16, k=2, tokens=600, dtype="bf16"), seed=2)
    model = _model(inp)
    x_host = inp.x.contiguous().pin_memory()
    y_ref = torch.empty_like(x_host).pin_memory()
    model.forward_host(x_host, y_ref, chunk=256)  # creates the copy streams before capture
    torch.cuda.synchronize()
    y_host = torch.empty_like(x_host).pin_memory()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        model.forward_host(x_host, y_host, chunk=256)
    for _ in range(2):
        y_host.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y_host, y_ref)
    del g


def test_host_call_rejects_short_workspace():
    import ternary_butterfly_experts_b200 as B
    inp = W.generate(W.custom("hw", d=64, n_experts=4, k=2, tokens=300, dtype="bf16"), seed=3)
    model = _model(inp)
    x_host = inp.x.contiguous().pin_memory()
    y_host = torch.empty_like(x_host).pin_memory()
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.BfmoeError) as ei:
        B.bfmoe_moe_forward_host(model.layer, x_host, model.w_gate, model.bias, 2, y_host, ws)
    assert ei.value.status == B.capi.BFMOE_EWORKSPACE
