"""CUDA path vs the float64 oracle, through the C ABI (needs a B200)."""
import numpy as np
import pytest

import workloads as W
from oracle import bfmoe_oracle as O
from tests.parity_util import compare, compare_routing_full, run_cuda

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_butterfly_experts_b200.build as b
    b.build()


def B():
    import ternary_butterfly_experts_b200 as m
    return m


# -- pack / unpack ------------------------------------------------------------

@pytest.mark.parametrize("d", [4, 16, 64, 512, 2048])
def test_pack_matches_oracle_bit_exact(d):
    rng = np.random.default_rng(d)
    w = rng.integers(-1, 2, size=(d, d)).astype(np.int8)
    packed = B().bfmoe_pack_base(torch.from_numpy(w).cuda())
    got = packed.cpu().numpy().view(np.uint32)
    ref = O.pack_base(w) if d <= 512 else None
    if ref is not None:
        assert np.array_equal(got, ref)
    # unpack to the bf16 matrix used by the tensor-core product: exact
    wb = B().bfmoe_unpack_base(packed, d).float().cpu().numpy()
    assert np.array_equal(wb, w.astype(np.float32))


def test_pack_rejects_non_ternary():
    w = torch.zeros((64, 64), dtype=torch.int8)
    w[3, 7] = 2
    with pytest.raises(B().BfmoeError) as ei:
        B().bfmoe_pack_base(w.cuda())
    assert ei.value.status == 2


# -- materialised experts ----------------------------------------------------------

@pytest.mark.parametrize("d", [4, 8, 64, 256])
def test_materialize_matches_oracle(d):
    wl = W.custom("m", d=d, n_experts=3, k=1, tokens=1, dtype="f32")
    inp = W.generate(wl, seed=d)
    layer = B().Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    for e in range(3):
        got = B().bfmoe_materialize_expert(layer, e).cpu().numpy()
        ref = O.expert_matrix(inp.w_base, inp.alpha, inp.theta[e], inp.phi[e])
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max() + 1e-7


def test_zero_angles_materialize_to_scaled_base():
    wl = W.custom("z", d=64, n_experts=2, k=1, tokens=1, dtype="f32")
    inp = W.generate(wl)
    z = np.zeros_like(inp.theta)
    layer = B().Layer.from_host(inp.w_base, 0.5, z, z)
    got = B().bfmoe_materialize_expert(layer, 1).cpu().numpy()
    assert np.array_equal(got, 0.5 * inp.w_base.astype(np.float32))


# -- router + buckets + forward, small shapes with ragged tails ------------------

SMALL = [
    # d, N, k, T, dtype
    (4, 3, 1, 5, "f32"),
    (8, 5, 2, 37, "f32"),
    (64, 8, 2, 256, "f32"),         # the tiny float32 workload's shape
    (128, 16, 4, 257, "f32"),
    (32, 4, 4, 100, "bf16"),
    (64, 8, 2, 300, "bf16"),        # tensor-core product, one 64-wide N tile
    (128, 32, 3, 131, "bf16"),
    (256, 64, 2, 1000, "bf16"),
    (512, 64, 2, 777, "bf16"),      # 2 N tiles, ragged M tail
    (1024, 16, 8, 129, "bf16"),
]


@pytest.mark.parametrize("d,N,k,T,dt", SMALL)
def test_forward_parity_small(d, N, k, T, dt):
    wl = W.custom("s", d=d, n_experts=N, k=k, tokens=T, dtype=dt, bias_var=0.5,
                  outlier_frac=0.02, outlier_scale=20.0)
    inp = W.generate(wl, seed=d + N + k + T)
    gpu = run_cuda(inp)
    compare(inp, gpu)


def test_tiny_f32_workload_full():
    inp = W.generate(W.WORKLOADS["tiny_f32"])
    compare(inp, run_cuda(inp))


def test_pages_example_workload_full():
    inp = W.generate(W.WORKLOADS["d512_n64"])
    stats = compare(inp, run_cuda(inp))
    print(f"d512_n64: {stats}")


def test_headline_workload_full():
    inp = W.generate(W.WORKLOADS["d512_n256"])
    stats = compare(inp, run_cuda(inp))
    print(f"d512_n256: {stats}")
    assert stats["max_rel_l2"] < 1e-2


@pytest.mark.parametrize("name", ["d1024_n256", "d2048_n1024"])
def test_large_workloads_full_routing_sampled_outputs(name):
    """The two largest workloads at full size: every token's routing against
    the oracle's float64 logits, the bucket arrays against the oracle's
    buckets, and the outputs of a token sample through the oracle's
    three-step experts (forming every expert densely would take too long)."""
    inp = W.generate(W.WORKLOADS[name])
    gpu = run_cuda(inp)
    T = inp.wl.tokens
    near, mism, gerr = compare_routing_full(inp, gpu)
    print(f"{name}: {near} near-tie tokens of {T} ({mism} routed differently), gate error {gerr:.2e}")
    sample = np.unique(np.concatenate([np.arange(4), np.random.default_rng(5).integers(0, T, 44), [T - 1]]))
    stats = compare(inp, gpu, tokens=sample)
    print(f"{name}: sampled outputs max rel L2 {stats['max_rel_l2']:.3e}")
    assert np.isfinite(gpu["y"]).all()


# -- the boundary's maximum sizes ------------------------------------------------------

def _compare_all_tokens_with_buckets(inp, gpu):
    """Every token through the oracle's per-token expert (no dense experts,
    for large d), plus the bucket arrays against the oracle's buckets."""
    c, o, r = O.buckets(gpu["idx"], inp.wl.n_experts)
    assert np.array_equal(gpu["counts"], c) and np.array_equal(gpu["offsets"], o)
    assert np.array_equal(gpu["rows"], r)
    compare(inp, gpu, tokens=np.arange(inp.wl.tokens))


@pytest.mark.parametrize("N,T,dt", [(16, 70, "f32"), (64, 301, "bf16")])
def test_forward_parity_d2048(N, T, dt):
    """d = 2048: one row per warp, the pre-rotation switching layouts through
    half a float32 row; several experts per warp range and a ragged tail."""
    wl = W.custom("d2k", d=2048, n_experts=N, k=2, tokens=T, dtype=dt, bias_var=0.5,
                  outlier_frac=0.005, outlier_scale=50.0)
    inp = W.generate(wl, seed=N + T)
    _compare_all_tokens_with_buckets(inp, run_cuda(inp))


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_maximum_d(dt):
    """d = 4096, the largest d the boundary accepts: 12 stages, one row per warp."""
    wl = W.custom("dmax", d=4096, n_experts=4, k=2, tokens=37, dtype=dt, bias_var=0.5)
    inp = W.generate(wl, seed=11)
    _compare_all_tokens_with_buckets(inp, run_cuda(inp))


def test_maximum_experts_and_k():
    """N = 4096 experts (the boundary's limit) with k = 8, the largest top-k."""
    wl = W.custom("nmax", d=64, n_experts=4096, k=8, tokens=300, dtype="bf16", bias_var=0.5)
    inp = W.generate(wl, seed=12)
    compare(inp, run_cuda(inp))


# -- edge cases ---------------------------------------------------------------------

def test_single_token_and_single_expert():
    for N, k in ((1, 1), (4, 4)):
        wl = W.custom("e", d=64, n_experts=N, k=k, tokens=1, dtype="bf16")
        inp = W.generate(wl, seed=N)
        compare(inp, run_cuda(inp))


def test_zero_tokens():
    m = B()
    wl = W.custom("e0", d=64, n_experts=4, k=2, tokens=1, dtype="bf16")
    inp = W.generate(wl)
    layer = m.Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    wg = torch.from_numpy(inp.w_gate).cuda()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    idx, gates, counts, offsets, rows = m.bfmoe_router_topk(x, wg, None, 2, ws)
    assert counts.cpu().numpy().sum() == 0 and offsets.cpu().numpy().sum() == 0
    y = m.bfmoe_forward(layer, x, 2, idx, gates, offsets, rows, ws)
    assert y.shape == (0, 64)


def test_skewed_routing_and_empty_experts():
    # a huge bias on two experts sends every token there; the rest stay empty
    wl = W.custom("sk", d=256, n_experts=32, k=2, tokens=600, dtype="bf16")
    inp = W.generate(wl, seed=3)
    inp.bias = np.zeros(32, np.float32)
    inp.bias[[5, 17]] = 100.0
    gpu = run_cuda(inp)
    assert gpu["counts"][5] == 600 and gpu["counts"][17] == 600
    compare(inp, gpu)


def test_identical_experts_give_one_dense_layer():
    wl = W.custom("id", d=128, n_experts=8, k=2, tokens=200, dtype="f32")
    inp = W.generate(wl, seed=9)
    inp.theta[:] = inp.theta[0]
    inp.phi[:] = inp.phi[0]
    gpu = run_cuda(inp)
    W0 = O.expert_matrix(inp.w_base, inp.alpha, inp.theta[0], inp.phi[0])
    ref = inp.x_f64() @ W0.T
    assert O.rel_l2_per_token(gpu["y"], ref).max() < 1e-5


def test_deterministic_bitwise():
    inp = W.generate(W.custom("det", d=512, n_experts=64, k=2, tokens=1000, dtype="bf16"), seed=1)
    a = run_cuda(inp)
    b = run_cuda(inp)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["rows"], b["rows"])


def test_bad_routing_is_reported_not_faulted():
    m = B()
    wl = W.custom("bad", d=64, n_experts=4, k=2, tokens=8, dtype="bf16")
    inp = W.generate(wl)
    gpu = run_cuda(inp)
    idx = torch.from_numpy(gpu["idx"]).cuda()
    idx[3, 1] = 99  # out of range expert
    gates = torch.from_numpy(gpu["gates"].astype(np.float32)).cuda()
    rows = torch.from_numpy(gpu["rows"]).cuda()
    offsets = torch.from_numpy(gpu["offsets"]).cuda()
    ws = m.workspace(64, 4, 8, 2, m.BFMOE_BF16)
    m.bfmoe_forward(gpu["layer"], gpu["x"], 2, idx, gates, offsets, rows, ws)
    with pytest.raises(m.BfmoeError) as ei:
        m.bfmoe_check_device_error()
    assert ei.value.status == 7
    m.bfmoe_check_device_error()  # cleared


# -- the combined call -------------------------------------------------------------

@pytest.mark.parametrize("d,N,k,T,dt", [(512, 64, 2, 777, "bf16"), (64, 8, 2, 256, "f32"), (32, 4, 3, 50, "bf16"),
                                         # many experts, and many chunks
                                         (256, 256, 2, 2000, "bf16"), (128, 256, 2, 40000, "bf16")])
def test_moe_forward_equals_router_then_forward(d, N, k, T, dt):
    """The combined call (whose router scatter also writes the fused kernel's
    padded bucket order) equals the router then the forward bit for bit."""
    m = B()
    wl = W.custom("mf", d=d, n_experts=N, k=k, tokens=T, dtype=dt, bias_var=0.5)
    inp = W.generate(wl, seed=d + T)
    gpu = run_cuda(inp)
    x = gpu["x"]
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = torch.from_numpy(inp.bias).cuda()
    code = m.BFMOE_BF16 if dt == "bf16" else m.BFMOE_F32
    ws = torch.empty(m.bfmoe_moe_workspace_size(d, N, T, k, code), dtype=torch.uint8, device="cuda")
    for _ in range(2):  # the second call reuses the side stream and events
        y, (idx, gates, counts, offsets, rows) = m.bfmoe_moe_forward(gpu["layer"], x, wg, bias, k, ws)
        m.bfmoe_check_device_error()
        assert np.array_equal(idx.cpu().numpy(), gpu["idx"])
        assert np.array_equal(rows.cpu().numpy(), gpu["rows"])
        assert np.array_equal(y.float().cpu().numpy().astype(np.float64), gpu["y"])


def test_moe_forward_in_a_cuda_graph():
    m = B()
    wl = W.custom("mg", d=512, n_experts=32, k=2, tokens=300, dtype="bf16", bias_var=0.5)
    inp = W.generate(wl, seed=5)
    gpu = run_cuda(inp)
    model = m.ButterflyMoE(gpu["layer"], torch.from_numpy(inp.w_gate).cuda(),
                           torch.from_numpy(inp.bias).cuda(), 2, 300, torch.bfloat16)
    x = gpu["x"]
    y = torch.empty_like(x)
    model(x, y=y)  # first call creates the side stream before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        model(x, y=y)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    m.bfmoe_check_device_error()
    assert np.array_equal(y.float().cpu().numpy().astype(np.float64), gpu["y"])
    del g


# -- prepared weight tables ------------------------------------------------------

@pytest.mark.parametrize("d,N,k,T,dt", [(512, 64, 2, 777, "bf16"), (1024, 16, 2, 200, "bf16"),
                                        (64, 8, 2, 256, "f32"), (32, 4, 3, 50, "bf16")])
def test_prepared_tables_give_identical_results(d, N, k, T, dt):
    """bfmoe_prepare_layer once, then the calls read the tables: bit for bit
    the per-call results, for the fused path, the separate kernels and the
    small-d path."""
    m = B()
    wl = W.custom("pt", d=d, n_experts=N, k=k, tokens=T, dtype=dt, bias_var=0.5)
    inp = W.generate(wl, seed=d + N)
    gpu = run_cuda(inp)
    layer = gpu["layer"]
    x = gpu["x"]
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = torch.from_numpy(inp.bias).cuda()
    code = m.BFMOE_BF16 if dt == "bf16" else m.BFMOE_F32
    layer.prepare()
    try:
        ws = m.workspace(d, N, T, k, code)
        idx = torch.from_numpy(gpu["idx"]).cuda()
        gates = torch.from_numpy(gpu["gates"].astype(np.float32)).cuda()
        offsets = torch.from_numpy(gpu["offsets"]).cuda()
        rows = torch.from_numpy(gpu["rows"]).cuda()
        y = m.bfmoe_forward(layer, x, k, idx, gates, offsets, rows, ws)
        ws2 = torch.empty(m.bfmoe_moe_workspace_size(d, N, T, k, code), dtype=torch.uint8, device="cuda")
        y2, _ = m.bfmoe_moe_forward(layer, x, wg, bias, k, ws2)
        m.bfmoe_check_device_error()
        for yy in (y, y2):
            assert np.array_equal(yy.float().cpu().numpy().astype(np.float64), gpu["y"])
    finally:
        layer.unprepare()


@pytest.mark.parametrize("d,N,k,T", [(512, 256, 2, 3000), (1024, 64, 2, 700)])
def test_prepared_gate_parts_give_identical_results(d, N, k, T):
    """Router weights split once (bfmoe_prepare_gate): the combined call and
    the host call equal the per-call split bit for bit."""
    m = B()
    wl = W.custom("pg", d=d, n_experts=N, k=k, tokens=T, dtype="bf16", bias_var=0.5)
    inp = W.generate(wl, seed=d + N)
    layer = m.Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi)
    x = inp.x.cuda().contiguous()
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = torch.from_numpy(inp.bias).cuda()
    ws = torch.empty(m.bfmoe_moe_workspace_size(d, N, T, k, m.BFMOE_BF16), dtype=torch.uint8, device="cuda")
    model = m.ButterflyMoE(layer, wg, bias, k, T, torch.bfloat16)
    x_host = inp.x.contiguous().pin_memory()

    def host_call():
        y_host = torch.empty(x.shape, dtype=torch.bfloat16).pin_memory()
        model.forward_host(x_host, y_host)
        torch.cuda.synchronize()
        return y_host

    y0, r0 = m.bfmoe_moe_forward(layer, x, wg, bias, k, ws)
    y0, i0 = y0.clone(), r0[0].clone()
    yh0 = host_call()
    layer.prepare_gate(wg)
    try:
        y1, r1 = m.bfmoe_moe_forward(layer, x, wg, bias, k, ws)
        m.bfmoe_check_device_error()
        assert torch.equal(r1[0], i0) and torch.equal(y1, y0)
        # the host call cuts the tokens into chunks: compared with itself
        assert torch.equal(host_call(), yh0)
    finally:
        layer.unprepare_gate()
