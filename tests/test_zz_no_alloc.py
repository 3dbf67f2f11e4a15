"""The router entry point for callers that cannot allocate device memory at
call time (a plug-in handed only its input and output buffers, code running
while the framework owns the allocator).  It takes no workspace and uses the
library's built-in scratch array; its results must equal those of the
workspace entry point.  This file is collected last, so a stop at the first
failure has already run every other test."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import ternary_butterfly_experts_b200.build as b
    b.build()
    import ternary_butterfly_experts_b200 as m
    return m


def _inputs(wl, seed):
    inp = W.generate(wl, seed=seed)
    x = inp.x.cuda().contiguous()
    wg = torch.from_numpy(inp.w_gate).cuda()
    bias = None if inp.bias is None else torch.from_numpy(inp.bias).cuda()
    return x, wg, bias


def _host(out):
    return [t.cpu().numpy() for t in out]


def _code(B, wl):
    return B.BFMOE_BF16 if wl.dtype == "bf16" else B.BFMOE_F32


def _check_same(B, wl, seed):
    x, wg, bias = _inputs(wl, seed)
    ws = B.workspace(wl.d, wl.n_experts, wl.tokens, wl.k, _code(B, wl))
    ref = _host(B.bfmoe_router_topk(x, wg, bias, wl.k, ws))
    got = _host(B.bfmoe_router_topk_noalloc(x, wg, bias, wl.k))
    B.bfmoe_check_device_error()
    assert np.array_equal(got[0], ref[0])                       # idx
    assert np.abs(got[1] - ref[1]).max() <= 1e-5                # gates
    for a, b in zip(got[2:], ref[2:]):                          # counts, offsets, rows
        assert np.array_equal(a, b)


def test_noalloc_router_matches_workspace_router_two_calls(B):
    # calls in a row with different sizes and both router paths (tensor
    # cores for bf16 with d % 64 == 0; CUDA cores, which also keep the
    # float32 logits in the array, for float32 tokens and d < 64): the
    # shared scratch carries nothing from one call to the next
    cases = [W.custom("na1", d=512, n_experts=64, k=2, tokens=1000, dtype="bf16", bias_var=0.5),
             W.custom("na2", d=256, n_experts=40, k=4, tokens=777, dtype="bf16",
                      outlier_frac=0.02, outlier_scale=20.0),
             W.custom("na3", d=128, n_experts=96, k=3, tokens=901, dtype="f32", bias_var=0.5),
             W.custom("na4", d=32, n_experts=12, k=2, tokens=333, dtype="bf16")]
    for i, wl in enumerate(cases):
        _check_same(B, wl, seed=11 + i)


def test_noalloc_router_accepts_sizes_just_under_its_scratch(B):
    # the float32 router keeps T*N float32 logits in the array: the largest T
    # whose router scratch still fits is accepted and computed correctly
    d, N, k = 64, 1024, 2
    lim = B.capi.BFMOE_NOALLOC_SCRATCH_BYTES
    lo, hi = 1, 1 << 16
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if B.bfmoe_router_scratch_size(d, N, mid, k, B.BFMOE_F32) <= lim:
            lo = mid
        else:
            hi = mid - 1
    assert lim - B.bfmoe_router_scratch_size(d, N, lo, k, B.BFMOE_F32) < 1 << 20
    assert B.bfmoe_router_scratch_size(d, N, lo + 1, k, B.BFMOE_F32) > lim
    _check_same(B, W.custom("na5", d=d, n_experts=N, k=k, tokens=lo, dtype="f32"), seed=21)


def test_noalloc_router_rejects_sizes_beyond_its_scratch(B):
    L = B.capi.lib()
    d, N, T, k = 2048, 1024, 131072, 4
    need = B.bfmoe_router_scratch_size(d, N, T, k, B.BFMOE_F32)
    assert need > B.capi.BFMOE_NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    rc = L.bfmoe_router_topk_noalloc(p, B.BFMOE_F32, T, d, p, None, N, k, p, p, p, p, p, None)
    assert rc == B.capi.BFMOE_EUNSUPPORTED
    assert b"scratch" in L.bfmoe_last_error()
