"""Run the CUDA path through the C ABI and compare it with the oracle.

Comparison rules:
* routing indices bit-exact, except near-tie tokens (oracle float64 logits of
  neighbouring ranks among the first k+1 within 1e-5), which are counted;
* every token's GPU selection, near tie or not, must be a valid top-k of the
  oracle's float64 logits: k distinct experts in range whose j-th largest
  logit is within 1e-5 of the j-th largest of all N (for every rank j), in
  slots whose logits descend (within 1e-5);
* buckets bit-exact against the oracle's buckets of the GPU's own routing;
* gates within gate_tol(d) = 1e-5 * max(1, d / 512) of the oracle's softmax
  over the GPU-selected experts: the gates are float32 softmaxes of float32
  logits, whose rounding grows with d (measured on B200: 2e-6 at d = 512,
  9e-6 at d = 1024, 2.3e-5 at d = 2048 with logits up to |l| ~ 25);
* outputs: per-token relative L2 against the oracle evaluated with the GPU's
  routing (so near-tie tokens still check the arithmetic), at most 1e-5 on
  the float32 path and 1e-2 on the bfloat16 path.
"""
from __future__ import annotations

import numpy as np

from oracle import bfmoe_oracle as O

TOL = {"f32": 1e-5, "bf16": 1e-2}


def gate_tol(d):
    return 1e-5 * max(1.0, d / 512)


def run_cuda(inp, device="cuda", check_errors=True):
    import torch
    import ternary_butterfly_experts_b200 as B

    wl = inp.wl
    layer = B.Layer.from_host(inp.w_base, inp.alpha, inp.theta, inp.phi, device=device)
    x = inp.x.to(device).contiguous()
    wg = torch.from_numpy(inp.w_gate).to(device)
    bias = None if inp.bias is None else torch.from_numpy(inp.bias).to(device)
    code = B.BFMOE_BF16 if wl.dtype == "bf16" else B.BFMOE_F32
    ws = B.workspace(wl.d, wl.n_experts, x.shape[0], wl.k, code, device)
    idx, gates, counts, offsets, rows = B.bfmoe_router_topk(x, wg, bias, wl.k, ws)
    y = B.bfmoe_forward(layer, x, wl.k, idx, gates, offsets, rows, ws)
    if check_errors:
        B.bfmoe_check_device_error()
    torch.cuda.synchronize()
    return {
        "idx": idx.cpu().numpy(), "gates": gates.cpu().numpy().astype(np.float64),
        "counts": counts.cpu().numpy(), "offsets": offsets.cpu().numpy(), "rows": rows.cpu().numpy(),
        "y": y.float().cpu().numpy().astype(np.float64), "layer": layer, "x": x,
    }


def check_routing(logits, idx_g, k):
    """Routing of the GPU against the oracle's float64 ``logits`` [T, N].

    Tokens that are not near ties must match the oracle's top-k exactly.  Every
    token's selection must be a valid top-k (see the module docstring), which
    is what still binds the near-tie tokens.  Returns (near [T] bool,
    mismatched [T] bool)."""
    T, N = logits.shape
    idx_o, near = O.topk(logits, k)
    idx_g = np.asarray(idx_g).astype(np.int64).reshape(T, k)
    mism = (idx_g != idx_o).any(axis=1)
    bad = mism & ~near
    assert not bad.any(), f"{int(bad.sum())} non-tie tokens routed differently, e.g. {np.nonzero(bad)[0][:5]}"
    assert ((idx_g >= 0) & (idx_g < N)).all(), "expert index out of range"
    srt = np.sort(idx_g, axis=1)
    assert (np.diff(srt, axis=1) != 0).all(), "a token selects the same expert twice"
    sel = np.take_along_axis(logits, idx_g, axis=1)
    # rank by rank: the j-th largest selected logit is never above the j-th
    # largest of all N, and must not be below it by more than the tie band
    top = np.take_along_axis(logits, idx_o.astype(np.int64), axis=1)
    low = -np.sort(-sel, axis=1) < top - O.NEAR_TIE
    assert not low.any(), (f"{int(low.any(axis=1).sum())} tokens select experts that are not a top-{k} within "
                           f"{O.NEAR_TIE}, e.g. {np.nonzero(low.any(axis=1))[0][:5]}")
    if k > 1:
        up = np.diff(sel, axis=1) > O.NEAR_TIE
        assert not up.any(), f"slots not in descending logit order, e.g. token {np.nonzero(up.any(axis=1))[0][:5]}"
    return near, mism


def compare(inp, gpu, tokens=None, tol=None):
    """Check the GPU results against the oracle.  With ``tokens`` given, only
    those tokens are evaluated by the oracle (sampled mode for full sizes).
    Returns a dict of statistics (near ties, max relative error)."""
    wl = inp.wl
    tol = TOL[wl.dtype] if tol is None else tol
    x = inp.x_f64()
    sel = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    xs = x[sel]
    logits = O.router_logits(xs, inp.w_gate, inp.bias)
    idx_g = gpu["idx"][sel].astype(np.int64)
    near, mism = check_routing(logits, idx_g, wl.k)
    g_ref = O.gates_for(logits, idx_g)
    gerr = np.abs(gpu["gates"][sel] - g_ref).max()
    assert gerr < gate_tol(wl.d), f"gate error {gerr}"
    if tokens is None:
        c, o, r = O.buckets(gpu["idx"], wl.n_experts)
        assert np.array_equal(gpu["counts"], c), "bucket counts differ"
        assert np.array_equal(gpu["offsets"], o), "bucket offsets differ"
        assert np.array_equal(gpu["rows"], r), "bucket rows differ"
        y_ref = O.forward(xs, inp.w_base, inp.alpha, inp.theta, inp.phi, idx_g, g_ref)
    else:
        y_ref = O.forward_tokens(xs, inp.w_base, inp.alpha, inp.theta, inp.phi, idx_g, g_ref)
    rel = O.rel_l2_per_token(gpu["y"][sel], y_ref)
    assert rel.max() <= tol, f"max per-token relative L2 {rel.max():.3e} > {tol} (token {sel[rel.argmax()]})"
    return {"near_ties": int(near.sum()), "mismatched_near_ties": int(mism.sum()),
            "max_rel_l2": float(rel.max()), "mean_rel_l2": float(rel.mean()), "gate_err": float(gerr)}


def compare_routing_full(inp, gpu, block=8192):
    """Full-size routing check: every token's indices and gates against the
    oracle's float64 logits (computed in token blocks to bound host memory),
    and the bucket arrays against the oracle's buckets of the GPU's routing.
    Returns (near-tie count, mismatched near-tie count, max gate error)."""
    wl = inp.wl
    T = wl.tokens
    near_n = mism_n = 0
    gerr = 0.0
    for a in range(0, T, block):
        b = min(T, a + block)
        xs = inp.x[a:b].float().double().numpy()
        logits = O.router_logits(xs, inp.w_gate, inp.bias)
        idx_g = gpu["idx"][a:b].astype(np.int64)
        near, mism = check_routing(logits, idx_g, wl.k)
        near_n += int(near.sum())
        mism_n += int(mism.sum())
        gerr = max(gerr, float(np.abs(gpu["gates"][a:b] - O.gates_for(logits, idx_g)).max()))
    assert gerr < gate_tol(wl.d), f"gate error {gerr}"
    c, o, r = O.buckets(gpu["idx"], wl.n_experts)
    assert np.array_equal(gpu["counts"], c), "bucket counts differ"
    assert np.array_equal(gpu["offsets"], o), "bucket offsets differ"
    assert np.array_equal(gpu["rows"], r), "bucket rows differ"
    return near_n, mism_n, gerr
