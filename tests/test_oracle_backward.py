"""Pins of the oracle's backward pass (CPU): every gradient against central
finite differences of the oracle's forward (itself pinned in
test_oracle_pins.py), on small sizes whose top-k margins are wide enough
that the perturbations never change the routing."""
import numpy as np
import pytest

from oracle import bfmoe_oracle as O

H = 1e-6


def _case(d=8, N=3, k=2, T=6, seed=0, bias=True):
    rng = np.random.default_rng(seed)
    L = int(np.log2(d))
    while True:
        x = rng.normal(size=(T, d))
        w = rng.integers(-1, 2, size=(d, d)).astype(np.float64)
        th = rng.uniform(-np.pi, np.pi, size=(N, L, d // 2))
        ph = rng.uniform(-np.pi, np.pi, size=(N, L, d // 2))
        wg = rng.normal(0, 1 / np.sqrt(d), size=(N, d))
        b = rng.normal(0, 0.5, size=N) if bias else None
        gy = rng.normal(size=(T, d))
        l = O.router_logits(x, wg, b)
        srt = -np.sort(-l, axis=1)
        if k < N and (srt[:, k - 1] - srt[:, k]).min() < 1e-2:
            continue  # keep routing stable under the perturbations
        return dict(x=x, w=w, alpha=0.3, th=th, ph=ph, wg=wg, b=b, k=k, gy=gy)


def _loss(c):
    idx, g, _, _ = O.route(c["x"], c["wg"], c["b"], c["k"])
    y = O.forward(c["x"], c["w"], c["alpha"], c["th"], c["ph"], idx, g)
    return float(np.sum(y * c["gy"]))


def _fd(c, key):
    base = c[key]
    if np.isscalar(base):
        c1, c2 = dict(c), dict(c)
        c1[key], c2[key] = base + H, base - H
        return (_loss(c1) - _loss(c2)) / (2 * H)
    out = np.zeros_like(base)
    for i in np.ndindex(base.shape):
        p, m = base.copy(), base.copy()
        p[i] += H
        m[i] -= H
        c1, c2 = dict(c), dict(c)
        c1[key], c2[key] = p, m
        out[i] = (_loss(c1) - _loss(c2)) / (2 * H)
    return out


def _grads(c):
    return O.backward(c["x"], c["w"], c["alpha"], c["th"], c["ph"], c["wg"], c["b"], c["k"], c["gy"])


@pytest.mark.parametrize("seed,bias,k", [(0, True, 2), (1, False, 1), (2, True, 3)])
def test_backward_matches_finite_differences(seed, bias, k):
    c = _case(seed=seed, bias=bias, k=k)
    g = _grads(c)
    pairs = [("x", "dx"), ("th", "dtheta"), ("ph", "dphi"), ("w", "dw_base"), ("alpha", "dalpha"),
             ("wg", "dw_gate")] + ([("b", "dbias")] if bias else [])
    for key, gk in pairs:
        fd = _fd(c, key)
        an = np.asarray(g[gk])
        scale = max(1.0, float(np.abs(fd).max()))
        assert np.abs(an - fd).max() <= 1e-7 * scale, (key, np.abs(an - fd).max())


def test_backward_d16_angles_and_base():
    # one more size (4 stages), angles and base only (the slowest to difference)
    c = _case(d=16, N=2, k=1, T=3, seed=4)
    g = _grads(c)
    for key, gk in (("th", "dtheta"), ("ph", "dphi"), ("w", "dw_base")):
        fd = _fd(c, key)
        assert np.abs(g[gk] - fd).max() <= 1e-7 * max(1.0, np.abs(fd).max()), key


def test_unused_experts_get_zero_angle_gradients():
    c = _case(N=4, k=1, seed=5)
    g = _grads(c)
    used = np.unique(g["idx"])
    for e in range(4):
        if e not in used:
            assert not g["dtheta"][e].any() and not g["dphi"][e].any()
            assert not g["dw_gate"][e].any()


def test_zero_angles_reduce_to_a_scaled_dense_layer():
    # with B = I the expert is alpha W: dx = alpha W^T (sum_j g_j) gy plus the
    # router term, and dW = alpha gy^T x summed with the gates
    c = _case(seed=6)
    c["th"][:] = 0
    c["ph"][:] = 0
    g = _grads(c)
    idx, gates, _, _ = O.route(c["x"], c["wg"], c["b"], c["k"])
    gsum = gates.sum(axis=1)[:, None]
    dW = c["alpha"] * ((gsum * c["gy"]).T @ c["x"])
    assert np.allclose(g["dw_base"], dW, atol=1e-12)


def test_stage_derivative_is_the_difference_quotient_of_the_stage():
    rng = np.random.default_rng(8)
    d = 8
    for s in range(3):
        ang = rng.uniform(-np.pi, np.pi, d // 2)
        for r in range(d // 2):
            p, m = ang.copy(), ang.copy()
            p[r] += H
            m[r] -= H
            fd = (O.stage_matrix(d, s, p) - O.stage_matrix(d, s, m)) / (2 * H)
            assert np.abs(O.stage_derivative(d, s, ang, r) - fd).max() < 1e-8


def test_angle_gradient_equals_the_dense_factorisation():
    # the stage-by-stage contraction against the dense prefix/suffix products
    rng = np.random.default_rng(9)
    d, L = 16, 4
    ang = rng.uniform(-np.pi, np.pi, (L, d // 2))
    X = rng.normal(size=(3, d))
    G = rng.normal(size=(3, d))
    S = [O.stage_matrix(d, s, ang[s]) for s in range(L)]
    got = O.butterfly_angle_grad(ang, X, G)
    for s in range(L):
        P = np.eye(d)
        for q in range(s):
            P = S[q] @ P
        Q = np.eye(d)
        for q in range(s + 1, L):
            Q = S[q] @ Q
        for r in range(d // 2):
            dB = Q @ O.stage_derivative(d, s, ang[s], r) @ P
            assert abs(got[s, r] - np.einsum("ti,ij,tj->", G, dB, X)) < 1e-12
