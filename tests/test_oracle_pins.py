"""Pins of the float64 oracle to facts that do not come from the oracle itself:
hand-worked examples, closed forms, library routines and brute force.

Sources: ButterflyMoE technical summary (gist.science), section 2.1 (expert
parametrisation, ternary base, butterfly rotations), section 2.2 (memory
O(d^2 + N d log d)), section 2.3 (three-step inference); the word "rotation"
(orthogonal transform) in section 2.1 pins orthogonality and norm
preservation.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special

from oracle import bfmoe_oracle as O


def _angles(d, entries):
    L = O.n_stages(d)
    a = np.zeros((L, d // 2))
    for s, r, v in entries:
        a[int(s), int(r)] = v
    return a


@pytest.fixture(scope="module")
def worked(golden_dir):
    with open(os.path.join(golden_dir, "butterfly_worked_examples.json")) as f:
        return json.load(f)


# -- P1: zero angles -> identity -------------------------------------------

@pytest.mark.parametrize("d", [2, 4, 8, 64, 256])
def test_zero_angles_give_identity(d):
    L = O.n_stages(d)
    B = O.butterfly_matrix(np.zeros((L, d // 2)))
    assert np.array_equal(B, np.eye(d))
    rng = np.random.default_rng(1)
    W = rng.integers(-1, 2, size=(d, d))
    z = np.zeros((L, d // 2))
    assert np.array_equal(O.expert_matrix(W, 0.25, z, z), 0.25 * W)


# -- P2: rotations are orthogonal with det +1 ---------------------------------

@pytest.mark.parametrize("d", [2, 4, 8, 16, 64, 256])
def test_butterfly_is_rotation(d):
    rng = np.random.default_rng(d)
    a = rng.uniform(-np.pi, np.pi, size=(O.n_stages(d), d // 2))
    B = O.butterfly_matrix(a)
    assert np.abs(B.T @ B - np.eye(d)).max() < 1e-12
    sign, logdet = np.linalg.slogdet(B)
    assert sign == 1.0 and abs(logdet) < 1e-10


# -- P3: hand-worked signed permutations (pairing, order, sign, transpose) ----

def test_worked_examples(worked):
    for case in worked["cases"]:
        d = case["d"]
        a = _angles(d, case["angles"])
        x = np.arange(1, d + 1, dtype=np.float64)
        B = O.butterfly_matrix(a)
        assert np.abs(B @ x - np.array(case["Bx"])).max() < 1e-12, case["note"]
        assert np.abs(O.butterfly_apply(a, x[None])[0] - case["Bx"]).max() < 1e-12
        if "BTx" in case:
            assert np.abs(B.T @ x - np.array(case["BTx"])).max() < 1e-12
            assert np.abs(O.butterfly_apply(a, x[None], transpose=True)[0]
                          - case["BTx"]).max() < 1e-12


def test_worked_expert(worked):
    c = worked["expert_case"]
    d = c["d"]
    a = _angles(d, c["angles"])
    W = np.array([[((4 * o + i) % 3) - 1 for i in range(d)] for o in range(d)])
    assert np.array_equal(W, np.array(c["w_base"]))
    assert np.abs(O.butterfly_matrix(a) - np.array(c["B"])).max() < 1e-12
    We = O.expert_matrix(W, c["alpha"], a, a)
    assert np.abs(We - np.array(c["W_e"])).max() < 1e-12


# -- closed forms: Kronecker structure and 2-D rotations ------------------------

def _rot(a):
    return np.array([[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]])


@pytest.mark.parametrize("d", [2, 4, 8, 32])
def test_equal_angles_is_kronecker_power(d):
    # All rotations equal a: stage s acts on index bit s, so B is R(a)^{(x)L}.
    a = 0.7313
    L = O.n_stages(d)
    B = O.butterfly_matrix(np.full((L, d // 2), a))
    K = np.array([[1.0]])
    for _ in range(L):
        K = np.kron(K, _rot(a))
    assert np.abs(B - K).max() < 1e-12


@pytest.mark.parametrize("d,s", [(8, 0), (8, 1), (8, 2), (16, 2), (32, 3)])
def test_stage_angle_indexing_closed_form(d, s):
    # One stage, angle of rotation r = f(high part) + g(low part) with the
    # rotation index r = high * 2^s + low: the stage matrix is, per high block,
    # [[C, -S], [S, C]] with C, S diagonal over the low index.
    h = 1 << s
    n_high = d // (2 * h)
    rng = np.random.default_rng(7 + d + s)
    ang = rng.uniform(-np.pi, np.pi, size=(n_high, h))
    S = O.stage_matrix(d, s, ang.reshape(-1))
    blocks = []
    for hi in range(n_high):
        C = np.diag(np.cos(ang[hi]))
        Sn = np.diag(np.sin(ang[hi]))
        blocks.append(np.block([[C, -Sn], [Sn, C]]))
    assert np.abs(S - scipy.linalg.block_diag(*blocks)).max() < 1e-12


def test_stage_is_exponential_of_generators():
    # Each stage is the product of commuting Givens rotations, so it equals
    # expm of the sum of their skew generators (library routine).
    rng = np.random.default_rng(3)
    for d in (4, 8, 16):
        for s in range(O.n_stages(d)):
            a = rng.uniform(-1.5, 1.5, size=d // 2)
            G = np.zeros((d, d))
            h = 1 << s
            r = 0
            for i in range(d):
                if i & h:
                    continue
                j = i + h
                G[j, i] += a[r]
                G[i, j] -= a[r]
                r += 1
            assert np.abs(O.stage_matrix(d, s, a) - scipy.linalg.expm(G)).max() < 1e-12


def test_d2_expert_by_complex_rotation():
    # d = 2: B(a) is the plane rotation by a, i.e. multiplication by e^{ia}.
    rng = np.random.default_rng(11)
    for _ in range(20):
        th, ph = rng.uniform(-np.pi, np.pi, size=2)
        W = rng.integers(-1, 2, size=(2, 2))
        x = rng.normal(size=2)
        u = np.exp(-1j * th) * complex(x[0], x[1])
        z = 0.5 * (W @ np.array([u.real, u.imag]))
        y = np.exp(1j * ph) * complex(z[0], z[1])
        got = O.expert_matrix(W, 0.5, [[th]], [[ph]]) @ x
        assert abs(got[0] - y.real) < 1e-12 and abs(got[1] - y.imag) < 1e-12


# -- P4: stage-wise application equals the dense product -----------------------

@pytest.mark.parametrize("d", [2, 4, 16, 64, 512])
def test_stagewise_equals_dense(d):
    rng = np.random.default_rng(d + 5)
    a = rng.uniform(-np.pi, np.pi, size=(O.n_stages(d), d // 2))
    X = rng.normal(size=(3, d))
    B = O.butterfly_matrix(a)
    assert np.abs(O.butterfly_apply(a, X) - X @ B.T).max() < 1e-12
    assert np.abs(O.butterfly_apply(a, X, transpose=True) - X @ B).max() < 1e-12


def test_three_step_inference_equals_materialised_expert():
    rng = np.random.default_rng(17)
    d = 64
    W = rng.integers(-1, 2, size=(d, d))
    th = rng.uniform(-np.pi, np.pi, size=(6, 32))
    ph = rng.uniform(-np.pi, np.pi, size=(6, 32))
    X = rng.normal(size=(5, d))
    a = O.expert_apply(W, 0.125, th, ph, X)
    b = X @ O.expert_matrix(W, 0.125, th, ph).T
    assert np.abs(a - b).max() < 1e-12


# -- P8: norm preservation -----------------------------------------------------

def test_norm_preserved():
    rng = np.random.default_rng(23)
    for d in (8, 128, 1024):
        a = rng.uniform(-np.pi, np.pi, size=(O.n_stages(d), d // 2))
        X = rng.normal(size=(4, d))
        for tr in (False, True):
            Y = O.butterfly_apply(a, X, transpose=tr)
            n0 = np.linalg.norm(X, axis=1)
            assert np.abs(np.linalg.norm(Y, axis=1) - n0).max() < 1e-13 * n0.max() * 10


# -- P5: stored-parameter count and packed size --------------------------------

def test_param_count_closed_form():
    assert O.param_count(512, 64) == (262144, 294912)
    assert O.param_count(512, 256) == (262144, 1179648)
    for d, n in ((64, 8), (1024, 256), (2048, 1024)):
        t, a = O.param_count(d, n)
        assert t == d * d and a == n * d * int(math.log2(d))
        W = np.zeros((d, d), dtype=np.int8)
        if d <= 64:
            assert O.pack_base(W).nbytes == d * d // 4


# -- P6: 2-bit pack -------------------------------------------------------------

def test_pack_hand_example(golden_dir):
    with open(os.path.join(golden_dir, "ternary_pack_example.json")) as f:
        g = json.load(f)
    row = np.array([g["row"]], dtype=np.int8)
    p = O.pack_base(row)
    assert p.shape == (1, 1)
    assert int(p[0, 0]) == int(g["word_hex"], 16)


def test_pack_roundtrip_and_reject():
    rng = np.random.default_rng(29)
    for d in (4, 16, 48, 64):
        W = rng.integers(-1, 2, size=(d, d)).astype(np.int8)
        assert np.array_equal(O.unpack_base(O.pack_base(W), d), W)
    with pytest.raises(ValueError):
        O.pack_base(np.array([[0, 2, 0, 0]]))
    with pytest.raises(ValueError):
        O.unpack_base(np.array([[0b10]], dtype=np.uint32), 4)


# -- P9: router -----------------------------------------------------------------

def test_topk_brute_force():
    rng = np.random.default_rng(31)
    for N, k in ((5, 1), (5, 2), (8, 3), (4, 4)):
        # integers make exact ties common
        l = rng.integers(-3, 4, size=(40, N)).astype(np.float64)
        idx, near = O.topk(l, k)
        for t in range(40):
            ranked = sorted(range(N), key=lambda e: (-l[t, e], e))
            assert list(idx[t]) == ranked[:k]
            vals = [l[t, e] for e in ranked[:min(k + 1, N)]]
            tie = any(vals[i] - vals[i + 1] < O.NEAR_TIE for i in range(len(vals) - 1))
            assert near[t] == tie


def test_gates_equal_softmax_topk_renormalised():
    rng = np.random.default_rng(37)
    l = rng.normal(size=(50, 16)) * 3
    for k in (1, 2, 4):
        idx, _ = O.topk(l, k)
        g = O.gates_for(l, idx)
        p = scipy.special.softmax(l, axis=1)
        ps = np.take_along_axis(p, idx.astype(np.int64), axis=1)
        assert np.abs(g - ps / ps.sum(axis=1, keepdims=True)).max() < 1e-14
        assert np.abs(g.sum(axis=1) - 1).max() < 1e-14
        assert (np.diff(g, axis=1) <= 1e-15).all()  # slots in descending order


def test_logits_include_bias():
    rng = np.random.default_rng(41)
    x = rng.normal(size=(3, 4))
    W = rng.normal(size=(5, 4))
    b = rng.normal(size=5)
    l = O.router_logits(x, W, b)
    for t, e in itertools.product(range(3), range(5)):
        assert abs(l[t, e] - (sum(x[t, i] * W[e, i] for i in range(4)) + b[e])) < 1e-12


# -- buckets: brute force ---------------------------------------------------------

def test_buckets_brute_force():
    rng = np.random.default_rng(43)
    T, N, k = 37, 6, 3
    idx = np.array([rng.permutation(N)[:k] for _ in range(T)], dtype=np.int32)
    counts, offsets, rows = O.buckets(idx, N)
    expect = []
    for e in range(N):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    expect.append(t * k + j)
    assert list(rows) == expect
    assert list(counts) == [int((idx == e).sum()) for e in range(N)]
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert list(np.diff(offsets)) == list(counts)


# -- P7: invariants of the whole forward ----------------------------------------------

def _small_inputs(seed, d=16, N=5, T=9):
    rng = np.random.default_rng(seed)
    W = rng.integers(-1, 2, size=(d, d)).astype(np.int8)
    L = O.n_stages(d)
    th = rng.uniform(-np.pi, np.pi, size=(N, L, d // 2))
    ph = rng.uniform(-np.pi, np.pi, size=(N, L, d // 2))
    x = rng.normal(size=(T, d))
    Wg = rng.normal(size=(N, d))
    return W, th, ph, x, Wg


def test_identical_experts_ignore_routing():
    W, th, ph, x, Wg = _small_inputs(47)
    th[:] = th[0]
    ph[:] = ph[0]
    W0 = O.expert_matrix(W, 0.3, th[0], ph[0])
    for k in (1, 2, 3):
        idx, g, _, _ = O.route(x, Wg, None, k)
        y = O.forward(x, W, 0.3, th, ph, idx, g)
        assert np.abs(y - x @ W0.T).max() < 1e-12


def test_top1_is_single_expert_and_linear():
    W, th, ph, x, Wg = _small_inputs(53)
    idx, g, _, _ = O.route(x, Wg, None, 1)
    assert np.all(g == 1.0)
    y = O.forward(x, W, 0.3, th, ph, idx, g)
    for t in range(x.shape[0]):
        We = O.expert_matrix(W, 0.3, th[idx[t, 0]], ph[idx[t, 0]])
        assert np.abs(y[t] - We @ x[t]).max() < 1e-12
    # linear in x for fixed routing
    y2 = O.forward(2.5 * x, W, 0.3, th, ph, idx, g)
    assert np.abs(y2 - 2.5 * y).max() < 1e-12


def test_forward_dense_equals_sampled_three_step():
    W, th, ph, x, Wg = _small_inputs(59, d=32, N=6, T=11)
    idx, g, _, _ = O.route(x, Wg, None, 2)
    y = O.forward(x, W, 0.2, th, ph, idx, g)
    ys = O.forward_tokens(x[[0, 4, 10]], W, 0.2, th, ph, idx[[0, 4, 10]], g[[0, 4, 10]])
    assert np.abs(y[[0, 4, 10]] - ys).max() < 1e-12


def test_forward_brute_force_loops():
    # Tiny case with every product written as explicit loops over scalars.
    d, N, T, k = 4, 3, 5, 2
    W, th, ph, x, Wg = _small_inputs(61, d=d, N=N, T=T)
    idx, g, _, _ = O.route(x, Wg, None, k)
    y = O.forward(x, W, 0.5, th, ph, idx, g)
    for t in range(T):
        acc = [0.0] * d
        for j in range(k):
            e = idx[t, j]
            Bt = O.butterfly_matrix(th[e])
            Bp = O.butterfly_matrix(ph[e])
            u = [sum(Bt[i2, i] * x[t, i2] for i2 in range(d)) for i in range(d)]  # B^T x
            z = [0.5 * sum(int(W[o, i]) * u[i] for i in range(d)) for o in range(d)]
            v = [sum(Bp[a, o] * z[o] for o in range(d)) for a in range(d)]
            for a in range(d):
                acc[a] += g[t, j] * v[a]
        assert np.abs(y[t] - np.array(acc)).max() < 1e-12


def test_rel_l2_metric():
    y = np.array([[3.0, 4.0], [0.0, 0.0]])
    yr = np.array([[3.0, 0.0], [0.0, 0.0]])
    r = O.rel_l2_per_token(y, yr)
    assert abs(r[0] - 4.0 / 3.0) < 1e-15 and r[1] == 0.0
