"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch each one: a wrong Givens sign, a reversed stage order, a wrong rotation
index, B(-theta) in place of B(theta)^T, a dropped scale, a wrong tie-break,
unnormalised gates, a transposed base and a wrong bit order in the 2-bit code.
"""
import math

import numpy as np
import pytest

import tests.test_oracle_pins as pins
from oracle import bfmoe_oracle as O


def _fails(fn, *args):
    try:
        fn(*args)
    except (AssertionError, ValueError, IndexError):
        return True
    return False


@pytest.fixture
def worked(golden_dir):
    import json, os
    with open(os.path.join(golden_dir, "butterfly_worked_examples.json")) as f:
        return json.load(f)


def test_wrong_givens_sign_is_caught(monkeypatch, worked):
    good = O.stage_matrix
    monkeypatch.setattr(O, "stage_matrix", lambda d, s, a: good(d, s, a).T)
    assert _fails(pins.test_worked_examples, worked)


def test_reversed_stage_order_is_caught(monkeypatch, worked):
    def bad(angles):
        angles = np.asarray(angles, dtype=np.float64)
        L, half = angles.shape
        B = np.eye(2 * half)
        for s in range(L):
            B = B @ O.stage_matrix(2 * half, s, angles[s])
        return B
    monkeypatch.setattr(O, "butterfly_matrix", bad)
    assert _fails(pins.test_worked_examples, worked)


def test_wrong_rotation_index_is_caught(monkeypatch, worked):
    monkeypatch.setattr(O, "rotation_index", lambda i, s: (i >> 1) % (1 << s) if s else i >> 1)
    assert _fails(pins.test_worked_examples, worked)


def test_negated_angles_instead_of_transpose_is_caught(monkeypatch, worked):
    good = O.butterfly_apply

    def bad(angles, X, transpose=False):
        if transpose:
            return good(-np.asarray(angles), X, transpose=False)
        return good(angles, X)
    monkeypatch.setattr(O, "butterfly_apply", bad)
    assert _fails(pins.test_worked_examples, worked)


def test_dropped_alpha_is_caught(monkeypatch):
    good = O.expert_matrix
    monkeypatch.setattr(O, "expert_matrix", lambda W, a, t, p: good(W, 1.0, t, p))
    assert _fails(pins.test_forward_brute_force_loops)


def test_untransposed_input_rotation_is_caught(monkeypatch):
    def bad(W, alpha, th, ph):
        return float(alpha) * (O.butterfly_matrix(ph) @ np.asarray(W, float) @ O.butterfly_matrix(th))
    monkeypatch.setattr(O, "expert_matrix", bad)
    assert _fails(pins.test_forward_brute_force_loops)


def test_transposed_base_is_caught(monkeypatch):
    def bad(W, alpha, th, ph):
        return float(alpha) * (O.butterfly_matrix(ph) @ np.asarray(W, float).T @ O.butterfly_matrix(th).T)
    monkeypatch.setattr(O, "expert_matrix", bad)
    assert _fails(pins.test_forward_brute_force_loops)


def test_highest_index_tie_break_is_caught(monkeypatch):
    def bad(logits, k):
        T, N = logits.shape
        order = np.lexsort((-np.broadcast_to(np.arange(N), logits.shape), -logits), axis=-1)
        return order[:, :k].astype(np.int32), np.zeros(T, bool)
    monkeypatch.setattr(O, "topk", bad)
    assert _fails(pins.test_topk_brute_force)


def test_unnormalised_gates_are_caught(monkeypatch):
    def bad(logits, idx):
        z = np.exp(logits - logits.max(axis=1, keepdims=True))
        p = z / z.sum(axis=1, keepdims=True)
        return np.take_along_axis(p, idx.astype(np.int64), axis=1)
    monkeypatch.setattr(O, "gates_for", bad)
    assert _fails(pins.test_gates_equal_softmax_topk_renormalised)


def test_msb_first_pack_is_caught(monkeypatch, golden_dir):
    def bad(w):
        w = np.asarray(w)
        d = w.shape[1]
        out = np.zeros((w.shape[0], O.words_per_row(d)), dtype=np.uint32)
        for o in range(w.shape[0]):
            for i in range(d):
                out[o, i // 16] |= np.uint32(O.CODE[int(w[o, i])] << (30 - 2 * (i % 16)))
        return out
    monkeypatch.setattr(O, "pack_base", bad)
    assert _fails(pins.test_pack_hand_example, golden_dir)


def test_missing_bias_is_caught(monkeypatch):
    monkeypatch.setattr(O, "router_logits",
                        lambda x, W, b: np.asarray(x, float) @ np.asarray(W, float).T)
    assert _fails(pins.test_logits_include_bias)


# -- backward pass: planted mistakes must fail the finite-difference pins ------

def test_backward_wrong_rotation_derivative_is_caught(monkeypatch):
    import tests.test_oracle_backward as bw
    good = O.rotation_derivative
    monkeypatch.setattr(O, "rotation_derivative", lambda a: good(a).T)
    assert _fails(bw.test_backward_matches_finite_differences, 0, True, 2)


def test_backward_untransposed_base_is_caught(monkeypatch):
    import tests.test_oracle_backward as bw
    good = O.backward

    def bad(*a, **k):
        g = good(*a, **k)
        g["dw_base"] = g["dw_base"].T
        return g
    monkeypatch.setattr(O, "backward", bad)
    assert _fails(bw.test_backward_matches_finite_differences, 0, True, 2)


def test_backward_without_router_term_is_caught(monkeypatch):
    import tests.test_oracle_backward as bw
    good = O.backward

    def bad(*a, **k):
        g = good(*a, **k)
        g["dw_gate"] = np.zeros_like(g["dw_gate"])
        return g
    monkeypatch.setattr(O, "backward", bad)
    assert _fails(bw.test_backward_matches_finite_differences, 0, True, 2)
