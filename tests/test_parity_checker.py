"""The parity checker itself, on the CPU: routings that are wrong in ways a
top-k kernel could get wrong must fail it, also on near-tie tokens where
several selections are valid.  The 'GPU' results here are made by the oracle
and then altered, so only the routing check can catch them."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import bfmoe_oracle as O
from tests.parity_util import check_routing, compare


def _near_tie_inputs():
    # d=8, N=4, k=2: token 0 gets logits (1.0, 0.5, 0.5 + 5e-6, -1.0), a near
    # tie between ranks 2 and 3; token 1 has no tie
    wl = W.custom("tie", d=8, n_experts=4, k=2, tokens=2, dtype="f32")
    inp = W.generate(wl, seed=0)
    inp.w_gate = np.zeros((4, 8), np.float32)
    inp.w_gate[:, 0] = np.array([1.0, 0.5, 0.500005, -1.0], np.float32)
    inp.w_gate[:, 1] = np.array([0.0, 2.0, 1.0, 3.0], np.float32)
    inp.bias = None
    x = np.zeros((2, 8), np.float32)
    x[0, 0] = 1.0
    x[1, 1] = 1.0
    inp.x = torch.from_numpy(x)
    return inp


def _fake_gpu(inp, idx):
    idx = np.asarray(idx, np.int32)
    x = inp.x_f64()
    logits = O.router_logits(x, inp.w_gate, inp.bias)
    g = O.gates_for(logits, idx)
    c, o, r = O.buckets(idx, inp.wl.n_experts)
    y = O.forward(x, inp.w_base, inp.alpha, inp.theta, inp.phi, idx, g)
    return {"idx": idx, "gates": g, "counts": c, "offsets": o, "rows": r, "y": y}


def test_inputs_have_the_intended_near_tie():
    inp = _near_tie_inputs()
    logits = O.router_logits(inp.x_f64(), inp.w_gate, inp.bias)
    idx, near = O.topk(logits, 2)
    assert near.tolist() == [True, False]
    assert idx.tolist() == [[0, 2], [3, 1]]


@pytest.mark.parametrize("idx", [[[0, 2], [3, 1]], [[0, 1], [3, 1]]])
def test_valid_choices_on_a_near_tie_pass(idx):
    inp = _near_tie_inputs()
    stats = compare(inp, _fake_gpu(inp, idx))
    assert stats["near_ties"] == 1


@pytest.mark.parametrize("idx", [
    [[0, 3], [3, 1]],   # an expert far below the k-th logit on the near-tie token
    [[2, 0], [3, 1]],   # slots out of logit order on the near-tie token
    [[1, 2], [3, 1]],   # the clear winner dropped on the near-tie token
    [[0, 0], [3, 1]],   # the same expert twice
    [[0, 2], [1, 3]],   # slot order swapped on a token without a tie
    [[0, 2], [3, 2]],   # a wrong expert on a token without a tie
])
def test_invalid_choices_fail(idx):
    inp = _near_tie_inputs()
    with pytest.raises(AssertionError):
        compare(inp, _fake_gpu(inp, idx))


def test_out_of_range_expert_fails():
    logits = np.array([[1.0, 0.5, 0.5 + 5e-6, -1.0]])
    with pytest.raises(AssertionError):
        check_routing(logits, np.array([[0, 7]]), 2)
