"""Plain float64 CPU oracle of the ButterflyMoE expert forward.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module.  It is slow on purpose and shares no code
with the CUDA path: it builds every butterfly as a product of dense stage
matrices, forms each expert densely, routes naively and multiplies densely.

What it computes, and where each piece is defined:

* Expert i is ``W_i = B(phi_i) . W_base . B(theta_i)^T``, with ``W_base`` one
  ternary {-1, 0, +1} matrix shared by every expert and ``B(.)`` a per-expert
  learned butterfly rotation with O(d log d) parameters (gist.science,
  "ButterflyMoE: sub-linear ternary experts via structured butterfly orbits",
  technical summary section 2.1; same statement in the arXiv abstract quoted
  on the signalfieldnotes ButterflyMoE article and on the umar.mx record).
* Inference never forms ``W_i``: it applies ``B(theta_i)^T`` to x, multiplies
  by the ternary base, then applies ``B(phi_i)`` (technical summary, section
  2.3).  :func:`expert_apply` follows those three steps; :func:`forward`
  uses the formed matrix; a pin checks that the two agree.
* Memory is O(d^2 + N d log d) (technical summary, section 2.2);
  :func:`param_count` gives the exact stored-parameter count.
* Routing is standard mixture-of-experts selection (signalfieldnotes
  article, glossary entry "Mixtures of Experts").  The pages give no router
  formula; this oracle uses a float32 gate matrix and optional bias, logits
  ``x W_g^T + b``, top-k by descending logit with the lower expert index
  winning ties, and gates equal to a softmax over the k selected logits
  (the same as softmax over all N, top-k, renormalise).

Readings where the pages are silent (butterfly pairing, stage order, Givens
sign, the meaning of ``B^T``, the scale ``alpha``, the 2-bit code) are stated
at each function.  Every function here is pinned by a ``-m "not gpu"`` test
against a closed form, a hand-worked example, a library routine or brute
force.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

NEAR_TIE = 1e-5  # logit gap below which two experts count as tied


# ---------------------------------------------------------------------------
# Butterfly rotations
# ---------------------------------------------------------------------------

def n_stages(d: int) -> int:
    if d < 2 or d & (d - 1):
        raise ValueError("d must be a power of two >= 2")
    return d.bit_length() - 1


def rotation_index(i: int, s: int) -> int:
    """Index, within stage ``s``, of the rotation that acts on element ``i``
    (whose bit ``s`` is clear) and its partner ``i + 2**s``.

    Reading (the pages only say "butterfly structure"): rotations of a stage
    are numbered in ascending order of their lower element.
    """
    h = 1 << s
    return (i >> (s + 1)) * h + (i & (h - 1))


def stage_matrix(d: int, s: int, angles_s: np.ndarray) -> np.ndarray:
    """Dense d x d matrix of butterfly stage ``s`` (stride ``h = 2**s``).

    For each i with bit s clear and j = i + h, with a = angles_s[r(i)]:
    [y_i, y_j] = [[cos a, -sin a], [sin a, cos a]] [x_i, x_j]
    (counter-clockwise Givens rotation; the pages fix no sign).
    """
    h = 1 << s
    S = np.zeros((d, d), dtype=np.float64)
    a = np.asarray(angles_s, dtype=np.float64)
    for i in range(d):
        if i & h:
            continue
        j = i + h
        r = rotation_index(i, s)
        c, sn = math.cos(a[r]), math.sin(a[r])
        S[i, i] = c
        S[i, j] = -sn
        S[j, i] = sn
        S[j, j] = c
    return S


def butterfly_matrix(angles: np.ndarray) -> np.ndarray:
    """B = S_{L-1} ... S_1 S_0 as a product of dense stage matrices.

    ``angles`` is [L, d/2].  Stage 0 (stride 1) acts first on a column vector.
    """
    angles = np.asarray(angles, dtype=np.float64)
    L, half = angles.shape
    d = 2 * half
    if n_stages(d) != L:
        raise ValueError("angles must be [log2 d, d/2]")
    B = np.eye(d)
    for s in range(L):
        B = stage_matrix(d, s, angles[s]) @ B
    return B


def butterfly_apply(angles: np.ndarray, X: np.ndarray, transpose: bool = False) -> np.ndarray:
    """Apply B (or B^T) to each row of X stage by stage, in O(d log d) per row.

    ``B^T`` is the literal transpose of :func:`butterfly_matrix`: stages in
    the order L-1 ... 0, each with its 2x2 block transposed.  (Not B(-angles),
    which would keep the forward stage order.)
    """
    angles = np.asarray(angles, dtype=np.float64)
    L, half = angles.shape
    d = 2 * half
    Y = np.array(X, dtype=np.float64, copy=True)
    order = range(L - 1, -1, -1) if transpose else range(L)
    for s in order:
        h = 1 << s
        lo = np.array([i for i in range(d) if not i & h])
        hi = lo + h
        r = np.array([rotation_index(int(i), s) for i in lo])
        c = np.cos(angles[s][r])
        sn = np.sin(angles[s][r])
        if transpose:
            sn = -sn
        xi = Y[..., lo].copy()
        xj = Y[..., hi].copy()
        Y[..., lo] = c * xi - sn * xj
        Y[..., hi] = sn * xi + c * xj
    return Y


# ---------------------------------------------------------------------------
# Experts
# ---------------------------------------------------------------------------

def expert_matrix(w_base: np.ndarray, alpha: float, theta_e: np.ndarray,
                  phi_e: np.ndarray) -> np.ndarray:
    """W_e = alpha * B(phi_e) . W_base . B(theta_e)^T, formed densely.

    ``W_base[o, i]``: o is the output row, i the input column (y = W x).
    ``alpha`` is the one float32 scale of the ternary base (the pages only
    say "1.58 bits per weight"; the scale is a reading).
    """
    W = np.asarray(w_base, dtype=np.float64)
    return float(alpha) * (butterfly_matrix(phi_e) @ W @ butterfly_matrix(theta_e).T)


def expert_apply(w_base: np.ndarray, alpha: float, theta_e: np.ndarray,
                 phi_e: np.ndarray, X: np.ndarray) -> np.ndarray:
    """The three-step, non-materialising expert: rows of X through
    B(theta)^T, then the ternary base times alpha, then B(phi)."""
    U = butterfly_apply(theta_e, X, transpose=True)
    Z = float(alpha) * (U @ np.asarray(w_base, dtype=np.float64).T)
    return butterfly_apply(phi_e, Z, transpose=False)


def param_count(d: int, n_experts: int) -> Tuple[int, int]:
    """(ternary weights, rotation angles) stored: d^2 and 2 N (d/2) log2 d."""
    return d * d, 2 * n_experts * (d // 2) * n_stages(d)


# ---------------------------------------------------------------------------
# Routing
# ---------------------------------------------------------------------------

def router_logits(x: np.ndarray, w_gate: np.ndarray,
                  bias: Optional[np.ndarray]) -> np.ndarray:
    """l = x W_g^T (+ b), in float64 from the stored values."""
    l = np.asarray(x, dtype=np.float64) @ np.asarray(w_gate, dtype=np.float64).T
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)[None, :]
    return l


def topk(logits: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    """Top-k experts per token by descending logit, lower index first on ties.

    Returns (idx [T, k] int32, near_tie [T] bool).  A token is a near tie when
    two neighbours among its first min(k+1, N) sorted logits differ by less
    than NEAR_TIE: then another selection or slot order is equally valid.
    """
    T, N = logits.shape
    if not 1 <= k <= N:
        raise ValueError("need 1 <= k <= N")
    experts = np.broadcast_to(np.arange(N), logits.shape)
    order = np.lexsort((experts, -logits), axis=-1)
    idx = order[:, :k].astype(np.int32)
    m = min(k + 1, N)
    top = np.take_along_axis(logits, order[:, :m], axis=1)
    near = (np.diff(-top, axis=1) < NEAR_TIE).any(axis=1) if m > 1 else np.zeros(T, bool)
    return idx, near


def gates_for(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g_j = exp(l_{e_j} - l_{e_0}) / sum_j' exp(l_{e_j'} - l_{e_0})."""
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    z = np.exp(sel - sel[:, :1])
    return z / z.sum(axis=1, keepdims=True)


def route(x, w_gate, bias, k):
    """Naive router: (idx [T,k] int32, gates [T,k] f64, near_tie [T] bool, logits)."""
    l = router_logits(x, w_gate, bias)
    idx, near = topk(l, k)
    return idx, gates_for(l, idx), near, l


def buckets(idx: np.ndarray, n_experts: int):
    """Token-to-expert buckets.

    Routed row r = t*k + j.  ``counts[e]`` rows go to expert e; ``offsets`` is
    the exclusive prefix sum of counts (length N+1); ``rows`` lists, expert by
    expert, that expert's rows in ascending token order.
    """
    flat = np.asarray(idx).reshape(-1)
    counts = np.zeros(n_experts, dtype=np.int32)
    parts = []
    for e in range(n_experts):
        r = np.nonzero(flat == e)[0]
        counts[e] = r.size
        parts.append(r)
    offsets = np.zeros(n_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    rows = np.concatenate(parts).astype(np.int32) if parts else np.zeros(0, np.int32)
    return counts, offsets, rows


# ---------------------------------------------------------------------------
# Forward
# ---------------------------------------------------------------------------

def forward(x, w_base, alpha, theta, phi, idx, gates) -> np.ndarray:
    """y_t = sum_j g_{t,j} W_{e_{t,j}} x_t with every used W_e formed densely."""
    X = np.asarray(x, dtype=np.float64)
    T, d = X.shape
    k = idx.shape[1]
    y = np.zeros((T, d), dtype=np.float64)
    flat = idx.reshape(-1)
    for e in np.unique(flat):
        W_e = expert_matrix(w_base, alpha, theta[e], phi[e])
        r = np.nonzero(flat == e)[0]
        t, j = r // k, r % k
        y_part = X[t] @ W_e.T
        np.add.at(y, t, gates[t, j][:, None] * y_part)
    return y


def forward_tokens(x_rows, w_base, alpha, theta, phi, idx_rows, gates_rows) -> np.ndarray:
    """Same output for a sample of tokens (rows of x with their routing), by
    the three-step expert of :func:`expert_apply`; for full-size workloads
    where forming every expert densely would take too long."""
    X = np.asarray(x_rows, dtype=np.float64)
    y = np.zeros_like(X)
    for t in range(X.shape[0]):
        for j in range(idx_rows.shape[1]):
            e = int(idx_rows[t, j])
            v = expert_apply(w_base, alpha, theta[e], phi[e], X[t:t + 1])
            y[t] += gates_rows[t, j] * v[0]
    return y


# ---------------------------------------------------------------------------
# 2-bit ternary storage
# ---------------------------------------------------------------------------

CODE = {0: 0b00, 1: 0b01, -1: 0b11}   # 0b10 is not a valid code


def words_per_row(d: int) -> int:
    return max(1, (d + 15) // 16)


def pack_base(w: np.ndarray) -> np.ndarray:
    """Row-major 2-bit codes, 16 per uint32, lowest column in the lowest bits.

    The pages store the base at "1.58 bits per weight" (log2 3, technical
    summary section 2.1); this storage spends 2 bits: 0 -> 00, +1 -> 01,
    -1 -> 11.
    """
    w = np.asarray(w)
    d = w.shape[1]
    if not np.isin(w, (-1, 0, 1)).all():
        raise ValueError("not ternary")
    out = np.zeros((w.shape[0], words_per_row(d)), dtype=np.uint32)
    for o in range(w.shape[0]):
        for i in range(d):
            out[o, i // 16] |= np.uint32(CODE[int(w[o, i])] << (2 * (i % 16)))
    return out


def unpack_base(packed: np.ndarray, d: int) -> np.ndarray:
    inv = {0b00: 0, 0b01: 1, 0b11: -1}
    packed = np.asarray(packed, dtype=np.uint32)
    w = np.zeros((packed.shape[0], d), dtype=np.int8)
    for o in range(packed.shape[0]):
        for i in range(d):
            code = (int(packed[o, i // 16]) >> (2 * (i % 16))) & 3
            if code not in inv:
                raise ValueError("invalid 2-bit code")
            w[o, i] = inv[code]
    return w


def rel_l2_per_token(y: np.ndarray, y_ref: np.ndarray) -> np.ndarray:
    """||y_t - y*_t||_2 / max(||y*_t||_2, 1e-30) for every token t."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    num = np.linalg.norm(y - y_ref, axis=1)
    den = np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    return num / den


# ---------------------------------------------------------------------------
# Backward pass (training the rotations with the ternary base)
# ---------------------------------------------------------------------------
#
# The pages train the angles jointly with the quantised base (technical
# summary, section 2.4; arXiv abstract on the signalfieldnotes article: the
# rotations are learned with quantisation-aware training).  They give no
# formula; the gradients below are the chain rule of the forward above, for
# a loss L with dL/dy = gy.  The ternary base gets the straight-through
# estimate: dL/dW_base as if W_base were a real matrix (the usual estimator
# for a quantised weight; its use to update a latent full-precision base is
# the trainer's business).  The top-k selection is piecewise constant, so the
# router's gradient flows through the k selected logits only.

def rotation_derivative(a: float) -> np.ndarray:
    """d/da of the Givens block [[cos a, -sin a], [sin a, cos a]]."""
    return np.array([[-math.sin(a), -math.cos(a)], [math.cos(a), -math.sin(a)]])


def stage_derivative(d: int, s: int, angles_s: np.ndarray, r: int) -> np.ndarray:
    """d S_s / d a_r as a dense matrix: zero except the 2 x 2 block of
    rotation r, :func:`rotation_derivative` of its angle."""
    h = 1 << s
    a = float(np.asarray(angles_s, dtype=np.float64)[r])
    D = np.zeros((d, d))
    blk = rotation_derivative(a)
    for i in range(d):
        if i & h or rotation_index(i, s) != r:
            continue
        j = i + h
        D[np.ix_([i, j], [i, j])] = blk
    return D


def stage_apply(angles_s: np.ndarray, X: np.ndarray, s: int, transpose: bool = False) -> np.ndarray:
    """Rows of X times stage s (or its transpose): one step of
    :func:`butterfly_apply`."""
    d = X.shape[-1]
    h = 1 << s
    a = np.asarray(angles_s, dtype=np.float64)
    lo = np.array([i for i in range(d) if not i & h])
    hi = lo + h
    r = np.array([rotation_index(int(i), s) for i in lo])
    c, sn = np.cos(a[r]), np.sin(a[r])
    if transpose:
        sn = -sn
    Y = np.array(X, dtype=np.float64, copy=True)
    Y[..., lo] = c * X[..., lo] - sn * X[..., hi]
    Y[..., hi] = sn * X[..., lo] + c * X[..., hi]
    return Y


def butterfly_angle_grad(angles: np.ndarray, inp: np.ndarray, gout: np.ndarray) -> np.ndarray:
    """Sum over rows of <gout, (d B / d a_{s,r}) inp> for every angle, from
    the factorisation B = S_{L-1} ... S_0:
    d B / d a_{s,r} = (S_{L-1} ... S_{s+1}) (d S_s / d a_r) (S_{s-1} ... S_0),
    so the term is b^T (d S_s / d a_r) a with a = S_{s-1} ... S_0 inp (the
    stage's input) and b = (S_{L-1} ... S_{s+1})^T gout; only the 2 x 2 block
    of rotation r contributes.  ``inp`` and ``gout`` are [rows, d]; returns
    [L, d/2]."""
    angles = np.asarray(angles, dtype=np.float64)
    L, half = angles.shape
    d = 2 * half
    X = np.asarray(inp, dtype=np.float64)
    ins = [X]
    for s in range(L - 1):
        ins.append(stage_apply(angles[s], ins[-1], s))
    out = np.zeros((L, half))
    Bg = np.asarray(gout, dtype=np.float64)
    for s in range(L - 1, -1, -1):
        A = ins[s]
        h = 1 << s
        for i in range(d):
            if i & h:
                continue
            j = i + h
            r = rotation_index(i, s)
            D = rotation_derivative(angles[s][r])
            pa = A[:, [i, j]]
            pb = Bg[:, [i, j]]
            out[s, r] = float(np.einsum("ti,ij,tj->", pb, D, pa))
        Bg = stage_apply(angles[s], Bg, s, transpose=True)
    return out


def backward(x, w_base, alpha, theta, phi, w_gate, bias, k, gy):
    """Gradients of L with dL/dy = gy through the whole layer (router
    included), with the routing of :func:`route`.  Returns a dict with dx,
    dtheta, dphi (like theta), dw_base [d, d] (straight-through), dalpha,
    dw_gate [N, d] and dbias [N] (None without a bias)."""
    X = np.asarray(x, dtype=np.float64)
    GY = np.asarray(gy, dtype=np.float64)
    W = np.asarray(w_base, dtype=np.float64)
    T, d = X.shape
    N = np.asarray(w_gate).shape[0]
    idx, g, _, _ = route(X, w_gate, bias, k)
    dx = np.zeros_like(X)
    dtheta = np.zeros(np.shape(theta))
    dphi = np.zeros(np.shape(phi))
    dW = np.zeros((d, d))
    dalpha = 0.0
    dg = np.zeros((T, k))
    for e in np.unique(idx):
        Bt = butterfly_matrix(theta[e])
        Bp = butterfly_matrix(phi[e])
        t, j = np.nonzero(idx == e)
        U = X[t] @ Bt                     # rows u = B(theta)^T x
        Z = float(alpha) * (U @ W.T)      # rows z = alpha W u
        V = Z @ Bp.T                      # rows v = B(phi) z
        dg[t, j] = np.einsum("ti,ti->t", V, GY[t])
        dV = g[t, j][:, None] * GY[t]     # dL/dv
        dZ = dV @ Bp                      # B(phi)^T dv
        dU = float(alpha) * (dZ @ W)      # alpha W^T dz
        dW += float(alpha) * (dZ.T @ U)
        dalpha += float(np.einsum("ti,ti->", dZ, U @ W.T))
        np.add.at(dx, t, dU @ Bt.T)       # B(theta) du
        dphi[e] = butterfly_angle_grad(phi[e], Z, dV)
        # u = B(theta)^T x: <du, dB^T/da x> = <dB/da du, x>
        dtheta[e] = butterfly_angle_grad(theta[e], dU, X[t])
    # router: g = softmax of the selected logits
    dl = g * (dg - np.sum(g * dg, axis=1, keepdims=True))
    dw_gate = np.zeros((N, d))
    dbias = np.zeros(N)
    for jj in range(k):
        np.add.at(dw_gate, idx[:, jj], dl[:, jj][:, None] * X)
        np.add.at(dbias, idx[:, jj], dl[:, jj])
        dx += dl[:, jj][:, None] * np.asarray(w_gate, dtype=np.float64)[idx[:, jj]]
    return {"dx": dx, "dtheta": dtheta, "dphi": dphi, "dw_base": dW, "dalpha": dalpha,
            "dw_gate": dw_gate, "dbias": dbias if bias is not None else None,
            "idx": idx, "gates": g}
