"""Shared test helpers: small networks from layer lists, exact ranges on 2-D inputs,
uniform/vertex sampling of an L-inf box, and the LP relaxation used as an outside pin.

None of this is product code and none of it is oracle arithmetic: the exact-range
enumerator and the LP solve a *different* problem (the true range, the triangle
relaxation) that the oracle's bounds must enclose.
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np

from linear_bound_propagation_b200.synth import Node, INPUT, DENSE, RELU

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def net_from_layers(layers):
    """Dense ReLU network from [{"W": ..., "b": ...}, ...]; ReLU between consecutive layers."""
    W0 = np.asarray(layers[0]["W"], np.float32)
    net = [Node(INPUT, shape=(W0.shape[1],))]
    for i, L in enumerate(layers):
        net.append(Node(DENSE, src=len(net) - 1, W=np.asarray(L["W"], np.float32),
                        b=np.asarray(L["b"], np.float32)))
        if i + 1 < len(layers):
            net.append(Node(RELU, src=len(net) - 1))
    return net


def load_hand_examples():
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        return json.load(f)["examples"]


def relu_ids(net):
    return [v for v, nd in enumerate(net) if nd.op == "relu"]


def box_samples(centre, eps, n_uniform, n_vertex, rng):
    centre = np.asarray(centre, np.float64)
    d = centre.shape[0]
    U = centre + eps * (2.0 * rng.random((n_uniform, d)) - 1.0)
    V = centre + eps * rng.choice([-1.0, 1.0], size=(n_vertex, d))
    return np.concatenate([U, V])


def exact_range_2d(layers, C, centre, eps):
    """True min and max of C f(x) over a 2-D box for a dense ReLU net, by enumerating
    every activation pattern: on each pattern's region (box ∩ sign half-planes, a convex
    polygon) f is affine, so its extremes sit at polygon vertices, found here as all
    pairwise intersections of constraint lines that satisfy every constraint."""
    Ws = [np.asarray(L["W"], np.float64) for L in layers]
    bs = [np.asarray(L["b"], np.float64) for L in layers]
    C = np.asarray(C, np.float64)
    c = np.asarray(centre, np.float64)
    hidden = [W.shape[0] for W in Ws[:-1]]
    lines0 = [(np.array([1.0, 0.0]), -(c[0] - eps), 1), (np.array([1.0, 0.0]), -(c[0] + eps), -1),
              (np.array([0.0, 1.0]), -(c[1] - eps), 1), (np.array([0.0, 1.0]), -(c[1] + eps), -1)]
    lo = np.full(C.shape[0], np.inf)
    hi = np.full(C.shape[0], -np.inf)
    for pattern in itertools.product([0, 1], repeat=sum(hidden)):
        cons = list(lines0)  # (a, b0, sign): sign * (a.x + b0) >= 0
        A = np.eye(2)
        a0 = np.zeros(2)
        pos = 0
        for li, n in enumerate(hidden):
            Z = Ws[li] @ A
            z0 = Ws[li] @ a0 + bs[li]
            s = np.array(pattern[pos:pos + n], np.float64)
            pos += n
            for j in range(n):
                cons.append((Z[j], z0[j], 1 if s[j] else -1))
            A = s[:, None] * Z
            a0 = s * z0
        Aout = C @ (Ws[-1] @ A)
        aout = C @ (Ws[-1] @ a0 + bs[-1])
        verts = []
        for (p, q) in itertools.combinations(range(len(cons)), 2):
            M = np.stack([cons[p][0], cons[q][0]])
            if abs(np.linalg.det(M)) < 1e-12:
                continue
            x = np.linalg.solve(M, -np.array([cons[p][1], cons[q][1]]))
            if all(sg * (a @ x + b0) >= -1e-9 for (a, b0, sg) in cons):
                verts.append(x)
        if not verts:
            continue
        vals = np.stack([Aout @ x + aout for x in verts])
        lo = np.minimum(lo, vals.min(axis=0))
        hi = np.maximum(hi, vals.max(axis=0))
    return lo, hi


def triangle_lp_min(layers, crow, centre, eps, l1, u1):
    """Minimum of crow . f(x) for a one-hidden-layer net under the triangle (Planet)
    relaxation of each ReLU, by scipy's LP solver. Variables: x (d), z (n), h (n)."""
    from scipy.optimize import linprog
    W1 = np.asarray(layers[0]["W"], np.float64)
    b1 = np.asarray(layers[0]["b"], np.float64)
    W2 = np.asarray(layers[1]["W"], np.float64)
    b2 = np.asarray(layers[1]["b"], np.float64)
    n, d = W1.shape
    nv = d + 2 * n
    cobj = np.zeros(nv)
    cobj[d + n:] = crow @ W2
    Aeq = np.zeros((n, nv))
    beq = np.zeros(n)
    Aeq[:, :d] = W1
    Aeq[:, d:d + n] = -np.eye(n)
    beq[:] = -b1
    Aub, bub = [], []
    for j in range(n):
        lj, uj = l1[j], u1[j]
        zj, hj = d + j, d + n + j
        if uj <= 0:
            r = np.zeros(nv); r[hj] = 1; Aub.append(r); bub.append(0.0)
            r = np.zeros(nv); r[hj] = -1; Aub.append(r); bub.append(0.0)
        elif lj >= 0:
            r = np.zeros(nv); r[hj] = 1; r[zj] = -1; Aub.append(r); bub.append(0.0)
            r = np.zeros(nv); r[hj] = -1; r[zj] = 1; Aub.append(r); bub.append(0.0)
        else:
            r = np.zeros(nv); r[hj] = -1; Aub.append(r); bub.append(0.0)          # h >= 0
            r = np.zeros(nv); r[hj] = -1; r[zj] = 1; Aub.append(r); bub.append(0.0)  # h >= z
            s = uj / (uj - lj)
            r = np.zeros(nv); r[hj] = 1; r[zj] = -s; Aub.append(r); bub.append(-s * lj)  # h <= s z - s l
    bounds = [(centre[i] - eps, centre[i] + eps) for i in range(d)] + [(None, None)] * (2 * n)
    res = linprog(cobj, A_ub=np.array(Aub), b_ub=np.array(bub), A_eq=Aeq, b_eq=beq, bounds=bounds,
                  method="highs")
    assert res.status == 0, res.message
    return res.fun + crow @ b2
