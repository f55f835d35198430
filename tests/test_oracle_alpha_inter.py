"""Pins of the oracle's alpha-CROWN for intermediate bounds (``verify(..., alpha_inter_iters=...)``, the per-neuron
alpha tensors of [SNNV §3, §4.3] applied to the intermediate passes) against what the mathematics fixes:

* a one-neuron closed form for the ascent itself: the lower bound of relu(z) over z in [l, u] is 0, which the
  adaptive slope (1 when u >= -l) misses and the ascent reaches once Adam has driven the slope to 0;
* the triangle LP: with one hidden layer before the bounded node, a lower bound from any slopes in [0, 1] is at
  most the minimum of the triangle relaxation's LP (scipy), and the optimised slopes reach it (the relaxation's
  dual is the slope choice);
* soundness: every refined bound holds on sampled inputs, and the refined bounds are never looser than the
  plain ones;
* zero steps change nothing, bit for bit.

Each planted mistake at the end must be caught by one of these checks."""
from __future__ import annotations

import inspect
import textwrap

import numpy as np
import pytest

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._helpers import box_samples, net_from_layers, relu_ids


def _chain(weights, biases):
    return net_from_layers([{"W": np.asarray(w, np.float32), "b": np.asarray(b, np.float32)}
                            for w, b in zip(weights, biases)])


def check_one_neuron_closed_form():
    """x in [c - eps, c + eps], z1 = x, z2 = w relu(z1) + b. Over the box z2 lies exactly in b + w * [0, u1]
    (w > 0) or b + w * [u1, 0] (w < 0), with u1 = c + eps > 0 > l1 = c - eps and u1 >= -l1. The bound of the rows
    [1; -1] over z2 with the relaxation of [l1, u1]: the side where the lower slope enters starts, at the adaptive
    slope 1, at b + w l1 (or b - |w| l1 for the upper side) and 20 Adam steps of 0.1 drive the slope to 0 and reach
    the exact value; the other side is exact from the start (``ascend`` on the network up to z2)."""
    for c, eps, w, b in ((0.1, 0.5, 2.0, 0.3), (0.1, 0.5, -1.5, 1.0), (0.05, 0.25, 0.75, -0.2)):
        net = _chain([[[1.0]], [[w]], [[1.0]]], [[0.0], [b], [0.0]])
        sub = net[:relu_ids(net)[1]]
        e = np.float64(np.float32(eps))
        cf = np.float64(np.float32(c))
        l1, u1 = np.array([cf - e]), np.array([cf + e])
        relax = {relu_ids(net)[0]: O.relax_params(l1, u1)}
        rows = np.array([[1.0], [-1.0]])
        best, start = O.ascend(sub, np.array([c], np.float32), float(np.float32(eps)), rows, relax, 20, 0.1)
        wf, bf = np.float64(np.float32(w)), np.float64(np.float32(b))
        lo, hi = (bf, bf + wf * u1[0]) if w > 0 else (bf + wf * u1[0], bf)
        if abs(best[0] - lo) > 1e-12 or abs(-best[1] - hi) > 1e-12:
            return False, f"w={w}: optimised [{best[0]}, {-best[1]}] vs exact [{lo}, {hi}]"
        loose = start[0] if w > 0 else -start[1]
        if abs(loose - (bf + abs(wf) * l1[0] * (1 if w > 0 else -1))) > 1e-12:
            return False, f"w={w}: start {loose} is not the adaptive slope's bound"
    return True, ""


def _triangle_lp(W1, b1, c, eps, l1, u1, row, sign):
    """min sign * (row . h) over x in the box, z = W1 x + b1, h in the triangle relaxation of ReLU on [l1, u1]."""
    from scipy.optimize import linprog
    d, n = W1.shape[1], W1.shape[0]
    # variables [x (d), h (n)]; z is substituted
    cost = np.concatenate([np.zeros(d), sign * row])
    A, bb = [], []
    for j in range(n):
        wj, bj = W1[j], b1[j]
        if u1[j] <= 0.0:  # h = 0
            A.append(np.concatenate([np.zeros(d), np.eye(n)[j]]))
            bb.append(0.0)
            A.append(np.concatenate([np.zeros(d), -np.eye(n)[j]]))
            bb.append(0.0)
            continue
        # h >= 0 and h >= z
        A.append(np.concatenate([np.zeros(d), -np.eye(n)[j]]))
        bb.append(0.0)
        A.append(np.concatenate([wj, -np.eye(n)[j]]))
        bb.append(-bj)
        if l1[j] >= 0.0:  # h <= z
            A.append(np.concatenate([-wj, np.eye(n)[j]]))
            bb.append(bj)
        else:  # h <= u (z - l) / (u - l)
            s = u1[j] / (u1[j] - l1[j])
            A.append(np.concatenate([-s * wj, np.eye(n)[j]]))
            bb.append(s * (bj - l1[j]))
    bounds = [(ci - eps, ci + eps) for ci in c] + [(None, None)] * n
    r = linprog(cost, A_ub=np.array(A), b_ub=np.array(bb), bounds=bounds, method="highs")
    assert r.status == 0
    return sign * r.fun


def check_triangle_lp(seed=31):
    """4-8-6-2 nets: for every neuron of the second affine node still unstable after the plain pass, the
    refined bounds lie inside the triangle LP's range (sound against it) and within 5e-3 of it after 300 steps
    of 0.05."""
    rng = np.random.default_rng(seed)
    gaps, n_checked = [], 0
    for trial in range(4):
        W1 = (rng.standard_normal((8, 4)) * 0.7).astype(np.float32)
        b1 = (rng.standard_normal(8) * 0.2).astype(np.float32)
        W2 = (rng.standard_normal((6, 8)) * 0.7).astype(np.float32)
        b2 = (rng.standard_normal(6) * 0.2).astype(np.float32)
        W3 = (rng.standard_normal((2, 6)) * 0.7).astype(np.float32)
        net = _chain([W1, W2, W3], [b1, b2, np.zeros(2, np.float32)])
        c = rng.random(4).astype(np.float32)
        eps = float(np.float32(0.4))
        C = np.ones((1, 1, 2), np.float32)
        k1, k2 = relu_ids(net)
        plain = O.verify(net, c[None], eps, C)
        res = O.verify(net, c[None], eps, C, alpha_inter_iters=300, alpha_inter_lr=0.05)
        l1, u1 = (x[0] for x in res.pre_bounds[k1])  # exact IBP range of the first layer
        pl, pu = (x[0] for x in plain.pre_bounds[k2])
        rl, ru = (x[0] for x in res.pre_bounds[k2])
        W1d, b1d, W2d, b2d = (a.astype(np.float64) for a in (W1, b1, W2, b2))
        cd = c.astype(np.float64)
        for j in np.nonzero((pl < 0.0) & (pu > 0.0))[0]:
            lo = _triangle_lp(W1d, b1d, cd, np.float64(eps), l1, u1, W2d[j], 1.0) + b2d[j]
            hi = _triangle_lp(W1d, b1d, cd, np.float64(eps), l1, u1, W2d[j], -1.0) + b2d[j]
            tol = 1e-9 * (1 + abs(lo) + abs(hi))
            if rl[j] > lo + tol or ru[j] < hi - tol:
                return False, f"trial {trial} neuron {j}: [{rl[j]}, {ru[j]}] inside the LP range [{lo}, {hi}]"
            gaps += [lo - rl[j], ru[j] - hi]
            n_checked += 1
    if n_checked < 4:
        return False, f"only {n_checked} unstable neurons"
    if max(gaps) > 5e-3:
        return False, f"optimised slopes stop {max(gaps):.4g} short of the LP bound"
    return True, gaps


def check_sound_and_tighter(seed=32):
    """Random 5-10-10-10-3 nets: every refined pre-activation bound holds on 10^4 uniform and 10^3 vertex samples,
    the final lower bounds hold too, and no refined bound is looser than the plain one."""
    rng = np.random.default_rng(seed)
    improved = 0
    for trial in range(3):
        net = synth.mlp([5, 10, 10, 10, 3], rng)
        centres = rng.random((2, 5)).astype(np.float32)
        C = synth.margin_spec(np.array([0, 1]), 3)
        eps = float(np.float32(0.2))
        plain = O.verify(net, centres, eps, C)
        res = O.verify(net, centres, eps, C, alpha_inter_iters=8, alpha_inter_lr=0.1)
        for k in relu_ids(net):
            (pl, pu), (rl, ru) = plain.pre_bounds[k], res.pre_bounds[k]
            if np.any(rl < pl) or np.any(ru > pu):
                return False, f"trial {trial} relu {k}: a refined bound is looser than the plain one"
            improved += int(np.sum(rl > pl + 1e-9) + np.sum(ru < pu - 1e-9))
        for b in range(2):
            xs = box_samples(centres[b], eps, 10000, 1000, np.random.default_rng(trial))
            outs = O.forward(net, xs)
            for k in relu_ids(net):
                z = outs[net[k].src]
                l, u = res.pre_bounds[k][0][b], res.pre_bounds[k][1][b]
                if np.any(z < l - 1e-9) or np.any(z > u + 1e-9):
                    return False, f"trial {trial} centre {b} relu {k}: a sample leaves the refined bounds"
            y = outs[-1] @ C[b].astype(np.float64).T
            if np.any(y.min(axis=0) < res.lb[b] - 1e-9):
                return False, f"trial {trial} centre {b}: a sample is below the final bound"
    if improved < 10:
        return False, f"only {improved} bounds tightened"
    return True, ""


def check_zero_steps_is_plain(seed=33):
    rng = np.random.default_rng(seed)
    net = synth.mlp([6, 12, 12, 4], rng)
    centres = rng.random((3, 6)).astype(np.float32)
    C = synth.margin_spec(np.array([0, 1, 2]), 4)
    a = O.verify(net, centres, 0.1, C)
    b = O.verify(net, centres, 0.1, C, alpha_inter_iters=0)
    same = all(np.array_equal(a.pre_bounds[k][i], b.pre_bounds[k][i]) for k in a.pre_bounds for i in (0, 1))
    return (same and np.array_equal(a.lb, b.lb)), "zero steps changed a bound"


CHECKS = [check_one_neuron_closed_form, check_triangle_lp, check_sound_and_tighter, check_zero_steps_is_plain]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_alpha_inter_pin(check):
    ok, detail = check()
    assert ok, detail


MUTATIONS = [
    ("verify", "l1[idx] = np.maximum(l1[idx], best[:m])", "l1[idx] = np.maximum(l1[idx], best[m:])",
     check_sound_and_tighter),
    ("verify", "u1[idx] = np.minimum(u1[idx], -best[m:])", "u1[idx] = np.minimum(u1[idx], best[m:])",
     check_sound_and_tighter),
    ("verify", "np.concatenate([eye[idx], -eye[idx]])", "np.concatenate([eye[idx], eye[idx]])",
     check_sound_and_tighter),
    ("verify", "alpha_inter_iters, alpha_inter_lr, sg)", "0, alpha_inter_lr, sg)", check_triangle_lp),
    ("ascend", "return x + lr * mh / (np.sqrt(vh) + 1e-8), m1, m2", "return x - lr * mh / (np.sqrt(vh) + 1e-8), m1, m2",
     check_one_neuron_closed_form),
    ("verify", "idx = np.nonzero((l1 < 0.0) & (u1 > 0.0))[0]", "idx = np.nonzero((l1 < 0.0) & (u1 > 0.0))[0][:1]",
     check_triangle_lp),
    ("ascend", "alpha[k] = np.clip(a, 0.0, 1.0)", "alpha[k] = np.clip(a, 0.0, 2.0)", check_triangle_lp),
]


@pytest.mark.parametrize("fname,old,new,check", MUTATIONS, ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTATIONS)])
def test_alpha_inter_mutation_is_caught(monkeypatch, fname, old, new, check):
    src = textwrap.dedent(inspect.getsource(getattr(O, fname)))
    assert src.count(old) == 1, f"mutation target not unique in {fname}: {old!r}"
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant {fname}>", "exec"), O.__dict__, ns)
    monkeypatch.setattr(O, fname, ns[fname])
    try:
        ok, _ = check()
    except Exception:
        ok = False
    assert not ok, f"{check.__name__} did not catch {old!r} -> {new!r}"
