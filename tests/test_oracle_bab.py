"""Pins for the oracle's split constraints, beta multipliers and branch-and-bound search, against things
other than the oracle itself:

* soundness on the subdomain: sampled inputs that satisfy the splits stay inside every bound;
* closed form: with every hidden neuron of a one-hidden-layer net split, the network is one affine map
  and the CROWN bound is its exact minimum over the box;
* LP duality (scipy's linprog): any beta >= 0 gives a bound below the minimum over the split region
  (weak duality), and optimised multipliers reach it (strong duality of the linear program);
* central differences for the beta gradient, on a dense chain and on a residual graph;
* exact ranges of 2-D nets: the search never verifies a false property and verifies true ones;
* planted mistakes in the new code, each caught by one of the checks above.
"""
from __future__ import annotations

import inspect
import itertools
import textwrap

import numpy as np
import pytest

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._helpers import box_samples, exact_range_2d, net_from_layers, relu_ids
from tests._random_nets import random_mlp, random_net


def _signs_at(net, x, frac, rng):
    """Split signs for a random `frac` of every ReLU's neurons, each taken from z at the input x (so the
    subdomain holds x and is not empty)."""
    outs = O.forward(net, np.asarray(x, np.float64)[None, :])
    sp = {}
    for k in relu_ids(net):
        z = outs[net[k].src][0]
        pick = rng.random(z.size) < frac
        sp[k] = np.where(pick, np.where(z >= 0.0, 1, -1), 0).astype(np.int8)
    return sp


def _small_nets(rng):
    return [
        (synth.mlp([5, 10, 10, 4], rng), 0.15),
        (synth.cnn_cfg3(rng, image=(2, 8, 8), c1=3, c2=3, hidden=8, classes=3), 0.08),
        (synth.resnet_cfg4(rng, image=(2, 8, 8), widths=(2, 3, 3), fc=6, classes=3), 0.05),
    ]


def check_split_subdomain_sound(seed=20):
    rng = np.random.default_rng(seed)
    for i, (net, eps) in enumerate(_small_nets(rng)):
        n0 = int(np.prod(net[0].shape))
        classes = int(net[-1].W.shape[0])
        c = rng.random(n0).astype(np.float32)
        x0 = c + eps * (2 * rng.random(n0) - 1)
        sp = _signs_at(net, x0, 0.3, rng)
        C = synth.margin_spec(np.array([0]), classes)
        res = O.verify(net, c[None], eps, C, both_sides=True, splits={k: s[None] for k, s in sp.items()})
        xs = np.concatenate([box_samples(c, eps, 20000, 2000, rng), x0[None, :]])
        outs = O.forward(net, xs)
        keep = np.ones(xs.shape[0], bool)
        for k, s in sp.items():
            z = outs[net[k].src]
            keep &= np.all((s[None, :] == 0) | (s[None, :] * z >= 0.0), axis=1)
        if keep.sum() < 1:
            return False, f"net {i}: no sample inside the subdomain"
        y = outs[-1][keep] @ C[0].astype(np.float64).T
        tol = 1e-9 * (1 + np.abs(y).max())
        if np.any(y < res.lb[0] - tol) or np.any(y > res.ub[0] + tol):
            return False, f"net {i}: spec bound violated inside the subdomain"
        for k in relu_ids(net):
            z = outs[net[k].src][keep]
            l, u = res.pre_bounds[k]
            if np.any(z < l[0] - tol) or np.any(z > u[0] + tol):
                return False, f"net {i}: bound of relu {k} violated inside the subdomain"
        if not any(np.any(s != 0) for s in sp.values()):
            return False, "no split drawn"
    return True, ""


def _one_hidden(rng, d, n, k):
    layers = [{"W": rng.standard_normal((n, d)).astype(np.float32), "b": (0.3 * rng.standard_normal(n)).astype(np.float32)},
              {"W": rng.standard_normal((k, n)).astype(np.float32), "b": (0.3 * rng.standard_normal(k)).astype(np.float32)}]
    return layers, net_from_layers(layers)


def check_full_split_closed_form(seed=21):
    rng = np.random.default_rng(seed)
    for trial in range(4):
        layers, net = _one_hidden(rng, 6, 8, 3)
        c = rng.random(6).astype(np.float32)
        eps = float(np.float32(0.4))
        x0 = c + eps * (2 * rng.random(6) - 1)
        sp = _signs_at(net, x0, 1.0, rng)
        k = relu_ids(net)[0]
        Cm = rng.standard_normal((3, 3)).astype(np.float32)
        res = O.verify(net, c[None], eps, Cm[None], splits={k: sp[k][None]})
        W1, b1 = layers[0]["W"].astype(np.float64), layers[0]["b"].astype(np.float64)
        W2, b2 = layers[1]["W"].astype(np.float64), layers[1]["b"].astype(np.float64)
        D = np.diag((sp[k] > 0).astype(np.float64))
        A = Cm.astype(np.float64) @ W2 @ D @ W1
        a0 = Cm.astype(np.float64) @ (W2 @ D @ b1 + b2)
        exact = A @ c.astype(np.float64) - np.float64(np.float32(eps)) * np.abs(A).sum(axis=1) + a0
        if not np.allclose(res.lb_crown[0], exact, rtol=0, atol=1e-9):
            return False, f"trial {trial}: full-split bound {res.lb_crown[0]} != affine minimum {exact}"
    return True, ""


def _region_lp_min(layers, crow, c, eps, sp):
    """min crow . f(x) over {x in the box, s_j z_j(x) >= 0} for a fully split one-hidden-layer net (f is
    affine there), by scipy's LP solver."""
    from scipy.optimize import linprog
    W1, b1 = layers[0]["W"].astype(np.float64), layers[0]["b"].astype(np.float64)
    W2, b2 = layers[1]["W"].astype(np.float64), layers[1]["b"].astype(np.float64)
    D = np.diag((sp > 0).astype(np.float64))
    a = crow @ W2 @ D @ W1
    a0 = crow @ (W2 @ D @ b1 + b2)
    s = sp.astype(np.float64)
    A_ub = -(s[:, None] * W1)  # s_j (W1 x + b1)_j >= 0
    b_ub = s * b1
    e = np.float64(np.float32(eps))
    r = linprog(a, A_ub=A_ub, b_ub=b_ub, bounds=[(ci - e, ci + e) for ci in c.astype(np.float64)], method="highs")
    assert r.status == 0
    return r.fun + a0


def check_beta_duality_lp(seed=22):
    rng = np.random.default_rng(seed)
    gaps = []
    for trial in range(3):
        layers, net = _one_hidden(rng, 4, 7, 2)
        c = rng.random(4).astype(np.float32)
        eps = 0.5
        x0 = c + eps * (2 * rng.random(4) - 1)
        sp = _signs_at(net, x0, 1.0, rng)
        k = relu_ids(net)[0]
        crow = np.array([[1.0, -1.0]], np.float32)
        lp = _region_lp_min(layers, crow[0].astype(np.float64), c, eps, sp[k])
        res = O.verify(net, c[None], eps, crow[None], splits={k: sp[k][None]})
        relax = {k: O.relax_params(res.pre_bounds[k][0][0], res.pre_bounds[k][1][0])}
        for _ in range(20):  # weak duality at random multipliers
            beta = {k: rng.exponential(1.0, (1, sp[k].size))}
            lb = O.spec_bound_alpha(net, c, eps, crow, relax, {k: np.zeros((1, sp[k].size))}, sp, beta)[0][0]
            if lb > lp + 1e-9 * (1 + abs(lp)):
                return False, f"trial {trial}: bound {lb} above the region minimum {lp} at beta >= 0"
        best = O.alpha_crown(net, c[None], eps, crow[None], iters=300, lr=0.05, splits={k: sp[k][None]})[0][0, 0]
        if best > lp + 1e-9 * (1 + abs(lp)):
            return False, f"trial {trial}: optimised bound {best} above the region minimum {lp}"
        gaps.append(lp - best)
        if lp - best > 5e-3 * (1 + abs(lp)):
            return False, f"trial {trial}: optimised multipliers stop {lp - best:.4g} below the region minimum"
    return True, gaps


def _fd_beta(net, c, eps, C, relax, a, sp, beta, pairs, h=1e-6):
    lb, g, gb = O.spec_bound_alpha(net, c, eps, C, relax, a, sp, beta)
    for k, r, i in pairs:
        bp = {kk: v.copy() for kk, v in beta.items()}
        bm = {kk: v.copy() for kk, v in beta.items()}
        bp[k][r, i] += h
        bm[k][r, i] -= h
        fd = (O.spec_bound_alpha(net, c, eps, C, relax, a, sp, bp)[0][r] -
              O.spec_bound_alpha(net, c, eps, C, relax, a, sp, bm)[0][r]) / (2 * h)
        if abs(fd - gb[k][r, i]) > 1e-6 * (1 + abs(fd)):
            return False, f"beta gradient mismatch relu {k} row {r} neuron {i}: {gb[k][r, i]} vs {fd}"
    for k in sp:
        if np.any(gb[k][:, sp[k] == 0] != 0.0):
            return False, "nonzero beta gradient on a free neuron"
    return True, ""


def check_beta_fd_gradient(seed=23):
    rng = np.random.default_rng(seed)
    cases = [(synth.mlp([6, 9, 8, 4], rng), (1, 6), 0.2),
             (synth.resnet_cfg4(rng, image=(2, 8, 8), widths=(2, 3, 3), fc=5, classes=3), (1, 128), 0.05)]
    for net, shape, eps in cases:
        c = rng.random(shape[1]).astype(np.float64).astype(np.float32)
        x0 = c + eps * (2 * rng.random(shape[1]) - 1)
        sp = _signs_at(net, x0, 0.4, rng)
        classes = int(net[-1].W.shape[0])
        C = synth.margin_spec(np.array([0]), classes)
        res = O.verify(net, c[None], eps, C, splits={k: s[None] for k, s in sp.items()})
        relax = {k: O.relax_params(res.pre_bounds[k][0][0], res.pre_bounds[k][1][0]) for k in relu_ids(net)}
        R = C.shape[1]
        a = {k: rng.random((R, relax[k][0].size)) for k in relax}
        beta = {k: rng.exponential(0.5, (R, sp[k].size)) for k in sp}
        pairs = [(k, r, i) for k in sp for i in np.nonzero(sp[k])[0][:6] for r in range(R)]
        if len(pairs) < 6:
            return False, "too few split neurons for the check to mean anything"
        ok, det = _fd_beta(net, c, eps, C[0], relax, a, sp, beta, pairs)
        if not ok:
            return False, det
    return True, ""


def check_bab_exact_2d(seed=24):
    """Random 2-w-w-3 nets (w = 3, 4), margin rows of the centre's class, each at the first radius whose
    plain bound over the whole box is not positive: the search says "verified" only when the exact
    minimum is > 0 and "falsified" only when it is < 0, and at least once it verifies by splitting. (It
    need not settle every true property: with a fixed number of ascent steps per subdomain, a subdomain
    with no unstable neuron left can stay below its exact minimum, which ends the search "unknown"; the
    duality check pins the limit.)"""
    rng = np.random.default_rng(seed)
    split_wins = 0
    for trial in range(16):
        w = 3 + trial % 2
        dims = [2, w, w, 3]
        layers = [{"W": (rng.standard_normal((dims[i + 1], dims[i])) * 0.8).astype(np.float32),
                   "b": (rng.standard_normal(dims[i + 1]) * 0.3).astype(np.float32)} for i in range(3)]
        net = net_from_layers(layers)
        c = rng.random(2).astype(np.float32)
        y = O.forward(net, c[None].astype(np.float64))[-1][0]
        C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
        for eps in (0.15, 0.2, 0.3, 0.4):
            eps = float(np.float32(eps))
            if O.verify(net, c[None], eps, C[None]).lb.min() <= 0.0:
                break
        lo, _ = exact_range_2d(layers, C, c, eps)
        r = O.bab(net, c, eps, C, max_domains=400, batch=16, iters=40, lr=0.1)
        if r.status == "verified" and lo.min() <= 0.0:
            return False, f"trial {trial}: verified a property whose exact minimum is {lo.min()}"
        if r.status == "falsified" and lo.min() >= 0.0:
            return False, f"trial {trial}: falsified a property whose exact minimum is {lo.min()}"
        if r.status == "verified" and r.domains > 1:
            split_wins += 1
    if split_wins < 1:
        return False, "no property needed splitting"
    return True, ""


def check_bab_sampled(seed=0):
    """4-10-10-3 nets at three radii: whenever the search says "verified", no sampled input of the box
    has a negative row; at least one property is verified only after splitting."""
    rng = np.random.default_rng(seed)
    wins = 0
    for t in range(4):
        net = synth.mlp([4, 10, 10, 3], rng)
        c = rng.random(4).astype(np.float32)
        y = O.forward(net, c[None].astype(np.float64))[-1][0]
        C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
        for eps in (0.1, 0.2, 0.3):
            eps = float(np.float32(eps))
            r = O.bab(net, c, eps, C, max_domains=200, batch=16, iters=20, lr=0.1)
            if r.status == "verified":
                xs = box_samples(c, eps, 20000, 2000, np.random.default_rng(t))
                if (O.forward(net, xs)[-1] @ C.astype(np.float64).T).min() <= 0.0:
                    return False, f"net {t} eps {eps}: verified but a sample is negative"
                wins += r.domains > 1
    if wins < 1:
        return False, "no property needed splitting"
    return True, ""


def check_minimiser_vertex(seed=25):
    """4-8-8-3 nets at three radii, every margin row: the vertex x*_r lies in the box, the row's linear lower
    bound lam_r . x + const_r takes there its minimum over all 16 vertices of the box (brute force), that
    minimum is the CROWN bound ``verify`` reports, and the row's exact value at x*_r is not below it."""
    rng = np.random.default_rng(seed)
    for t in range(6):
        net = synth.mlp([4, 8, 8, 3], rng)
        c = rng.random(4).astype(np.float32)
        y = O.forward(net, c[None].astype(np.float64))[-1][0]
        C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
        for eps in (0.05, 0.2, 0.5):
            eps = float(np.float32(eps))
            _, lam, cst, xs = O.minimiser_vertices(net, c, eps, C)
            crown = O.verify(net, c[None], eps, C[None]).lb_crown[0]
            cen = c.astype(np.float64)
            V = np.array(list(itertools.product(*[(ci - eps, ci + eps) for ci in cen])))
            brute = (V @ lam.T + cst[None, :]).min(axis=0)
            at = np.einsum("ri,ri->r", lam, xs) + cst
            val = np.einsum("ri,ri->r", O.forward(net, xs)[-1], C.astype(np.float64))
            tol = 1e-12 * (1 + np.abs(brute))
            if np.abs(xs - cen[None, :]).max() > eps * (1 + 1e-15):
                return False, f"net {t} eps {eps}: a vertex outside the box"
            if np.any(np.abs(at - brute) > tol) or np.any(np.abs(at - crown) > tol):
                return False, f"net {t} eps {eps}: vertex value {at} vs brute force {brute} vs CROWN {crown}"
            if np.any(val < at - tol):
                return False, f"net {t} eps {eps}: the linear bound exceeds the row at its vertex"
    return True, ""


def check_attack_exact_2d(seed=26):
    """Random 2-w-w-3 nets, margin rows of the centre's class, radii 0.1-0.8, the search given one subdomain
    (so only the centre and the vertices can decide): it says "falsified" only when the exact minimum over the
    box (enumerated activation regions) is < 0, and does so for at least 3/4 of the properties whose exact
    minimum is below -0.02 (the vertex is a heuristic; 34 of 38 here)."""
    rng = np.random.default_rng(seed)
    hits = false_props = 0
    for trial in range(40):
        w = 3 + trial % 2
        dims = [2, w, w, 3]
        layers = [{"W": (rng.standard_normal((dims[i + 1], dims[i])) * 0.8).astype(np.float32),
                   "b": (rng.standard_normal(dims[i + 1]) * 0.3).astype(np.float32)} for i in range(3)]
        net = net_from_layers(layers)
        c = rng.random(2).astype(np.float32)
        y = O.forward(net, c[None].astype(np.float64))[-1][0]
        C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
        for eps in (0.1, 0.2, 0.4, 0.8):
            eps = float(np.float32(eps))
            lo, _ = exact_range_2d(layers, C, c, eps)
            r = O.bab(net, c, eps, C, max_domains=1, batch=2, iters=0)
            if r.status == "falsified" and lo.min() >= 0.0:
                return False, f"trial {trial} eps {eps}: falsified a property whose exact minimum is {lo.min()}"
            if lo.min() < -0.02:
                false_props += 1
                hits += r.status == "falsified" and r.domains == 0
    if hits * 4 < false_props * 3:
        return False, f"only {hits} of {false_props} false properties falsified without splitting"
    return True, ""


CHECKS = [check_split_subdomain_sound, check_full_split_closed_form, check_beta_duality_lp,
          check_beta_fd_gradient, check_bab_exact_2d, check_bab_sampled, check_minimiser_vertex,
          check_attack_exact_2d]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_bab_pin(check):
    ok, detail = check()
    assert ok, detail


MUTATIONS = [
    ("spec_bound_alpha", "lam_z = lam_z - np.asarray(beta_rows[v], F)", "lam_z = lam_z + np.asarray(beta_rows[v], F)",
     check_beta_duality_lp),
    ("spec_bound_alpha", "bgrads[v] = -Gz * sg[None, :]", "bgrads[v] = Gz * sg[None, :]", check_beta_fd_gradient),
    ("split_clamp", "np.where(s > 0, np.maximum(l, 0.0), l)", "np.where(s > 0, np.minimum(l, 0.0), l)",
     check_full_split_closed_form),
    ("split_clamp", "np.where(s < 0, np.minimum(u, 0.0), u)", "np.where(s < 0, np.maximum(u, 0.0), u)",
     check_full_split_closed_form),
    ("ascend", "beta[k] = np.maximum(x, 0.0)", "beta[k] = x", check_beta_duality_lp),
    ("verify", "split_clamp(*ibp_b[net[k].src], splits.get(k))", "split_clamp(*ibp_b[net[k].src], None)",
     check_full_split_closed_form),
    ("minimiser_vertices", "centre[None, :] - F(eps) * np.sign(lam_in)", "centre[None, :] + F(eps) * np.sign(lam_in)",
     check_minimiser_vertex),
    ("minimiser_vertices", "centre[None, :] - F(eps) * np.sign(lam_in)", "centre[None, :] - F(eps) * lam_in",
     check_minimiser_vertex),
    ("minimiser_vertices", "backward(net, len(net) - 1, C, relax)", "backward(net, len(net) - 1, -C, relax)",
     check_minimiser_vertex),
    ("minimiser_attack", "forward(net, xs)[-1] @ np.asarray(C, F).T", "forward(net, xs)[-1] @ np.asarray(-C, F).T",
     check_attack_exact_2d),
    ("bab", "if ya.size and np.any(ya < 0.0):", "if ya.size and np.all(ya < 0.0):", check_attack_exact_2d),
]


@pytest.mark.parametrize("fname,old,new,check", MUTATIONS, ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTATIONS)])
def test_split_mutation_is_caught(monkeypatch, fname, old, new, check):
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


def test_every_subdomain_bound_takes_the_requested_ascent_steps(monkeypatch):
    """Regression: the search's bound for every subdomain, the whole box and every child alike, runs
    alpha_crown with the requested number of Adam steps (a loop counter once shadowed it)."""
    seen = []
    real = O.alpha_crown

    def spy(*a, **kw):
        seen.append(kw.get("iters"))
        return real(*a, **kw)

    monkeypatch.setattr(O, "alpha_crown", spy)
    rng = np.random.default_rng(3)
    net = synth.mlp([4, 10, 10, 3], rng)
    c = rng.random(4).astype(np.float32)
    y = O.forward(net, c[None].astype(np.float64))[-1][0]
    C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
    r = O.bab(net, c, float(np.float32(0.3)), C, max_domains=40, batch=8, iters=7, lr=0.1)
    assert r.iterations >= 2 and len(seen) == r.iterations + 1
    assert set(seen) == {7}


@pytest.mark.parametrize("seed", list(range(12)))
def test_split_bounds_sound_on_random_architectures(seed):
    """Subdomain soundness of split-constrained bounds (both sides, every intermediate bound) on the random
    CNN / residual / dense networks of the GPU fuzz suite: every sampled input that satisfies the splits
    stays inside every bound."""
    net = random_net(seed)[0] if seed % 2 == 0 else random_mlp(seed)[0]
    rng = np.random.default_rng(60_000 + seed)
    n0 = int(np.prod(net[0].shape))
    classes = int(net[-1].W.shape[0])
    eps = float(np.float32(rng.choice([0.01, 0.05])))
    c = rng.random(n0).astype(np.float32)
    x0 = c + eps * (2 * rng.random(n0) - 1)
    sp = _signs_at(net, x0, 0.3, rng)
    C = synth.margin_spec(np.array([int(rng.integers(0, classes))]), classes)
    res = O.verify(net, c[None], eps, C, both_sides=True, splits={k: s[None] for k, s in sp.items()})
    xs = np.concatenate([box_samples(c, eps, 3000, 300, rng), x0[None, :]])
    outs = O.forward(net, xs)
    keep = np.ones(xs.shape[0], bool)
    for k, s in sp.items():
        keep &= np.all((s[None, :] == 0) | (s[None, :] * outs[net[k].src] >= 0.0), axis=1)
    assert keep[-1], "the point the splits were taken from lies in the subdomain"
    y = outs[-1][keep] @ C[0].astype(np.float64).T
    tol = 1e-9 * (1 + np.abs(y).max())
    assert np.all(y >= res.lb[0] - tol) and np.all(y <= res.ub[0] + tol)
    for k in relu_ids(net):
        z = outs[net[k].src][keep]
        l, u = res.pre_bounds[k]
        assert np.all(z >= l[0] - tol) and np.all(z <= u[0] + tol), f"relu {k}"


@pytest.mark.parametrize("seed", list(range(6)))
def test_beta_gradient_central_differences_on_random_architectures(seed):
    """d lb / d beta against central differences on random CNN / residual / dense networks, for a seeded
    sample of (row, split neuron) pairs of every ReLU layer with splits."""
    net = random_net(seed)[0] if seed % 2 == 0 else random_mlp(seed)[0]
    rng = np.random.default_rng(70_000 + seed)
    n0 = int(np.prod(net[0].shape))
    classes = int(net[-1].W.shape[0])
    eps = float(np.float32(0.03))
    c = rng.random(n0).astype(np.float32)
    x0 = c + eps * (2 * rng.random(n0) - 1)
    sp = _signs_at(net, x0, 0.4, rng)
    C = synth.margin_spec(np.array([int(rng.integers(0, classes))]), classes)
    res = O.verify(net, c[None], eps, C, splits={k: s[None] for k, s in sp.items()})
    relax = {k: O.relax_params(res.pre_bounds[k][0][0], res.pre_bounds[k][1][0]) for k in relu_ids(net)}
    R = C.shape[1]
    a = {k: rng.random((R, relax[k][0].size)) for k in relax}
    beta = {k: rng.exponential(0.5, (R, sp[k].size)) for k in sp}
    pairs = [(k, int(r), int(i)) for k in sp for i in rng.permutation(np.nonzero(sp[k])[0])[:4]
             for r in rng.permutation(R)[:2]]
    if not pairs:
        pytest.skip("no split neuron drawn")
    ok, det = _fd_beta(net, c, eps, C[0], relax, a, sp, beta, pairs)
    assert ok, det


def _small_props():
    rng = np.random.default_rng(0)
    out = []
    for t in range(24):
        net = synth.mlp([4, 10, 10, 3], rng)
        c = rng.random(4).astype(np.float32)
        y = O.forward(net, c[None].astype(np.float64))[-1][0]
        C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
        for eps in (0.1, 0.2, 0.3):
            out.append((net, c, float(np.float32(eps)), C))
    return out


def check_warm_start_settles_more():
    """72 properties of 4-10-10-3 nets, 3 ascent steps per subdomain, 200 subdomains: children that start from
    their parent's slopes and multipliers settle more properties than children that start afresh (36 against 31
    verified), and every "verified" of either holds on sampled inputs (sound whatever the start)."""
    counts = {}
    for warm in (False, True):
        n = 0
        for net, c, eps, C in _small_props():
            r = O.bab(net, c, eps, C, max_domains=200, batch=8, iters=3, lr=0.1, warm_start=warm)
            if r.status == "verified":
                n += 1
                xs = box_samples(c, eps, 4000, 400, np.random.default_rng(1))
                if (O.forward(net, xs)[-1] @ C.astype(np.float64).T).min() <= 0.0:
                    return False, f"warm={warm}: verified a property with a negative sample"
        counts[warm] = n
    if counts[True] < counts[False] + 3:
        return False, f"warm start verified {counts[True]}, cold {counts[False]}"
    return True, counts


def test_warm_start_settles_more():
    ok, detail = check_warm_start_settles_more()
    assert ok, detail


@pytest.mark.parametrize("old,new", [
    ("starts = [saved.get(key[:-1]) if warm_start and key else None for key in keys]",
     "starts = [saved.get(key) if warm_start and key else None for key in keys]"),
    ("saved[key] = st", "saved[key] = (st[0], None)"),
])
def test_warm_start_mutation_is_caught(monkeypatch, old, new):
    src = textwrap.dedent(inspect.getsource(O.bab))
    assert src.count(old) == 1
    ns = {}
    exec(compile(src.replace(old, new), "<mutant bab>", "exec"), O.__dict__, ns)
    monkeypatch.setattr(O, "bab", ns["bab"])
    ok, _ = check_warm_start_settles_more()
    assert not ok
