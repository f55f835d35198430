"""Pins for the oracle's alpha-CROWN functions: the analytic gradient against central differences,
the hand-derivable optimum of a 1-D example, soundness of optimised bounds, the adaptive start equal to
the CROWN bound, and planted gradient mistakes caught by the finite-difference check."""
import inspect
import textwrap

import numpy as np
import pytest

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._helpers import box_samples, load_hand_examples, net_from_layers, relu_ids


def _setup(seed=0, widths=(6, 9, 8, 4), eps=0.2):
    rng = np.random.default_rng(seed)
    net = synth.mlp(list(widths), rng)
    c = rng.random((1, widths[0])).astype(np.float32)
    C = synth.margin_spec(np.array([1]), widths[-1])
    res = O.verify(net, c, eps, C)
    relax = {k: O.relax_params(res.pre_bounds[k][0][0], res.pre_bounds[k][1][0]) for k in relu_ids(net)}
    return rng, net, c, C, eps, res, relax


def check_fd_gradient(seed=0):
    rng, net, c, C, eps, res, relax = _setup(seed)
    R = C.shape[1]
    a = {k: rng.random((R, relax[k][0].size)) for k in relax}
    lb, g = O.spec_bound_alpha(net, c[0], eps, C[0], relax, a)
    h = 1e-6
    for k in relax:
        unst = (relax[k][1] > 0) & (relax[k][1] < 1)
        for i in range(a[k].shape[1]):
            for r in range(R):
                ap = {kk: v.copy() for kk, v in a.items()}
                am = {kk: v.copy() for kk, v in a.items()}
                ap[k][r, i] += h
                am[k][r, i] -= h
                fd = (O.spec_bound_alpha(net, c[0], eps, C[0], relax, ap)[0][r] -
                      O.spec_bound_alpha(net, c[0], eps, C[0], relax, am)[0][r]) / (2 * h)
                if abs(fd - g[k][r, i]) > 1e-6 * (1 + abs(fd)):
                    return False, f"gradient mismatch relu {k} row {r} neuron {i}: {g[k][r, i]} vs {fd}"
                if not unst[i] and g[k][r, i] != 0.0:
                    return False, "nonzero gradient on a stable neuron"
    return True, ""


def _setup_conv(seed=0, eps=0.15):
    """A small convolutional chain: conv 3x3 s1 p1, ReLU, conv 2x2 s2, ReLU, dense, ReLU, dense."""
    rng = np.random.default_rng(100 + seed)
    net = [synth.Node(synth.INPUT, shape=(2, 6, 6))]
    v = synth._relu(net, synth._conv(net, rng, 0, 2, 3, 3, 1, 1))
    v = synth._relu(net, synth._conv(net, rng, v, 3, 4, 2, 2, 0))
    v = synth._relu(net, synth._dense(net, rng, v, 4 * 3 * 3, 5))
    synth._dense(net, rng, v, 5, 3)
    c = rng.random((1, 2 * 6 * 6)).astype(np.float32)
    C = synth.margin_spec(np.array([0]), 3)
    res = O.verify(net, c, eps, C)
    relax = {k: O.relax_params(res.pre_bounds[k][0][0], res.pre_bounds[k][1][0]) for k in relu_ids(net)}
    return rng, net, c, C, eps, res, relax


def check_fd_gradient_conv(seed=0):
    rng, net, c, C, eps, res, relax = _setup_conv(seed)
    R = C.shape[1]
    a = {k: rng.random((R, relax[k][0].size)) for k in relax}
    lb, g = O.spec_bound_alpha(net, c[0], eps, C[0], relax, a)
    h = 1e-6
    n_checked = 0
    for k in relax:
        unst = (relax[k][1] > 0) & (relax[k][1] < 1)
        for i in range(a[k].shape[1]):
            for r in range(R):
                ap = {kk: v.copy() for kk, v in a.items()}
                am = {kk: v.copy() for kk, v in a.items()}
                ap[k][r, i] += h
                am[k][r, i] -= h
                fd = (O.spec_bound_alpha(net, c[0], eps, C[0], relax, ap)[0][r] -
                      O.spec_bound_alpha(net, c[0], eps, C[0], relax, am)[0][r]) / (2 * h)
                if abs(fd - g[k][r, i]) > 1e-6 * (1 + abs(fd)):
                    return False, f"conv gradient mismatch relu {k} row {r} neuron {i}: {g[k][r, i]} vs {fd}"
                if not unst[i] and g[k][r, i] != 0.0:
                    return False, "nonzero gradient on a stable neuron"
                n_checked += int(unst[i])
    if n_checked < 10:
        return False, "too few unstable neurons for the check to mean anything"
    return True, ""


def _setup_residual(seed=0, eps=0.05):
    rng = np.random.default_rng(200 + seed)
    net = synth.resnet_cfg4(rng, image=(2, 8, 8), widths=(2, 3, 3), fc=4, classes=3)
    c = rng.random((1, 2 * 8 * 8)).astype(np.float32)
    C = synth.margin_spec(np.array([1]), 3)
    res = O.verify(net, c, eps, C)
    relax = {k: O.relax_params(res.pre_bounds[k][0][0], res.pre_bounds[k][1][0]) for k in relu_ids(net)}
    return rng, net, c, C, eps, res, relax


def check_fd_gradient_residual(seed=0, samples=40):
    """Central differences on a residual net (identity and 1x1-convolution shortcuts) for a seeded sample
    of (row, unstable neuron) pairs of every ReLU layer."""
    rng, net, c, C, eps, res, relax = _setup_residual(seed)
    R = C.shape[1]
    a = {k: rng.random((R, relax[k][0].size)) for k in relax}
    lb, g = O.spec_bound_alpha(net, c[0], eps, C[0], relax, a)
    if not np.allclose(O.spec_bound_alpha(net, c[0], eps, C[0], relax,
                                          {k: np.repeat(relax[k][0][None, :], R, axis=0) for k in relax})[0],
                       res.lb_crown[0], rtol=1e-12, atol=1e-12):
        return False, "adaptive slopes do not reproduce the CROWN bound on a residual net"
    h = 1e-6
    n_checked = 0
    for k in relax:
        unst = np.nonzero((relax[k][1] > 0) & (relax[k][1] < 1))[0]
        for i in rng.permutation(unst)[:samples]:
            for r in range(R):
                ap = {kk: v.copy() for kk, v in a.items()}
                am = {kk: v.copy() for kk, v in a.items()}
                ap[k][r, i] += h
                am[k][r, i] -= h
                fd = (O.spec_bound_alpha(net, c[0], eps, C[0], relax, ap)[0][r] -
                      O.spec_bound_alpha(net, c[0], eps, C[0], relax, am)[0][r]) / (2 * h)
                if abs(fd - g[k][r, i]) > 1e-6 * (1 + abs(fd)):
                    return False, f"residual gradient mismatch relu {k} row {r} neuron {i}: {g[k][r, i]} vs {fd}"
                n_checked += 1
    if n_checked < 20:
        return False, "too few unstable neurons for the check to mean anything"
    return True, ""


def check_adaptive_start_is_crown_conv(seed=1):
    rng, net, c, C, eps, res, relax = _setup_conv(seed)
    a = {k: np.repeat(relax[k][0][None, :], C.shape[1], axis=0) for k in relax}
    lb, _ = O.spec_bound_alpha(net, c[0], eps, C[0], relax, a)
    if not np.allclose(lb, res.lb_crown[0], rtol=1e-12, atol=1e-12):
        return False, "adaptive slopes do not reproduce the CROWN bound on a convolutional chain"
    return True, ""


def check_adaptive_start_is_crown(seed=1):
    rng, net, c, C, eps, res, relax = _setup(seed)
    a = {k: np.repeat(relax[k][0][None, :], C.shape[1], axis=0) for k in relax}
    lb, _ = O.spec_bound_alpha(net, c[0], eps, C[0], relax, a)
    if not np.allclose(lb, res.lb_crown[0], rtol=1e-12, atol=1e-12):
        return False, "adaptive slopes do not reproduce the CROWN bound"
    return True, ""


def check_hand_optimum():
    # y = ReLU(x), x in [-1, 1]: lb(alpha) = -alpha, maximised at alpha = 0 with lb = 0
    ex = [e for e in load_hand_examples() if e["name"] == "relu_1d"][0]
    net = net_from_layers(ex["layers"])
    best, start = O.alpha_crown(net, np.asarray([ex["centre"]], np.float32), ex["eps"],
                                np.asarray(ex["C"], np.float32)[None], iters=60, lr=0.1)
    if abs(start[0, 0] - (-1.0)) > 1e-12 or abs(best[0, 0]) > 1e-3:
        return False, f"hand optimum: start {start}, best {best}"
    return True, ""


def check_optimised_sound(seed=2):
    rng = np.random.default_rng(seed)
    net = synth.mlp([8, 16, 16, 5], rng)
    c = rng.random((3, 8)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 5, 3), 5)
    best, start = O.alpha_crown(net, c, 0.1, C, iters=15, lr=0.2)
    if np.any(best < start - 1e-12):
        return False, "best bound below the start"
    for b in range(3):
        xs = box_samples(c[b], 0.1, 4000, 400, rng)
        y = O.forward(net, xs)[-1] @ C[b].astype(np.float64).T
        if np.any(y < best[b] - 1e-9):
            return False, "optimised bound violated by a sample"
    if not np.any(best > start + 1e-6):
        return False, "optimisation improved nothing (test net too easy?)"
    return True, ""


CHECKS = [check_fd_gradient, check_adaptive_start_is_crown, check_hand_optimum, check_optimised_sound,
          check_fd_gradient_conv, check_adaptive_start_is_crown_conv, check_fd_gradient_residual]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_alpha_pin(check):
    ok, detail = check()
    assert ok, detail


MUTATIONS = [
    ("G[v] = G[nd.src] @ nd.W.astype(F).T + nd.b.astype(F)[None, :]", "G[v] = G[nd.src] @ nd.W.astype(F).T",
     check_fd_gradient),
    ("G[v] = Gz * slope + np.where(lam_h < 0.0, t[None, :], 0.0)", "G[v] = Gz * slope", check_fd_gradient),
    ("G = {0: c[None, :] - F(eps) * np.sign(lam_in)}", "G = {0: c[None, :] + F(eps) * np.sign(lam_in)}",
     check_fd_gradient),
    ("np.where(unst[None, :] & (lam_h >= 0.0), Gz * lam_h, 0.0)", "np.where(unst[None, :], Gz * lam_h, 0.0)",
     check_fd_gradient),
    ("nd.pad) + nd.b.astype(F)[None, :, None, None]", "nd.pad)", check_fd_gradient_conv),
    ("Gz = conv2d(G[nd.src].reshape((R,) + sh[nd.src]), nd.W, nd.stride, nd.pad)",
     "Gz = conv2d(G[nd.src].reshape((R,) + sh[nd.src]), nd.W[:, :, ::-1, ::-1], nd.stride, nd.pad)",
     check_fd_gradient_conv),
    ("G[v] = G[nd.src] + G[nd.src2]", "G[v] = G[nd.src]", check_fd_gradient_residual),
]


@pytest.mark.parametrize("old,new,check", MUTATIONS)
def test_gradient_mutation_is_caught(monkeypatch, old, new, check):
    src = textwrap.dedent(inspect.getsource(O.spec_bound_alpha))
    assert src.count(old) == 1
    ns = {}
    exec(compile(src.replace(old, new), "<mutant>", "exec"), O.__dict__, ns)
    monkeypatch.setattr(O, "spec_bound_alpha", ns["spec_bound_alpha"])
    caught = False
    for seed in range(3):
        ok, _ = check(seed)
        caught |= not ok
    assert caught
