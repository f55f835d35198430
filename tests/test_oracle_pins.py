"""Pins for the fp64 oracle: each check ties it to something other than itself --
library routines, closed forms, attained vertices, hand-derived examples, exact
ranges by enumeration, an LP, sampling. The ``check_*`` functions return
(ok, detail) so the mutation tests can plant mistakes in the oracle and show that
some pin catches each one.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._helpers import (box_samples, exact_range_2d, load_hand_examples, net_from_layers,
                            relu_ids, triangle_lp_min)


# ----------------------------------------------------------------------------- checks

def check_conv_vs_torch(seed=0):
    rng = np.random.default_rng(seed)
    for (ci, co, h, k, s, p) in [(3, 5, 9, 4, 2, 1), (2, 3, 8, 3, 1, 1), (4, 6, 7, 1, 2, 0), (3, 2, 6, 3, 2, 1)]:
        x = rng.standard_normal((2, ci, h, h))
        W = rng.standard_normal((co, ci, k, k)).astype(np.float32)
        ref = torch.nn.functional.conv2d(torch.from_numpy(x), torch.from_numpy(W.astype(np.float64)),
                                         stride=s, padding=p).numpy()
        got = O.conv2d(x, W, s, p)
        if got.shape != ref.shape or not np.allclose(got, ref, rtol=1e-12, atol=1e-12):
            return False, f"conv2d mismatch at {(ci, co, h, k, s, p)}"
        y = rng.standard_normal(ref.shape)
        g = O.conv2d_adjoint(y, W, s, p, (h, h))
        op = (ref.shape[2] - 1) * s - 2 * p + k
        ref_t = torch.nn.functional.conv_transpose2d(torch.from_numpy(y), torch.from_numpy(W.astype(np.float64)),
                                                     stride=s, padding=p, output_padding=h - op).numpy()
        if g.shape != ref_t.shape or not np.allclose(g, ref_t, rtol=1e-12, atol=1e-12):
            return False, f"conv2d_adjoint mismatch at {(ci, co, h, k, s, p)}"
    return True, ""


def check_forward_vs_torch(seed=1):
    rng = np.random.default_rng(seed)
    net = synth.resnet_cfg4(rng, image=(2, 8, 8), widths=(3, 4, 5), fc=7, classes=4)
    x = rng.random((3, 128))
    outs = O.forward(net, x)
    # torch re-statement of the same graph with library ops
    t = [None] * len(net)
    sh = synth.node_shapes(net)
    for v, nd in enumerate(net):
        if nd.op == "input":
            t[v] = torch.from_numpy(x)
        elif nd.op == "dense":
            t[v] = torch.nn.functional.linear(t[nd.src].reshape(3, -1), torch.from_numpy(nd.W.astype(np.float64)),
                                              torch.from_numpy(nd.b.astype(np.float64)))
        elif nd.op == "conv":
            t[v] = torch.nn.functional.conv2d(t[nd.src].reshape((3,) + sh[nd.src]),
                                              torch.from_numpy(nd.W.astype(np.float64)),
                                              torch.from_numpy(nd.b.astype(np.float64)), stride=nd.stride,
                                              padding=nd.pad).reshape(3, -1)
        elif nd.op == "relu":
            t[v] = torch.relu(t[nd.src])
        elif nd.op == "add":
            t[v] = t[nd.src] + t[nd.src2]
    for v in range(len(net)):
        if not np.allclose(outs[v], t[v].reshape(3, -1).numpy(), rtol=1e-12, atol=1e-12):
            return False, f"forward mismatch at node {v}"
    return True, ""


def _verify_example(ex):
    net = net_from_layers(ex["layers"])
    rel = relu_ids(net)
    alphas = None
    if ex.get("alpha"):
        alphas = {rel[int(k)]: np.asarray([v], np.float64) for k, v in ex["alpha"].items()}
    C = np.asarray(ex["C"], np.float32)[None]
    res = O.verify(net, np.asarray([ex["centre"]], np.float32), ex["eps"], C, alphas=alphas, both_sides=True)
    return net, res


def check_hand_examples():
    for ex in load_hand_examples():
        net, res = _verify_example(ex)
        got = {"lb_ibp": res.lb_ibp[0, 0], "ub_ibp": res.ub_ibp[0, 0], "lb_crown": res.lb_crown[0, 0],
               "ub_crown": res.ub_crown[0, 0], "lb": res.lb[0, 0], "ub": res.ub[0, 0]}
        rel = relu_ids(net)
        if len(rel) > 1:
            got["pre2_l"] = res.pre_bounds[rel[1]][0][0, 0]
            got["pre2_u"] = res.pre_bounds[rel[1]][1][0, 0]
        for key, want in ex["expect"].items():
            if key.startswith("exact"):
                continue
            if abs(got[key] - want) > 1e-12:
                return False, f"{ex['name']}: {key} = {got[key]} != {want}"
        if "exact_min" in ex["expect"]:
            lo, hi = exact_range_2d(ex["layers"], ex["C"], ex["centre"], ex["eps"])
            if abs(lo[0] - ex["expect"]["exact_min"]) > 1e-9 or abs(hi[0] - ex["expect"]["exact_max"]) > 1e-9:
                return False, f"{ex['name']}: exact range {lo, hi}"
    return True, ""


def check_linear_network(seed=2):
    """No ReLU: CROWN equals the closed form over the composed affine map and is attained."""
    rng = np.random.default_rng(seed)
    dims = [5, 7, 6, 4]
    net = [synth.Node("input", shape=(5,))]
    for i in range(3):
        net.append(synth.Node("dense", src=len(net) - 1, W=rng.standard_normal((dims[i + 1], dims[i])).astype(np.float32),
                              b=rng.standard_normal(dims[i + 1]).astype(np.float32)))
    c = rng.random((2, 5)).astype(np.float32)
    eps = 0.3
    C = rng.standard_normal((1, 3, 4)).astype(np.float32)
    res = O.verify(net, c, eps, C, both_sides=True)
    # composed map by forward evaluation on the unit vectors (no matrix algebra of the oracle)
    f0 = O.forward(net, np.zeros((1, 5)))[-1][0]
    Wc = np.stack([O.forward(net, np.eye(5)[i:i + 1])[-1][0] - f0 for i in range(5)], axis=1)  # [4, 5]
    for b in range(2):
        G = C[0].astype(np.float64) @ Wc
        closed_lb = G @ c[b] + C[0] @ f0 - eps * np.abs(G).sum(1)
        if not np.allclose(res.lb_crown[b], closed_lb, rtol=1e-10, atol=1e-10):
            return False, "linear lb closed form"
        xstar = c[b][None, :] - eps * np.sign(G)  # one vertex per row
        vals = np.einsum("rn,rn->r", C[0], O.forward(net, xstar)[-1])
        if not np.allclose(vals, res.lb_crown[b], rtol=1e-10, atol=1e-10):
            return False, "linear lb not attained"
        if np.any(res.lb_ibp[b] > res.lb_crown[b] + 1e-10):
            return False, "IBP tighter than exact on a linear net"
    return True, ""


def check_first_layer_exact(seed=3):
    """One affine layer: IBP per-neuron bounds are attained at a vertex of the box."""
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((6, 4)).astype(np.float32)
    b = rng.standard_normal(6).astype(np.float32)
    net = [synth.Node("input", shape=(4,)), synth.Node("dense", src=0, W=W, b=b)]
    c = rng.random((1, 4)).astype(np.float32)
    eps = 0.2
    cs, rs = O.ibp(net, c, eps)
    lo, hi = cs[1] - rs[1], cs[1] + rs[1]
    c64 = c[0].astype(np.float64)
    xs = c64[None, :] - eps * np.sign(W.astype(np.float64))  # minimiser of each neuron
    vals = np.diagonal(O.forward(net, xs)[1])
    if not np.allclose(vals, lo[0], rtol=1e-12, atol=1e-12):
        return False, "IBP lower not attained"
    xs = c64[None, :] + eps * np.sign(W.astype(np.float64))
    vals = np.diagonal(O.forward(net, xs)[1])
    if not np.allclose(vals, hi[0], rtol=1e-12, atol=1e-12):
        return False, "IBP upper not attained"
    return True, ""


def check_relax_valid(seed=4):
    """Relaxation lines enclose ReLU on [l, u]; the chord touches at both ends."""
    rng = np.random.default_rng(seed)
    l = rng.standard_normal(500) * 2
    u = l + rng.random(500) * 3
    for alpha in (None, rng.random(500) * 1.6 - 0.3):
        lo, up, t = O.relax_params(l, u, alpha)
        z = l[None, :] + (u - l)[None, :] * np.linspace(0, 1, 33)[:, None]
        h = np.maximum(z, 0)
        if np.any(lo * z > h + 1e-12) or np.any(up * z + t < h - 1e-12):
            return False, "relaxation does not enclose ReLU"
        unst = (l < 0) & (u > 0)
        if not np.allclose((up * u + t)[unst], u[unst]) or not np.allclose((up * l + t)[unst], 0.0, atol=1e-12):
            return False, "chord does not touch"
        if alpha is None and not np.array_equal(lo[unst], (u[unst] >= -l[unst]).astype(float)):
            return False, "adaptive alpha rule"
    lo, up, t = O.relax_params(np.array([-1.0, 1.0, -2.0, -1.0]), np.array([1.0, 2.0, -1.0, 0.0]))
    if not (np.array_equal(lo, [1, 1, 0, 0]) and np.array_equal(up, [0.5, 1, 0, 0]) and np.array_equal(t, [0.5, 0, 0, 0])):
        return False, f"special cases {lo, up, t}"
    return True, ""


def _random_mlp(rng, widths):
    return synth.mlp(widths, rng)


def check_one_hidden_alpha0(seed=5):
    """One hidden layer, alpha = 0: CROWN lb >= IBP lb row by row (first-layer bounds exact)."""
    rng = np.random.default_rng(seed)
    for trial in range(4):
        net = _random_mlp(rng, [6, 10, 5])
        c = rng.random((3, 6)).astype(np.float32)
        C = synth.margin_spec(rng.integers(0, 5, 3), 5)
        alphas = {relu_ids(net)[0]: np.zeros((3, 10))}
        res = O.verify(net, c, 0.15, C, alphas=alphas)
        if np.any(res.lb_crown < res.lb_ibp - 1e-10):
            return False, "alpha=0 one-hidden CROWN looser than IBP"
    return True, ""


def check_all_stable_exact(seed=6):
    """Tiny eps: every neuron stable, the net is affine on the box, CROWN is exact and attained."""
    rng = np.random.default_rng(seed)
    for widths in ([5, 8, 8, 4], [4, 4, 4, 4]):
        net = _random_mlp(rng, widths)
        c = rng.random((2, widths[0])).astype(np.float32)
        eps = 1e-7
        C = rng.standard_normal((1, 3, widths[-1])).astype(np.float32)
        res = O.verify(net, c, eps, C, both_sides=True)
        for b in range(2):
            rel = {}
            for k in relu_ids(net):
                l, u = res.pre_bounds[k]
                if np.any((l[b] < 0) & (u[b] > 0)):
                    return False, "not all stable; choose another seed"
                rel[k] = O.relax_params(l[b], u[b])
            lam, cst = O.backward(net, len(net) - 1, C[0].astype(np.float64), rel)
            xs = c[b][None, :] - eps * np.sign(lam)
            vals = np.einsum("rn,rn->r", C[0], O.forward(net, xs)[-1])
            if not np.allclose(vals, res.lb_crown[b], rtol=0, atol=1e-9):
                return False, f"stable net: lb {res.lb_crown[b]} not attained {vals}"
            f = C[0] @ O.forward(net, c[b:b + 1].astype(np.float64))[-1][0]
            if np.any(np.abs(res.lb_crown[b] - f) > 1e-5) or np.any(np.abs(res.ub_crown[b] - f) > 1e-5):
                return False, "stable net bounds far from f(c)"
    return True, ""


def _sound_on(net, centres, eps, C, n_uniform, n_vertex, seed, crown_relus=None):
    rng = np.random.default_rng(seed)
    res = O.verify(net, centres, eps, C, crown_relus=crown_relus, both_sides=True)
    rel_ids = relu_ids(net)
    for b in range(centres.shape[0]):
        xs = box_samples(centres[b], eps, n_uniform, n_vertex, rng)
        rel = {k: O.relax_params(res.pre_bounds[k][0][b], res.pre_bounds[k][1][b]) for k in rel_ids}
        Cb = C[b if C.shape[0] > 1 else 0].astype(np.float64)
        lam, cst = O.backward(net, len(net) - 1, Cb, rel)
        xs = np.concatenate([xs, centres[b][None, :] - eps * np.sign(lam)])
        outs = O.forward(net, xs)
        y = outs[-1] @ Cb.T
        tol = 1e-9 * (1 + np.abs(y).max())
        if np.any(y < res.lb[b] - tol) or np.any(y > res.ub[b] + tol):
            return False, f"spec bound violated at centre {b}"
        if np.any(xs @ lam.T + cst > y + tol):
            return False, f"linear lower function above f at centre {b}"
        for k in rel_ids:
            z = outs[net[k].src]
            l, u = res.pre_bounds[k]
            if np.any(z < l[b] - tol) or np.any(z > u[b] + tol):
                return False, f"intermediate bound of relu {k} violated at centre {b}"
    return True, res


def check_soundness_small_configs(seed=7):
    rng = np.random.default_rng(seed)
    cases = [
        (synth.mlp([8, 32, 32, 4], rng), 0.05, synth.identity_spec(4), None),
        (synth.mlp([20, 16, 16, 16, 5], rng), 0.05, synth.margin_spec(rng.integers(0, 5, 3), 5), None),
        (synth.cnn_cfg3(rng, image=(2, 8, 8), c1=3, c2=4, hidden=10, classes=4), 0.05,
         synth.margin_spec(rng.integers(0, 4, 3), 4), None),
        (synth.resnet_cfg4(rng, image=(2, 8, 8), widths=(3, 4, 5), fc=12, classes=5), 0.02,
         synth.margin_spec(rng.integers(0, 5, 3), 5), None),
        (synth.mlp([12] + [10] * 5 + [6], rng), 0.05, synth.margin_spec(rng.integers(0, 6, 3), 6), "last2"),
    ]
    for i, (net, eps, C, mode) in enumerate(cases):
        n0 = int(np.prod(net[0].shape))
        centres = rng.random((C.shape[0] if C.shape[0] > 1 else 2, n0)).astype(np.float32)
        crown = relu_ids(net)[-2:] if mode == "last2" else None
        ok, det = _sound_on(net, centres, eps, C, 10000, 1000, seed + i, crown)
        if not ok:
            return False, f"case {i}: {det}"
    return True, ""


def check_exact_2d(seed=8):
    """Random 2-w-w-k nets: lb <= exact min <= exact max <= ub, and the bounds are not vacuous."""
    rng = np.random.default_rng(seed)
    for trial in range(6):
        w = 3 + trial % 2
        layers = []
        dims = [2, w, w, 3]
        for i in range(3):
            layers.append({"W": (rng.standard_normal((dims[i + 1], dims[i])) * 0.8).astype(np.float32).tolist(),
                           "b": (rng.standard_normal(dims[i + 1]) * 0.3).astype(np.float32).tolist()})
        net = net_from_layers(layers)
        centre = rng.random(2).astype(np.float32)
        eps = 0.4
        C = np.eye(3, dtype=np.float32)
        res = O.verify(net, centre[None], eps, C[None], both_sides=True)
        lo, hi = exact_range_2d(layers, C, centre, eps)
        if np.any(res.lb[0] > lo + 1e-9) or np.any(res.ub[0] < hi - 1e-9):
            return False, f"trial {trial}: bound tighter than exact range"
    return True, ""


def check_lp_sandwich(seed=9):
    """One hidden layer: CROWN lb <= triangle-LP min <= sampled min."""
    rng = np.random.default_rng(seed)
    for trial in range(4):
        layers = [{"W": rng.standard_normal((7, 4)).astype(np.float32), "b": (rng.standard_normal(7) * 0.2).astype(np.float32)},
                  {"W": rng.standard_normal((3, 7)).astype(np.float32), "b": (rng.standard_normal(3) * 0.2).astype(np.float32)}]
        net = net_from_layers(layers)
        c = rng.random(4).astype(np.float32)
        eps = 0.3
        C = np.eye(3, dtype=np.float32)
        res = O.verify(net, c[None], eps, C[None])
        k = relu_ids(net)[0]
        l1, u1 = res.pre_bounds[k][0][0], res.pre_bounds[k][1][0]
        xs = box_samples(c, eps, 4000, 200, rng)
        y = O.forward(net, xs)[-1]
        for r in range(3):
            lp = triangle_lp_min(layers, C[r].astype(np.float64), c.astype(np.float64), eps, l1, u1)
            if res.lb_crown[0, r] > lp + 1e-7 or lp > y[:, r].min() + 1e-7:
                return False, f"LP sandwich broken: crown {res.lb_crown[0, r]} lp {lp} sample {y[:, r].min()}"
    return True, ""


def check_eps_monotone(seed=10):
    """IBP is inclusion-monotone: shrinking eps never loosens its bounds (interval
    arithmetic). CROWN with the adaptive slope is not (the slope can switch as the
    intermediate bounds move), so only IBP is held to it. eps = 0 gives f(c) exactly."""
    rng = np.random.default_rng(seed)
    net = synth.mlp([10, 12, 12, 4], rng)
    c = rng.random((3, 10)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, 4, 3), 4)
    prev = None
    for eps in (0.2, 0.1, 0.05, 0.01):
        res = O.verify(net, c, eps, C, both_sides=True)
        if prev is not None and (np.any(res.lb_ibp < prev.lb_ibp - 1e-10) or np.any(res.ub_ibp > prev.ub_ibp + 1e-10)):
            return False, "shrinking eps loosened an IBP bound"
        prev = res
    res = O.verify(net, c, 0.0, C, both_sides=True)
    f = np.einsum("brn,bn->br", C, O.forward(net, c.astype(np.float64))[-1])
    if not (np.allclose(res.lb, f, atol=1e-12) and np.allclose(res.ub, f, atol=1e-12)
            and np.allclose(res.lb_crown, f, atol=1e-12)):
        return False, "eps = 0 does not give f(c)"
    return True, ""


def _one_neuron_net(w):
    """y = ReLU(w x) on x in [-1, 1]: input -> dense [[w]] -> ReLU -> dense [[1]], zero biases."""
    return net_from_layers([{"W": [[w]], "b": [0.0]}, {"W": [[1.0]], "b": [0.0]}])


def check_adam_closed_form():
    """alpha-CROWN's ascent against Adam's closed form (Kingma & Ba 2015, Algorithm 1, bias-corrected).

    On y = ReLU(w x), x in [-1, 1], the pre-activation interval [-w, w] sits at the adaptive tie, so the
    start slope is 1, and the specification bound is lb(alpha) = -w alpha, whose gradient -w does not
    change while alpha stays in [0, 1]. With a constant gradient g the bias-corrected moments are exactly
    m_hat = g and v_hat = g^2 after every step k (m_k = (1 - b1^k) g, v_k = (1 - b2^k) g^2), so each step
    moves alpha by lr * g / (|g| + 1e-8) and after k steps alpha_k = 1 - k lr w / (w + 1e-8). The bound
    improves with every step, so the best over the iterates is -w alpha_k. w = 1e-4 makes the 1e-8
    term visible (|g| is comparable to it), which fixes where the epsilon sits."""
    for w, lr in ((2.0, 0.1), (1e-4, 0.1), (0.5, 0.25)):
        net = _one_neuron_net(w)
        w32 = float(np.float32(w))
        c = np.zeros((1, 1), np.float32)
        C = np.ones((1, 1, 1), np.float32)
        for k in range(0, 4):
            best, start = O.alpha_crown(net, c, 1.0, C, iters=k, lr=lr)
            a_k = max(0.0, 1.0 - k * lr * w32 / (w32 + 1e-8))
            want = -w32 * a_k
            if not abs(start[0, 0] + w32) <= 1e-15:
                return False, f"w={w}: adaptive start {start[0, 0]} != {-w32}"
            if not abs(best[0, 0] - want) <= 1e-12 * (1.0 + abs(want)):
                return False, f"w={w} lr={lr} after {k} steps: best {best[0, 0]} != closed form {want}"
    return True, ""


def check_crown_subset(seed=11):
    """IBP substitution for the unselected ReLUs: a ReLU outside crown_relus keeps its IBP bounds bit for
    bit, and a selected one takes, on its IBP-unstable neurons, the intersection with a standalone CROWN
    pass from rows [I; -I] over its pre-activation node, run with the relaxations of the earlier ReLUs.
    The selected passes must also change something (else 'refine nothing' would pass)."""
    rng = np.random.default_rng(seed)
    net = synth.mlp([12] + [10] * 5 + [6], rng)
    relus = relu_ids(net)
    sel = relus[-2:]
    c = rng.random((2, 12)).astype(np.float32)
    C = synth.margin_spec(np.array([1, 4]), 6)
    eps = 0.05
    res = O.verify(net, c, eps, C, crown_relus=sel)
    tightened = 0
    for b in range(2):
        relax = {}
        for k in relus:
            p = net[k].src
            l_ibp, u_ibp = res.ibp_bounds[p][0][b], res.ibp_bounds[p][1][b]
            l, u = res.pre_bounds[k][0][b], res.pre_bounds[k][1][b]
            if k not in sel:
                if not (np.array_equal(l, l_ibp) and np.array_equal(u, u_ibp)):
                    return False, f"unselected relu {k} does not keep its IBP bounds"
            else:
                n = l.size
                eye = np.eye(n)
                lbs = O.crown_pass(net, p, np.concatenate([eye, -eye]), relax, c[b], eps)
                unst = (l_ibp < 0) & (u_ibp > 0)
                l_want = np.where(unst, np.maximum(l_ibp, lbs[:n]), l_ibp)
                u_want = np.where(unst, np.minimum(u_ibp, -lbs[n:]), u_ibp)
                if not (np.allclose(l, l_want, rtol=0, atol=1e-12) and np.allclose(u, u_want, rtol=0, atol=1e-12)):
                    return False, f"selected relu {k}: bounds differ from a standalone CROWN pass"
                tightened += int(np.sum((l > l_ibp) | (u < u_ibp)))
            relax[k] = O.relax_params(l, u)
    if tightened == 0:
        return False, "no selected bound was tightened"
    return True, ""


ALL_CHECKS = [check_conv_vs_torch, check_forward_vs_torch, check_hand_examples, check_linear_network,
              check_first_layer_exact, check_relax_valid, check_one_hidden_alpha0, check_all_stable_exact,
              check_soundness_small_configs, check_exact_2d, check_lp_sandwich, check_eps_monotone,
              check_adam_closed_form, check_crown_subset]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=[c.__name__ for c in ALL_CHECKS])
def test_oracle_pin(check):
    ok, detail = check()
    assert ok, detail


def test_alpha_nan_rejected():
    with pytest.raises(ValueError):
        O.relax_params(np.array([-1.0]), np.array([1.0]), np.array([np.nan]))


def test_wide_mlp_crown_layers_are_the_last_two():
    """The wide MLP workload refines z7 and z8 (the last two of its eight hidden ReLU layers) by CROWN and
    keeps IBP for z1..z6 (IBP substitution for the middle layers)."""
    w = synth.workload(5, B=1)
    dense = [v for v, nd in enumerate(w.net) if nd.op == "dense"]
    assert len(dense) == 9
    want = [v for v, nd in enumerate(w.net) if nd.op == "relu" and nd.src in (dense[6], dense[7])]
    assert w.crown_relus == want and len(want) == 2
