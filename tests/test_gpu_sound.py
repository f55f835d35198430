"""GPU checks of the sound-in-fp32 mode (vf_opts.sound): its bounds never pass the exact-arithmetic
minimum (or maximum) over the box, where that is known exactly -- all-stable networks, whose CROWN bound
is attained at a vertex, and 2-D networks by enumeration -- and never pass a sampled network value; they
stay within a small budget of the fp64 oracle's bounds of the same method."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._helpers import exact_range_2d, net_from_layers
from tests._parity import ambiguous_centres

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(net, centres, eps, C, **kw):
    g = vf.Net(net)
    out = g.verify(_dev(centres), eps, _dev(C), **kw)
    torch.cuda.synchronize()
    g.check()
    return g, {k: v.cpu().numpy().astype(np.float64) for k, v in out.items()}


@pytest.mark.parametrize("which", ["mlp", "mlp784"])
def test_sound_bound_below_attained_minimum(which):
    """Tiny radius: every neuron stable, the network affine on the box, so the exact minimum of each row
    is the oracle's CROWN bound (fp64, attained at a vertex). The plain fp32 path lands on either side of
    it by rounding; the sound path must stay below it, within a small budget."""
    rng = np.random.default_rng(31)
    if which == "mlp":
        net = synth.mlp([20, 48, 48, 32, 6], rng)
        B, classes = 12, 6
        centres = rng.random((B, 20)).astype(np.float32)
    else:
        w = synth.workload(2, B=8)
        net, centres, classes, B = w.net, w.centres, 10, 8
    C = synth.margin_spec(rng.integers(0, classes, B), classes)
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]
    for eps in (1e-6, 1e-7, 1e-8, 1e-9):  # the largest radius at which every neuron is stable
        eps = float(np.float32(eps))
        ora = O.verify(net, centres, eps, C, both_sides=True)
        if not any(np.any((ora.pre_bounds[k][0] < 0) & (ora.pre_bounds[k][1] > 0)) for k in relus):
            break
    else:
        pytest.fail("no radius with every neuron stable")
    exact_lo, exact_hi = ora.lb_crown, ora.ub_crown
    scale = 1e-12 * (np.abs(exact_lo) + 1.0)
    _, plain = _run(net, centres, eps, C, both_sides=True)
    _, snd = _run(net, centres, eps, C, both_sides=True, sound=True)
    assert np.all(snd["lb"] <= exact_lo + scale), "sound lower bound above the exact minimum"
    assert np.all(snd["ub"] >= exact_hi - scale), "sound upper bound below the exact maximum"
    # the budget is the rigorous K u per dot product of K terms (no cancellation assumed): about 1e-3 of the
    # bound on small nets and 1e-2 on the 784-256x3-10 network
    assert np.all(exact_lo - snd["lb"] <= 2e-2 * (np.abs(exact_lo) + 1.0))
    assert np.all(snd["ub"] - exact_hi <= 2e-2 * (np.abs(exact_hi) + 1.0))
    # the check bites: rounding puts some plain fp32 bounds on the wrong side of the exact value
    assert np.sum(plain["lb"] > exact_lo + scale) + np.sum(plain["ub"] < exact_hi - scale) > 0


def test_sound_bounds_contain_exact_2d_range():
    rng = np.random.default_rng(32)
    for trial in range(6):
        w = 3 + trial % 2
        dims = [2, w, w, 3]
        layers = [{"W": (rng.standard_normal((dims[i + 1], dims[i])) * 0.8).astype(np.float32),
                   "b": (rng.standard_normal(dims[i + 1]) * 0.3).astype(np.float32)} for i in range(3)]
        net = net_from_layers(layers)
        c = rng.random(2).astype(np.float32)
        eps = float(np.float32(rng.choice([0.05, 0.2, 0.4])))
        C = np.eye(3, dtype=np.float32)
        lo, hi = exact_range_2d(layers, C, c, eps)
        _, snd = _run(net, c[None], eps, C[None], both_sides=True, sound=True)
        assert np.all(snd["lb"][0] <= lo) and np.all(snd["ub"][0] >= hi), f"trial {trial}"


@pytest.mark.parametrize("kind", ["mlp", "cnn", "resnet"])
def test_sound_bounds_contain_samples_and_track_oracle(kind):
    rng = np.random.default_rng(33)
    if kind == "mlp":
        net = synth.mlp([16, 32, 32, 24, 5], rng)
        eps, classes, shape = 0.05, 5, (16,)
    elif kind == "cnn":
        net = synth.cnn_cfg3(rng, image=(3, 8, 8), c1=4, c2=6, hidden=16, classes=4)
        eps, classes, shape = 0.02, 4, (3, 8, 8)
    else:
        net = synth.resnet_cfg4(rng, image=(3, 8, 8), widths=(3, 4, 5), fc=8, classes=4)
        eps, classes, shape = 0.01, 4, (3, 8, 8)
    eps = float(np.float32(eps))
    B = 3
    n0 = int(np.prod(shape))
    centres = rng.random((B, n0)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, classes, B), classes)
    g, snd = _run(net, centres, eps, C, both_sides=True, want_pre=True, sound=True)
    ora = O.verify(net, centres, eps, C, both_sides=True)
    ok = ~ambiguous_centres(ora, net)
    for b in range(B):
        xs = centres[b].astype(np.float64) + eps * np.concatenate(
            [2 * rng.random((4000, n0)) - 1, rng.choice([-1.0, 1.0], (1000, n0))])
        outs = O.forward(net, xs)
        y = outs[-1] @ C[b].astype(np.float64).T
        tol = 1e-12 * (np.abs(y).max() + 1.0)
        assert np.all(y >= snd["lb"][b] - tol) and np.all(y <= snd["ub"][b] + tol), f"centre {b}"
        for k in [v for v, nd in enumerate(net) if nd.op == "relu"]:
            p = net[k].src
            z = outs[p]
            l = g.node_block(torch.from_numpy(snd["pre_lb"]), p, B).numpy()[b]
            u = g.node_block(torch.from_numpy(snd["pre_ub"]), p, B).numpy()[b]
            t = 1e-12 * (np.abs(z).max() + 1.0)
            assert np.all(z >= l - t) and np.all(z <= u + t), f"centre {b} relu {k}"
        if ok[b]:
            d = ora.lb[b] - snd["lb"][b]
            assert np.all(d <= 1e-3 * (np.abs(ora.lb[b]) + 1.0)), f"centre {b}: sound bound far below the oracle's"


def test_sound_mode_is_verify_only():
    w = synth.workload(2, B=2)
    g = vf.Net(w.net)
    o, keep = g._opts()
    o.sound = 1
    B, R = 2, w.C.shape[1]
    lb = torch.empty(B, R, device="cuda")
    code = vf.lib().vf_alpha_crown(g.h, vf._ptr(_dev(w.centres)), B, float(w.eps), vf._ptr(_dev(w.C)), R, 0,
                                   vf.ctypes.byref(o), 1, 0.1, vf._ptr(lb), None, None, vf._stream_ptr())
    assert code == vf.VF_ERR_UNSUPPORTED
