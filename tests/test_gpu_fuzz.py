"""GPU parity on seeded random small networks: plain and residual CNNs with random kernel sizes, strides and
paddings, dense heads, and dense ReLU chains of random widths, with random batch sizes, radii, CROWN-refined
layer subsets and bound sides. Each network exercises a different mix of the
executor's paths (receptive-field windows and their merges at residual adds, whole-map rows, unstable-only
compaction, tensor-core and FFMA contractions); every result is compared with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import ambiguous_centres, max_violation, sound_on_samples
from tests._random_nets import random_mlp, random_net

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")

SEEDS = list(range(24))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _dense_kernel(monkeypatch, seed):
    """Even seeds force the tensor cores on every dense launch the shapes allow (VF_DENSE_KERNEL=tc); odd
    seeds keep the default choice, which sends launches of few tiles to the K-split FFMA kernel."""
    if seed % 2 == 0:
        monkeypatch.setenv("VF_DENSE_KERNEL", "tc")
    else:
        monkeypatch.delenv("VF_DENSE_KERNEL", raising=False)


@pytest.mark.parametrize("seed", SEEDS)
def test_random_network_matches_oracle(monkeypatch, seed):
    _dense_kernel(monkeypatch, seed)
    net, shape, classes = random_net(seed)
    rng = np.random.default_rng(20_000 + seed)
    B = int(rng.integers(1, 4))
    n0 = int(np.prod(shape))
    centres = rng.random((B, n0)).astype(np.float32)
    eps = float(np.float32(rng.choice([0.002, 0.01, 0.03])))
    C = synth.margin_spec(rng.integers(0, classes, B), classes)
    both = bool(rng.random() < 0.5)
    ora = O.verify(net, centres, eps, C, both_sides=both)
    g = vf.Net(net)
    out = g.verify(_dev(centres), eps, _dev(C), both_sides=both, want_pre=True)
    torch.cuda.synchronize()
    g.check()
    out = {k: v.cpu().numpy() for k, v in out.items()}
    assert max_violation(out["lb_ibp"], ora.lb_ibp) <= 1.0
    amb = ambiguous_centres(ora, net)
    for b in range(B):
        viol = max_violation(out["lb"][b], ora.lb[b])
        if both:
            viol = max(viol, max_violation(out["ub"][b], ora.ub[b]))
        for k in [v for v, nd in enumerate(net) if nd.op == "relu"]:
            p = net[k].src
            gl = g.node_block(torch.from_numpy(out["pre_lb"]), p, B).numpy()[b]
            gu = g.node_block(torch.from_numpy(out["pre_ub"]), p, B).numpy()[b]
            viol = max(viol, max_violation(gl, ora.pre_bounds[k][0][b]), max_violation(gu, ora.pre_bounds[k][1][b]))
        if viol > 1.0:
            assert amb[b], f"seed {seed} centre {b}: violation {viol:.2f} without an adaptive-slope tie"
            assert sound_on_samples(net, centres[b:b + 1], eps, C[b:b + 1], out["lb"][b:b + 1],
                                    out["ub"][b:b + 1] if both else None)


@pytest.mark.parametrize("seed", list(range(16)))
def test_random_mlp_matches_oracle(monkeypatch, seed):
    """Random dense ReLU chains (widths that do and do not meet the tensor-core shape rules), random batch
    sizes that leave ragged tiles, random subsets of layers refined by CROWN (the rest keep IBP bounds)
    and both bound sides."""
    _dense_kernel(monkeypatch, seed)
    net, widths = random_mlp(seed)
    rng = np.random.default_rng(40_000 + seed)
    B = int(rng.integers(1, 41))
    centres = rng.random((B, widths[0])).astype(np.float32)
    eps = float(np.float32(rng.choice([0.005, 0.02, 0.08])))
    classes = widths[-1]
    C = synth.margin_spec(rng.integers(0, classes, B), classes)
    both = bool(rng.random() < 0.5)
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]
    crown = [v for v in relus if rng.random() < 0.7]
    ora = O.verify(net, centres, eps, C, crown_relus=crown, both_sides=both)
    g = vf.Net(net)
    out = g.verify(_dev(centres), eps, _dev(C), crown_relus=crown, both_sides=both, want_pre=True)
    torch.cuda.synchronize()
    g.check()
    out = {k: v.cpu().numpy() for k, v in out.items()}
    assert max_violation(out["lb_ibp"], ora.lb_ibp) <= 1.0
    amb = ambiguous_centres(ora, net)
    for b in range(B):
        viol = max_violation(out["lb"][b], ora.lb[b])
        if both:
            viol = max(viol, max_violation(out["ub"][b], ora.ub[b]))
        for k in relus:
            p = net[k].src
            gl = g.node_block(torch.from_numpy(out["pre_lb"]), p, B).numpy()[b]
            gu = g.node_block(torch.from_numpy(out["pre_ub"]), p, B).numpy()[b]
            viol = max(viol, max_violation(gl, ora.pre_bounds[k][0][b]), max_violation(gu, ora.pre_bounds[k][1][b]))
        if viol > 1.0:
            assert amb[b], f"seed {seed} centre {b}: violation {viol:.2f} without an adaptive-slope tie"
            assert sound_on_samples(net, centres[b:b + 1], eps, C[b:b + 1], out["lb"][b:b + 1],
                                    out["ub"][b:b + 1] if both else None)


def _alpha_blocks(g, B, R):
    off, blocks = 0, {}
    for k in g.relu_ids:
        blocks[k] = (off, g.sizes[k])
        off += B * R * g.sizes[k]
    return blocks


@pytest.mark.parametrize("seed", list(range(12)))
def test_random_alpha_gradient_matches_oracle(seed):
    """alpha-CROWN bound and slope gradient at random slopes on random networks (CNN chains, residual
    graphs and dense chains alike), against the oracle's reverse-mode gradient."""
    net = random_net(seed)[0] if seed % 2 == 0 else random_mlp(seed)[0]
    rng = np.random.default_rng(50_000 + seed)
    B = int(rng.integers(1, 4))
    n0 = int(np.prod(net[0].shape))
    classes = int(net[-1].W.shape[0])
    centres = rng.random((B, n0)).astype(np.float32)
    eps = float(np.float32(rng.choice([0.005, 0.02])))
    C = synth.margin_spec(rng.integers(0, classes, B), classes)
    R = C.shape[1]
    g = vf.Net(net)
    alpha = rng.random(g.alpha_size(B, R)).astype(np.float32)
    lb, grad = g.alpha_grad(_dev(centres), eps, _dev(C), _dev(alpha))
    torch.cuda.synchronize()
    g.check()
    lb, grad = lb.cpu().numpy(), grad.cpu().numpy()
    res = O.verify(net, centres, eps, C)
    amb = ambiguous_centres(res, net)
    blocks = _alpha_blocks(g, B, R)
    for b in range(B):
        if amb[b]:
            continue
        relax = {k: O.relax_params(res.pre_bounds[k][0][b], res.pre_bounds[k][1][b]) for k in g.relu_ids}
        a = {k: alpha[o + b * R * n: o + (b + 1) * R * n].reshape(R, n).astype(np.float64) for k, (o, n) in blocks.items()}
        olb, og = O.spec_bound_alpha(net, centres[b], eps, C[b], relax, a)
        assert max_violation(lb[b], olb) <= 1.0, f"seed {seed} centre {b}"
        for k, (o, n) in blocks.items():
            gg = grad[o + b * R * n: o + (b + 1) * R * n].reshape(R, n)
            v = np.abs(gg - og[k]) / (1e-4 * (np.abs(og[k]) + 1.0))
            assert v.max() <= 10.0, f"seed {seed} centre {b} relu {k}: {v.max():.2f}"
