"""GPU parity of branch-and-bound split constraints, their multipliers beta and the search
(vf_verify_batch, vf_alpha_beta_grad and vf_alpha_crown with opts.split; vf_bab_verify) against the
fp64 oracle, on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._parity import ambiguous_centres, max_violation
from tests.test_gpu_alpha import _assert_off_rows_at_kinks

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _viol(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(got - ref) / (1e-4 * (np.abs(ref) + 1.0))


def _case(kind, B=3, seed=0):
    rng = np.random.default_rng(700 + seed)
    if kind == "mlp":
        net = synth.mlp([12, 24, 24, 20, 5], rng)
        eps, classes = 0.1, 5
    elif kind == "cnn":
        net = synth.cnn_cfg3(rng, image=(3, 8, 8), c1=4, c2=6, hidden=16, classes=4)
        eps, classes = 0.03, 4
    elif kind == "resnet":
        net = synth.resnet_cfg4(rng, image=(3, 8, 8), widths=(3, 4, 5), fc=8, classes=4)
        eps, classes = 0.02, 4
    else:  # the 784-256x3-10 dense network of the headline workload, a few centres
        w = synth.workload(2, B=B)
        return w.net, w.centres, w.C, w.eps
    n0 = int(np.prod(net[0].shape))
    centres = rng.random((B, n0)).astype(np.float32)
    C = synth.margin_spec(rng.integers(0, classes, B), classes)
    return net, centres, C, float(np.float32(eps))


def _signs(net, centres, eps, frac, rng, consistent=True):
    """Per centre, split signs for a random `frac` of each ReLU layer's neurons: the sign of z at a random
    point of the centre's box (a subdomain holding that point), or random signs (possibly empty ones)."""
    B, n0 = centres.shape
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]
    sp = {}
    for b in range(B):
        x0 = centres[b].astype(np.float64) + eps * (2 * rng.random(n0) - 1)
        outs = O.forward(net, x0[None, :])
        for k in relus:
            z = outs[net[k].src][0]
            sg = np.where(z >= 0.0, 1, -1) if consistent else rng.choice([-1, 1], z.size)
            sp.setdefault(k, np.zeros((B, z.size), np.int8))[b] = np.where(rng.random(z.size) < frac, sg, 0)
    return sp


@pytest.mark.parametrize("consistent", [True, False], ids=["holding-a-point", "random-signs"])
@pytest.mark.parametrize("kind", ["mlp", "cnn", "resnet", "mlp784"])
def test_split_bounds_match_oracle(kind, consistent):
    net, centres, C, eps = _case(kind)
    rng = np.random.default_rng(11)
    sp = _signs(net, centres, eps, 0.3, rng, consistent)
    both = kind in ("mlp", "resnet")
    ora = O.verify(net, centres, eps, C, both_sides=both, splits=sp)
    g = vf.Net(net)
    out = g.verify(_dev(centres), eps, _dev(C), both_sides=both, want_pre=True,
                   splits={k: _dev(v) for k, v in sp.items()})
    torch.cuda.synchronize()
    g.check()
    out = {k: v.cpu().numpy() for k, v in out.items()}
    B = centres.shape[0]
    amb = ambiguous_centres(ora, net)
    assert max_violation(out["lb_ibp"], ora.lb_ibp) <= 1.0
    checked = 0
    for b in range(B):
        if amb[b]:
            continue
        viol = max_violation(out["lb"][b], ora.lb[b])
        if both:
            viol = max(viol, max_violation(out["ub"][b], ora.ub[b]))
        for k in g.relu_ids:
            p = net[k].src
            gl = g.node_block(torch.from_numpy(out["pre_lb"]), p, B).numpy()[b]
            gu = g.node_block(torch.from_numpy(out["pre_ub"]), p, B).numpy()[b]
            viol = max(viol, max_violation(gl, ora.pre_bounds[k][0][b]), max_violation(gu, ora.pre_bounds[k][1][b]))
        assert viol <= 1.0, f"centre {b}: {viol:.2f}"
        checked += 1
    assert checked >= 1


def _blocks(g, B, R):
    off, blocks = 0, {}
    for k in g.relu_ids:
        blocks[k] = (off, g.sizes[k])
        off += B * R * g.sizes[k]
    return blocks


@pytest.mark.parametrize("kind", ["mlp", "cnn", "resnet"])
def test_alpha_beta_gradient_matches_oracle(kind):
    net, centres, C, eps = _case(kind, B=2, seed=1)
    rng = np.random.default_rng(12)
    sp = _signs(net, centres, eps, 0.3, rng)
    B, R = centres.shape[0], C.shape[1]
    g = vf.Net(net)
    alpha = rng.random(g.alpha_size(B, R)).astype(np.float32)
    beta = rng.exponential(0.5, g.alpha_size(B, R)).astype(np.float32)
    lb, ga, gb = g.alpha_beta_grad(_dev(centres), eps, _dev(C), _dev(alpha), _dev(beta),
                                   {k: _dev(v) for k, v in sp.items()})
    torch.cuda.synchronize()
    g.check()
    lb, ga, gb = lb.cpu().numpy(), ga.cpu().numpy(), gb.cpu().numpy()
    res = O.verify(net, centres, eps, C, splits=sp)
    amb = ambiguous_centres(res, net)
    blocks = _blocks(g, B, R)
    checked = 0
    for b in range(B):
        if amb[b]:
            continue
        relax = {k: O.relax_params(res.pre_bounds[k][0][b], res.pre_bounds[k][1][b]) for k in g.relu_ids}
        cut = lambda arr, o, n: arr[o + b * R * n: o + (b + 1) * R * n].reshape(R, n)  # noqa: E731
        a = {k: cut(alpha, o, n).astype(np.float64) for k, (o, n) in blocks.items()}
        bt = {k: cut(beta, o, n).astype(np.float64) for k, (o, n) in blocks.items()}
        olb, og, obg = O.spec_bound_alpha(net, centres[b], eps, C[b], relax, a, {k: sp[k][b] for k in sp}, bt)
        assert _viol(lb[b], olb).max() <= 1.0, f"centre {b}"
        for k, (o, n) in blocks.items():
            assert _viol(cut(ga, o, n), og[k]).max() <= 1.0, f"centre {b} relu {k}: slope gradient"
            assert _viol(cut(gb, o, n), obg[k]).max() <= 1.0, f"centre {b} relu {k}: beta gradient"
            assert np.all(cut(gb, o, n)[:, sp[k][b] == 0] == 0.0)
        checked += 1
    assert checked >= 1


def test_alpha_crown_with_splits_tracks_oracle():
    net, centres, C, eps = _case("mlp", B=4, seed=2)
    rng = np.random.default_rng(13)
    sp = _signs(net, centres, eps, 0.3, rng)
    g = vf.Net(net)
    out = g.alpha_crown(_dev(centres), eps, _dev(C), iters=10, lr=0.1, splits={k: _dev(v) for k, v in sp.items()})
    torch.cuda.synchronize()
    g.check()
    lb, lb0 = out["lb"].cpu().numpy(), out["lb_start"].cpu().numpy()
    assert np.all(lb >= lb0)
    res = O.verify(net, centres, eps, C, splits=sp)
    ok = ~ambiguous_centres(res, net)
    assert _viol(lb0[ok], res.lb_crown[ok]).max() <= 1.0
    best, _ = O.alpha_crown(net, centres, eps, C, iters=10, lr=0.1, splits=sp)
    # every row matches the oracle's trajectory or sits at a kink of it (its oracle value jumps under a 1e-6
    # relative change of eps)
    _assert_off_rows_at_kinks(net, centres, eps, C, lb, best, ok, iters=10, splits=sp)
    # sound on the subdomains: sampled inputs that satisfy a centre's splits stay above its bound
    for b in range(centres.shape[0]):
        xs = centres[b] + eps * (2 * rng.random((20000, centres.shape[1])) - 1)
        outs = O.forward(net, xs)
        keep = np.ones(len(xs), bool)
        for k, s in sp.items():
            keep &= np.all((s[b][None, :] == 0) | (s[b][None, :] * outs[net[k].src] >= 0.0), axis=1)
        y = outs[-1][keep] @ C[b].astype(np.float64).T
        assert np.all(y >= lb[b] - 1e-4 * (np.abs(y) + 1.0))


def _bab_cases():
    rng = np.random.default_rng(0)
    cases = []
    for t in range(4):
        net = synth.mlp([4, 10, 10, 3], rng)
        c = rng.random(4).astype(np.float32)
        y = O.forward(net, c[None].astype(np.float64))[-1][0]
        C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
        for eps in (0.1, 0.2, 0.3):
            cases.append((f"mlp4-{t}-{eps}", net, c, float(np.float32(eps)), C))
    return cases


def test_bab_matches_oracle():
    """The same search on the device and in the oracle ends with the same decision on every case; every
    "verified" holds on sampled inputs."""
    agree, total, wins = 0, 0, 0
    for name, net, c, eps, C in _bab_cases():
        g = vf.Net(net)
        r = g.bab(_dev(c), eps, _dev(C), max_domains=200, batch=16, alpha_iters=20, lr=0.1)
        torch.cuda.synchronize()
        g.check()
        o = O.bab(net, c, eps, C, max_domains=200, batch=16, iters=20, lr=0.1)
        total += 1
        agree += r["status"] == o.status
        assert r["status"] == o.status, f"{name}: device {r} vs oracle {o}"
        if r["status"] == "verified":
            wins += r["domains"] > 1
            xs = c + eps * (2 * np.random.default_rng(1).random((20000, c.size)) - 1)
            assert (O.forward(net, xs)[-1] @ C.astype(np.float64).T).min() > 0.0, name
    assert wins >= 1


def test_bab_headline_network_small_budget():
    """vf_bab_verify on the 784-256x3-10 network: margin rows of each centre's own top class (so the
    centre is no counterexample) at two radii, the search against the oracle's on a small budget."""
    w = synth.workload(2, B=2)
    g = vf.Net(w.net)
    y = O.forward(w.net, w.centres.astype(np.float64))[-1]
    for b in range(2):
        C = synth.margin_spec(np.array([int(np.argmax(y[b]))]), 10)[0]
        for eps in (w.eps, float(np.float32(w.eps / 8))):
            r = g.bab(_dev(w.centres[b]), eps, _dev(C), max_domains=48, batch=16, alpha_iters=10, lr=0.1)
            torch.cuda.synchronize()
            g.check()
            o = O.bab(w.net, w.centres[b], eps, C, max_domains=48, batch=16, iters=10, lr=0.1)
            assert r["status"] == o.status, f"centre {b} eps {eps}: device {r} vs oracle {o}"
            assert r["domains"] <= 48


def test_bab_rejects_bad_options():
    net, centres, C, eps = _case("mlp", B=1)
    g = vf.Net(net)
    for kw in (dict(batch=3), dict(batch=0), dict(max_domains=0), dict(alpha_iters=-1)):
        with pytest.raises(vf.VfError) as e:
            g.bab(_dev(centres[0]), eps, _dev(C[0]), **kw)
        assert e.value.code == vf.VF_ERR_ARG


def test_bab_with_intermediate_alpha():
    """Branch and bound with alpha-CROWN intermediate bounds (slopes and the split multipliers of earlier layers)
    in every subdomain, on the 72 small properties of the decision test: the device ends with the oracle's status
    (same options) on at least 90% of them, every "verified" holds on sampled inputs, and the properties that the
    option turns from "unknown" to "verified" in the oracle are verified on the device as well."""
    from tests.test_gpu_edge_cases import _bab_problems
    agree = total = 0
    gained = []
    for name, net, c, eps, C in _bab_problems():
        g = vf.Net(net)
        r = g.bab(_dev(c), eps, _dev(C), max_domains=120, batch=8, alpha_iters=0, alpha_inter_iters=5)
        torch.cuda.synchronize()
        g.check()
        o = O.bab(net, c, eps, C, max_domains=120, batch=8, iters=0, alpha_inter_iters=5)
        total += 1
        agree += r["status"] == o.status
        if r["status"] == "verified":
            xs = c + eps * (2 * np.random.default_rng(2).random((20000, c.size)) - 1)
            assert (O.forward(net, xs)[-1] @ C.astype(np.float64).T).min() > 0.0, name
        if o.status == "verified" and O.bab(net, c, eps, C, max_domains=120, batch=8, iters=0).status == "unknown":
            gained.append((name, r["status"]))
    assert agree >= 0.9 * total, f"{agree} of {total} statuses agree"
    assert gained and all(s == "verified" for _, s in gained), gained


def _starts(g, net, B, R, rng, sp):
    """Seeded start slopes in [0, 1] with a fifth of the entries negative (no start), and start multipliers, in
    the alpha_out layout; plus the same as the oracle's per-centre (slopes, multipliers) dicts."""
    relus = g.relu_ids
    a = rng.random(g.alpha_size(B, R)).astype(np.float32)
    a[rng.random(a.size) < 0.2] = -1.0
    bt = (rng.random(g.alpha_size(B, R)) * 0.5).astype(np.float32)
    per_centre, off = [({}, {}) for _ in range(B)], 0
    for k in relus:
        n = g.sizes[k]
        blk_a = a[off: off + B * R * n].reshape(B, R, n)
        blk_b = bt[off: off + B * R * n].reshape(B, R, n)
        for b in range(B):
            per_centre[b][0][k] = blk_a[b].astype(np.float64)
            if k in sp:
                per_centre[b][1][k] = blk_b[b].astype(np.float64)
        off += B * R * n
    return a, bt, per_centre


def test_alpha_crown_start_states_match_oracle():
    """vf_alpha_crown from given start slopes and multipliers (the warm start of branch and bound) against the
    oracle's ascent from the same start: at zero steps the bound element-wise (a negative slope entry starts from
    the adaptive slope); after four steps every row, except at kinks of the ascent; the returned last multipliers
    are >= 0, keep their start value on free neurons (their gradient is zero) and are zero on layers without
    splits."""
    net, centres, C, eps = _case("mlp", B=4, seed=3)
    rng = np.random.default_rng(17)
    sp = _signs(net, centres, eps, 0.3, rng)
    g = vf.Net(net)
    B, R = centres.shape[0], C.shape[1]
    a, bt, starts = _starts(g, net, B, R, rng, sp)
    oracle_starts = []
    res = O.verify(net, centres, eps, C, splits=sp)
    for b in range(B):
        relax = {k: O.relax_params(res.pre_bounds[k][0][b], res.pre_bounds[k][1][b]) for k in g.relu_ids}
        # the oracle takes a slope start per entry: a negative device entry means the relaxation's slope
        a0 = {k: np.where(v < 0, np.repeat(relax[k][0][None, :], R, axis=0), v) for k, v in starts[b][0].items()}
        oracle_starts.append((a0, starts[b][1]))
    spd = {k: _dev(v) for k, v in sp.items()}
    for iters in (0, 4):
        out = g.alpha_crown(_dev(centres), eps, _dev(C), iters=iters, lr=0.1, splits=spd, alpha_init=_dev(a),
                            beta_init=_dev(bt), want_beta=True)
        torch.cuda.synchronize()
        g.check()
        lb = out["lb"].cpu().numpy()
        best, start = O.alpha_crown(net, centres, eps, C, iters=iters, lr=0.1, splits=sp, starts=oracle_starts)
        ok = ~ambiguous_centres(res, net)
        assert ok.sum() >= 2
        assert _viol(out["lb_start"].cpu().numpy()[ok], start[ok]).max() <= 1.0, iters
        if iters == 0:
            assert _viol(lb[ok], best[ok]).max() <= 1.0
        else:
            _assert_off_rows_at_kinks(net, centres, eps, C, lb, best, ok, iters=iters, splits=sp,
                                      starts=oracle_starts)
        beta = out["beta"].cpu().numpy()
        assert np.all(beta >= 0.0)
        off = 0
        for k in g.relu_ids:
            n = g.sizes[k]
            blk = beta[off: off + B * R * n].reshape(B, R, n)
            if k in sp:
                free = np.broadcast_to((sp[k] == 0)[:, None, :], blk.shape)
                start_b = np.maximum(bt[off: off + B * R * n].reshape(B, R, n), 0.0)
                assert np.array_equal(blk[free], start_b[free]), k
            else:
                assert np.all(blk == 0.0), k
            off += B * R * n


def test_bab_warm_start_on_device():
    """The 72 small properties with 3 ascent steps per subdomain: children that start from their parent's
    slopes and multipliers settle more properties on the device than children that start afresh (as in the
    oracle: 36 against 31), the device's statuses agree with the oracle's warm search on at least 90% of them,
    and every "verified" holds on sampled inputs."""
    from tests.test_gpu_edge_cases import _bab_problems
    counts = {True: 0, False: 0}
    agree = total = 0
    for name, net, c, eps, C in _bab_problems():
        g = vf.Net(net)
        for warm in (True, False):
            r = g.bab(_dev(c), eps, _dev(C), max_domains=200, batch=8, alpha_iters=3, lr=0.1, warm_start=warm)
            torch.cuda.synchronize()
            g.check()
            if r["status"] == "verified":
                counts[warm] += 1
                xs = c + eps * (2 * np.random.default_rng(3).random((20000, c.size)) - 1)
                assert (O.forward(net, xs)[-1] @ C.astype(np.float64).T).min() > 0.0, (name, warm)
            if warm:
                o = O.bab(net, c, eps, C, max_domains=200, batch=8, iters=3, lr=0.1)
                total += 1
                agree += r["status"] == o.status
    assert counts[True] >= counts[False] + 3, counts
    assert agree >= 0.9 * total, f"{agree} of {total}"
