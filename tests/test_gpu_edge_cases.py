"""The method's edge cases on the device, through the C ABI, against values the definitions fix and
against the fp64 oracle:

* the hand-derived examples of tests/golden/hand_examples.json (1-D and 2-D ReLU networks, an
  intermediate-bound pass, active and inactive neurons, given slopes), including the exact adaptive-slope
  tie u = -l, where the reading (alpha = 1 iff u >= -l) fixes the branch and fp32 and fp64 must both take it;
* a zero radius, where every bound is the network's value at the centre;
* one centre with one specification row;
* the first alpha-CROWN ascent step, element by element;
* the branch-and-bound search's decisions (branching neuron of every bounded subdomain, subdomain count,
  rounds, depth) against the oracle's search on properties where no decision sits near a tie.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.lbp as O
from linear_bound_propagation_b200 import synth
from tests._helpers import load_hand_examples, net_from_layers, relu_ids
from tests._parity import ambiguous_centres, max_violation

pytestmark = pytest.mark.gpu

vf = pytest.importorskip("linear_bound_propagation_b200.vf")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _close(got, want):
    return abs(float(got) - float(want)) <= 1e-4 * (abs(float(want)) + 1.0)


@pytest.mark.parametrize("ex", load_hand_examples(), ids=lambda e: e["name"])
def test_hand_example_on_device(ex):
    """vf_verify_batch (both sides) gives the printed final and IBP bounds; vf_crown_backward +
    vf_concretize from the device's own pre-activation bounds give the printed CROWN bounds. In relu_1d and
    relu_2d_sum the pre-activation interval is [-u, u] exactly, so the CROWN lower bound (-1, -2) is the
    alpha = 1 branch; alpha = 0 would give 0."""
    net = net_from_layers(ex["layers"])
    rel = relu_ids(net)
    centre = np.asarray([ex["centre"]], np.float32)
    C = np.asarray(ex["C"], np.float32)[None]
    alpha = None
    if ex.get("alpha"):
        alpha = {rel[int(k)]: _dev(np.asarray([v], np.float32)) for k, v in ex["alpha"].items()}
    g = vf.Net(net)
    out = g.verify(_dev(centre), ex["eps"], _dev(C), alpha=alpha, both_sides=True, want_pre=True)
    lam_lo, cst_lo = g.crown_backward(len(net) - 1, _dev(C), out["pre_lb"], out["pre_ub"], 1, alpha=alpha)
    lam_up, cst_up = g.crown_backward(len(net) - 1, _dev(-C), out["pre_lb"], out["pre_ub"], 1, alpha=alpha)
    lb_cr = vf.concretize(lam_lo, cst_lo, _dev(centre), ex["eps"])
    ub_cr = -vf.concretize(lam_up, cst_up, _dev(centre), ex["eps"])
    torch.cuda.synchronize()
    g.check()
    got = {"lb": out["lb"][0, 0], "ub": out["ub"][0, 0], "lb_ibp": out["lb_ibp"][0, 0],
           "lb_crown": lb_cr[0, 0], "ub_crown": ub_cr[0, 0]}
    if len(rel) > 1:
        p = net[rel[1]].src
        got["pre2_l"] = g.node_block(out["pre_lb"], p, 1)[0, 0]
        got["pre2_u"] = g.node_block(out["pre_ub"], p, 1)[0, 0]
    for key, want in ex["expect"].items():
        if key in got:
            assert _close(got[key].item(), want), f"{ex['name']}: {key} = {got[key].item()} != {want}"
    assert bool(out["verified"][0, 0]) == (ex["expect"]["lb"] > 0)


@pytest.mark.parametrize("config,B", [(1, 5), (2, 5), (3, 2)])
def test_zero_radius_gives_the_value_at_the_centre(config, B):
    """eps = 0: the box is one point, so IBP, every intermediate bound and the CROWN bounds collapse to
    the network's value there; lb = ub = C f(c) (fp64 forward of the oracle)."""
    w = synth.workload(config, B=B)
    g = vf.Net(w.net)
    out = g.verify(_dev(w.centres), 0.0, _dev(w.C), both_sides=True, want_pre=True)
    torch.cuda.synchronize()
    g.check()
    fw = O.forward(w.net, w.centres.astype(np.float64))
    Cf = np.broadcast_to(w.C, (B,) + w.C.shape[1:]).astype(np.float64)
    f = np.einsum("brn,bn->br", Cf, fw[-1])
    assert max_violation(out["lb"].cpu().numpy(), f) <= 1.0
    assert max_violation(out["ub"].cpu().numpy(), f) <= 1.0
    assert max_violation(out["lb_ibp"].cpu().numpy(), f) <= 1.0
    for k in relu_ids(w.net):
        p = w.net[k].src
        assert max_violation(g.node_block(out["pre_lb"], p, B).cpu().numpy(), fw[p]) <= 1.0
        assert max_violation(g.node_block(out["pre_ub"], p, B).cpu().numpy(), fw[p]) <= 1.0


@pytest.mark.parametrize("config", [2, 3, 5])
def test_one_centre_one_row(config):
    """B = 1 and R = 1 (one margin row), against the oracle element by element."""
    w = synth.workload(config, B=1)
    C = np.ascontiguousarray(w.C[:, :1, :])
    ora = O.verify(w.net, w.centres, w.eps, C, crown_relus=w.crown_relus, both_sides=True)
    g = vf.Net(w.net)
    out = g.verify(_dev(w.centres), w.eps, _dev(C), crown_relus=w.crown_relus, both_sides=True)
    torch.cuda.synchronize()
    g.check()
    assert out["lb"].shape == (1, 1)
    if not ambiguous_centres(ora, w.net)[0]:
        assert max_violation(out["lb"].cpu().numpy(), ora.lb) <= 1.0
        assert max_violation(out["ub"].cpu().numpy(), ora.ub) <= 1.0


@pytest.mark.parametrize("config,B", [(1, 64), (2, 16), (3, 3)])
def test_first_alpha_step_elementwise(config, B):
    """One projected Adam step from the adaptive slopes: the best bound over the two iterates matches the
    oracle's on every row of every centre without an adaptive-slope near-tie. A slope whose gradient sign
    differs between fp32 and fp64 moves the other way, but such a gradient is within rounding of 0 and so
    is its effect on the bound after one step."""
    w = synth.workload(config, B=B)
    g = vf.Net(w.net)
    out = g.alpha_crown(_dev(w.centres), w.eps, _dev(w.C), iters=1, lr=0.1)
    torch.cuda.synchronize()
    g.check()
    lb = out["lb"].cpu().numpy()
    res = O.verify(w.net, w.centres, w.eps, w.C)
    ok = ~ambiguous_centres(res, w.net)
    best, _ = O.alpha_crown(w.net, w.centres, w.eps, w.C, iters=1, lr=0.1)
    assert ok.sum() >= B // 2
    assert max_violation(lb[ok], best[ok]) <= 1.0


# ------------------------------------------------------------------------------------- branch and bound

def _bab_problems():
    rng = np.random.default_rng(0)
    out = []
    for t in range(24):
        net = synth.mlp([4, 10, 10, 3], rng)
        c = rng.random(4).astype(np.float32)
        y = O.forward(net, c[None].astype(np.float64))[-1][0]
        C = synth.margin_spec(np.array([int(np.argmax(y))]), 3)[0]
        for eps in (0.1, 0.2, 0.3):
            out.append((f"mlp4-{t}-{eps}", net, c, float(np.float32(eps)), C))
    return out


NEAR = 1e-3  # relative gap below which a decision taken on bounds that match to 1e-4 may flip


def _oracle_search_log(monkeypatch, net, c, eps, C, max_domains, batch):
    """The oracle's search with every bounded subdomain recorded in the order bounded: its splits, the
    (lowest row bound, empty, branching neuron) result, the top-two branching-score gap and whether an
    adaptive slope sat near its tie. Recorded by wrapping the oracle's verify and search functions."""
    relus = relu_ids(net)
    sizes = [int(np.prod(O.shapes(net)[net[k].src])) for k in relus]
    base = {k: int(sum(sizes[:i])) for i, k in enumerate(relus)}
    verify_log, results, attack = [], [], {}
    real_verify, real_search = O.verify, O.bab_search
    real_vertices, real_attack = O.minimiser_vertices, O.minimiser_attack

    def vertices(*a, **kw):
        out = real_vertices(*a, **kw)
        attack["lb"], attack["lam"] = out[0], out[1]
        attack["amb"] = bool(ambiguous_centres(verify_log[-1], net)[0])
        return out

    def attack_values(*a, **kw):
        y = real_attack(*a, **kw)
        attack["y"] = y
        return y

    def verify(*a, **kw):
        res = real_verify(*a, **kw)
        verify_log.append(res)
        return res

    def search(evaluate, max_d, bt):
        def ev(domains):
            r = evaluate(domains)
            res = verify_log[-1]
            amb = ambiguous_centres(res, net)
            for i, (d, x) in enumerate(zip(domains, r)):
                sc = np.concatenate([O.branch_scores(res.pre_bounds[k][0][i], res.pre_bounds[k][1][i]) for k in relus])
                top = np.sort(sc[np.isfinite(sc)])[::-1]
                gap = (top[0] - top[1]) / max(abs(top[0]), 1e-30) if top.size > 1 else np.inf
                results.append({"splits": dict(d), "lb": x[0], "empty": x[1], "choice": x[2], "score_gap": gap,
                                "amb": bool(amb[i])})
            return r
        return real_search(ev, max_d, bt)

    monkeypatch.setattr(O, "verify", verify)
    monkeypatch.setattr(O, "bab_search", search)
    monkeypatch.setattr(O, "minimiser_vertices", vertices)
    monkeypatch.setattr(O, "minimiser_attack", attack_values)
    try:
        o = O.bab(net, c, eps, C, max_domains=max_domains, batch=batch, iters=0)
    finally:
        monkeypatch.setattr(O, "verify", real_verify)
        monkeypatch.setattr(O, "bab_search", real_search)
        monkeypatch.setattr(O, "minimiser_vertices", real_vertices)
        monkeypatch.setattr(O, "minimiser_attack", real_attack)
    trace = [-1 if r["choice"] is None else base[r["choice"][0]] + r["choice"][1] for r in results]
    return o, results, trace, attack


def _attack_near_tie(attack):
    """The vertex attack's decision sits near a tie: a whole-box row bound (which decides whether the attack
    runs) or a row value at a vertex within the tolerance of 0, an adaptive slope of the whole box near its
    tie, or a coefficient of lam_in so small against its row that the device's fp32 sign of it may differ."""
    if "lb" not in attack:
        return False
    if attack["amb"] or np.any(np.abs(attack["lb"]) <= NEAR * (1 + np.abs(attack["lb"]))):
        return True
    y = attack.get("y")
    if y is None or y.size == 0:
        return False
    lam = attack["lam"]
    small = np.abs(lam) <= NEAR * np.abs(lam).max(axis=1, keepdims=True)
    return bool(np.any(np.abs(y) <= NEAR * (1 + np.abs(y).max())) or np.any(small & (lam != 0.0)))


def _near_tie(results):
    """A decision of the search sits near a tie: a branching argmax, a closing test lb > 0, an
    adaptive slope, or the best-first order between two subdomains open at the same time."""
    for r in results:
        if r["amb"] or r["score_gap"] <= NEAR or abs(r["lb"]) <= NEAR * (1 + abs(r["lb"])):
            return True
    # equal bounds (a split that leaves the bound unchanged repeats its parent's arithmetic) are ordered by
    # creation on both sides; only distinct bounds closer than the tolerance may swap
    lbs = sorted(set(r["lb"] for r in results if not r["empty"] and r["lb"] <= 0.0))
    return any(b - a <= NEAR * (1 + abs(a)) for a, b in zip(lbs, lbs[1:]))


def test_bab_decisions_bit_exact(monkeypatch):
    """vf_bab_verify (bounds of vf_verify_batch alone, no ascent) against the oracle's search: on every
    property whose decisions all sit clear of their ties, the same status; when falsified, by the same step
    (the centre or the vertex attack, both before any subdomain is bounded); otherwise the same neuron is
    chosen for every bounded subdomain in the same order, and the subdomain count, rounds and depth are
    equal (index work: exact)."""
    compared = deep = falsified = 0
    for name, net, c, eps, C in _bab_problems():
        o, results, trace, attack = _oracle_search_log(monkeypatch, net, c, eps, C, max_domains=120, batch=8)
        g = vf.Net(net)
        r = g.bab(_dev(c), eps, _dev(C), max_domains=120, batch=8, alpha_iters=0, lr=0.1, trace=True)
        torch.cuda.synchronize()
        g.check()
        tie = _near_tie(results) or _attack_near_tie(attack)
        assert r["status"] == o.status or tie, f"{name}: device {r['status']} vs oracle {o.status}"
        if o.status == "falsified":
            falsified += not tie
            assert r["domains"] == o.domains or tie, name
            continue
        if tie:
            continue
        assert r["trace"] == trace, f"{name}: branching sequence differs"
        assert (r["domains"], r["rounds"], r["max_depth"]) == (o.domains, o.iterations, o.max_depth), name
        compared += 1
        deep += r["rounds"] >= 2
    assert compared >= 8 and deep >= 2, f"only {compared} properties free of near-ties ({deep} with 2+ rounds)"
    assert falsified >= 8, f"only {falsified} falsified properties free of near-ties"


def test_empty_batches_are_no_ops():
    """No centres or no specification rows: every entry point returns VF_OK without touching its outputs (the
    output buffers keep a sentinel), and the handle keeps working."""
    import ctypes
    w = synth.workload(2, B=2)
    g = vf.Net(w.net)
    L = vf.lib()
    cen, C = _dev(w.centres), _dev(w.C)
    sentinel = torch.full((64,), 7.0, device="cuda")
    p = sentinel.data_ptr()
    o = vf.Opts()
    for B, R in ((0, 9), (2, 0), (0, 0)):
        assert L.vf_verify_batch(g.h, cen.data_ptr(), B, w.eps, C.data_ptr(), R, 0, ctypes.byref(o), p, None, None,
                                 None, None) == vf.VF_OK
        assert L.vf_alpha_crown(g.h, cen.data_ptr(), B, w.eps, C.data_ptr(), R, 0, ctypes.byref(o), 3, 0.1, p, None,
                                None, None) == vf.VF_OK
        assert L.vf_concretize(p, None, cen.data_ptr(), w.eps, B, R, 784, p, None) == vf.VF_OK
    assert L.vf_ibp(g.h, cen.data_ptr(), 0, w.eps, p, p, None) == vf.VF_OK
    torch.cuda.synchronize()
    g.check()
    assert torch.all(sentinel == 7.0)
    out = g.verify(cen, w.eps, C)  # still usable
    torch.cuda.synchronize()
    assert torch.isfinite(out["lb"]).all()
