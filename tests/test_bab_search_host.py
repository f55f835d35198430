"""The branch-and-bound search's host logic, bit for bit: the library's search (vf_bab_search, the loop
vf_bab_verify runs) and the oracle's (oracle.lbp.bab_search) are driven by the same deterministic bound
function, and must ask for the same subdomains in the same order and end with the same result. No GPU:
the search itself touches no device."""
from __future__ import annotations

import numpy as np
import pytest

import oracle.lbp as O
from linear_bound_propagation_b200 import vf


def _mock(n_neurons, seed, empty_pairs=(), base=-1.0, lo=-0.05, hi=0.3):
    """A bound function of the split set alone: a base bound plus a fixed fp32 gain per (neuron, sign),
    summed in neuron order; the next neuron to split is the first unsplit one in a fixed permutation;
    a listed pair of splits marks a subdomain empty. Records every batch it is asked for."""
    rng = np.random.default_rng(seed)
    gain = rng.uniform(lo, hi, size=(n_neurons, 2)).astype(np.float32)
    perm = [int(p) for p in rng.permutation(n_neurons)]
    calls = []

    def evaluate(domains):
        calls.append([tuple(d.items()) for d in domains])
        out = []
        for d in domains:
            lb = np.float32(base)
            for nrn in sorted(d):
                lb = np.float32(lb + gain[nrn, (d[nrn] + 1) // 2])
            empty = any(d.get(a) == sa and d.get(b) == sb for a, sa, b, sb in empty_pairs)
            nxt = next((p for p in perm if p not in d), None)
            out.append((float(lb), bool(empty), nxt))
        return out

    return evaluate, calls


CASES = [
    # (neurons, seed, max_domains, batch, empty pairs, base)
    (6, 0, 1, 2, (), -1.0),
    (6, 0, 2, 2, (), -1.0),
    (6, 1, 3, 4, (), -1.0),
    (6, 2, 40, 4, (), -1.0),
    (6, 3, 200, 8, (), -1.0),
    (8, 4, 500, 16, ((1, 1, 2, -1),), -0.6),
    (5, 5, 1000, 8, (), -0.2),
    (4, 6, 1000, 2, ((0, -1, 3, 1),), -2.0),
    (10, 7, 300, 64, (), -0.8),
    (6, 8, 10, 4, (), 0.5),  # verified by the whole box
]


@pytest.mark.parametrize("case", CASES, ids=[f"n{c[0]}-s{c[1]}-d{c[2]}-b{c[3]}" for c in CASES])
def test_library_search_matches_oracle_search(case):
    n, seed, max_domains, batch, pairs, base = case
    ev_lib, calls_lib = _mock(n, seed, pairs, base)
    ev_ora, calls_ora = _mock(n, seed, pairs, base)
    r = vf.bab_search(ev_lib, max_domains, batch)
    o = O.bab_search(ev_ora, max_domains, batch)
    assert calls_lib == calls_ora
    assert (r["status"], r["domains"], r["rounds"], r["max_depth"]) == (o.status, o.domains, o.iterations, o.max_depth)
    assert np.float32(r["lb"]) == np.float32(o.lb)


def test_search_outcomes_cover_every_ending():
    """The cases above reach all three endings: verified, unknown at the budget, unknown at a subdomain
    with nothing left to split."""
    seen = set()
    for n, seed, max_domains, batch, pairs, base in CASES:
        ev, _ = _mock(n, seed, pairs, base)
        o = O.bab_search(ev, max_domains, batch)
        if o.status == "verified":
            seen.add("verified")
        elif o.domains + 1 >= max_domains or (max_domains - o.domains) < 2:
            seen.add("budget")
        else:
            seen.add("unsplittable")
    assert seen == {"verified", "budget", "unsplittable"}, seen


def test_search_reports_bound_function_errors():
    def bad(domains):
        raise RuntimeError("bound failed")

    with pytest.raises(RuntimeError):
        vf.bab_search(bad, 10, 4)
    with pytest.raises(vf.VfError):
        vf.bab_search(lambda d: [(0.0, False, None)] * len(d), 0, 4)
