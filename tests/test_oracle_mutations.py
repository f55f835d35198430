"""Plant plausible mistakes in the oracle (CPU only) and check that some pin catches each.

Each mutation edits one expression of one oracle function's source text, swaps the
edited function into the oracle module for the duration of the test, and runs the
pin checks until one fails (an exception inside a check also counts as caught).
"""
from __future__ import annotations

import inspect
import textwrap

import pytest

import oracle.lbp as O
from tests import test_oracle_pins as P

FAST_FIRST = [P.check_hand_examples, P.check_linear_network, P.check_first_layer_exact, P.check_relax_valid,
              P.check_conv_vs_torch, P.check_forward_vs_torch, P.check_all_stable_exact,
              P.check_one_hidden_alpha0, P.check_eps_monotone, P.check_exact_2d, P.check_lp_sandwich,
              P.check_adam_closed_form, P.check_crown_subset, P.check_soundness_small_configs]

MUTATIONS = [
    ("relax_params", "t[unstable] = -s * l[unstable]", "t[unstable] = s * l[unstable]"),
    ("relax_params", "np.where(u[unstable] >= -l[unstable], 1.0, 0.0)", "np.where(u[unstable] > -l[unstable], 1.0, 0.0)"),
    ("relax_params", "up[unstable] = s", "up[unstable] = 1.0 - s"),
    ("relax_params", "lo[active] = 1.0", "lo[active] = 0.0"),
    ("backward", "const = const + lam @ nd.b.astype(F)", "const = const"),
    ("backward", "put(nd.src, lam @ nd.W.astype(F))", "put(nd.src, lam @ nd.W.astype(F).T)"),
    ("backward", "put(nd.src, pos * lo + neg * up)", "put(nd.src, pos * up + neg * lo)"),
    ("backward", "const = const + neg @ t", "const = const - neg @ t"),
    ("backward", "put(nd.src2, lam)", "pass"),
    ("backward", "const = const + lam4.reshape(R, co, -1).sum(axis=2) @ nd.b.astype(F)", "const = const"),
    ("concretize", "- F(eps) * np.abs(lam_in).sum(axis=1)", "+ F(eps) * np.abs(lam_in).sum(axis=1)"),
    ("concretize", "np.abs(lam_in).sum(axis=1)", "lam_in.sum(axis=1)"),
    ("ibp", "r = rs[nd.src] @ np.abs(Wf).T", "r = rs[nd.src] @ Wf.T"),
    ("ibp", "c, r = (hi + lo) / 2.0, (hi - lo) / 2.0", "c, r = (hi + lo) / 2.0, (hi + lo) / 2.0"),
    ("ibp", "c, r = cs[nd.src] + cs[nd.src2], rs[nd.src] + rs[nd.src2]", "c, r = cs[nd.src] + cs[nd.src2], rs[nd.src]"),
    ("conv2d_adjoint", "Wf[:, :, p, q]", "Wf[:, :, k - 1 - p, k - 1 - q]"),
    ("conv2d", "xp[:, :, p:p + stride * (Ho - 1) + 1:stride, q:q + stride * (Wo - 1) + 1:stride]",
     "xp[:, :, q:q + stride * (Ho - 1) + 1:stride, p:p + stride * (Wo - 1) + 1:stride]"),
    ("verify", "np.where(unst, np.maximum(l0, l_cr), l0)", "np.where(unst, np.minimum(l0, l_cr), l0)"),
    ("verify", "l_cr, u_cr = lbs[:n], -lbs[n:]", "l_cr, u_cr = lbs[:n], lbs[n:]"),
    ("verify", "np.einsum(\"brn,bn->br\", np.abs(Cfull), zr)\n    ub_ibp", "np.einsum(\"brn,bn->br\", Cfull, zr)\n    ub_ibp"),
    ("verify", "ub_cr[b] = -lbs[R:]", "ub_cr[b] = lbs[R:]"),
    ("verify", "lb = np.maximum(lb_ibp, lb_cr)", "lb = np.minimum(lb_ibp, lb_cr)"),
    ("verify", "if k in crown_set and not _first_affine_on_input(net, p):",
     "if k not in crown_set and not _first_affine_on_input(net, p):"),
    ("verify", "crown_set = set(relus if crown_relus is None else crown_relus)",
     "crown_set = set(relus if crown_relus is None else [r - 2 for r in crown_relus])"),
    ("verify", "pre[k][0][b] = np.where(unst, np.maximum(l0, l_cr), l0)", "pass"),
    ("ascend", "mh = m1 / (1 - b1 ** (it + 1))", "mh = m1 / (1 - b1 ** it)"),
    ("ascend", "mh = m1 / (1 - b1 ** (it + 1))", "mh = m1 / (1 - b1 ** (it + 2))"),
    ("ascend", "np.sqrt(vh) + 1e-8", "np.sqrt(vh + 1e-8)"),
    ("ascend", "lr * mh / (np.sqrt(vh) + 1e-8)", "lr * mh / (vh + 1e-8)"),
    ("ascend", "m2 = b2 * m2 + (1 - b2) * g * g", "m2 = b2 * m2 + (1 - b2) * np.abs(g)"),
]


def _mutate(monkeypatch, fname, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(O, fname)))
    assert src.count(old) == 1, f"mutation target not unique in {fname}: {old!r}"
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant {fname}>", "exec"), O.__dict__, ns)
    monkeypatch.setattr(O, fname, ns[fname])


@pytest.mark.parametrize("fname,old,new", MUTATIONS, ids=[f"{m[0]}:{i}" for i, m in enumerate(MUTATIONS)])
def test_mutation_is_caught(monkeypatch, fname, old, new):
    _mutate(monkeypatch, fname, old, new)
    for check in FAST_FIRST:
        try:
            ok, _ = check()
        except Exception:
            ok = False
        if not ok:
            return
    pytest.fail(f"no pin caught the mutation {old!r} -> {new!r} in {fname}")


def test_unmutated_oracle_passes_every_check():
    for check in FAST_FIRST:
        ok, detail = check()
        assert ok, (check.__name__, detail)
