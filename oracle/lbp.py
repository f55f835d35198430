"""Plain fp64 statement of the hot path: IBP, ReLU relaxation, CROWN back-substitution,
concretisation over an L-infinity box, intermediate-bound passes and the final decision.

TEST INFRASTRUCTURE (see the package docstring): only tests, the smoke check and
the benchmark's CPU-baseline leg use this module.

Page: "Scaling Neural Network Verification with Tensor Parallelism and Fully
Sharded Data Parallelism" (gist.science summary of arXiv 2606.09377), cited as
[SNNV <section>]:
  * [SNNV §1]   the task: prove a property for every input of a domain, with the
                weights and the linear relaxation matrices A of IBP / CROWN /
                alpha-CROWN held on one accelerator;
  * [SNNV §2.1] CROWN's backward pass needs intermediate bounds to fix the ReLU
                relaxation slopes lambda_i; IBP is the cheap, looser but still sound
                substitute for them;
  * [SNNV §3], [SNNV §4.3] per-neuron alpha tensors (the ReLU lower slopes);
  * [SNNV §4.2] soundness means a one-sided over-approximation.

Everything is computed in float64 from the fp32 inputs promoted exactly. The
oracle works centre by centre, and within a centre on all specification rows at
once; matrix products use numpy's matmul as a library step. Rows are independent,
so a pass may be split into row blocks purely to bound memory.

Network format: a list of nodes in topological order (``src`` < own index), node 0
the input; ops ``input``, ``dense`` (W [n_out, n_in], b), ``conv`` (W [Co, Ci, k, k],
b [Co], stride, pad), ``relu``, ``add`` (src + src2). Activations are flattened in
C order (channel, row, column).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

F = np.float64


# ----------------------------------------------------------------------------- shapes

def shapes(net) -> List[tuple]:
    out = []
    for nd in net:
        if nd.op == "input":
            out.append(tuple(nd.shape))
        elif nd.op == "dense":
            out.append((nd.W.shape[0],))
        elif nd.op == "conv":
            c, h, w = out[nd.src]
            k = nd.W.shape[2]
            out.append((nd.W.shape[0], (h + 2 * nd.pad - k) // nd.stride + 1,
                        (w + 2 * nd.pad - k) // nd.stride + 1))
        elif nd.op in ("relu", "add"):
            out.append(out[nd.src])
        else:
            raise ValueError(nd.op)
    return out


def _size(shape) -> int:
    return int(np.prod(shape))


# ----------------------------------------------------------------------------- convolution

def conv2d(x: np.ndarray, W: np.ndarray, stride: int, pad: int) -> np.ndarray:
    """Cross-correlation by its definition, without bias.

    out[n, o, i, j] = sum_{c, p, q} W[o, c, p, q] * x[n, c, i*stride - pad + p, j*stride - pad + q],
    with x read as zero outside the image. x: [N, Ci, H, W] -> [N, Co, Ho, Wo].
    """
    N, Ci, H, Wd = x.shape
    Co, _, k, _ = W.shape
    Ho = (H + 2 * pad - k) // stride + 1
    Wo = (Wd + 2 * pad - k) // stride + 1
    xp = np.zeros((N, Ci, H + 2 * pad, Wd + 2 * pad), F)
    xp[:, :, pad:pad + H, pad:pad + Wd] = x
    out = np.zeros((N, Co, Ho, Wo), F)
    Wf = W.astype(F)
    for p in range(k):
        for q in range(k):
            patch = xp[:, :, p:p + stride * (Ho - 1) + 1:stride, q:q + stride * (Wo - 1) + 1:stride]
            out += np.einsum("nchw,oc->nohw", patch, Wf[:, :, p, q], optimize=True)
    return out


def conv2d_adjoint(y: np.ndarray, W: np.ndarray, stride: int, pad: int, in_hw) -> np.ndarray:
    """Adjoint (transpose) of :func:`conv2d`: <conv2d(x), y> = <x, conv2d_adjoint(y)> for all x, y.

    y: [N, Co, Ho, Wo] -> [N, Ci, H, W]. Each output position scatters its
    coefficient back onto the input positions it read.
    """
    N, Co, Ho, Wo = y.shape
    _, Ci, k, _ = W.shape
    H, Wd = in_hw
    gp = np.zeros((N, Ci, H + 2 * pad, Wd + 2 * pad), F)
    Wf = W.astype(F)
    for p in range(k):
        for q in range(k):
            gp[:, :, p:p + stride * (Ho - 1) + 1:stride, q:q + stride * (Wo - 1) + 1:stride] += \
                np.einsum("nohw,oc->nchw", y, Wf[:, :, p, q], optimize=True)
    return gp[:, :, pad:pad + H, pad:pad + Wd]


# ----------------------------------------------------------------------------- forward

def forward(net, x: np.ndarray) -> List[np.ndarray]:
    """Plain fp64 evaluation; x [N, n0]. Returns every node's output, flattened [N, n_v]."""
    sh = shapes(net)
    x = np.asarray(x, F)
    N = x.shape[0]
    outs: List[np.ndarray] = []
    for v, nd in enumerate(net):
        if nd.op == "input":
            o = x
        elif nd.op == "dense":
            o = outs[nd.src] @ nd.W.astype(F).T + nd.b.astype(F)
        elif nd.op == "conv":
            xs = outs[nd.src].reshape((N,) + sh[nd.src])
            o = conv2d(xs, nd.W, nd.stride, nd.pad) + nd.b.astype(F)[None, :, None, None]
            o = o.reshape(N, -1)
        elif nd.op == "relu":
            o = np.maximum(outs[nd.src], 0.0)
        elif nd.op == "add":
            o = outs[nd.src] + outs[nd.src2]
        outs.append(o)
    return outs


# ----------------------------------------------------------------------------- IBP

def split_clamp(l: np.ndarray, u: np.ndarray, s: Optional[np.ndarray]):
    """Pre-activation interval of ReLU neurons inside a branch-and-bound subdomain [SNNV §2.2, §3, §4.3:
    complete verification by beta-CROWN with branch-and-bound; the page names the method only].

    Reading: a split fixes the sign of one ReLU's pre-activation z_i on a subdomain of the input box.
    s[i] = +1 is the subdomain where z_i >= 0 (its interval becomes [max(l, 0), u]); s[i] = -1 the one
    where z_i <= 0 (interval [l, min(u, 0)]); 0 leaves the neuron free. Nothing else changes: bounds
    computed over the whole box stay valid on any part of it. An interval left empty (l > u) means
    the subdomain holds no input, so every bound on it is vacuously sound.
    """
    l = np.asarray(l, F)
    u = np.asarray(u, F)
    if s is None:
        return l, u
    s = np.asarray(s)
    return np.where(s > 0, np.maximum(l, 0.0), l), np.where(s < 0, np.minimum(u, 0.0), u)


def ibp(net, centres: np.ndarray, eps: float, splits: Optional[Dict[int, np.ndarray]] = None):
    """Interval bound propagation in centre/radius form [SNNV §2.1, §4.2].

    The input box is centre c, radius eps (no clipping to any data range: the page
    only speaks of "a specified domain" [SNNV §1]; the plain reading is the L-inf ball).
    Affine node: centre' = W c + b, radius' = |W| r (the exact image of a box under an
    affine map, coordinate-wise). ReLU: clamp both ends, then back to centre/radius.
    Add: centres add, radii add. Under split constraints (relu node -> [B, n] signs, see
    ``split_clamp``) a ReLU first clamps its input interval; a neuron split to z <= 0 outputs
    exactly 0.

    Returns (centre, radius) lists over nodes, each [B, n_v] float64.
    """
    sh = shapes(net)
    c0 = np.asarray(centres, F)
    B = c0.shape[0]
    cs: List[np.ndarray] = []
    rs: List[np.ndarray] = []
    for v, nd in enumerate(net):
        if nd.op == "input":
            c, r = c0, np.full_like(c0, F(eps))
        elif nd.op == "dense":
            Wf = nd.W.astype(F)
            c = cs[nd.src] @ Wf.T + nd.b.astype(F)
            r = rs[nd.src] @ np.abs(Wf).T
        elif nd.op == "conv":
            ci = cs[nd.src].reshape((B,) + sh[nd.src])
            ri = rs[nd.src].reshape((B,) + sh[nd.src])
            c = (conv2d(ci, nd.W, nd.stride, nd.pad) + nd.b.astype(F)[None, :, None, None]).reshape(B, -1)
            r = conv2d(ri, np.abs(nd.W.astype(F)), nd.stride, nd.pad).reshape(B, -1)
        elif nd.op == "relu":
            sp = None if splits is None else splits.get(v)
            l, u = split_clamp(cs[nd.src] - rs[nd.src], cs[nd.src] + rs[nd.src], sp)
            lo = np.maximum(l, 0.0)
            hi = np.maximum(u, 0.0)
            if sp is not None:
                off = np.asarray(sp) < 0
                lo, hi = np.where(off, 0.0, lo), np.where(off, 0.0, hi)
            c, r = (hi + lo) / 2.0, (hi - lo) / 2.0
        elif nd.op == "add":
            c, r = cs[nd.src] + cs[nd.src2], rs[nd.src] + rs[nd.src2]
        cs.append(c)
        rs.append(r)
    return cs, rs


# ----------------------------------------------------------------------------- relaxation

def relax_params(l: np.ndarray, u: np.ndarray, alpha: Optional[np.ndarray] = None):
    """Linear relaxation of h = ReLU(z) for l <= z <= u [SNNV §2.1: slopes lambda_i; §3: alpha].

    Returns (lo, up, t): lower relaxation h >= lo * z, upper relaxation h <= up * z + t.
      * u <= 0 (inactive, tested first): lo = up = t = 0 (h = 0 exactly);
      * else l >= 0 (active):            lo = up = 1, t = 0 (h = z exactly);
      * else (unstable, l < 0 < u):      up = u / (u - l), t = -up * l (the chord), and
                                          lo = alpha clamped to [0, 1] when alpha is given,
                                          otherwise the adaptive choice lo = 1 if u >= -l else 0.
    """
    l = np.asarray(l, F)
    u = np.asarray(u, F)
    lo = np.zeros_like(l)
    up = np.zeros_like(l)
    t = np.zeros_like(l)
    inactive = u <= 0.0
    active = (~inactive) & (l >= 0.0)
    unstable = (~inactive) & (~active)
    lo[active] = 1.0
    up[active] = 1.0
    s = u[unstable] / (u[unstable] - l[unstable])
    up[unstable] = s
    t[unstable] = -s * l[unstable]
    if alpha is None:
        lo[unstable] = np.where(u[unstable] >= -l[unstable], 1.0, 0.0)
    else:
        a = np.asarray(alpha, F)
        if np.isnan(a).any():
            raise ValueError("alpha contains NaN")
        lo[unstable] = np.clip(a[unstable], 0.0, 1.0)
    return lo, up, t


# ----------------------------------------------------------------------------- CROWN

def backward(net, start: int, lam0: np.ndarray, relax: Dict[int, tuple], const0=None):
    """Back-substitute lower-bound rows from node ``start`` to the input [SNNV §1, §2.1].

    lam0 [R, n_start]: the rows' coefficients over node ``start``'s output. For every
    row the result (lam_in [R, n0], const [R]) satisfies, for each x in the domain,
    lam0 . node_start(x) >= lam_in . x + const, given the relaxations in ``relax``
    (relu node -> (lo, up, t) vectors for this centre).

    Nodes are visited in reverse topological order; a node's coefficient matrix is
    complete once all its consumers (which have larger indices) have been visited.
      dense z = W h + b:  const += lam . b;  lam_h += lam W
      conv:               const += sum over (c, i, j) of lam[c, i, j] * b[c];  lam_h += conv^T(lam)
      relu h = ReLU(z):   positive coefficients take the lower relaxation, negative ones the
                          upper: lam_z = lo * max(lam, 0) + up * min(lam, 0);
                          const += min(lam, 0) . t
      add y = a + b:      lam_a += lam; lam_b += lam
    """
    sh = shapes(net)
    R = lam0.shape[0]
    pend: Dict[int, np.ndarray] = {start: np.asarray(lam0, F)}
    const = np.zeros(R, F) if const0 is None else np.asarray(const0, F).copy()

    def put(v, m):
        if v in pend:
            pend[v] = pend[v] + m
        else:
            pend[v] = m

    for v in range(start, -1, -1):
        if v not in pend:
            continue
        lam = pend.pop(v)
        nd = net[v]
        if nd.op == "input":
            return lam, const
        if nd.op == "dense":
            const = const + lam @ nd.b.astype(F)
            put(nd.src, lam @ nd.W.astype(F))
        elif nd.op == "conv":
            co = nd.W.shape[0]
            lam4 = lam.reshape((R,) + sh[v])
            const = const + lam4.reshape(R, co, -1).sum(axis=2) @ nd.b.astype(F)
            put(nd.src, conv2d_adjoint(lam4, nd.W, nd.stride, nd.pad, sh[nd.src][1:]).reshape(R, -1))
        elif nd.op == "relu":
            lo, up, t = relax[v]
            pos = np.maximum(lam, 0.0)
            neg = np.minimum(lam, 0.0)
            const = const + neg @ t
            put(nd.src, pos * lo + neg * up)
        elif nd.op == "add":
            put(nd.src, lam)
            put(nd.src2, lam)
    raise AssertionError("input node not reached")


def concretize(lam_in: np.ndarray, const: np.ndarray, centre: np.ndarray, eps: float) -> np.ndarray:
    """Minimum of lam_in . x + const over the box |x - centre|_inf <= eps [SNNV §1]:
    lam_in . centre - eps * sum |lam_in| + const (attained at x = centre - eps * sign(lam_in))."""
    c = np.asarray(centre, F)
    return lam_in @ c - F(eps) * np.abs(lam_in).sum(axis=1) + const


def crown_pass(net, start: int, lam0: np.ndarray, relax, centre, eps, row_block: int = 4096):
    """backward + concretize for a block of rows; rows are independent, so large passes
    are evaluated ``row_block`` rows at a time (memory only: each row's arithmetic is unchanged)."""
    R = lam0.shape[0]
    out = np.empty(R, F)
    for r0 in range(0, R, row_block):
        r1 = min(R, r0 + row_block)
        lam_in, cst = backward(net, start, lam0[r0:r1], relax)
        out[r0:r1] = concretize(lam_in, cst, centre, eps)
    return out


# ----------------------------------------------------------------------------- full verify

@dataclasses.dataclass
class OracleResult:
    lb: np.ndarray            # [B, R] final lower bound max(IBP, CROWN)
    ub: Optional[np.ndarray]  # [B, R] final upper bound min(IBP, CROWN) (both sides only)
    lb_ibp: np.ndarray        # [B, R]
    ub_ibp: np.ndarray        # [B, R]
    lb_crown: np.ndarray      # [B, R]
    ub_crown: Optional[np.ndarray]
    verified: np.ndarray      # [B, R] bool, lb > 0
    pre_bounds: Dict[int, tuple]  # relu node -> (l, u) [B, n] used for its relaxation
    ibp_bounds: Dict[int, tuple]  # every node -> (l, u) [B, n] from the single IBP pass


def _first_affine_on_input(net, p: int) -> bool:
    nd = net[p]
    return nd.op in ("dense", "conv") and nd.src == 0


def verify(net, centres, eps, C, crown_relus: Optional[Sequence[int]] = None,
           alphas: Optional[Dict[int, np.ndarray]] = None, both_sides: bool = False,
           row_block: int = 4096, splits: Optional[Dict[int, np.ndarray]] = None,
           alpha_inter_iters: int = 0, alpha_inter_lr: float = 0.1) -> OracleResult:
    """IBP, then CROWN intermediate bounds, then the specification pass and decision.

    Readings taken where the page is silent (it names the methods only, [SNNV §1, §2.1]):
      * one IBP pass over the whole network with the plain IBP bounds (later layers
        are not re-propagated from refined bounds);
      * for each ReLU node k in topological order whose pre-activation node p is in
        ``crown_relus`` (None = every ReLU): a CROWN pass from rows [I; -I] over p gives
        l_cr (first half) and -u_cr (second half); IBP-unstable neurons (l < 0 < u) take
        l = max(l_ibp, l_cr), u = min(u_ibp, u_cr); IBP-stable neurons keep the IBP bounds
        (their relaxation is exact either way). When p is a single affine node fed by
        the input, IBP already gives the exact range and no pass is run;
      * every other ReLU keeps its IBP bounds (the IBP substitution of [SNNV §2.1]);
      * specification rows C_b [R, n_L] act on the last node: the CROWN lower bound
        comes from back-substituting C_b; the IBP bound from C applied to the last
        node's interval, C c - |C| r; the final lower bound is the larger (both are sound)
        and a row is verified iff it is > 0 [SNNV §1]. Upper bounds, when asked for,
        are -lower(-C) and C c + |C| r, the final one the smaller;
      * alpha (relu node -> [B, n]) is shared by all rows and passes; missing = adaptive;
      * splits (relu node -> [B, n] in {-1, 0, +1}): each centre's row is one subdomain; the IBP
        pass and the IBP bounds of split neurons are clamped (``split_clamp``), which makes those
        neurons IBP-stable, so they take no CROWN refinement and their relaxation is exact;
      * alpha_inter_iters > 0 (alpha-CROWN for the intermediate bounds; the page names the per-neuron alpha
        tensors [SNNV §3, §4.3], the reading is ours): right after the CROWN pass of a ReLU k whose source p
        is a dense node, the neurons of p still unstable (l < 0 < u) take rows [e_j; -e_j] over p and
        ``ascend`` (alpha_inter_iters Adam steps of size alpha_inter_lr, per-row slopes of every earlier
        ReLU, split multipliers where splits are given) on the network up to p with the relaxations of the
        earlier ReLUs; l_j = max(l_j, best of e_j), u_j = min(u_j, -best of -e_j). The ascent starts at the
        relaxation's slopes, so its best is never below the pass it refines. Layers after k relax with the
        refined bounds.
    """
    centres = np.asarray(centres, F)
    B = centres.shape[0]
    C = np.asarray(C, F)
    R = C.shape[1]
    sh = shapes(net)
    L = len(net) - 1
    cs, rs = ibp(net, centres, eps, splits)
    ibp_b = {v: (cs[v] - rs[v], cs[v] + rs[v]) for v in range(len(net))}
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]
    crown_set = set(relus if crown_relus is None else crown_relus)
    alphas = alphas or {}
    splits = splits or {}

    pre = {k: tuple(x.copy() for x in split_clamp(*ibp_b[net[k].src], splits.get(k))) for k in relus}
    lb_cr = np.empty((B, R), F)
    ub_cr = np.empty((B, R), F) if both_sides else None
    for b in range(B):
        relax: Dict[int, tuple] = {}
        for k in relus:
            p = net[k].src
            if k in crown_set and not _first_affine_on_input(net, p):
                n = _size(sh[p])
                eye = np.eye(n, dtype=F)
                lbs = crown_pass(net, p, np.concatenate([eye, -eye]), relax, centres[b], eps, row_block)
                l_cr, u_cr = lbs[:n], -lbs[n:]
                l0, u0 = pre[k][0][b], pre[k][1][b]
                unst = (l0 < 0.0) & (u0 > 0.0)
                pre[k][0][b] = np.where(unst, np.maximum(l0, l_cr), l0)
                pre[k][1][b] = np.where(unst, np.minimum(u0, u_cr), u0)
                if alpha_inter_iters > 0 and net[p].op == "dense":
                    l1, u1 = pre[k][0][b], pre[k][1][b]
                    idx = np.nonzero((l1 < 0.0) & (u1 > 0.0))[0]
                    if idx.size:
                        sub = net[:p + 1]
                        sg = {j: np.asarray(splits[j][b]) for j in relus if j < p and j in splits} or None
                        best, _ = ascend(sub, centres[b], eps, np.concatenate([eye[idx], -eye[idx]]), relax,
                                         alpha_inter_iters, alpha_inter_lr, sg)
                        m = idx.size
                        l1[idx] = np.maximum(l1[idx], best[:m])
                        u1[idx] = np.minimum(u1[idx], -best[m:])
            a = alphas.get(k)
            relax[k] = relax_params(pre[k][0][b], pre[k][1][b], None if a is None else a[b])
        Cb = C[b if C.shape[0] > 1 else 0]
        rows = np.concatenate([Cb, -Cb]) if both_sides else Cb
        lbs = crown_pass(net, L, rows, relax, centres[b], eps, row_block)
        lb_cr[b] = lbs[:R]
        if both_sides:
            ub_cr[b] = -lbs[R:]
    Cfull = np.broadcast_to(C, (B,) + C.shape[1:])
    zc, zr = cs[L], rs[L]
    lb_ibp = np.einsum("brn,bn->br", Cfull, zc) - np.einsum("brn,bn->br", np.abs(Cfull), zr)
    ub_ibp = np.einsum("brn,bn->br", Cfull, zc) + np.einsum("brn,bn->br", np.abs(Cfull), zr)
    lb = np.maximum(lb_ibp, lb_cr)
    ub = np.minimum(ub_ibp, ub_cr) if both_sides else None
    return OracleResult(lb=lb, ub=ub, lb_ibp=lb_ibp, ub_ibp=ub_ibp, lb_crown=lb_cr, ub_crown=ub_cr,
                        verified=lb > 0.0, pre_bounds=pre, ibp_bounds=ibp_b)


# ----------------------------------------------------------------------------- alpha-CROWN

def _dense_chain(net):
    """Node ids of the affine nodes of a chain input -> affine -> relu -> ... -> dense, where each affine
    node is dense or a convolution, else None."""
    if net[0].op != "input" or net[-1].op != "dense":
        return None
    for v in range(1, len(net)):
        nd = net[v]
        if nd.src != v - 1 or nd.op not in ("dense", "conv", "relu"):
            return None
        if (nd.op != "relu") == (v % 2 == 0):
            return None
    return [v for v in range(len(net)) if net[v].op != "relu" and v > 0]


def spec_bound_alpha(net, centre, eps, rows, relax, alpha_rows, split_signs=None, beta_rows=None):
    """Lower bounds of `rows` (R x n_L) over the box, with one lower slope per (row, unstable neuron)
    [SNNV §3, §4.3: per-neuron alpha tensors], and their gradients with respect to those slopes.

    relax: relu node -> (lo, up, t) vectors (the intermediate-bound relaxation); alpha_rows: relu node
    -> [R, n] slopes in [0, 1], used in place of `lo` for unstable neurons (0 < up < 1). Returns
    (lb [R], grads {relu node: [R, n]}, zero where the neuron is stable).

    Split constraints (beta-CROWN [SNNV §2.2, §4.3], reading: the Lagrangian form of a split): on a
    subdomain where s_i z_i >= 0 (split_signs: relu node -> [n] signs, 0 = free) the rows' function is
    bounded below by itself minus beta_i s_i z_i for any beta_i >= 0 (beta_rows: relu node -> [R, n]), so
    the coefficients over the ReLU's input z gain -beta_i s_i before the back-substitution goes on. With
    beta_rows given the return is (lb, grads, beta_grads), d lb / d beta_i = -s_i G_z,i.

    Forward: the back-substitution of `backward` with row-specific lower slopes. Gradient: reverse
    mode through that chain (layer order from the input up): with G the gradient of lb with respect
    to the coefficients over a node's output,
      input:   G = centre - eps * sign(lam_in)             (from lam . centre - eps |lam|)
      dense:   G_z = G_h W^T + b                           (lam_h = lam_z W,  const += lam_z . b)
      conv:    G_z = conv(G_h) + b per channel             (lam_h = conv^T(lam_z), const += sum lam_z b)
      add:     G_y = G_a + G_b                             (lam_a += lam_y, lam_b += lam_y)
      relu:    dlb/dalpha_i = G_z,i * lam_h,i * [lam_h,i >= 0]   for unstable i
               G_h = G_z * slope + [lam_h < 0] * t         (lam_z = slope * lam_h, const += min(lam_h, 0) t)
    """
    sh = shapes(net)
    L = len(net) - 1
    R = np.asarray(rows).shape[0]
    const = np.zeros(R, F)
    pend: Dict[int, np.ndarray] = {L: np.asarray(rows, F)}
    saved = {}  # relu node -> (lam_h, slope, unstable) used on the way down

    def put(v, m):
        pend[v] = pend[v] + m if v in pend else m

    for v in range(L, 0, -1):
        if v not in pend:
            continue
        lam = pend.pop(v)
        nd = net[v]
        if nd.op == "dense":
            const = const + lam @ nd.b.astype(F)
            put(nd.src, lam @ nd.W.astype(F))
        elif nd.op == "conv":
            lam4 = lam.reshape((R,) + sh[v])
            const = const + lam4.reshape(R, nd.W.shape[0], -1).sum(axis=2) @ nd.b.astype(F)
            put(nd.src, conv2d_adjoint(lam4, nd.W, nd.stride, nd.pad, sh[nd.src][1:]).reshape(R, -1))
        elif nd.op == "relu":
            lo, up, t = relax[v]
            unst = (up > 0.0) & (up < 1.0)
            lo_rows = np.where(unst[None, :], np.asarray(alpha_rows[v], F), lo[None, :])
            slope = np.where(lam >= 0.0, lo_rows, up[None, :])
            const = const + np.minimum(lam, 0.0) @ t
            saved[v] = (lam, slope, unst)
            lam_z = lam * slope
            if beta_rows is not None and v in split_signs:
                lam_z = lam_z - np.asarray(beta_rows[v], F) * np.asarray(split_signs[v], F)[None, :]
            put(nd.src, lam_z)
        else:  # add: both branches receive the rows
            put(nd.src, lam)
            put(nd.src2, lam)
    lam_in = pend[0]
    c = np.asarray(centre, F)
    lb = lam_in @ c - F(eps) * np.abs(lam_in).sum(axis=1) + const
    # G[v]: gradient of lb with respect to the coefficients over node v's output, in topological order
    G = {0: c[None, :] - F(eps) * np.sign(lam_in)}
    grads, bgrads = {}, {}
    for v in range(1, L + 1):
        nd = net[v]
        if nd.op == "dense":
            G[v] = G[nd.src] @ nd.W.astype(F).T + nd.b.astype(F)[None, :]
        elif nd.op == "conv":
            Gz = conv2d(G[nd.src].reshape((R,) + sh[nd.src]), nd.W, nd.stride, nd.pad) + nd.b.astype(F)[None, :, None, None]
            G[v] = Gz.reshape(R, -1)
        elif nd.op == "relu":
            Gz = G[nd.src]
            if v not in saved:  # not an ancestor of the last node: its slopes do not enter lb
                grads[v] = np.zeros((R, _size(sh[v])), F)
                bgrads[v] = np.zeros((R, _size(sh[v])), F)
                G[v] = np.zeros_like(Gz)
                continue
            lam_h, slope, unst = saved[v]
            t = relax[v][2]
            grads[v] = np.where(unst[None, :] & (lam_h >= 0.0), Gz * lam_h, 0.0)
            sg = np.zeros(Gz.shape[1], F) if split_signs is None or v not in split_signs else \
                np.asarray(split_signs[v], F)
            bgrads[v] = -Gz * sg[None, :]
            G[v] = Gz * slope + np.where(lam_h < 0.0, t[None, :], 0.0)
        else:
            G[v] = G[nd.src] + G[nd.src2]
    if beta_rows is not None:
        return lb, grads, bgrads
    return lb, grads


def ascend(net, centre, eps, rows, relax, iters, lr, split_signs=None, betas=(0.9, 0.999), alpha0=None, beta0=None,
           return_state=False):
    """Projected gradient ascent (Adam, step lr, moments ``betas``) on per-row lower slopes of the bound of
    ``rows`` over ``net``'s last node for one centre [SNNV §1 alpha-CROWN; §3 alpha tensors], starting from the
    slopes of ``relax`` (or from ``alpha0``: relu node -> [R, n], clamped to [0, 1]); with split signs (relu node
    -> [n]) the split multipliers beta are optimised with them (from 0, or from ``beta0`` where it has the node,
    projected to beta >= 0; see ``spec_bound_alpha``). Adam's moments start at zero. Returns (best lb over the
    iterates [R], lb at the start [R]), plus the last iterate's (slopes, multipliers) with ``return_state``."""
    b1, b2 = betas
    R = np.asarray(rows).shape[0]
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]

    def adam(x, m1, m2, g, it):
        m1 = b1 * m1 + (1 - b1) * g
        m2 = b2 * m2 + (1 - b2) * g * g
        mh = m1 / (1 - b1 ** (it + 1))
        vh = m2 / (1 - b2 ** (it + 1))
        return x + lr * mh / (np.sqrt(vh) + 1e-8), m1, m2

    alpha = {k: (np.repeat(relax[k][0][None, :], R, axis=0) if alpha0 is None else
                 np.clip(np.asarray(alpha0[k], F), 0.0, 1.0)) for k in relus}
    m1 = {k: np.zeros_like(a) for k, a in alpha.items()}
    m2 = {k: np.zeros_like(a) for k, a in alpha.items()}
    sg = split_signs or None
    beta = None if sg is None else {k: (np.maximum(np.asarray(beta0[k], F), 0.0) if beta0 is not None and k in beta0
                                        else np.zeros((R, len(sg[k])), F)) for k in sg}
    bm1 = None if sg is None else {k: np.zeros_like(x) for k, x in beta.items()}
    bm2 = None if sg is None else {k: np.zeros_like(x) for k, x in beta.items()}
    start = best = None
    for it in range(iters + 1):
        out = spec_bound_alpha(net, centre, eps, rows, relax, alpha, sg, beta)
        lb, g = out[0], out[1]
        if it == 0:
            start, best = lb, lb.copy()
        else:
            best = np.maximum(best, lb)
        if it == iters:
            break
        for k in relus:
            a, m1[k], m2[k] = adam(alpha[k], m1[k], m2[k], g[k], it)
            alpha[k] = np.clip(a, 0.0, 1.0)
        if beta is not None:
            for k in beta:
                gb = np.where(sg[k][None, :] != 0, out[2][k], 0.0)
                x, bm1[k], bm2[k] = adam(beta[k], bm1[k], bm2[k], gb, it)
                beta[k] = np.maximum(x, 0.0)
    if return_state:
        return best, start, alpha, beta
    return best, start


def alpha_crown(net, centres, eps, C, iters=10, lr=0.1, crown_relus=None, betas=(0.9, 0.999), splits=None,
                alpha_inter_iters=0, alpha_inter_lr=0.1, starts=None, return_state=False):
    """Projected gradient ascent (Adam) on per-row lower slopes of the specification pass, starting
    from the adaptive slopes, keeping each row's best bound [SNNV §1 alpha-CROWN; §3 alpha tensors]
    (``ascend`` per centre). Intermediate bounds are those of `verify` (with ``alpha_inter_iters`` > 0, those of
    its intermediate ascent). Returns (best lb [B, R], lb at the adaptive start [B, R]).

    With split constraints (relu node -> [B, n] signs) the multipliers beta of the split neurons
    (beta-CROWN, see ``spec_bound_alpha``) are optimised together with the slopes: one per (row, split
    neuron), starting at 0, the same Adam step, projected to beta >= 0.

    starts (or None): per centre None or (slopes, multipliers) to start from instead (``ascend``'s alpha0 and
    beta0); with ``return_state`` the last iterates per centre are returned as a third element."""
    res = verify(net, centres, eps, C, crown_relus=crown_relus, splits=splits, alpha_inter_iters=alpha_inter_iters,
                 alpha_inter_lr=alpha_inter_lr)
    B, R = res.lb.shape
    C = np.asarray(C, F)
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]
    best = np.empty((B, R), F)
    start = np.empty((B, R), F)
    state = []
    for b in range(B):
        relax = {k: relax_params(res.pre_bounds[k][0][b], res.pre_bounds[k][1][b]) for k in relus}
        rows = C[b if C.shape[0] > 1 else 0]
        sg = None if not splits else {k: np.asarray(splits[k][b]) for k in relus if k in splits}
        a0, b0 = starts[b] if starts is not None and starts[b] is not None else (None, None)
        best[b], start[b], a_fin, b_fin = ascend(net, centres[b], eps, rows, relax, iters, lr, sg, betas, a0, b0,
                                                 return_state=True)
        state.append((a_fin, b_fin))
    if return_state:
        return best, start, state
    return best, start


# ----------------------------------------------------------------------------- branch and bound

def branch_scores(l: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Branching score of ReLU neurons from their pre-activation bounds (reading: the page names
    branch-and-bound only [SNNV §3, §4.3]). An unstable neuron (l < 0 < u) scores the intercept of its
    upper relaxation, -u l / (u - l), the widest vertical gap between the chord and the ReLU; a stable
    one scores -inf and is never split.

    The score decides an index (the neuron to split), so it is taken in the precision the device takes
    it in: the bounds rounded to fp32 and the score evaluated in fp32 arithmetic, in the same order."""
    l = np.asarray(l, F).astype(np.float32)
    u = np.asarray(u, F).astype(np.float32)
    sc = np.full(l.shape, -np.inf, np.float32)
    un = (l < 0.0) & (u > 0.0)
    sc[un] = (-u[un] * l[un]) / (u[un] - l[un])
    return sc


@dataclasses.dataclass
class BabResult:
    status: str       # "verified", "falsified" or "unknown"
    domains: int      # subdomains whose bounds were computed, the whole box included
    iterations: int   # batched evaluations after the whole box
    max_depth: int    # most splits in one evaluated subdomain
    lb: float         # lowest row bound over the subdomains still open at the end (+inf if none)


def bab(net, centre, eps, C, max_domains: int = 1000, batch: int = 16, crown_relus=None, iters: int = 20,
        lr: float = 0.1, alpha_inter_iters: int = 0, alpha_inter_lr: float = 0.1, warm_start: bool = True) -> BabResult:
    """Branch and bound over ReLU splits on top of ``verify`` [SNNV §2.2, §3, §4.3: beta-CROWN with
    branch-and-bound for complete verification; the page names the method only].

    Property: every row of C [R, n_L] is positive at every input of the box centre +- eps.
    A subdomain's row bound is the larger of ``verify``'s bound and the best bound of ``alpha_crown``
    (``iters`` Adam steps of size ``lr`` on the slopes and on the split multipliers beta); with
    ``alpha_inter_iters`` > 0 both take their intermediate bounds from ``verify``'s intermediate ascent (slopes
    and the split multipliers of earlier layers). With ``warm_start`` (reading; the page names the method only) a
    child's ascent starts from its parent's last slopes and multipliers (its new split's multiplier from 0); the
    whole box starts from the adaptive slopes.
    Reading of the search (one plain best-first variant):
      1. the centre is evaluated first, then every row's CROWN minimiser vertex of the whole box
         (``minimiser_attack``); a row < 0 at any of these inputs is a counterexample ("falsified");
      2. the whole box is bounded; if every row's lower bound is > 0 it is "verified";
      3. otherwise the open subdomains are kept with their lowest row bound; each round takes the
         (at most batch // 2) open subdomains with the lowest bound (ties: created first), splits each
         on its highest-scoring neuron (``branch_scores`` over all ReLU layers, ties: first layer, then
         lowest index) into z <= 0 and z >= 0 (in that order), and bounds all children together;
      4. a child is closed when its bounds are contradictory (some l > u: it holds no input) or all its
         rows are > 0; a child with no unstable neuron left and a row <= 0 cannot be split further and
         ends the search ("unknown"), as does a spent budget of ``max_domains`` bounded subdomains;
      5. no open subdomain left: "verified".
    """
    C = np.asarray(C, F)
    centre = np.asarray(centre, F)
    relus = [v for v, nd in enumerate(net) if nd.op == "relu"]
    sizes = [_size(shapes(net)[net[k].src]) for k in relus]
    y = (forward(net, centre[None, :])[-1][0] @ C.T).astype(np.float32)  # a decision: fp32, as on the device
    if np.any(y < 0.0):
        return BabResult("falsified", 0, 0, 0, float(y.min()))
    ya = minimiser_attack(net, centre, eps, C, crown_relus)
    if ya.size and np.any(ya < 0.0):
        return BabResult("falsified", 0, 0, 0, float(ya.min()))

    saved = {}  # a bounded subdomain's splits, in the order made -> its last slopes and multipliers

    def evaluate(domains):
        sp = {k: np.zeros((len(domains), n), np.int8) for k, n in zip(relus, sizes)}
        for i, d in enumerate(domains):
            for (k, j), sign in d.items():
                sp[k][i, j] = sign
        cen = np.repeat(centre[None, :], len(domains), axis=0)
        res = verify(net, cen, eps, C[None], crown_relus=crown_relus, splits=sp, alpha_inter_iters=alpha_inter_iters,
                     alpha_inter_lr=alpha_inter_lr)
        lb = res.lb
        if iters > 0:
            keys = [tuple(d.items()) for d in domains]
            starts = [saved.get(key[:-1]) if warm_start and key else None for key in keys]
            best, _, state = alpha_crown(net, cen, eps, C[None], iters=iters, lr=lr, crown_relus=crown_relus,
                                         splits=sp, alpha_inter_iters=alpha_inter_iters, alpha_inter_lr=alpha_inter_lr,
                                         starts=starts, return_state=True)
            lb = np.maximum(lb, best)
            for key, st in zip(keys, state):
                saved[key] = st
        out = []
        for i in range(len(domains)):
            empty = any(np.any(res.pre_bounds[k][0][i] > res.pre_bounds[k][1][i]) for k in relus)
            best, choice = -np.inf, None
            for k in relus:
                sc = branch_scores(res.pre_bounds[k][0][i], res.pre_bounds[k][1][i])
                j = int(np.argmax(sc))
                if sc[j] > best:
                    best, choice = sc[j], (k, j)
            # the closing test and the best-first order are decisions too: taken on fp32 values
            out.append((float(np.float32(lb[i].min())), empty, choice))
        return out

    return bab_search(evaluate, max_domains, batch)


def minimiser_vertices(net, centre, eps, C, crown_relus=None):
    """Each row's CROWN minimiser vertex of the box centre +- eps (reading; the page names branch-and-bound
    only [SNNV §3, §4.3]): back-substituting row r of C with the relaxations of ``verify``'s intermediate
    bounds gives C_r f(x) >= lam_r . x + const_r on the box, and the linear function is smallest at
    x*_r = centre - eps * sign(lam_r) (sign(0) = 0: the centre's coordinate). Returns (lb, lam_in [R, n0],
    const [R], x* [R, n0]) with lb [R] the whole box's row bounds (larger of IBP and CROWN)."""
    centre = np.asarray(centre, F)
    C = np.asarray(C, F)
    res = verify(net, centre[None, :], eps, C[None], crown_relus=crown_relus)
    relax = {k: relax_params(res.pre_bounds[k][0][0], res.pre_bounds[k][1][0])
             for k, nd in enumerate(net) if nd.op == "relu"}
    lam_in, const = backward(net, len(net) - 1, C, relax)
    return res.lb[0], lam_in, const, centre[None, :] - F(eps) * np.sign(lam_in)


def minimiser_attack(net, centre, eps, C, crown_relus=None) -> np.ndarray:
    """Candidate counterexamples of a property: the fp32 values C f(x*_r) [R candidates, R rows] at every
    row's minimiser vertex (``minimiser_vertices``). A negative entry is a genuine counterexample, an input of
    the box with a negative row. Only a row that the whole box does not prove positive can be negative at its
    vertex, so when every row's bound is > 0 nothing is evaluated (an empty result). The values decide, so
    they are taken in fp32 as on the device."""
    lb, _, _, xs = minimiser_vertices(net, centre, eps, C, crown_relus)
    if np.all(lb > 0.0):
        return np.zeros((0, len(lb)), np.float32)
    return (forward(net, xs)[-1] @ np.asarray(C, F).T).astype(np.float32)


def bab_search(evaluate, max_domains: int, batch: int) -> BabResult:
    """Steps 2-5 of ``bab`` with any bound function: evaluate(list of subdomains) -> one (lowest row bound,
    holds no input, neuron to split next or None) per subdomain. A subdomain is a dict neuron -> sign in
    the order its splits were made (its parent's, then the new one)."""
    (lb0, _, choice0), = evaluate([{}])
    if lb0 > 0.0:
        return BabResult("verified", 1, 0, 0, np.inf)
    if choice0 is None:
        return BabResult("unknown", 1, 0, 0, lb0)
    open_ = [(lb0, 0, {}, choice0)]  # (lowest row bound, creation number, splits, branching neuron)
    domains, iters, depth, seq = 1, 0, 0, 1
    while open_:
        take = min(len(open_), batch // 2, (max_domains - domains) // 2)
        if take <= 0:
            break
        open_.sort(key=lambda d: (d[0], d[1]))
        parents, open_ = open_[:take], open_[take:]
        children = []
        for _, _, sp, nb in parents:
            for sign in (-1, 1):
                d = dict(sp)
                d[nb] = sign
                children.append(d)
        results = evaluate(children)
        domains += len(children)
        iters += 1
        for d, (lbd, empty, nb) in zip(children, results):
            depth = max(depth, len(d))
            num, seq = seq, seq + 1
            if empty or lbd > 0.0:
                continue
            if nb is None:
                return BabResult("unknown", domains, iters, depth, lbd)
            open_.append((lbd, num, d, nb))
    if not open_:
        return BabResult("verified", domains, iters, depth, np.inf)
    return BabResult("unknown", domains, iters, depth, min(d[0] for d in open_))
