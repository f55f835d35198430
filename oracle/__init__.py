"""fp64 CPU oracle for linear bound propagation (IBP + CROWN with alpha-slope ReLU relaxation).

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the package-level
smoke check and the benchmark's CPU-baseline leg may import or run anything
under this directory. The CUDA path never calls it and shares no code with it;
both are fed by the seeded generator in ``linear_bound_propagation_b200.synth``
(which draws numbers only).

Source page for the method: "Scaling Neural Network Verification with Tensor
Parallelism and Fully Sharded Data Parallelism" (gist.science summary of arXiv
2606.09377). The page names IBP, CROWN and alpha-CROWN, the linear relaxation
matrices A, the ReLU relaxation slopes and the per-neuron alpha tensors, but
prints none of their equations, no worked example and no bound value. The
functions in ``lbp.py`` therefore follow the plainest standard reading of those
named methods; each reading is stated where it is taken.

Parity status per function (what pins it, all in tests/test_oracle_*.py):
  ibp, forward, conv2d, conv2d_adjoint  -- pinned (library conv, adjoint identity,
                                           exact ranges, soundness sampling)
  relax_params                          -- pinned (hand 1-D/2-D examples, special cases)
  backward, concretize                  -- pinned (linear and all-stable closed forms,
                                           attained vertices, hand examples, LP sandwich,
                                           pointwise L(x) <= f(x))
  verify (intermediate + spec passes)   -- pinned (2-D exact ranges, soundness,
                                           one-hidden-layer ordering, monotonicity in eps)
  spec_bound_alpha, ascend, alpha_crown -- pinned (central differences, hand optimum, Adam's closed-form
                                           first steps, soundness of optimised bounds)
  verify(alpha_inter_iters=...)         -- pinned (one-neuron closed form of the ascent, the triangle LP
                                           bounding and reached by the optimised intermediate bounds,
                                           soundness by sampling, never looser than plain)
  split_clamp, splits in ibp / verify,  -- pinned (soundness on the subdomain by sampling, the
  beta in spec_bound_alpha / alpha_crown   full-split affine closed form, weak and strong LP
                                           duality, central differences for beta)
  branch_scores, bab, bab_search        -- pinned (exact 2-D ranges and sampling: never a wrong
                                           "verified" or "falsified"; splitting verifies
                                           properties the whole-box bound leaves open)
  minimiser_vertices, minimiser_attack  -- pinned (brute force over the box's vertices: the vertex attains
                                           the CROWN bound; exact 2-D ranges: only false properties are
                                           falsified, most clearly false ones without a split)
"""
from .lbp import (  # noqa: F401
    shapes, conv2d, conv2d_adjoint, forward, ibp, relax_params, backward, concretize,
    crown_pass, verify, OracleResult, spec_bound_alpha, ascend, alpha_crown, split_clamp, branch_scores, bab,
    bab_search, BabResult, minimiser_vertices, minimiser_attack,
)
