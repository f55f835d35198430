"""B200-native linear bound propagation (IBP + CROWN with alpha-slope ReLU relaxation).

The compute path is the CUDA library ``libvf.so`` built from ``csrc/`` (sm_100a);
:mod:`linear_bound_propagation_b200.vf` is its thin ctypes binding. Importing this
package does not load the library; the first call into :mod:`.vf` does, and
raises if the library is missing.
"""
__all__ = ["synth", "vf"]
