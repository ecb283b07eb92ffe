"""B200-native MoE routing hot path.

Import :mod:`expert_load_balancing_tcgen05_b200.moe` for the library binding
(it loads ``libmoeroute.so`` and fails loudly if it is missing) and
:mod:`expert_load_balancing_tcgen05_b200.workloads` for the seeded synthetic
inputs.  Importing the package itself loads nothing.
"""
__all__ = ["moe", "workloads"]
