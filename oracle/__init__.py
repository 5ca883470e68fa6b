"""CPU oracle for the routed NVFP4 MoE site -- TEST INFRASTRUCTURE ONLY.

A plain, slow fp64 restatement of what the site computes, used to prove the
CUDA path. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference legs may import it; the library never does, and the
two share no code (only the seeded generator in
``routed_nvfp4_expert_b200.synthetic``, which holds none of the arithmetic).
"""
from . import formats, site  # noqa: F401
