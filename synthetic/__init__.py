"""Seeded synthetic inputs for the global self-attention layer over N views.

This module only draws numbers and lays them out as tokens.  It holds none of
the attention method's arithmetic (no pooling, no scores, no softmax, no gate):
both the CPU oracle and the CUDA library are fed from it, and nothing else is
shared between them.

Token layout (the problem statement of the Speed3R pages, "Background and
problem definition"): frame f contributes ``S`` special tokens followed by its
``Hp x Wp`` patch tokens in row-major order; frames are concatenated.  Q, K, V
are ``[T, H, D]`` bf16 with ``T = N * (S + Hp * Wp)``.
"""

from .workloads import (  # noqa: F401
    Workload,
    WORKLOADS,
    Inputs,
    generate,
    gaussian_inputs,
    scene_inputs,
)
