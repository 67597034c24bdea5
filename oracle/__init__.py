"""fp64 CPU oracle of the TileQ MoE-layer forward.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the layer computes, written from the TileQ paper
("TileQ: Efficient Low-Rank Quantization of Mixture-of-Experts with 2D
Tiling").  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference arm of ``bench.py`` may import it.  The CUDA library never calls
it, shares no code with it, and fails loudly instead of falling back to it.

Parity status of each function is listed in ``oracle.tileq.PINS``.
"""
from .tileq import *  # noqa: F401,F403
