"""Seeded synthetic inputs for absorbed MLA decode.

This package is shared by the CPU oracle's tests and by the CUDA path's tests
and benchmark. It holds none of the method's arithmetic: it only draws seeded
random numbers, rounds them to bf16 storage, and lays them out (paged pool,
block table, per-step query and new-token rows).
"""

from .inputs import *  # noqa: F401,F403
