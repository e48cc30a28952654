"""Absorbed Multi-Head Latent Attention decode for B200 (sm_100a).

The product is the C-ABI library ``libmla.so`` (header ``include/mla.h``),
built from the CUDA sources under ``csrc/``. ``mla`` is its ctypes binding
(same function names); ``runtime`` drives whole decode steps through it.
"""

from . import mla  # noqa: F401
