"""CPU fp64 oracle for absorbed MLA decode (test infrastructure only).

Only tests, the package smoke check and the benchmark's CPU-baseline leg use
this package; the CUDA product path never imports it.
"""
