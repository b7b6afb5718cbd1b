"""fp64 CPU oracle for the packed variable-length attention forward pass.

Test infrastructure: only the tests, the smoke check and the benchmark's
CPU-baseline leg use it.  It shares no code with the CUDA product path.
"""
