"""Float64 CPU oracle for the GDN forward pass (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline / reference
leg may import this package.  It shares no code with the CUDA library.
"""
