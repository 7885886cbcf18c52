"""CPU checker for the LoopVQ path (test infrastructure only).

Only tests, the package smoke check and the benchmark's CPU-baseline leg use
this package.  It shares no code with the CUDA library.
"""
