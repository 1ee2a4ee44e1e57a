"""fp64 CPU oracle for the prunable 2-bit KV decode path.

TEST INFRASTRUCTURE ONLY: only the test suite, the package smoke check and the
CPU-baseline leg of the benchmark may import it.  It shares no code with the
CUDA library.
"""
