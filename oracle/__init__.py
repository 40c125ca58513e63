"""Oracle for the ZeRO partitioned mixed-precision Adam step.

TEST INFRASTRUCTURE ONLY: a plain single-threaded CPU statement of the step
(zero_ref.c) with a numpy/ctypes face (zero_ref.py). The test suite, the
package's smoke check and the benchmark's CPU-baseline leg may use it; the
CUDA library and its Python binding never import it.
"""
