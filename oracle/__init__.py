"""CPU oracle for the selective-SSM mixer core (test infrastructure only).

Only tests, the package smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library and its Python binding never do.
"""
