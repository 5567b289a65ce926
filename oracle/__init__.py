"""CPU oracle for the Lighthouse layer (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path never does.
"""
