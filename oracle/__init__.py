"""CPU oracle for the DMS inference path.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may use this package; the product path never does.
"""
