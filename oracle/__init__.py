"""fp64 CPU oracle for jagged HSTU attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the CPU-baseline
leg of the benchmark, never by the product path.
"""
