"""CPU fp64 oracle for RIPE caching and verification attention.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the package smoke check and by
the benchmark's CPU-baseline leg, never by the library's product path.
"""
