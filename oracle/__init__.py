"""fp64 CPU oracle for the CSA/HCA hybrid-attention hot path.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the library's product path.
"""
