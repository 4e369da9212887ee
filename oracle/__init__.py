"""CPU oracle for the centroid-residual KV-cache codec and compressed-history
attention.  TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and
the benchmark's CPU-baseline leg, never by the library."""
