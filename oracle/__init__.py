"""CPU oracle for the MoE layer step.  TEST INFRASTRUCTURE ONLY: imported by the
tests, the smoke check and the benchmark's CPU-baseline leg, never by the library."""
