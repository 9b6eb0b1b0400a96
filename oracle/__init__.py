"""Float64 CPU oracle for the partially synchronized row-parallel layer (test infrastructure
only: imported by the tests, the smoke check and the bench's CPU-baseline leg, never by the
product path)."""
