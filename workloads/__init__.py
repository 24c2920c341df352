"""Seeded synthetic input generators shared by the tests, the benchmark and
the oracle harness (no method arithmetic lives here)."""
