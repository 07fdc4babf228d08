"""Seeded synthetic workloads and input generators (shared by tests, the benchmark and the
oracle's tests; holds none of the method's arithmetic)."""
from . import configs, gen  # noqa: F401
