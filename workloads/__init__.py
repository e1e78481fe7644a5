"""Seeded synthetic QSA workloads shared by the tests and the benchmark."""
from . import synth, configs  # noqa: F401
