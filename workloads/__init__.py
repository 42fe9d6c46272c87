"""Seeded synthetic workloads shared by the tests, the oracle and the benchmark."""

from .synth import HYPER, Workload, make, make_random, sweep_batch, sweep_shape  # noqa: F401
