"""Seeded synthetic workloads shared by the tests, the oracle and the benchmark."""

from .synth import (HYPER, Workload, make, make_block_permuted, make_random,  # noqa: F401
                    make_sweep_blocks, sweep_batch, sweep_block_shape, sweep_shape)
