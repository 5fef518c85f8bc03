"""Seeded synthetic inputs and workload shapes shared by the oracle tests, the GPU
tests and the benchmark.  Holds no arithmetic of the method itself."""
from . import configs, gen  # noqa: F401
