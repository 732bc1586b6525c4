"""fp64 CPU oracle of the DeepSeekMoE layer (test infrastructure only).

Only the tests, the package's smoke check and the benchmark's CPU-baseline leg
may import this package. It shares no code with the CUDA path.
"""
from . import moe_oracle, fp8  # noqa: F401
