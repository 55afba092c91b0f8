"""CPU oracle for the fused FP8 ReLU^2 MLP block.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` use it.  It shares no code with the CUDA
library (no kernels, headers, helpers, tables or constant generators), and
it imports nothing from ``fp8_relu_mlp_b200``.
"""
from . import ref  # noqa: F401
