"""CPU oracle (float64, NumPy) for the fused Hadamard rotate + quantize path.

Test infrastructure: imported only by the tests, the smoke check and the CPU
baseline leg of the benchmark.  It shares no code with the CUDA library.
"""
from .hadamard_oracle import *  # noqa: F401,F403
from .hadamard_oracle import __all__  # noqa: F401
