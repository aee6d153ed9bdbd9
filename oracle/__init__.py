"""CPU oracle (test infrastructure only).

Plain, slow, fp64 restatement of what the attention forward and its backward
pass compute, plus the FP8 preparation (exact rotation, block quantisation
decided in the kernel's fp32 precision).
Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline leg may import
this package; the CUDA library and its binding never do, and this package never
imports them.
"""
from .attention import attention_fp64, attention_probs_fp64  # noqa: F401
from .attention_bwd import attention_bwd_fp64  # noqa: F401
from .fp8 import (e4m3_decode, e4m3_encode, prepare_fp8, dequantize,  # noqa: F401
                  rotate, quantize_tiles)
