"""B200-native DualQuant dual-scale BCD weight-quantization solver.

The solver runs as hand-written CUDA kernels for sm_100a behind the C ABI in
``include/dq.h`` (``libdq.so``); :mod:`.binding` marshals torch tensors to it.
Importing the package does not load the library; the first call does, and it
raises if the library is missing or no CUDA device is present.
"""
from .binding import (DQError, Format, dq_act_quant, dq_rtn, dq_solve, dq_solve_batched, dq_solve_static, output_nbytes,  # noqa: F401
                      load_library, solve, rtn, workspace_bytes)
