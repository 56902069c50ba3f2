"""B200-native (sm_100a) Kimi Delta Attention forward pass.

The compute lives in ``libkda.so`` (CUDA kernels behind the C ABI declared in
``include/kda.h``); ``gated_delta_rule_70_b200.kda`` is its ctypes binding and
``gated_delta_rule_70_b200.workloads`` draws the seeded synthetic inputs.
"""

from .kda import (KdaError, KdaLibraryError, decode_multi, decode_step, kernel_times,  # noqa: F401
                  kernel_timing, load_library, prefill, prefill_workspace_size, prologue, recurrence,
                  recurrence_workspace_size, status_string)
