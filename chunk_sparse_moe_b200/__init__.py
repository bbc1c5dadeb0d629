"""BlockFFN chunk-union layer forward on B200 (sm_100a).

Python binding of libblockffn.so: ``route``, ``chunk_union``, ``forward`` take
CUDA torch tensors, check them, and pass raw device pointers and the current
CUDA stream to the C ABI (include/blockffn.h).  All arithmetic runs in the
library's kernels; PyTorch only provides device memory and streams.
"""
from .api import (BlockFFNError, Workspace, chunk_union, debug_set_trace, debug_skip_flag, device_status,
                  forward,
                  num_sms, residual_layernorm, route, set_wait_limit_ns, version, workspace_bytes)

__all__ = ["BlockFFNError", "Workspace", "chunk_union", "debug_set_trace", "debug_skip_flag", "residual_layernorm",
           "device_status",
           "forward", "num_sms", "route", "set_wait_limit_ns", "version", "workspace_bytes"]
