"""B200-native (sm_100a) fused causal attention, forward and backward.

The library is a C ABI (include/forge_attn.h) over hand-written CUDA kernels
(csrc/).  ``_lib`` binds the ABI under its own names; ``attention`` adds a
torch-tensor front end; ``workloads`` holds the benchmark shapes and seeded
inputs.  Importing this package does not load the CUDA library; the first call
does, and fails loudly if it is missing.
"""
from . import workloads  # noqa: F401
from ._lib import ForgeAttnError, library_path, load  # noqa: F401
from .attention import (attn_bwd, attn_fwd, check_device_error, to_fp16,  # noqa: F401
                        workspace_bytes)
