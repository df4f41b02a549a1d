"""libkda: Kimi Delta Attention forward (chunked prefill and recurrent decode)
as hand-written sm_100a CUDA behind a C ABI (include/kda.h).

``kda`` is the ctypes binding; ``build`` compiles the library in-tree;
``synth`` draws the seeded synthetic inputs used by tests and benchmarks.
"""
from .kda import (KdaError, chunk_fwd, kda_chunk_fwd, kda_chunk_fwd_plan, kda_chunk_fwd_workspace_size,  # noqa: F401
                  kda_get_device_status, kda_recurrent_step, kda_status_string, kda_version, load_library,
                  recurrent_step)
