"""B200-native Kimi Delta Attention (KDA) forward: chunkwise prefill and
single-step decode, as CUDA kernels for sm_100a behind the C ABI in
``include/kda.h``.  This package holds the ctypes binding (``kda``), the
in-tree build (``build``) and the seeded synthetic inputs (``inputs``)."""
from .kda import (KdaError, chunk_fwd, chunk_fwd_host, chunk_fwd_noalloc, decode_step,  # noqa: F401
                  gdn_chunk_fwd, gdn_decode_step, inject_timeout, load, release_workspace,
                  set_wait_limit, status_string, stream_status, workspace_bytes)

__all__ = ["chunk_fwd", "chunk_fwd_host", "chunk_fwd_noalloc", "decode_step", "gdn_chunk_fwd",
           "gdn_decode_step", "stream_status", "status_string", "workspace_bytes", "release_workspace",
           "set_wait_limit", "inject_timeout", "load", "KdaError"]
