"""Condensate ("Topological") attention for NVIDIA B200 (sm_100a).

The computation lives in the CUDA library `libcondensate_attn.so` behind the
C ABI declared in `include/condensate_attn.h`; this package is its ctypes
binding and the build step that produces it.
"""
from .binding import (  # noqa: F401
    CA_BF16, CA_F32, CA_OK, CondensateError, LIB_PATH,
    condensate_attn_decode, condensate_attn_decode_chunks,
    condensate_attn_decode_shard_attend, condensate_attn_decode_shard_combine,
    condensate_attn_decode_shard_select,
    condensate_attn_decode_shard_workspace_size,
    condensate_attn_prefill, condensate_attn_status,
    condensate_attn_workspace_size, condensate_attn_workspace_size_ex, load,
    status_string,
)
from .sharded import decode_sharded, shard_bounds  # noqa: F401,E402
