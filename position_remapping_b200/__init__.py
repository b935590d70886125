"""ropeattn: causal attention with RoPE at remapped positions on B200 (sm_100a).

The compute path is the C-ABI library ``libropeattn.so`` (include/ropeattn.h);
``position_remapping_b200.ropeattn`` binds it. Attribute access below loads the
library lazily so that ``position_remapping_b200.inputs`` stays importable
without it; any compute call without the library raises ImportError.
"""
from .inputs import (BIFOCAL, ENDPROMPT, NOPE, PAIR_ADJACENT, PAIR_HALF, PERIODIC, STANDARD,  # noqa: F401
                     MapParams, Workload, WORKLOADS, make_qkv)

_API = ("prefill", "prefill_chunk", "cache_write", "decode", "decode_cache", "prefill_three_call", "decode_unfused",
        "wait_selftest", "posmap", "status", "version", "prefill_workspace_size", "prefill_chunk_workspace_size",
        "decode_workspace_size", "RopeAttnError")


def __getattr__(name):
    if name in _API:
        from . import ropeattn
        return getattr(ropeattn, name)
    raise AttributeError(name)
