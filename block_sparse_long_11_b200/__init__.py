"""MoBA (Mixture of Block Attention) causal prefill forward on B200 (sm_100a).

The compute lives in libmoba.so (hand-written CUDA, C ABI in include/moba.h);
this package is its thin binding.  Importing it does not load the library;
the first call does, and raises if the library has not been built.
"""
from ._lib import (EXPORTS, LIB_PATH, MobaError, Workspace, decode_kbar_cache,
                   default_chunk_tokens, lib, moba_backward, moba_check, moba_decode,
                   moba_decode_init,
                   moba_forward, moba_forward_full, moba_full_workspace_size, moba_gate,
                   moba_gate_noalloc, moba_status_string, moba_workspace_size)

__all__ = ["EXPORTS", "LIB_PATH", "MobaError", "Workspace", "default_chunk_tokens", "lib",
           "decode_kbar_cache", "moba_backward", "moba_check", "moba_decode", "moba_decode_init",
           "moba_forward", "moba_forward_full", "moba_full_workspace_size",
           "moba_gate", "moba_gate_noalloc", "moba_status_string", "moba_workspace_size"]
