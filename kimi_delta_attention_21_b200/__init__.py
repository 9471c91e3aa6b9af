"""B200 (sm_100a) Kimi Delta Attention layer forward.

The compute lives in ``libkda.so`` (hand-written CUDA behind the C ABI of
``include/kda.h``); this package only marshals torch tensors into it.
"""
from ._lib import KDAError, load as load_library  # noqa: F401
from .api import (chunk_bwd, chunk_fwd, chunk_workspace_bytes, decode_step, dplr_chunk_fwd,  # noqa: F401
                  dplr_recurrent_fwd, gate,
                  gdn_chunk_fwd, kda_decode,
                  kda_forward, norm_gate, out_norm_gate_proj, out_proj, recurrent_bwd)

__all__ = ["chunk_bwd", "chunk_fwd", "chunk_workspace_bytes", "decode_step", "dplr_chunk_fwd", "dplr_recurrent_fwd", "gate", "gdn_chunk_fwd", "kda_decode",
           "kda_forward", "norm_gate", "out_norm_gate_proj", "out_proj", "recurrent_bwd", "KDAError", "load_library"]
