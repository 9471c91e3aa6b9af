"""Head-sharded (tensor-parallel) KDA layer forward across GPUs.

The layer is independent per head up to the output projection, and the
projection is a sum over heads (y = sum_h x_h W_o[:, h*D_v:(h+1)*D_v]^T, the
"KDA Recurrence" page's head concat followed by the projection).  So each rank
owns a contiguous block of heads and the matching D_v-column block of W_o: it
runs the chunk engine on its heads and projects them (row-parallel
projection), and one all-reduce of the partial outputs (NCCL over NVLink /
NVSwitch between GPUs) gives every rank the layer output.  The final states
stay with the rank that owns their heads.

The partial projections are summed in fp32 (each rank's bf16 partial is
widened before the reduction), so the reduction adds no rounding beyond the
partials' own.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced block of heads [h0, h1) owned by `rank` of `world`
    (the first H % world ranks take one extra head)."""
    if not (0 <= rank < world) or H < 1:
        raise ValueError(f"bad head split: H={H}, world={world}, rank={rank}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def wo_columns(h0: int, h1: int, D_v: int) -> Tuple[int, int]:
    """The W_o columns [c0, c1) that multiply heads [h0, h1) (head-major concat)."""
    return h0 * D_v, h1 * D_v


def shard(x, h0: int, h1: int, head_axis: int = 2):
    """Heads [h0, h1) of a (B, S, H, ...) tensor (or (B, S, H) for beta), contiguous."""
    idx = [slice(None)] * x.ndim
    idx[head_axis] = slice(h0, h1)
    out = x[tuple(idx)]
    return out.contiguous() if hasattr(out, "contiguous") else out.copy()


def reduce_partial_outputs(y_partial, group=None):
    """Sum the ranks' partial layer outputs in fp32 (torch.distributed all_reduce
    on `group`); returns the fp32 sum.  At world size 1 it is the identity."""
    import torch
    import torch.distributed as dist
    y = y_partial.float()
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


def tp_forward(local_layer: Callable, rank: int, world: int, H: int, D_v: int, group=None):
    """One head-sharded layer forward: `local_layer(h0, h1, c0, c1)` returns this
    rank's partial output (its heads' normalised, gated activations projected by
    W_o[:, c0:c1]) and its heads' final states; the partials are all-reduced.
    Returns (y fp32, final states of heads [h0, h1), (h0, h1))."""
    h0, h1 = head_range(H, world, rank)
    c0, c1 = wo_columns(h0, h1, D_v)
    y_part, s_local = local_layer(h0, h1, c0, c1)
    return reduce_partial_outputs(y_part, group), s_local, (h0, h1)


def kda_forward_tp(query, key, value, decay_logits, write_strength, output_gate_logits, output_projection_cols,
                   initial_state=None, g_min=-5.0, eps=1e-6, *, H: int, rank: int, world: int, group=None,
                   out_dtype=None):
    """Head-sharded layer forward on this rank's GPU.

    The per-head inputs are this rank's shard, heads ``head_range(H, world, rank)``
    of the full (B,S,H,.) tensors (what a tensor-parallel input projection
    produces); ``output_projection_cols`` is the matching (D_model, H_r*D_v)
    column block of W_o.  Every rank receives the full layer output
    (B, S, D_model) in ``out_dtype`` (default: the input dtype) and keeps the
    final states of its own heads (B, H_r, D_k, D_v) fp32.
    """
    import torch
    from .api import chunk_fwd, out_proj
    h0, h1 = head_range(H, world, rank)
    B, S, Hr, Dk = query.shape
    if Hr != h1 - h0:
        raise ValueError(f"rank {rank} of {world} owns heads [{h0}, {h1}) but got {Hr} heads")
    Dv = value.shape[-1]
    if output_projection_cols.shape[1] != Hr * Dv:
        raise ValueError("output_projection_cols must hold this rank's H_r * D_v columns of W_o")

    def local(h0_, h1_, c0, c1):
        x, sf = chunk_fwd(query, key, value, write_strength.reshape(B, S, Hr), z=decay_logits, g_min=g_min,
                          initial_state=initial_state, gate_logits=output_gate_logits, eps=eps)
        return out_proj(x.view(B, S, Hr * Dv), output_projection_cols), sf

    y, sf, _ = tp_forward(local, rank, world, H, Dv, group)
    return y.to(out_dtype or query.dtype), sf
