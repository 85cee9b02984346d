"""Sequence sharding over a process group: every rank holds one contiguous
segment of the same sequences (rank order = token order) and computes the
outputs of its segment.

The only exchange is the segments' states (the recurrence's resume point,
"MiniMax-01与Lightning Attention", section 4.1): each rank computes K^T V of
its segment (la_segment_state), the states are all-gathered (B*Hkv*d*d*4
bytes per rank), each rank takes S0 plus the states of the ranks before it
(la_state_prefix) and runs la_forward_state from that state.  The arithmetic
runs in the library's kernels; this module only moves tensors.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def gather_states(state: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' states stacked in rank order: [world, *state.shape]."""
    world = dist.get_world_size(group)
    flat = state.contiguous().view(-1)
    out = torch.empty(world * flat.numel(), dtype=state.dtype, device=state.device)
    dist.all_gather_into_tensor(out, flat, group=group)  # rank r's elements at chunk r
    return out.view(world, *state.shape)


def forward_sequence_parallel(q, k, v, S0=None, group=None, chunk: int = 64, stream=None):
    """Outputs of this rank's segment q [B,Hq,n,d], k, v [B,Hkv,n,d] (bf16,
    CUDA) of sequences sharded over `group`; S0 [B,Hkv,d,d] fp32 (nullable)
    the state before the first segment, the same on every rank.  Returns
    (o, S): S is the state after this rank's segment (on the last rank the
    final state of the whole sequences)."""
    rank = dist.get_rank(group)
    states = gather_states(api.la_segment_state(k, v, chunk=chunk, stream=stream), group)
    S = api.la_state_prefix(states, rank, S0=S0, stream=stream)
    o = api.la_forward_state(q, k, v, S=S, chunk=chunk, stream=stream)
    return o, S
