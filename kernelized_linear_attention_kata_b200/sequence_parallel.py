"""Sequence-sharded chunked forward: one contiguous slice of the sequence per
rank, one exchange between the ranks.

The state of causal linear attention is a sum over tokens (the RNN view of
the "線形注意" definition; the scan across chunks of the KATA explainer,
section 2.3, taken one level up), so rank r's slice only needs the sum of the
states of the slices before it:

1. each rank computes its slice's state (S_r, z_r) in the library
   (``kata_chunked_state``);
2. the exclusive prefix over ranks, carry_r = sum_{r' < r} (S_r', z_r'), is
   one all-reduce: rank r' places its state in slots r' + 1 .. N - 1 of a
   zero [N, n] buffer, the collective sums the buffers, and rank r reads slot
   r (the additions happen inside the collective, NCCL over NVLink on GPUs);
3. each rank runs its forward from carry_r (``kata_fwd_chunked_from_state``);
   the last rank's final state is the whole sequence's.

Slices are in rank order along T; every rank holds the same B, H.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def exclusive_prefix_over_ranks(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of the ranks' `flat` tensors over the ranks before this one
    (zeros on rank 0), by one all-reduce of a [world, n] buffer. Without a
    process group there is one rank, and the carry is zero."""
    if not dist.is_initialized():
        return torch.zeros_like(flat)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    buf = torch.zeros((world, flat.numel()), dtype=flat.dtype, device=flat.device)
    buf[rank + 1:] = flat.reshape(1, -1)
    dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    return buf[rank].reshape(flat.shape)


def fwd_chunked_sequence_parallel(q, k, v, C, feature="psd", group=None, return_state=False,
                                  out=None):
    """This rank's outputs for its slice q, k, v [B, H, T_r, d] of a sequence
    cut along T in rank order (into `out` if given). With return_state, also
    the state after the slice (on the last rank: the state of the whole
    sequence)."""
    S_loc, z_loc = api.chunked_state(k, v, C, feature)
    nS = S_loc.numel()
    carry = exclusive_prefix_over_ranks(torch.cat([S_loc.reshape(-1), z_loc.reshape(-1)]), group)
    S0 = carry[:nS].view_as(S_loc)
    z0 = carry[nS:].view_as(z_loc)
    o = torch.empty_like(v) if out is None else out
    if return_state:
        S_out, z_out = torch.empty_like(S_loc), torch.empty_like(z_loc)
        api.kata_fwd_chunked(q, k, v, o, C, feature, S_out=S_out, z_out=z_out, S0=S0, z0=z0)
        return o, S_out, z_out
    api.kata_fwd_chunked(q, k, v, o, C, feature, S0=S0, z0=z0)
    return o
