"""Sequence-sharded SELECT step: one sequence's KV cache split by rows across the
ranks of a process group (rank order = row order), exact with respect to the
one-GPU step.

Every stage runs in libtsa (``tsa_shard_select``, ``tsa_shard_merge``,
``tsa_shard_attend``, ``tsa_shard_combine``); this module only moves the two
exchanged buffers between ranks with ``torch.distributed`` all-gathers:

1. each rank scores its rows and keeps its own top-k (score, global row) pairs;
2. all-gather of the candidates, then every rank merges them into the same
   global top-k (the global top-k rows are each among their shard's top-k);
3. each rank attends over the selected rows it holds: its normalised output and
   the base-2 log-sum-exp of its logits;
4. all-gather of those parts, then the exact split-K combine.

The exchanged bytes per step are small: R x units x k x 8 bytes of candidates
and R x B x Hq x (128 + 1) x 4 bytes of parts.  ``ops`` is the library binding;
tests on CPU pass a stand-in with the same four calls to check the exchange
over the gloo backend.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


def _gather(t: torch.Tensor, group, stream) -> torch.Tensor:
    """[world, *t.shape]: every rank's t in rank order (on `stream` when given)."""
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    if stream is not None:
        with torch.cuda.stream(stream):
            dist.all_gather(parts, t.contiguous(), group=group)
            return torch.stack(parts)
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def sharded_select_step(Q, K_shard, V_shard, shard_lens, k_per_seq, k_max: int, scale: float, row0: int, O, idx,
                        ws, group=None, ops=binding, stream=None):
    """One SELECT layer over a row-sharded cache.  This rank holds rows
    [row0, row0 + Ncap_r) of every unit in K_shard, V_shard [B, Hkv, Ncap_r, d]
    with shard_lens[b] = clamp(len_b - row0, 0, Ncap_r).  Writes the global
    top-k into idx [B, Hkv, k_max] and the attention output into O [B, Hq, d]
    (the same on every rank).  ws: ``ops.shard_workspace_size`` bytes.  stream: a
    torch.cuda.Stream (the all-gathers run on it too) or None (torch's current stream)."""
    B, Hq, d = Q.shape
    Hkv = K_shard.shape[1]
    dev = Q.device
    shape = ops.shape_of(Q, K_shard)
    cand_scores = torch.empty(B, Hkv, k_max, dtype=torch.float32, device=dev)
    cand_rows = torch.empty(B, Hkv, k_max, dtype=torch.int32, device=dev)
    ops.shard_select(Q, K_shard, shard_lens, k_per_seq, k_max, scale, row0, cand_scores, cand_rows, ws, stream)
    all_scores, all_rows = _gather(cand_scores, group, stream), _gather(cand_rows, group, stream)
    ops.shard_merge(all_scores, all_rows, shape, k_per_seq, k_max, idx, ws, stream)
    O_part = torch.empty(B, Hq, d, dtype=torch.float32, device=dev)
    lse_part = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ops.shard_attend(Q, K_shard, V_shard, shard_lens, idx, k_per_seq, k_max, row0, scale, O_part, lse_part, ws,
                     stream)
    ops.shard_combine(_gather(O_part, group, stream), _gather(lse_part, group, stream), shape, O, stream)
    return O, idx
