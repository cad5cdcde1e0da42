"""Seeded synthetic inputs for top-k context-sparse decode attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no scoring, no selection, no softmax).  Both the CUDA path
and the fp64 oracle consume what it returns, so it is the one piece they share.

Draw recipe (all draws from one ``torch.Generator`` seeded with ``seed``,
on the device given; the CPU and CUDA generators give different streams, so a
workload is identified by (seed, device)):

1. ``Q[B, Hq, d]``  ~ N(0, 1), rounded to bf16 (round-to-nearest-even).
2. For each sequence b in order: ``K[b]`` ~ N(0, 1) in fp32, then the planted
   heavy keys are added (below), then rounded to bf16.
3. For each sequence b in order: ``V[b]`` ~ N(0, 1), rounded to bf16.

Planted heavy keys: for each (b, kv-head) the generator picks
``round_half_up(frac * len_b)`` distinct rows uniformly in ``[0, len_b)`` and,
for each, one query head h of that kv-head's group uniformly; the row becomes
``3 * q_h / ||q_h||_2 + N(0, I)`` (the N(0, I) is the row's own draw from step 2).
This stands in for the "heavy hitter" keys that make real attention sparse.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

D_HEAD = 128


def round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


@dataclass
class DecodeInputs:
    """One decode layer's tensors (bf16 Q/K/V, int32 lengths)."""

    Q: torch.Tensor  # [B, Hq, d] bf16
    K: torch.Tensor  # [B, Hkv, Ncap, d] bf16
    V: torch.Tensor  # [B, Hkv, Ncap, d] bf16
    seq_lens: torch.Tensor  # [B] int32
    planted: list = field(default_factory=list)  # per (b, kvh): LongTensor of planted rows


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    return g


def draw_lengths(B: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """Per-sequence lengths uniform on the integers [lo, hi] (CPU generator)."""
    g = _gen(seed, "cpu")
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)


def decode_layer(B: int, Hq: int, Hkv: int, Ncap: int, seq_lens, *, plant_frac: float = 0.0,
                 seed: int = 0, device="cpu", d: int = D_HEAD, Q: torch.Tensor | None = None,
                 tail_fill: float | None = None) -> DecodeInputs:
    """Draw one layer's Q, K, V (recipe in the module docstring).

    ``seq_lens`` is an int or a length-B sequence; rows at or past ``len_b`` are
    still drawn (they are cache capacity) unless ``tail_fill`` is given, in
    which case K and V rows there are set to that value so that a kernel which
    reads past the valid length produces visibly wrong output.
    ``Q`` may be passed in (index-reuse stacks drift one query across layers);
    then step 1 is skipped.
    """
    assert Hq % Hkv == 0
    g = _gen(seed, device)
    dev = torch.device(device)
    if isinstance(seq_lens, int):
        lens = torch.full((B,), seq_lens, dtype=torch.int32)
    else:
        lens = torch.as_tensor(seq_lens, dtype=torch.int32).clone().cpu()
    assert lens.numel() == B and int(lens.max()) <= Ncap and int(lens.min()) >= 0
    if Q is None:
        Q = torch.randn(B, Hq, d, generator=g, device=dev).to(torch.bfloat16)
    else:
        Q = Q.to(dev)
    grp = Hq // Hkv
    K = torch.empty(B, Hkv, Ncap, d, dtype=torch.bfloat16, device=dev)
    V = torch.empty(B, Hkv, Ncap, d, dtype=torch.bfloat16, device=dev)
    planted = []
    qf = Q.float()
    for b in range(B):
        kb = torch.randn(Hkv, Ncap, d, generator=g, device=dev)
        n_b = int(lens[b])
        cnt = round_half_up(plant_frac * n_b) if plant_frac > 0 else 0
        for kvh in range(Hkv):
            if cnt > 0:
                rows = torch.randperm(n_b, generator=g, device=dev)[:cnt]
                heads = torch.randint(0, grp, (cnt,), generator=g, device=dev) + kvh * grp
                qh = qf[b, heads]  # [cnt, d]
                unit = qh / qh.norm(dim=-1, keepdim=True)
                kb[kvh, rows] += 3.0 * unit
                planted.append(rows.cpu())
            else:
                planted.append(torch.empty(0, dtype=torch.long))
        K[b] = kb.to(torch.bfloat16)
        del kb
    for b in range(B):
        V[b] = torch.randn(Hkv, Ncap, d, generator=g, device=dev).to(torch.bfloat16)
    if tail_fill is not None:
        for b in range(B):
            n_b = int(lens[b])
            K[b, :, n_b:] = tail_fill
            V[b, :, n_b:] = tail_fill
    return DecodeInputs(Q=Q, K=K, V=V, seq_lens=lens.to(dev), planted=planted)


def drift_query(Q: torch.Tensor, sigma: float, seed: int) -> torch.Tensor:
    """Next layer's query: bf16(q + sigma * N(0, 1)), drawn on Q's device."""
    g = _gen(seed, Q.device)
    noise = torch.randn(Q.shape, generator=g, device=Q.device)
    return (Q.float() + sigma * noise).to(torch.bfloat16)


def layer_index_lists(L: int, n_rows, k_rows, k_max: int, keep: float, seed: int) -> torch.Tensor:
    """L layers' index lists for len(n_rows) units: int32 [L, units, k_max], each
    list ascending then -1, as a decode step writes them.  Unit u draws
    min(k_rows[u], n_rows[u]) distinct rows of [0, n_rows[u]) uniformly for layer 0;
    each later layer keeps every row of the layer before with probability `keep`
    and fills up with rows the layer before did not hold, drawn uniformly (then,
    if those run out, with the rows it dropped) (CPU generator)."""
    g = _gen(seed, "cpu")
    units = len(n_rows)
    out = torch.full((L, units, k_max), -1, dtype=torch.int32)
    for u in range(units):
        n, k = int(n_rows[u]), min(int(k_rows[u]), int(n_rows[u]))
        cur = torch.randperm(n, generator=g)[:k]
        for l in range(L):
            if l > 0:
                take = torch.rand(k, generator=g) < keep
                kept, dropped = cur[take], cur[~take]
                pool = torch.randperm(n, generator=g)
                pool = torch.cat([pool[~torch.isin(pool, cur)], dropped])
                cur = torch.cat([kept, pool[:k - kept.numel()]])
            out[l, u, :k] = torch.sort(cur).values.to(torch.int32)
    return out
