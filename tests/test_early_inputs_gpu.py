"""Decode steps enqueued back to back on one stream and one workspace, with and
without TSA_EARLY_INPUTS (the caller's promise that the kernel just before a
step writes none of its lengths, k's, K, V or reused indices, so the step's
first kernel may read them before that kernel finishes).  Every layer's output
and every selected index set is checked against the fp64 oracle.

Also covers the attention's cp.async ring with more tiles per CTA than ring
stages (the ring is refilled), with both combines (cluster and workspace)."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import check_output, compare_idx
from top_sparse_attention_02_b200 import binding as tsa
from top_sparse_attention_02_b200 import inputs

import gpu_run as G

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)
EARLY = tsa.EARLY_INPUTS


def _layers(n, B, Hq, Hkv, N, lens, dev, seed):
    out = []
    for i in range(n):
        L = inputs.decode_layer(B, Hq, Hkv, N, lens, plant_frac=0.01, seed=seed + i, tail_fill=float("nan"))
        out.append((L, G.to_dev(L, dev)))
    return out


@pytest.mark.parametrize("Hq,Hkv,N,lens,k", [
    (32, 8, 20000, [20000], 3000),          # 3 tiles a CTA: the whole ring in flight
    (32, 8, 30000, [30000], 5000),          # 5 tiles a CTA: the ring is refilled
    (64, 8, 9000, [9000, 4000, 1], 2000),   # g = 8, ragged, a sequence of one token, k > len
    (8, 8, 12000, [12000, 11000], 1500),    # g = 1
])
def test_chained_steps_with_early_inputs(cuda_dev, Hq, Hkv, N, lens, k):
    """SELECT (early) -> REUSE (early) -> REUSE -> FULL (early) -> REUSE (early),
    one stream, one workspace, no host synchronisation in between."""
    B = len(lens)
    kreq = [k] * B
    lay = _layers(5, B, Hq, Hkv, N, lens, cuda_dev, seed=700 + N)
    d0 = lay[0][1]
    shape = tsa.shape_of(d0[0], d0[1])
    ws_bytes = max(tsa.workspace_size(shape, k, 1, m) for m in (tsa.SELECT, tsa.REUSE, tsa.FULL))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=cuda_dev)
    tsa.workspace_init(ws)
    kr = torch.tensor(kreq, dtype=torch.int32, device=cuda_dev)
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=cuda_dev)
    Os = [torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=cuda_dev) for _ in range(5)]
    plan = [(tsa.SELECT, EARLY), (tsa.REUSE, EARLY), (tsa.REUSE, 0), (tsa.FULL, EARLY), (tsa.REUSE, EARLY)]
    args = []
    for i, (mode, flags) in enumerate(plan):
        Q, K, V, ln = lay[i][1]
        args.append(tsa.step_args(Q, K, V, ln, Os[i], ws, mode=mode, scale=SCALE, k_max=k, k_per_seq=kr,
                                  idx_in=idx if mode == tsa.REUSE else None,
                                  idx_out=idx if mode == tsa.SELECT else None, flags=flags))
    for a in args:
        tsa.decode_step(a)
    tsa.check_device_status(ws)
    torch.cuda.synchronize()
    L0 = lay[0][0]
    gi = idx.cpu().numpy()
    S = oracle.scores(L0.Q, L0.K, L0.seq_lens, SCALE)
    counts = compare_idx(gi, S, lens, kreq)
    print(f"select: {counts}")
    for i, (mode, flags) in enumerate(plan):
        L = lay[i][0]
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, None if mode == tsa.FULL else gi,
                          None if mode == tsa.FULL else kreq, 0 if mode == tsa.FULL else k, 1, SCALE)
        check_output(Os[i].cpu().numpy(), ref, f"layer {i} ({'FSR'[mode]}, flags={flags})")


def test_chained_block_steps_with_early_inputs(cuda_dev):
    """Block mode: SELECT over block means (early), then REUSE of its blocks
    (early; contiguous 128-row tiles by TMA issued before the wait)."""
    B, Hq, Hkv, N, k = 2, 32, 8, 40000, 24
    lens = [40000, 17000]
    lay = _layers(2, B, Hq, Hkv, N, lens, cuda_dev, seed=801)
    (L0, d0), (L1, d1) = lay
    Km = G.block_means(d0[1], d0[3], 128)
    shape = tsa.shape_of(d0[0], d0[1])
    ws_bytes = max(tsa.workspace_size(shape, k, 128, m) for m in (tsa.SELECT, tsa.REUSE))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=cuda_dev)
    tsa.workspace_init(ws)
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=cuda_dev)
    O0 = torch.empty(B, Hq, 128, dtype=torch.float32, device=cuda_dev)
    O1 = torch.empty_like(O0)
    a0 = tsa.step_args(*d0[:3], d0[3], O0, ws, mode=tsa.SELECT, scale=SCALE, k_max=k, block=128, Kmean=Km,
                       idx_out=idx, flags=EARLY)
    a1 = tsa.step_args(*d1[:3], d1[3], O1, ws, mode=tsa.REUSE, scale=SCALE, k_max=k, block=128, idx_in=idx,
                       flags=EARLY)
    tsa.decode_step(a0)
    tsa.decode_step(a1)
    tsa.check_device_status(ws)
    gi = idx.cpu().numpy()
    nb = oracle.nblocks_of(L0.seq_lens, 128)
    S = oracle.block_scores(L0.Q, oracle.block_means(L0.K, L0.seq_lens, 128), nb, SCALE)
    compare_idx(gi, S, nb, [k, k])
    check_output(O0.cpu().numpy(), oracle.attn(L0.Q, L0.K, L0.V, L0.seq_lens, gi, [k, k], k, 128, SCALE), "select")
    check_output(O1.cpu().numpy(), oracle.attn(L1.Q, L1.K, L1.V, L1.seq_lens, gi, [k, k], k, 128, SCALE), "reuse")


def test_early_inputs_flag_is_the_only_new_bit(cuda_dev):
    L = inputs.decode_layer(1, 8, 2, 512, [512], seed=3)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    ws = G.ws_for(Q, K, 0, 1, tsa.FULL)
    O = torch.empty(1, 8, 128, dtype=torch.float32, device=cuda_dev)
    a = tsa.step_args(Q, K, V, ln, O, ws, mode=tsa.FULL, scale=SCALE, flags=4)
    with pytest.raises(tsa.TsaError) as e:
        tsa.decode_step(a)
    assert e.value.status == tsa.TSA_ERR_INVALID_ARG


def test_async_ring_with_workspace_combine(cuda_dev):
    """Three units with a long index list: many splits of several tiles each (the
    ring refilled), combined through the workspace (more than 8 splits)."""
    B, Hq, Hkv, N, k = 3, 8, 1, 40000, 20000
    lens = [40000, 39999, 25000]
    L = inputs.decode_layer(B, Hq, Hkv, N, lens, plant_frac=0.0, seed=77, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    rng = np.random.default_rng(5)
    idx = np.full((B, Hkv, k), -1, dtype=np.int32)
    kb = [k, k, 18000]
    for b in range(B):
        idx[b, 0, :kb[b]] = np.sort(rng.choice(lens[b], size=kb[b], replace=False))
    idx[0, 0, 100:140] = -1  # skipped entries inside a tile
    O, _ = G.run_attn(Q, K, V, ln, torch.from_numpy(idx).to(cuda_dev), kb, k, 1, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, kb, k, 1, SCALE)
    check_output(O.cpu().numpy(), ref, "ring + workspace combine")
