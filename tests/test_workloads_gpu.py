"""The five synthetic workloads at full size on the GPU, checked against the
oracle (every unit where the oracle finishes in seconds, else sampled units)."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import check_output, compare_idx, gather_units, sub_problem
from top_sparse_attention_02_b200 import binding as tsa
from top_sparse_attention_02_b200 import inputs, workloads

import gpu_run as G

pytestmark = pytest.mark.gpu


def _gen(w, dev, seed_offset=0, Q=None):
    if w.lens is not None:
        lens = inputs.draw_lengths(w.B, w.lens[0], w.lens[1], seed=w.seed + 1000)
    else:
        lens = [w.Ncap] * w.B
    return inputs.decode_layer(w.B, w.Hq, w.Hkv, w.Ncap, lens, plant_frac=w.plant_frac,
                               seed=w.seed + seed_offset, device=dev, Q=Q)


def _check_select_units(L, idx, O, kreq, k_max, units, scale, block=1):
    g = L.Q.shape[1] // L.K.shape[1]
    sp = sub_problem(L.Q, L.K, L.V, L.seq_lens, units, kreq=kreq)
    gi = gather_units(idx.cpu().numpy(), units, L.K.shape[1])  # [U, 1, k_max]
    if block == 1:
        S = oracle.scores(sp["Q"], sp["K"], sp["seq_lens"], scale)
        nrows = sp["seq_lens"].numpy()
    else:
        nrows = oracle.nblocks_of(sp["seq_lens"], block)
        S = oracle.block_scores(sp["Q"], oracle.block_means(sp["K"], sp["seq_lens"], block), nrows, scale)
    counts = compare_idx(gi, S, nrows, sp["kreq"])
    ref = oracle.attn(sp["Q"], sp["K"], sp["V"], sp["seq_lens"], gi, sp["kreq"], k_max, block, scale)
    check_output(gather_units(O.cpu().numpy(), units, L.K.shape[1], g), ref, "select")
    return counts


def _check_attn_units(L, idx, O, kreq, k_max, units, scale, block=1):
    g = L.Q.shape[1] // L.K.shape[1]
    sp = sub_problem(L.Q, L.K, L.V, L.seq_lens, units, kreq=kreq)
    gi = None if idx is None else gather_units(idx.cpu().numpy(), units, L.K.shape[1])
    ref = oracle.attn(sp["Q"], sp["K"], sp["V"], sp["seq_lens"], gi, sp.get("kreq"), k_max, block,
                      scale)
    check_output(gather_units(O.cpu().numpy(), units, L.K.shape[1], g), ref, "attn")


def test_llama8b_decode_layer(cuda_dev):
    w = workloads.LLAMA8B
    L = _gen(w, cuda_dev)
    kreq = w.k_per_seq(L.seq_lens.tolist())
    O, idx = G.step(L.Q, L.K, L.V, L.seq_lens, mode=tsa.SELECT, scale=w.scale, k_max=w.k, kreq=kreq)
    counts = _check_select_units(L, idx, O, kreq, w.k, range(w.B * w.Hkv), w.scale)
    print(f"llama8b: {counts}")
    assert counts["near_tie"] <= 0.2 * w.B * w.Hkv


def test_reuse128k_four_layers(cuda_dev):
    w = workloads.REUSE128K
    L0 = _gen(w, cuda_dev)
    kreq = w.k_per_seq(L0.seq_lens.tolist())
    O0, idx = G.step(L0.Q, L0.K, L0.V, L0.seq_lens, mode=tsa.SELECT, scale=w.scale, k_max=w.k,
                     kreq=kreq)
    counts = _check_select_units(L0, idx, O0, kreq, w.k, range(w.Hkv), w.scale)
    print(f"reuse128k layer 0: {counts}")
    Q = L0.Q
    del L0
    for layer in (1, 2, 3):
        Q = inputs.drift_query(Q, w.q_drift, seed=w.seed + 100 + layer)
        L = _gen(w, cuda_dev, seed_offset=layer, Q=Q)
        before = idx.clone()
        O, _ = G.step(L.Q, L.K, L.V, L.seq_lens, mode=tsa.REUSE, scale=w.scale, k_max=w.k, kreq=kreq,
                      idx_in=idx)
        assert torch.equal(idx, before)
        _check_attn_units(L, idx, O, kreq, w.k, range(w.Hkv), w.scale)
        del L


def test_large_batch_500x_sampled(cuda_dev):
    w = workloads.LARGE_BATCH
    L = _gen(w, cuda_dev)
    lens = L.seq_lens.tolist()
    kreq = w.k_per_seq(lens)
    k_max = max(kreq)
    O, idx = G.step(L.Q, L.K, L.V, L.seq_lens, mode=tsa.SELECT, scale=w.scale, k_max=k_max, kreq=kreq)
    rng = np.random.default_rng(0)
    units = sorted(rng.choice(w.B * w.Hkv, size=24, replace=False).tolist())
    units += [int(np.argmin(lens)) * w.Hkv, int(np.argmax(lens)) * w.Hkv + 7]
    counts = _check_select_units(L, idx, O, kreq, k_max, units, w.scale)
    print(f"large batch (26 sampled units): {counts}")
    # every unit: index layout is valid (ascending, in range, -1 padded)
    idx_np = idx.cpu().numpy()
    for b in range(w.B):
        kb = min(kreq[b], lens[b])
        row = idx_np[b]
        assert (row[:, kb:] == -1).all() and (np.diff(row[:, :kb], axis=1) > 0).all()
        assert (row[:, :kb] >= 0).all() and (row[:, :kb] < lens[b]).all()


def test_hybrid_block_stack_sampled(cuda_dev):
    w = workloads.HYBRID
    units = [0, 5, 11, 15]
    # layer 0: FULL
    L = _gen(w, cuda_dev, seed_offset=0)
    O, _ = G.step(L.Q, L.K, L.V, L.seq_lens, mode=tsa.FULL, scale=w.scale)
    _check_attn_units(L, None, O, None, 0, units, w.scale)
    del L
    # layer 2: SELECT in block mode, then layer 3 reuses its blocks
    L = _gen(w, cuda_dev, seed_offset=2)
    kreq = [w.k] * w.B
    Kmean = G.block_means(L.K, L.seq_lens, w.block)
    O, idx = G.step(L.Q, L.K, L.V, L.seq_lens, mode=tsa.SELECT, scale=w.scale, k_max=w.k,
                    block=w.block, kreq=kreq, Kmean=Kmean)
    counts = _check_select_units(L, idx, O, kreq, w.k, units, w.scale, block=w.block)
    print(f"hybrid block select (4 sampled units): {counts}")
    del L, Kmean
    L = _gen(w, cuda_dev, seed_offset=3)
    O, _ = G.step(L.Q, L.K, L.V, L.seq_lens, mode=tsa.REUSE, scale=w.scale, k_max=w.k, block=w.block,
                  kreq=kreq, idx_in=idx)
    _check_attn_units(L, idx, O, kreq, w.k, units, w.scale, block=w.block)


def test_hybrid_block_stack_all_layers_one_workspace(cuda_dev):
    """The whole 8-layer hybrid route (F F S R S R S R, 262144 tokens, top 32 of
    128-token blocks) enqueued back to back on one stream and ONE shared
    workspace, with no host synchronisation between layers; then every layer's
    O, and every SELECT layer's block indices, are checked against the oracle
    on sampled units (Flux Attention's hard per-layer routing; HyLRA's reuse of
    an earlier layer's blocks)."""
    w = workloads.HYBRID
    units = [0, 6, 9, 15]
    layers = [_gen(w, cuda_dev, seed_offset=li) for li in range(w.layers)]
    shape = tsa.shape_of(layers[0].Q, layers[0].K)
    kreq = [w.k] * w.B
    kr = torch.tensor(kreq, dtype=torch.int32, device=cuda_dev)
    ws_bytes = max(tsa.workspace_size(shape, w.k, w.block, m) for m in set(w.route))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=cuda_dev)
    tsa.workspace_init(ws)
    Os = [torch.full((w.B, w.Hq, 128), float("nan"), dtype=torch.float32, device=cuda_dev)
          for _ in range(w.layers)]
    idx = {li: torch.full((w.B, w.Hkv, w.k), -7, dtype=torch.int32, device=cuda_dev)
           for li, m in enumerate(w.route) if m == tsa.SELECT}
    Kmean = {li: G.block_means(layers[li].K, layers[li].seq_lens, w.block) for li in idx}
    args = []
    for li, (L, m) in enumerate(zip(layers, w.route)):
        args.append(tsa.step_args(L.Q, L.K, L.V, L.seq_lens, Os[li], ws, mode=m, scale=w.scale, k_max=w.k,
                                  block=w.block, k_per_seq=kr, Kmean=Kmean.get(li),
                                  idx_in=idx[w.reuse_from[li]] if m == tsa.REUSE else None,
                                  idx_out=idx.get(li)))
    for a in args:
        tsa.decode_step(a)
    tsa.check_device_status(ws)
    torch.cuda.synchronize()
    for li, (L, m) in enumerate(zip(layers, w.route)):
        if m == tsa.FULL:
            _check_attn_units(L, None, Os[li], None, 0, units, w.scale)
        elif m == tsa.SELECT:
            counts = _check_select_units(L, idx[li], Os[li], kreq, w.k, units, w.scale, block=w.block)
            print(f"hybrid layer {li} (select): {counts}")
        else:
            _check_attn_units(L, idx[w.reuse_from[li]], Os[li], kreq, w.k, units, w.scale, block=w.block)
