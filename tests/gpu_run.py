"""Run the CUDA path through the C ABI (via the binding) on torch tensors."""
from __future__ import annotations

import torch

from top_sparse_attention_02_b200 import binding as tsa


def to_dev(L, dev):
    return (L.Q.to(dev), L.K.to(dev), L.V.to(dev), L.seq_lens.to(dev).to(torch.int32))


def ws_for(Q, K, k_max, block, mode):
    return tsa.new_workspace(tsa.shape_of(Q, K), k_max, block, mode, Q.device)


def block_means(K, lens, block):
    B, Hkv, N, d = K.shape
    NB = (N + block - 1) // block
    Kmean = torch.zeros(B, Hkv, NB, d, dtype=torch.float32, device=K.device)
    ws = torch.zeros(256, dtype=torch.uint8, device=K.device)
    tsa.block_summarize(K, lens, block, Kmean, ws)
    tsa.check_device_status(ws)
    return Kmean


def step(Q, K, V, lens, *, mode, scale, k_max=0, block=1, kreq=None, Kmean=None, idx_in=None,
         ws=None, check=True, emit=False, flags=0):
    """One decode step; returns (O, idx) with idx None unless SELECT (or FULL with emit)."""
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    if ws is None:
        ws = ws_for(Q, K, k_max, block, mode)
    O = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device=Q.device)
    idx = None
    if mode == tsa.SELECT or emit:
        idx = torch.full((B, Hkv, k_max), -7, dtype=torch.int32, device=Q.device)
    kr = None if kreq is None else torch.as_tensor(kreq, dtype=torch.int32).to(Q.device)
    a = tsa.step_args(Q, K, V, lens, O, ws, mode=mode, scale=scale, k_max=k_max, block=block,
                      k_per_seq=kr, Kmean=Kmean, idx_in=idx_in, idx_out=idx, flags=flags)
    tsa.decode_step(a)
    if check:
        tsa.check_device_status(ws)
    torch.cuda.synchronize()
    return O, idx


def run_score(Q, K, lens, scale, block=1, Kmean=None, Ncap=None):
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    Ncap = Ncap or K.shape[2]
    rows = Ncap if block == 1 else (Ncap + block - 1) // block
    S = torch.full((B, Hkv, rows), float("nan"), dtype=torch.float32, device=Q.device)
    ws = torch.zeros(256, dtype=torch.uint8, device=Q.device)
    shape = tsa.tsa_shape(B, Hq, Hkv, Ncap, d)
    tsa.sparse_decode_score(Q, K if block == 1 else Kmean, lens, shape, block, scale, S, ws)
    tsa.check_device_status(ws)
    return S


def run_topk(S, lens, kreq, k_max, Hq, Ncap, block=1):
    B, Hkv, rows = S.shape
    idx = torch.full((B, Hkv, k_max), -7, dtype=torch.int32, device=S.device)
    ws = torch.zeros(256, dtype=torch.uint8, device=S.device)
    kr = None if kreq is None else torch.as_tensor(kreq, dtype=torch.int32).to(S.device)
    shape = tsa.tsa_shape(B, Hq, Hkv, Ncap, 128)
    tsa.topk_select(S, lens, kr, k_max, shape, block, idx, ws)
    tsa.check_device_status(ws)
    return idx


def run_attn(Q, K, V, lens, idx, kreq, k_max, block, scale, check=True):
    ws = ws_for(Q, K, k_max if idx is not None else 0, block, tsa.REUSE if idx is not None else tsa.FULL)
    O = torch.full(Q.shape, float("nan"), dtype=torch.float32, device=Q.device)
    kr = None if kreq is None else torch.as_tensor(kreq, dtype=torch.int32).to(Q.device)
    tsa.sparse_decode_attn(Q, K, V, lens, idx, kr, k_max, block, scale, O, ws)
    if check:
        tsa.check_device_status(ws)
    torch.cuda.synchronize()
    return O, ws
