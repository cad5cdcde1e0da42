"""Parity helpers: compare the CUDA path with the fp64 oracle.

Tolerances (from the problem statement of the decode path):
  - index sets equal, except at a near-tie: when the oracle's k-th and (k+1)-th
    scores differ by less than 1e-5 relative, the GPU set may differ only by
    rows whose oracle score lies within 1e-5 * |S_(k)| of S_(k); such units are
    counted and reported;
  - outputs within 2e-3 max-abs and 1e-3 relative-L2 (||O - O*|| / ||O*|| over
    the whole tensor), where O* is the oracle's attention over the GPU's own
    index set (so a legal near-tie swap does not count against the output).
"""
from __future__ import annotations

import numpy as np
import torch

NEAR_TIE_REL = 1e-5
O_MAX_ABS = 2e-3
O_REL_L2 = 1e-3


def check_idx_layout(idx: np.ndarray, kb: int, n: int):
    """Ascending, unique, in [0, n), then -1 padding."""
    head, tail = idx[:kb], idx[kb:]
    assert (tail == -1).all(), f"padding not -1: {tail[:8]}"
    assert (head >= 0).all() and (head < n).all(), "index out of range"
    assert (np.diff(head) > 0).all(), "indices not strictly ascending"


def compare_unit(gpu_row: np.ndarray, S: np.ndarray, n: int, kb: int) -> str:
    """'exact' | 'near_tie' (allowed) ; raises AssertionError otherwise."""
    check_idx_layout(gpu_row, kb, n)
    if kb == 0:
        return "exact"
    s = S[:n]
    order = np.lexsort((np.arange(n), -s))
    want = set(order[:kb].tolist())
    got = set(gpu_row[:kb].tolist())
    if want == got:
        return "exact"
    sk = s[order[kb - 1]]
    band = NEAR_TIE_REL * abs(sk)
    assert kb < n, "sets differ although every row is selected"
    gap = abs(sk - s[order[kb]])
    diff = want ^ got
    bad = [j for j in diff if abs(s[j] - sk) > band]
    assert gap < band and not bad, (
        f"index sets differ beyond the near-tie band: gap={gap:.3e} band={band:.3e}, "
        f"{len(diff)} rows differ, {len(bad)} outside the band")
    return "near_tie"


def compare_idx(gpu_idx: np.ndarray, S: np.ndarray, nrows, kreq, units=None) -> dict:
    """Compare [B,Hkv,k_max] GPU indices with oracle scores S [B,Hkv,rows]."""
    B, Hkv = gpu_idx.shape[:2]
    us = range(B * Hkv) if units is None else units
    counts = {"exact": 0, "near_tie": 0}
    for u in us:
        b, h = divmod(int(u), Hkv)
        n = int(nrows[b])
        kb = min(int(kreq[b]), n)
        counts[compare_unit(gpu_idx[b, h], S[b, h], n, kb)] += 1
    return counts


def check_output(O_gpu, O_ref, what=""):
    O_gpu = np.asarray(O_gpu, dtype=np.float64)
    O_ref = np.asarray(O_ref, dtype=np.float64)
    assert np.isfinite(O_gpu).all(), f"{what}: non-finite output"
    err = np.abs(O_gpu - O_ref)
    max_abs = float(err.max()) if err.size else 0.0
    nrm = float(np.linalg.norm(O_ref))
    rel = float(np.linalg.norm(O_gpu - O_ref) / nrm) if nrm > 0 else float(np.linalg.norm(O_gpu))
    assert max_abs <= O_MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {O_MAX_ABS}"
    assert rel <= O_REL_L2, f"{what}: rel-L2 {rel:.3e} > {O_REL_L2}"
    return max_abs, rel


def sub_problem(Q, K, V, seq_lens, units, kreq=None, idx=None):
    """The listed (b, kv-head) units as an independent CPU batch: B' = len(units),
    Hkv' = 1, Hq' = g.  Units do not interact, so the oracle on this batch is the
    oracle on those units of the full problem."""
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    qs, ks, vs, ls, kr, ix = [], [], [], [], [], []
    lens_cpu = seq_lens.cpu()
    for u in units:
        b, h = divmod(int(u), Hkv)
        qs.append(Q[b, h * g:(h + 1) * g].cpu())
        ks.append(K[b, h:h + 1].cpu())
        vs.append(V[b, h:h + 1].cpu())
        ls.append(int(lens_cpu[b]))
        if kreq is not None:
            kr.append(int(kreq[b]))
        if idx is not None:
            ix.append(np.asarray(idx[b, h:h + 1]))
    out = dict(Q=torch.stack(qs), K=torch.stack(ks), V=torch.stack(vs),
               seq_lens=torch.tensor(ls, dtype=torch.int32))
    if kreq is not None:
        out["kreq"] = kr
    if idx is not None:
        out["idx"] = np.stack(ix)
    return out


def gather_units(x: np.ndarray, units, Hkv: int, g: int = 1) -> np.ndarray:
    """Rows of a [B, Hkv*g, ...] array for the listed units, as [U, g, ...]."""
    out = []
    for u in units:
        b, h = divmod(int(u), Hkv)
        out.append(x[b, h * g:(h + 1) * g])
    return np.stack(out)
