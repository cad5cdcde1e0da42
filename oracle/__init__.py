"""fp64 CPU oracle for top-k context-sparse decode attention (ctypes wrapper).

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The product
path (the CUDA library and its binding) never does.

The arithmetic lives in ``oracle.c`` (plain C, double precision, OpenMP over
(sequence, kv-head) units).  This module only marshals arrays.  Pins that tie
the oracle to facts other than itself are in ``tests/test_oracle_pins.py``.

Parity status: every function here is pinned (closed forms, brute force on
tiny inputs, a library routine in a special case); none is "parity unpinned".
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")
_lib = None

i32p = ctypes.POINTER(ctypes.c_int32)
u16p = ctypes.POINTER(ctypes.c_uint16)
f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    I, D = ctypes.c_int, ctypes.c_double
    lib.oracle_scores.argtypes = [u16p, u16p, i32p, I, I, I, I, I, D, i32p, I, f64p]
    lib.oracle_block_means.argtypes = [u16p, i32p, I, I, I, I, I, i32p, I, f64p]
    lib.oracle_block_scores.argtypes = [u16p, f64p, i32p, I, I, I, I, I, D, i32p, I, f64p]
    lib.oracle_topk.argtypes = [f64p, i32p, i32p, I, I, I, I, i32p, I, i32p]
    lib.oracle_attn.argtypes = [u16p, u16p, u16p, i32p, i32p, i32p, I, I, I, I, I, I, I, D,
                                i32p, I, f64p]
    for f in ("oracle_scores", "oracle_block_means", "oracle_block_scores", "oracle_topk",
              "oracle_attn", "oracle_num_threads"):
        getattr(lib, f).restype = ctypes.c_int
    lib.oracle_set_threads.argtypes = [I]
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(_LIB)
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Temporarily route every call to another build of oracle.c (the mutation tests
    compile deliberately broken copies and check that the pins reject them)."""
    global _lib
    saved = _load()
    _lib = _bind(path)
    try:
        yield
    finally:
        _lib = saved


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def _bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy()).view(np.uint16)


def _i32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a: np.ndarray, typ):
    return a.ctypes.data_as(typ)


def _units(units):
    if units is None:
        return None, 0, None
    u = _i32(units)
    return u, int(u.size), _p(u, i32p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def scores(Q, K, seq_lens, scale: float, units=None) -> np.ndarray:
    """s[b,kvh,j] = max over the group's heads of scale*<q_h, k_j> (NaN past len_b)."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    q, k, L = _bits(Q), _bits(K), _i32(seq_lens)
    S = np.full((B, Hkv, Ncap), np.nan)
    ua, nu, up = _units(units)
    _check(_load().oracle_scores(_p(q, u16p), _p(k, u16p), _p(L, i32p), B, Hq, Hkv, Ncap, d,
                                 float(scale), up, nu, _p(S, f64p)), "scores")
    return S


def block_means(K, seq_lens, block: int, units=None) -> np.ndarray:
    """mu[b,kvh,beta] = mean of block beta's valid K rows (NaN for blocks with none)."""
    B, Hkv, Ncap, d = K.shape
    NB = (Ncap + block - 1) // block
    k, L = _bits(K), _i32(seq_lens)
    M = np.full((B, Hkv, NB, d), np.nan)
    ua, nu, up = _units(units)
    _check(_load().oracle_block_means(_p(k, u16p), _p(L, i32p), B, Hkv, Ncap, d, block, up, nu,
                                      _p(M, f64p)), "block_means")
    return M


def block_scores(Q, M: np.ndarray, nblocks, scale: float, units=None) -> np.ndarray:
    B, Hq, d = Q.shape
    _, Hkv, NB, _ = M.shape
    q, nb = _bits(Q), _i32(nblocks)
    Mc = np.ascontiguousarray(M, dtype=np.float64)
    S = np.full((B, Hkv, NB), np.nan)
    ua, nu, up = _units(units)
    _check(_load().oracle_block_scores(_p(q, u16p), _p(Mc, f64p), _p(nb, i32p), B, Hq, Hkv, NB, d,
                                       float(scale), up, nu, _p(S, f64p)), "block_scores")
    return S


def topk(S: np.ndarray, nrows, kreq, k_max: int, units=None) -> np.ndarray:
    """Exact top-k (ties to the lower index), ascending, -1 padded: int32 [B,Hkv,k_max]."""
    B, Hkv, cap = S.shape
    Sc = np.ascontiguousarray(S, dtype=np.float64)
    n, kr = _i32(nrows), _i32(kreq)
    idx = np.full((B, Hkv, k_max), -1, dtype=np.int32)
    ua, nu, up = _units(units)
    _check(_load().oracle_topk(_p(Sc, f64p), _p(n, i32p), _p(kr, i32p), B, Hkv, cap, k_max, up, nu,
                               _p(idx, i32p)), "topk")
    return idx


def attn(Q, K, V, seq_lens, idx, kreq, k_max: int, block: int, scale: float,
         units=None) -> np.ndarray:
    """Exact softmax attention over the selected rows (idx None = all valid rows): f64 [B,Hq,d]."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    q, k, v, L = _bits(Q), _bits(K), _bits(V), _i32(seq_lens)
    if idx is None:
        ip, kr, kp = None, _i32(np.zeros(B)), None
    else:
        ia = _i32(idx)
        assert ia.shape == (B, Hkv, k_max)
        ip = _p(ia, i32p)
        kr = _i32(kreq)
    O = np.full((B, Hq, d), np.nan)
    ua, nu, up = _units(units)
    _check(_load().oracle_attn(_p(q, u16p), _p(k, u16p), _p(v, u16p), _p(L, i32p), ip,
                               _p(kr, i32p), k_max, block, B, Hq, Hkv, Ncap, d, float(scale), up,
                               nu, _p(O, f64p)), "attn")
    return O


def index_overlap(idx):
    """Overlap of L layers' index sets (HyLRA, sec. 2.2: the similarity matrix M of
    top-k overlap ratios between a source layer i and a target layer j).

    idx: int [L, B, Hkv, k_max] (or [L, units, k_max]), each list ascending then -1.
    Returns (counts, M): counts int64 [L, L, units] = |I_i(u) ∩ I_j(u)| by numpy's
    set intersection; M float64 [L, L] lower triangular (row = target j, column =
    source i <= j): the mean, over the units whose target set is non-empty, of
    |I_i ∩ I_j| / |I_j| (1 if there is no such unit), 0 above the diagonal."""
    a = np.asarray(idx)
    L, k_max = a.shape[0], a.shape[-1]
    units = int(np.prod(a.shape[1:-1]))
    a = a.reshape(L, units, k_max)
    sets = [[a[l, u][a[l, u] >= 0] for u in range(units)] for l in range(L)]
    counts = np.zeros((L, L, units), dtype=np.int64)
    for i in range(L):
        for j in range(L):
            for u in range(units):
                counts[i, j, u] = np.intersect1d(sets[i][u], sets[j][u]).size
    M = np.zeros((L, L))
    for j in range(L):
        for i in range(j + 1):
            ratios = [counts[i, j, u] / sets[j][u].size for u in range(units) if sets[j][u].size > 0]
            M[j, i] = float(np.mean(ratios)) if ratios else 1.0
    return counts, M


def reuse_policy(M, theta: float, force_full=None):
    """HyLRA's offline policy (HyLRA, sec. 2.2) by exhaustive search, for small L.

    Every choice of full layers (layer 0 and the forced ones always full) is a
    policy; each other layer reuses the indices of the latest full layer before it
    and is allowed only if M[j][source] > theta.  Among the allowed policies: fewest
    full layers, then the largest similarity of the reusing layers (summed in layer
    order), then the smallest source sequence read from the last layer backwards.
    M is [L, L] with row = target layer.  Returns (source, n_full, total_sim)."""
    M = np.asarray(M, dtype=np.float64)
    L = M.shape[0]
    forced = [j == 0 or (force_full is not None and bool(force_full[j])) for j in range(L)]
    free = [j for j in range(1, L) if not forced[j]]
    best = None
    for mask in range(1 << len(free)):
        full = list(forced)
        for b, j in enumerate(free):
            if mask >> b & 1:
                full[j] = True
        src, cur, sim, ok = [], 0, 0.0, True
        for j in range(L):
            if full[j]:
                cur = j
            elif not M[j, cur] > theta:
                ok = False
                break
            else:
                sim += M[j, cur]
            src.append(cur)
        if not ok:
            continue
        key = (sum(full), -sim, src[::-1])
        if best is None or key < best[0]:
            best = (key, src, sum(full), sim)
    return np.array(best[1], dtype=np.int32), best[2], best[3]


def nblocks_of(seq_lens, block: int) -> np.ndarray:
    L = _i32(seq_lens)
    return ((L.astype(np.int64) + block - 1) // block).astype(np.int32)


def decode_step(Q, K, V, seq_lens, kreq, k_max: int, scale: float, mode: int = 1, block: int = 1,
                idx_in=None, units=None):
    """One layer: FULL (0) attends every valid row; SELECT (1) scores, selects and attends;
    REUSE (2) attends over ``idx_in`` unchanged.  Returns (O, idx, S) (idx/S None when unused)."""
    if mode == 0:
        return attn(Q, K, V, seq_lens, None, None, 0, 1, scale, units), None, None
    if mode == 2:
        return attn(Q, K, V, seq_lens, idx_in, kreq, k_max, block, scale, units), idx_in, None
    if block == 1:
        S = scores(Q, K, seq_lens, scale, units)
        nrows = _i32(seq_lens)
    else:
        M = block_means(K, seq_lens, block, units)
        nrows = nblocks_of(seq_lens, block)
        S = block_scores(Q, M, nrows, scale, units)
    idx = topk(S, nrows, kreq, k_max, units)
    O = attn(Q, K, V, seq_lens, idx, kreq, k_max, block, scale, units)
    return O, idx, S
