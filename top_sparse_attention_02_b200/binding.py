"""Thin Python binding of libtsa's C ABI (include/tsa.h), same names.

Argument marshalling only: every step of the decode path runs in the CUDA
kernels behind these calls.  Torch supplies device memory and streams.  There
is no CPU fallback: if libtsa.so is missing or cannot load, importing this
module raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtsa.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libtsa.so is not built ({_LIB_PATH}); run `python -m "
                      "top_sparse_attention_02_b200.build` (or __graft_entry__.build())")
_lib = ctypes.CDLL(_LIB_PATH)

TSA_OK, TSA_ERR_INVALID_ARG, TSA_ERR_UNSUPPORTED, TSA_ERR_WORKSPACE = 0, 1, 2, 3
TSA_ERR_CUDA, TSA_ERR_DEVICE_BOUNDS, TSA_ERR_DEVICE_TIMEOUT = 4, 5, 6
FULL, SELECT, REUSE = 0, 1, 2
STATUS_NAMES = {0: "TSA_OK", 1: "TSA_ERR_INVALID_ARG", 2: "TSA_ERR_UNSUPPORTED", 3: "TSA_ERR_WORKSPACE",
                4: "TSA_ERR_CUDA", 5: "TSA_ERR_DEVICE_BOUNDS", 6: "TSA_ERR_DEVICE_TIMEOUT"}


class tsa_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("Ncap", ctypes.c_int32), ("d", ctypes.c_int32)]


class tsa_step_args(ctypes.Structure):
    _fields_ = [("shape", tsa_shape), ("Q", ctypes.c_void_p), ("K", ctypes.c_void_p),
                ("V", ctypes.c_void_p), ("Kmean", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("k_per_seq", ctypes.c_void_p), ("k_max", ctypes.c_int32), ("block", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("scale", ctypes.c_float), ("idx_in", ctypes.c_void_p),
                ("idx_out", ctypes.c_void_p), ("O", ctypes.c_void_p), ("ws", ctypes.c_void_p),
                ("ws_bytes", ctypes.c_size_t), ("flags", ctypes.c_uint32)]


KV_HOST = 1  # tsa_step_args.flags: K and V in mapped page-locked host memory
EARLY_INPUTS = 2  # tsa_step_args.flags: the kernel before the step writes none of lens, k's, K, V, idx_in


_vp, _sz, _i32, _f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_float
_SIGS = {
    "tsa_workspace_size": (_sz, [tsa_shape, _i32, _i32, _i32]),
    "tsa_workspace_init": (ctypes.c_int, [_vp, _sz, _vp]),
    "tsa_block_summarize": (ctypes.c_int, [_vp, _vp, tsa_shape, _i32, _vp, _vp, _sz, _vp]),
    "sparse_decode_score": (ctypes.c_int, [_vp, _vp, _vp, tsa_shape, _i32, _f32, _vp, _vp, _sz, _vp]),
    "topk_select": (ctypes.c_int, [_vp, _vp, _vp, _i32, tsa_shape, _i32, _vp, _vp, _sz, _vp]),
    "sparse_decode_attn": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, tsa_shape, _f32,
                                          _vp, _vp, _sz, _vp]),
    "sparse_decode_attn_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, tsa_shape,
                                                  _f32, _vp, _vp]),
    "tsa_decode_step": (ctypes.c_int, [ctypes.POINTER(tsa_step_args), _vp]),
    "tsa_index_overlap": (ctypes.c_int, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "tsa_reuse_policy": (ctypes.c_int, [_vp, _i32, ctypes.c_double, _vp, _vp, _vp, _vp]),
    "tsa_shard_workspace_size": (_sz, [tsa_shape, _i32, _i32]),
    "tsa_shard_select": (ctypes.c_int, [_vp, _vp, _vp, tsa_shape, _vp, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "tsa_shard_merge": (ctypes.c_int, [_vp, _vp, _i32, tsa_shape, _vp, _i32, _vp, _vp, _sz, _vp]),
    "tsa_shard_attend": (ctypes.c_int, [_vp, _vp, _vp, _vp, tsa_shape, _vp, _vp, _i32, _i32, _f32, _vp, _vp, _vp,
                                        _sz, _vp]),
    "tsa_shard_combine": (ctypes.c_int, [_vp, _vp, _i32, tsa_shape, _vp, _vp]),
    "tsa_check_device_status": (ctypes.c_int, [_vp, _vp]),
    "tsa_last_error_string": (ctypes.c_char_p, []),
    "tsa_launch_count": (ctypes.c_uint64, []),
    "tsa_hbm_copy": (ctypes.c_int, [_vp, _vp, _sz, _vp]),
    "tsa_hbm_read": (ctypes.c_int, [_vp, _sz, _vp, _sz, _vp]),
    "tsa_hbm_gather": (ctypes.c_int, [_vp, _sz, _vp, _i32, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


class TsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def lib():
    """The loaded ctypes library (for callers that marshal raw pointers themselves)."""
    return _lib


def last_error() -> str:
    return (_lib.tsa_last_error_string() or b"").decode()


def _ok(st: int):
    if st != TSA_OK:
        raise TsaError(st, last_error())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def shape_of(Q: torch.Tensor, K: torch.Tensor) -> tsa_shape:
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    return tsa_shape(B, Hq, Hkv, Ncap, d)


def workspace_size(shape: tsa_shape, k_max: int, block: int, mode: int) -> int:
    n = _lib.tsa_workspace_size(shape, k_max, block, mode)
    if n == 0:
        raise TsaError(TSA_ERR_INVALID_ARG, last_error())
    return n


def workspace_init(ws: torch.Tensor, stream=None):
    _ok(_lib.tsa_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def new_workspace(shape: tsa_shape, k_max: int, block: int, mode: int, device) -> torch.Tensor:
    """Allocate (with torch) and zero a workspace for these arguments."""
    n = workspace_size(shape, k_max, block, mode)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    workspace_init(ws)
    return ws


def _wsargs(ws):
    return _ptr(ws), ws.numel() * ws.element_size()


def block_summarize(K, seq_lens, block: int, Kmean, ws, stream=None, shape=None):
    s = shape or tsa_shape(K.shape[0], K.shape[1], K.shape[1], K.shape[2], K.shape[3])
    _ok(_lib.tsa_block_summarize(_ptr(K), _ptr(seq_lens), s, block, _ptr(Kmean), *_wsargs(ws),
                                 _stream(stream)))


def sparse_decode_score(Q, keys, seq_lens, shape: tsa_shape, block: int, scale: float, scores, ws,
                        stream=None):
    _ok(_lib.sparse_decode_score(_ptr(Q), _ptr(keys), _ptr(seq_lens), shape, block, scale,
                                 _ptr(scores), *_wsargs(ws), _stream(stream)))


def topk_select(scores, seq_lens, k_per_seq, k_max: int, shape: tsa_shape, block: int, idx, ws,
                stream=None):
    _ok(_lib.topk_select(_ptr(scores), _ptr(seq_lens), _ptr(k_per_seq), k_max, shape, block,
                         _ptr(idx), *_wsargs(ws), _stream(stream)))


def sparse_decode_attn(Q, K, V, seq_lens, idx, k_per_seq, k_max: int, block: int, scale: float, O,
                       ws, stream=None, shape=None):
    s = shape or shape_of(Q, K)
    _ok(_lib.sparse_decode_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(seq_lens), _ptr(idx),
                                _ptr(k_per_seq), k_max, block, s, scale, _ptr(O), *_wsargs(ws),
                                _stream(stream)))


def sparse_decode_attn_noalloc(Q, K, V, seq_lens, idx, k_per_seq, k_max: int, block: int,
                               scale: float, O, stream=None, shape=None):
    """sparse_decode_attn with the library's fixed internal scratch instead of a workspace
    (for callers that cannot allocate one); calls on one device must not overlap."""
    s = shape or shape_of(Q, K)
    _ok(_lib.sparse_decode_attn_noalloc(_ptr(Q), _ptr(K), _ptr(V), _ptr(seq_lens), _ptr(idx),
                                        _ptr(k_per_seq), k_max, block, s, scale, _ptr(O),
                                        _stream(stream)))


def step_args(Q, K, V, seq_lens, O, ws, *, mode: int, scale: float, k_max: int = 0, block: int = 1,
              k_per_seq=None, Kmean=None, idx_in=None, idx_out=None, flags: int = 0) -> tsa_step_args:
    a = tsa_step_args()
    a.shape = shape_of(Q, K)
    a.Q, a.K, a.V, a.Kmean = _ptr(Q), _ptr(K), _ptr(V), _ptr(Kmean)
    a.seq_lens, a.k_per_seq = _ptr(seq_lens), _ptr(k_per_seq)
    a.k_max, a.block, a.mode, a.scale = k_max, block, mode, scale
    a.idx_in, a.idx_out, a.O = _ptr(idx_in), _ptr(idx_out), _ptr(O)
    a.ws, a.ws_bytes = _wsargs(ws)
    a.flags = flags
    return a


def decode_step(args: tsa_step_args, stream=None):
    _ok(_lib.tsa_decode_step(ctypes.byref(args), _stream(stream)))


def index_overlap(idx, counts, M, ws, stream=None):
    """Overlap of L layers' index lists idx [L, B, Hkv, k_max] (int32, device) into
    counts [L, L, B*Hkv] int32 and M [L, L] float64 (either may be None)."""
    L, units, k_max = idx.shape[0], math.prod(idx.shape[1:-1]), idx.shape[-1]
    _ok(_lib.tsa_index_overlap(_ptr(idx), L, units, k_max, _ptr(counts), _ptr(M), *_wsargs(ws),
                               _stream(stream)))


def reuse_policy(M, theta: float, force_full=None):
    """HyLRA's reuse policy from the similarity matrix M [L, L] (host, float64,
    row = target layer): returns (source [L] int32 numpy array, n_full, total_sim)."""
    import numpy as np

    Mh = np.ascontiguousarray(M.cpu().numpy() if isinstance(M, torch.Tensor) else M, dtype=np.float64)
    L = Mh.shape[0]
    assert Mh.shape == (L, L)
    ff = None if force_full is None else np.ascontiguousarray(np.asarray(force_full, dtype=np.uint8))
    src = np.empty(L, dtype=np.int32)
    nf = ctypes.c_int32()
    sim = ctypes.c_double()
    _ok(_lib.tsa_reuse_policy(Mh.ctypes.data, L, float(theta), None if ff is None else ff.ctypes.data,
                              src.ctypes.data, ctypes.byref(nf), ctypes.byref(sim)))
    return src, nf.value, sim.value


def shard_workspace_size(shard_shape: tsa_shape, k_max: int, n_shards: int) -> int:
    n = _lib.tsa_shard_workspace_size(shard_shape, k_max, n_shards)
    if n == 0:
        raise TsaError(TSA_ERR_INVALID_ARG, last_error())
    return int(n)


def shard_select(Q, K_shard, shard_lens, k_per_seq, k_max: int, scale: float, row0: int, cand_scores, cand_rows,
                 ws, stream=None):
    _ok(_lib.tsa_shard_select(_ptr(Q), _ptr(K_shard), _ptr(shard_lens), shape_of(Q, K_shard), _ptr(k_per_seq),
                              k_max, scale, row0, _ptr(cand_scores), _ptr(cand_rows), *_wsargs(ws), _stream(stream)))


def shard_merge(cand_scores, cand_rows, shape: tsa_shape, k_per_seq, k_max: int, idx, ws, stream=None):
    _ok(_lib.tsa_shard_merge(_ptr(cand_scores), _ptr(cand_rows), cand_scores.shape[0], shape, _ptr(k_per_seq),
                             k_max, _ptr(idx), *_wsargs(ws), _stream(stream)))


def shard_attend(Q, K_shard, V_shard, shard_lens, idx, k_per_seq, k_max: int, row0: int, scale: float, O_part,
                 lse_part, ws, stream=None):
    _ok(_lib.tsa_shard_attend(_ptr(Q), _ptr(K_shard), _ptr(V_shard), _ptr(shard_lens), shape_of(Q, K_shard),
                              _ptr(idx), _ptr(k_per_seq), k_max, row0, scale, _ptr(O_part), _ptr(lse_part),
                              *_wsargs(ws), _stream(stream)))


def shard_combine(O_parts, lse_parts, shape: tsa_shape, O, stream=None):
    _ok(_lib.tsa_shard_combine(_ptr(O_parts), _ptr(lse_parts), O_parts.shape[0], shape, _ptr(O), _stream(stream)))


def check_device_status(ws, stream=None):
    _ok(_lib.tsa_check_device_status(_ptr(ws), _stream(stream)))


def launch_count() -> int:
    return int(_lib.tsa_launch_count())


def hbm_copy(src, dst, nbytes: int, stream=None):
    _ok(_lib.tsa_hbm_copy(_ptr(src), _ptr(dst), nbytes, _stream(stream)))


def hbm_read(src, nbytes: int, ws, stream=None):
    _ok(_lib.tsa_hbm_read(_ptr(src), nbytes, *_wsargs(ws), _stream(stream)))


def hbm_gather(base, rows, ws, stream=None):
    """Gather the 256-byte rows `rows` (int32, device) of `base` (the probe; nothing is kept)."""
    nbytes = base.numel() * base.element_size()
    _ok(_lib.tsa_hbm_gather(_ptr(base), nbytes, _ptr(rows), rows.numel(), *_wsargs(ws), _stream(stream)))
