"""The C ABI without a GPU: the library loads, exports every declared symbol,
and rejects bad arguments on the host before anything is enqueued."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tsa.h")


@pytest.fixture(scope="module")
def tsa():
    from top_sparse_attention_02_b200 import build

    build.build()
    from top_sparse_attention_02_b200 import binding

    return binding


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b([A-Za-z_]\w*)\s*\([^;{]*\)\s*;", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("sparse_decode_score", "topk_select", "sparse_decode_attn", "tsa_decode_step",
                 "tsa_block_summarize", "tsa_workspace_size", "tsa_check_device_status",
                 "tsa_index_overlap", "tsa_reuse_policy"):
        assert want in names


def test_library_exports_every_declared_symbol(tsa):
    so = os.path.join(ROOT, "top_sparse_attention_02_b200", "libtsa.so")
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, f"{name} declared in tsa.h but not exported"
        assert getattr(tsa.lib(), name) is not None
    # the test-only knobs exist in libtsa_debug.so alone
    assert not any("debug" in n for n in exported), "the product library exports a debug knob"
    dbg = os.path.join(ROOT, "top_sparse_attention_02_b200", "libtsa_debug.so")
    if os.path.exists(dbg):
        out = subprocess.run(["nm", "-D", "--defined-only", dbg], capture_output=True, text=True,
                             check=True).stdout
        names = {line.split()[-1] for line in out.splitlines() if line.strip()}
        assert "tsa_debug_skip_tile" in names and set(declared_functions()) <= names


def _shape(tsa, B=1, Hq=8, Hkv=2, N=4096, d=128):
    return tsa.tsa_shape(B, Hq, Hkv, N, d)


def test_workspace_size_is_host_only_and_ordered(tsa):
    s = _shape(tsa)
    sel = tsa.workspace_size(s, 128, 1, tsa.SELECT)
    reu = tsa.workspace_size(s, 128, 1, tsa.REUSE)
    full = tsa.workspace_size(s, 0, 1, tsa.FULL)
    assert sel > reu >= 256 and full >= 256
    assert sel % 256 == 0 and reu % 256 == 0
    # SELECT adds the fp32 score buffer (units * Ncap * 4 bytes, 256-aligned); the
    # scorer's top-digit histograms (units * 2048 * 4 bytes) are in every layout
    assert sel - reu == 2 * 4096 * 4
    assert reu >= 256 + 2 * 2048 * 4 and full >= 256 + 2 * 2048 * 4
    # a full layer that also hands on its top-k adds the same score room
    assert tsa.workspace_size(s, 128, 1, tsa.FULL) - full == 2 * 4096 * 4
    assert tsa.workspace_size(s, 128, 128, tsa.FULL) - full == 256
    big = tsa.tsa_shape(1, 32, 8, 131072, 128)
    assert tsa.workspace_size(big, 2621, 1, tsa.SELECT) >= 8 * 131072 * 4


@pytest.mark.parametrize("shape,block,mode,msg", [
    ((1, 8, 2, 4096, 64), 1, 1, "head dimension"),
    ((1, 8, 3, 4096, 128), 1, 1, "multiple"),
    ((1, 12, 4, 4096, 128), 1, 1, "GQA group"),
    ((1, 8, 2, 4096, 128), 0, 1, "block"),
    ((1, 8, 2, 4096, 128), 1, 7, "mode"),
    ((-1, 8, 2, 4096, 128), 1, 1, "shape"),
])
def test_workspace_size_rejects(tsa, shape, block, mode, msg):
    assert tsa.lib().tsa_workspace_size(tsa.tsa_shape(*shape), 16, block, mode) == 0
    assert msg in tsa.last_error()


def _call_attn(tsa, *, Q=0x1000, K=0x2000, V=0x3000, lens=0x4000, idx=0x5000, k_max=16, block=1,
               shape=None, scale=0.1, O=0x6000, ws=0x10000, ws_bytes=1 << 30):
    # fake but aligned addresses: every one of these calls must fail validation,
    # so no address is ever dereferenced or handed to the device
    shape = shape or _shape(tsa)
    return tsa.lib().sparse_decode_attn(Q, K, V, lens, idx, None, k_max, block, shape, scale, O, ws,
                                        ws_bytes, None)


@pytest.mark.parametrize("kw,status,msg", [
    (dict(Q=None), 1, "NULL"),
    (dict(O=0x6004), 1, "aligned"),
    (dict(K=0x2008), 1, "aligned"),
    (dict(scale=0.0), 1, "scale"),
    (dict(scale=float("nan")), 1, "scale"),
    (dict(scale=-1.0), 1, "scale"),
    (dict(k_max=-1), 1, "k_max"),
    (dict(k_max=0), 1, "k_max"),
    (dict(block=0), 1, "block"),
    (dict(ws=None), 3, "NULL"),
    (dict(ws=0x10010), 3, "256-byte"),
    (dict(ws_bytes=100), 3, "needs"),
])
def test_attn_argument_errors(tsa, kw, status, msg):
    assert _call_attn(tsa, **kw) == status
    assert msg in tsa.last_error()


def test_unsupported_group(tsa):
    assert _call_attn(tsa, shape=tsa.tsa_shape(1, 48, 3, 64, 128)) == tsa.TSA_ERR_UNSUPPORTED


def test_score_and_topk_argument_errors(tsa):
    L = tsa.lib()
    s = _shape(tsa)
    assert L.sparse_decode_score(0x1000, None, 0x3000, s, 1, 0.1, 0x4000, 0x10000, 1 << 20, None) == 1
    assert L.sparse_decode_score(0x1000, 0x2000, 0x3000, s, 1, 0.1, 0x4000, 0x10000, 10, None) == 3
    assert L.topk_select(0x1000, 0x2000, None, -3, s, 1, 0x3000, 0x10000, 1 << 20, None) == 1
    huge = tsa.tsa_shape(1, 8, 2, 1 << 21, 128)
    assert L.topk_select(0x1000, 0x2000, None, 8, huge, 1, 0x3000, 0x10000, 1 << 20, None) == 2
    assert "cluster capacity" in tsa.last_error()


def test_decode_step_argument_errors(tsa):
    class T:  # stand-in tensors with fake aligned device addresses
        def __init__(self, addr, shape=()):
            self.addr, self.shape = addr, shape

        def data_ptr(self):
            return self.addr

    Q = T(0x1000, (1, 8, 128))
    K = T(0x2000, (1, 2, 4096, 128))
    ws = T(0x10000)
    ws.numel = lambda: 1 << 30
    ws.element_size = lambda: 1
    a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=tsa.SELECT, scale=0.1,
                      k_max=16, idx_out=None)
    assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 1 and "idx_out" in tsa.last_error()
    a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=tsa.REUSE, scale=0.1, k_max=16)
    assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 1 and "idx_in" in tsa.last_error()
    a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=tsa.SELECT, scale=0.1,
                      k_max=16, block=128, idx_out=T(0x7000))
    assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 1 and "Kmean" in tsa.last_error()
    a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=tsa.FULL, scale=0.1, k_max=0,
                      idx_out=T(0x7000))
    assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 1 and "k_max > 0" in tsa.last_error()
    a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=tsa.FULL, scale=0.1, k_max=16,
                      block=128, idx_out=T(0x7000))
    assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 1 and "Kmean" in tsa.last_error()
    a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=tsa.REUSE, scale=0.1, k_max=16,
                      idx_in=T(0x7000), flags=6)
    assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 1 and "flags" in tsa.last_error()
    # an offloaded cache: a layer that selects must score block means
    for mode, idx_out in ((tsa.SELECT, T(0x7000)), (tsa.FULL, T(0x7000))):
        a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=mode, scale=0.1, k_max=16,
                          idx_out=idx_out, flags=tsa.KV_HOST)
        assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 2 and "block means" in tsa.last_error()
    a = tsa.step_args(Q, K, T(0x3000), T(0x4000), T(0x5000), ws, mode=9, scale=0.1, k_max=16)
    assert tsa.lib().tsa_decode_step(ctypes.byref(a), None) == 1 and "mode" in tsa.last_error()
    assert tsa.lib().tsa_decode_step(None, None) == 1


def test_index_overlap_argument_errors(tsa):
    L = tsa.lib()
    assert L.tsa_index_overlap(0x1000, 0, 4, 8, 0x2000, 0x3000, 0x10000, 256, None) == 1
    assert "n_layers" in tsa.last_error()
    assert L.tsa_index_overlap(0x1000, 1025, 4, 8, 0x2000, 0x3000, 0x10000, 256, None) == 1
    assert L.tsa_index_overlap(0x1000, 3, -1, 8, 0x2000, 0x3000, 0x10000, 256, None) == 1
    assert L.tsa_index_overlap(None, 3, 4, 8, 0x2000, 0x3000, 0x10000, 256, None) == 1
    assert L.tsa_index_overlap(0x1000, 3, 4, 8, None, None, 0x10000, 256, None) == 1
    assert "NULL" in tsa.last_error()
    assert L.tsa_index_overlap(0x1000, 3, 4, 8, 0x2000, None, None, 256, None) == 3
    assert L.tsa_index_overlap(0x1000, 3, 4, 8, 0x2000, None, 0x10000, 100, None) == 3


def test_hbm_copy_argument_errors(tsa):
    assert tsa.lib().tsa_hbm_copy(0x1000, 0x2000, 17, None) == 1
    assert tsa.lib().tsa_hbm_copy(None, 0x2000, 16, None) == 1


def test_hbm_read_argument_errors(tsa):
    # rejected on the host, before any launch: size or pointer not 16-byte multiples, NULL, no workspace
    assert tsa.lib().tsa_hbm_read(0x1000, 17, 0x100000, 256, None) == 1
    assert tsa.lib().tsa_hbm_read(0x1008, 16, 0x100000, 256, None) == 1
    assert tsa.lib().tsa_hbm_read(None, 16, 0x100000, 256, None) == 1
    assert tsa.lib().tsa_hbm_read(0x1000, 16, None, 256, None) == 3
    assert tsa.lib().tsa_hbm_read(0x1000, 16, 0x100000, 255, None) == 3


def test_binding_raises_on_error(tsa):
    with pytest.raises(tsa.TsaError) as e:
        tsa.workspace_size(tsa.tsa_shape(1, 8, 2, 64, 96), 4, 1, tsa.SELECT)
    assert "head dimension" in str(e.value)


def test_reuse_policy_matches_exhaustive_search(tsa):
    """The library's dynamic program (a host function) against the oracle's
    exhaustive search over every choice of full layers."""
    import numpy as np

    import oracle

    rng = np.random.default_rng(17)
    for trial in range(300):
        L = int(rng.integers(1, 11))
        if trial % 3 == 0:  # coarse values: many exact ties
            M = rng.integers(0, 5, (L, L)) / 4.0
        else:
            M = rng.random((L, L))
        theta = float(rng.choice([0.0, 0.25, 0.5, 0.7, 0.9]))
        ff = (rng.random(L) < 0.15).astype(np.uint8) if trial % 2 else None
        got = tsa.reuse_policy(M, theta, ff)
        want = oracle.reuse_policy(M, theta, ff)
        assert got[0].tolist() == want[0].tolist(), (trial, M, theta, ff)
        assert got[1] == want[1] and got[2] == want[2]


def test_reuse_policy_argument_errors(tsa):
    import numpy as np

    L = tsa.lib()
    assert L.tsa_reuse_policy(None, 3, 0.5, None, 0x1000, None, None) == 1
    M = np.zeros((2, 2))
    assert L.tsa_reuse_policy(M.ctypes.data, 0, 0.5, None, 0x1000, None, None) == 1
    assert L.tsa_reuse_policy(M.ctypes.data, 2, float("nan"), None, 0x1000, None, None) == 1
    assert "NaN" in tsa.last_error()


def test_shard_entry_points_argument_errors(tsa):
    """The sequence-sharding calls: host-side checks only (fake aligned addresses)."""
    L = tsa.lib()
    s = _shape(tsa, B=2, Hq=8, Hkv=2, N=1000)
    n1 = tsa.shard_workspace_size(s, 64, 1)
    n64 = tsa.shard_workspace_size(s, 64, 64)  # the merge's candidates: 4 units x 64 shards x 64
    assert n1 >= 256 + 4 * 2048 * 4 and n1 % 256 == 0
    # the merge's scratch starts after the flag, the histograms and the split counters
    assert n64 >= (256 + 4 * 2048 * 4 + 256) + 2 * (4 * 64 * 64 * 4)
    assert L.tsa_shard_workspace_size(s, 64, 65) == 0 and "n_shards" in tsa.last_error()
    args = (0x1000, 0x2000, 0x3000, s, None, 64, 0.1, 0, 0x4000, 0x5000, 0x10000, 1 << 30, None)
    # every call below fails a host-side check before anything is launched
    bad = list(args)
    bad[7] = -5
    assert L.tsa_shard_select(*bad) == 1 and "row0" in tsa.last_error()
    bad = list(args)
    bad[5] = 0
    assert L.tsa_shard_select(*bad) == 1 and "k_max" in tsa.last_error()
    bad = list(args)
    bad[1] = 0x2008
    assert L.tsa_shard_select(*bad) == 1 and "aligned" in tsa.last_error()
    bad = list(args)
    bad[11] = 100
    assert L.tsa_shard_select(*bad) == 3
    assert L.tsa_shard_merge(0x1000, 0x2000, 0, s, None, 64, 0x3000, 0x10000, 1 << 30, None) == 1
    assert L.tsa_shard_merge(0x1000, None, 2, s, None, 64, 0x3000, 0x10000, 1 << 30, None) == 1
    huge = tsa.tsa_shape(2, 8, 2, 1000, 128)
    assert L.tsa_shard_merge(0x1000, 0x2000, 64, huge, None, 1 << 16, 0x3000, 0x10000, 1 << 40, None) == 2
    assert "capacity" in tsa.last_error()
    assert L.tsa_shard_attend(0x1000, 0x2000, 0x3000, 0x4000, s, 0x5000, None, 64, -1, 0.1, 0x6000, 0x7000,
                              0x10000, 1 << 30, None) == 1
    assert L.tsa_shard_attend(0x1000, 0x2000, 0x3000, 0x4000, s, None, None, 64, 0, 0.1, 0x6000, 0x7000,
                              0x10000, 1 << 30, None) == 1
    assert L.tsa_shard_combine(0x1000, 0x2000, 0, s, 0x3000, None) == 1
    assert L.tsa_shard_combine(0x1008, 0x2000, 2, s, 0x3000, None) == 1 and "aligned" in tsa.last_error()
