"""Failure detection without a GPU fault: a bounded device-side wait that runs
out is reported as TSA_ERR_DEVICE_TIMEOUT, and the context stays usable.

The library's waits on shared-memory barriers (the tcgen05 scorer's tile ring
and accumulators, the attention's contiguous-tile ring) give up after a fixed
number of polls, raise the device flag, stop, and wait (bounded) for the loads
they issued before the CTA leaves.  A test-only build of the same sources,
libtsa_debug.so, polls only ~1000 times and has one knob, tsa_debug_skip_tile,
that leaves one tile's load out in CTA (0, 0): nothing is ever armed or copied
for that tile, so the waits on it run out while no copy is in flight.  The
product library has neither (the CPU test checks it exports no debug symbol).
"""
import ctypes
import math
import os

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
DEBUG_LIB = os.path.join(os.path.dirname(tsa._LIB_PATH), "libtsa_debug.so")


@pytest.fixture(scope="module")
def dbg():
    if not os.path.exists(DEBUG_LIB):
        from top_sparse_attention_02_b200 import build

        build.build(debug=True)
    lib = ctypes.CDLL(DEBUG_LIB)  # its own copy of every symbol, separate from libtsa.so
    for name, (res, argt) in tsa._SIGS.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, argt
    lib.tsa_debug_skip_tile.restype = ctypes.c_int
    lib.tsa_debug_skip_tile.argtypes = [ctypes.c_int, ctypes.c_int]
    yield lib
    lib.tsa_debug_skip_tile(0, -1)
    lib.tsa_debug_skip_tile(1, -1)


def _status(lib, ws):
    return lib.tsa_check_device_status(tsa._ptr(ws), None)


def test_scorer_wait_runs_out_then_recovers(dbg, cuda_dev):
    B, Hq, Hkv, N = 1, 8, 2, 1024  # 8 CTAs a unit, one 128-row tile each
    L = inputs.decode_layer(B, Hq, Hkv, N, [N], plant_frac=0.01, seed=21)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    shape = tsa.tsa_shape(B, Hq, Hkv, N, 128)
    S = torch.zeros(B, Hkv, N, dtype=torch.float32, device=cuda_dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_dev)
    args = (tsa._ptr(Q), tsa._ptr(K), tsa._ptr(ln), shape, 1, SCALE, tsa._ptr(S), tsa._ptr(ws), 256, None)

    assert dbg.tsa_debug_skip_tile(0, 0) == 0
    assert dbg.sparse_decode_score(*args) == tsa.TSA_OK
    assert _status(dbg, ws) == tsa.TSA_ERR_DEVICE_TIMEOUT
    assert _status(dbg, ws) == tsa.TSA_OK  # the read cleared the flag

    # the same build, no tile left out: the scores are right again
    assert dbg.tsa_debug_skip_tile(0, -1) == 0
    assert dbg.sparse_decode_score(*args) == tsa.TSA_OK
    assert _status(dbg, ws) == tsa.TSA_OK
    ref = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
    np.testing.assert_allclose(S.cpu().numpy(), ref, rtol=2e-5, atol=2e-5)

    # and the product library in the same process: a whole SELECT step
    k = 64
    O, idx = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k)
    gi = idx.cpu().numpy()
    compare_idx(gi, ref, [N], [k])
    check_output(O.cpu().numpy(), oracle.attn(L.Q, L.K, L.V, L.seq_lens, gi, [k], k, 1, SCALE), "after timeout")


def test_attention_wait_runs_out_then_recovers(dbg, cuda_dev):
    B, Hq, Hkv, N = 1, 8, 2, 1024  # full attention: contiguous 128-row tiles by TMA, one a CTA
    L = inputs.decode_layer(B, Hq, Hkv, N, [N], seed=22)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    shape = tsa.tsa_shape(B, Hq, Hkv, N, 128)
    nws = tsa.workspace_size(shape, 0, 1, tsa.FULL)
    ws = torch.zeros(nws, dtype=torch.uint8, device=cuda_dev)
    O = torch.zeros(B, Hq, 128, dtype=torch.float32, device=cuda_dev)
    args = (tsa._ptr(Q), tsa._ptr(K), tsa._ptr(V), tsa._ptr(ln), None, None, 0, 1, shape, SCALE, tsa._ptr(O),
            tsa._ptr(ws), nws, None)

    assert dbg.tsa_debug_skip_tile(1, 0) == 0
    assert dbg.sparse_decode_attn(*args) == tsa.TSA_OK
    assert _status(dbg, ws) == tsa.TSA_ERR_DEVICE_TIMEOUT

    assert dbg.tsa_debug_skip_tile(1, -1) == 0
    assert dbg.sparse_decode_attn(*args) == tsa.TSA_OK
    assert _status(dbg, ws) == tsa.TSA_OK
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE)
    check_output(O.cpu().numpy(), ref, "debug build, no tile left out")

    O2, _ = G.run_attn(Q, K, V, ln, None, None, 0, 1, SCALE)  # the product library
    check_output(O2.cpu().numpy(), ref, "product library after the timeout")
