"""sparse_decode_attn_noalloc: the attention stage for callers that cannot give
the library a workspace (its scratch is a fixed device array in the library).

Collected last on purpose, so that a run stopping at the first failure has
already run every other test.  Each case calls the new entry point twice in a
row, through the C ABI, and compares it with sparse_decode_attn (which uses a
caller-allocated workspace) and with the fp64 oracle on the same indices,
within the tolerances the parity tests use.  The device's free memory is the
same before and after the warm calls: they allocate nothing."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import check_output
from top_sparse_attention_02_b200 import binding as tsa
from top_sparse_attention_02_b200 import inputs

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


def _case(dev, B, Hq, Hkv, N, lens, k_max, block, seed):
    L = inputs.decode_layer(B, Hq, Hkv, N, lens, plant_frac=0.01, seed=seed, device=dev)
    rng = np.random.default_rng(seed)
    nb = [n if block == 1 else -(-n // block) for n in lens]
    idx = np.full((B, Hkv, k_max), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            m = min(k_max, nb[b])
            idx[b, h, :m] = np.sort(rng.choice(nb[b], size=m, replace=False))
    kreq = torch.tensor([k_max] * B, dtype=torch.int32, device=dev)
    return L, torch.from_numpy(idx).to(dev), kreq, idx


def _with_workspace(L, idx, kreq, k_max, block):
    ws = tsa.new_workspace(tsa.shape_of(L.Q, L.K), k_max, block, tsa.REUSE, L.Q.device)
    O = torch.empty(L.Q.shape, dtype=torch.float32, device=L.Q.device)
    tsa.sparse_decode_attn(L.Q, L.K, L.V, L.seq_lens, idx, kreq, k_max, block, SCALE, O, ws)
    tsa.check_device_status(ws)
    return O


def _no_alloc(L, idx, kreq, k_max, block):
    O = torch.full(L.Q.shape, float("nan"), dtype=torch.float32, device=L.Q.device)
    tsa.sparse_decode_attn_noalloc(L.Q, L.K, L.V, L.seq_lens, idx, kreq, k_max, block, SCALE, O)
    torch.cuda.synchronize()
    return O


@pytest.mark.parametrize("B,Hq,Hkv,N,lens,k_max,block", [
    (1, 32, 8, 131072, [131072], 2621, 1),      # the 128K, 50x shape
    (3, 8, 2, 5000, [5000, 1, 777], 300, 1),    # ragged lengths, some k > len
    (2, 32, 8, 9000, [9000, 4100], 32, 128),    # block mode
])
def test_no_alloc_matches_workspace_entry_twice(cuda_dev, B, Hq, Hkv, N, lens, k_max, block):
    L, idx, kreq, idx_np = _case(cuda_dev, B, Hq, Hkv, N, lens, k_max, block, seed=B + N)
    ref = _with_workspace(L, idx, kreq, k_max, block).cpu().numpy()
    Lc = [t.cpu() for t in (L.Q, L.K, L.V, L.seq_lens)]
    want = oracle.attn(*Lc, idx_np, [k_max] * B, k_max, block, SCALE)
    _no_alloc(L, idx, kreq, k_max, block)  # warm: the first call on a device may load the module
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):  # the second call runs on the scratch the first one left behind
        got = _no_alloc(L, idx, kreq, k_max, block).cpu().numpy()
        check_output(got, ref, "no-alloc attention vs the workspace entry point")
        check_output(got, want, "no-alloc attention vs the oracle")
    assert torch.cuda.mem_get_info()[0] == free0, "a warm call changed the device's free memory"
    # a second, different problem right after: nothing carries over between calls
    L2, idx2, kreq2, idx2_np = _case(cuda_dev, B, Hq, Hkv, N, lens, k_max, block, seed=B + N + 1)
    ref2 = _with_workspace(L2, idx2, kreq2, k_max, block).cpu().numpy()
    got2 = _no_alloc(L2, idx2, kreq2, k_max, block).cpu().numpy()
    check_output(got2, ref2, "no-alloc, new inputs")
    L2c = [t.cpu() for t in (L2.Q, L2.K, L2.V, L2.seq_lens)]
    check_output(got2, oracle.attn(*L2c, idx2_np, [k_max] * B, k_max, block, SCALE), "no-alloc, new inputs, oracle")


def test_no_alloc_dense_mode_twice(cuda_dev):
    L, _, _, _ = _case(cuda_dev, 2, 32, 8, 20000, [20000, 333], 1, 1, seed=5)
    ws = tsa.new_workspace(tsa.shape_of(L.Q, L.K), 0, 1, tsa.FULL, cuda_dev)
    ref = torch.empty(L.Q.shape, dtype=torch.float32, device=cuda_dev)
    tsa.sparse_decode_attn(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE, ref, ws)
    want = oracle.attn(L.Q.cpu(), L.K.cpu(), L.V.cpu(), L.seq_lens.cpu(), None, None, 0, 1, SCALE)
    for _ in range(2):
        O = torch.empty_like(ref)
        tsa.sparse_decode_attn_noalloc(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE, O)
        torch.cuda.synchronize()
        check_output(O.cpu().numpy(), ref.cpu().numpy(), "no-alloc dense")
        check_output(O.cpu().numpy(), want, "no-alloc dense vs the oracle")


def test_no_alloc_rejects_shapes_beyond_its_scratch(cuda_dev):
    # 65528 units x 1 split x 4 heads x 528 bytes of partials is far beyond 8 MiB
    B, Hq, Hkv, N = 8191, 32, 8, 64
    shape = tsa.tsa_shape(B, Hq, Hkv, N, 128)
    Q = torch.zeros(16, dtype=torch.bfloat16, device=cuda_dev)  # never read: rejected first
    with pytest.raises(tsa.TsaError) as e:
        tsa.sparse_decode_attn_noalloc(Q, Q, Q, Q, Q, None, 64, 1, SCALE, Q, shape=shape)
    assert e.value.status == tsa.TSA_ERR_WORKSPACE
    assert "fixed array" in str(e.value)
