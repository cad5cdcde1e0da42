"""GPU vs oracle parity, stage by stage and for whole decode steps (needs a B200)."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import check_output, compare_idx, sub_problem
from top_sparse_attention_02_b200 import binding as tsa
from top_sparse_attention_02_b200 import inputs

import gpu_run as G

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


def layer(B, Hq, Hkv, N, lens=None, seed=0, plant=0.01, tail_fill=None):
    lens = lens if lens is not None else [N] * B
    return inputs.decode_layer(B, Hq, Hkv, N, lens, plant_frac=plant, seed=seed, tail_fill=tail_fill)


# ------------------------------------------------------------------ score stage

@pytest.mark.parametrize("Hq,Hkv,N,lens", [(8, 2, 4096, None), (32, 8, 1000, [1000, 999, 1, 0]),
                                           (8, 8, 333, None), (16, 8, 2048, [2048, 77]),
                                           (64, 8, 777, None)])
def test_score_stage(cuda_dev, Hq, Hkv, N, lens):
    B = len(lens) if lens else 1
    L = layer(B, Hq, Hkv, N, lens, seed=3, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    S = G.run_score(Q, K, ln, SCALE).cpu().numpy()
    ref = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
    for b in range(B):
        n = int(L.seq_lens[b])
        # fp32 sum of 128 exact bf16 products vs fp64: |err| <= 128 * 2^-24 * sum|terms|
        np.testing.assert_allclose(S[b, :, :n], ref[b, :, :n], rtol=2e-5, atol=2e-5)
        assert np.isnan(S[b, :, n:]).all(), "rows past len_b were written"


# ------------------------------------------------------------------ top-k stage (bit-exact)

def _topk_case(dev, S_np, lens, kreq, k_max, Hq=8, block=1, Ncap=None):
    S = torch.from_numpy(S_np.astype(np.float32)).to(dev)
    B, Hkv, rows = S.shape
    lens_t = torch.tensor(lens, dtype=torch.int32, device=dev)
    Ncap = Ncap or rows
    got = G.run_topk(S, lens_t, kreq, k_max, Hq if Hq % Hkv == 0 else Hkv, Ncap, block).cpu().numpy()
    nrows = lens if block == 1 else [-(-x // block) for x in lens]
    want = oracle.topk(S_np.astype(np.float32).astype(np.float64), nrows,
                       kreq if kreq is not None else [k_max] * B, k_max)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("rows", [1, 31, 100, 4096, 16385, 40000, 131072])
def test_topk_exact_random(cuda_dev, rows):
    rng = np.random.default_rng(rows)
    B, Hkv = 2, 2
    S = rng.standard_normal((B, Hkv, rows))
    lens = [rows, max(rows // 3, 1)]
    for k in sorted({1, 2, min(rows, 17), max(rows // 50, 1), max(rows - 1, 1), rows, rows + 5}):
        _topk_case(cuda_dev, S, lens, [k, k], k, Hq=Hkv * 4)


def test_topk_ties_signed_zeros_and_duplicates(cuda_dev):
    rng = np.random.default_rng(7)
    rows = 20000
    S = rng.integers(-4, 5, size=(1, 2, rows)).astype(np.float64) * 0.5  # heavy exact ties
    S[0, 0, ::7] = -0.0
    S[0, 1] = 0.0  # every score tied: lowest indices win
    S[0, 1, 5::11] = -0.0
    for k in (1, 10, 1234, 19999):
        _topk_case(cuda_dev, S, [rows], [k], k, Hq=8)
    S2 = -np.abs(rng.standard_normal((1, 2, 5000))) - 1.0  # all negative
    _topk_case(cuda_dev, S2, [5000], [100], 100)


def test_topk_many_units_and_wide_clusters(cuda_dev):
    """Launch shapes of the top-k: many units, a unit wider than 8 slices (a
    non-portable cluster of 16), and exact ties across a cluster of 3 (the
    boundary bin overflows rank 0's buffer)."""
    rng = np.random.default_rng(23)
    S = rng.standard_normal((40, 8, 20000))
    lens = rng.integers(1, 20001, size=40).tolist()
    kreq = [int(x) for x in rng.integers(1, 70, size=40)]
    _topk_case(cuda_dev, S, lens, kreq, 69, Hq=32)
    S = rng.standard_normal((1, 1, 250000))
    for k in (1, 6000, 249999):
        _topk_case(cuda_dev, S, [250000], [k], k, Hq=4)
    S = np.zeros((2, 1, 40000))
    S[1, 0, 20000:] = 1.0
    for k in (5, 12345, 30000):
        _topk_case(cuda_dev, S, [40000, 39000], [k, k], k, Hq=2)


def test_topk_one_cta_per_unit_ties_and_overflow(cuda_dev):
    """The one-CTA-per-unit top-k (many units, or units of <= 8192 rows): heavy
    exact ties, where the candidate list overflows and every later pass streams
    the scores again, and k close to the unit's length."""
    rng = np.random.default_rng(29)
    S = rng.integers(-2, 3, size=(2, 2, 6000)).astype(np.float64)
    S[0, 1] = 0.0
    S[1, 0, ::5] = -0.0
    for k in (1, 10, 1234, 5999):
        _topk_case(cuda_dev, S, [6000, 4321], [k, k], k, Hq=4)
    S = rng.integers(-1, 2, size=(20, 8, 3000)).astype(np.float64)  # 160 units
    lens = rng.integers(1, 3001, size=20).tolist()
    kreq = [int(x) for x in rng.integers(1, 3001, size=20)]
    _topk_case(cuda_dev, S, lens, kreq, 3000, Hq=16)


def test_topk_ragged_per_sequence_k(cuda_dev):
    rng = np.random.default_rng(11)
    B, Hkv, rows = 6, 3, 9000
    S = rng.standard_normal((B, Hkv, rows))
    lens = [9000, 8192, 1, 0, 4097, 333]
    kreq = [180, 17, 5, 3, 4097, 0]
    _topk_case(cuda_dev, S, lens, kreq, 4097, Hq=Hkv * 2)


# ------------------------------------------------------------------ attention stage

def _rand_idx(rng, B, Hkv, lens, k_max, kb):
    idx = np.full((B, Hkv, k_max), -1, dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            n = min(kb[b], lens[b])
            idx[b, h, :n] = np.sort(rng.choice(lens[b], size=n, replace=False))
    return idx


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (32, 8), (8, 8), (64, 8), (4, 2)])
def test_attn_stage_random_sets(cuda_dev, Hq, Hkv):
    rng = np.random.default_rng(Hq * 10 + Hkv)
    lens = [3000, 1, 700]
    L = layer(3, Hq, Hkv, 3000, lens, seed=5, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    kb = [611, 1, 700]
    idx = _rand_idx(rng, 3, Hkv, lens, 700, kb)
    O, _ = G.run_attn(Q, K, V, ln, torch.from_numpy(idx).to(cuda_dev), kb, 700, 1, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, kb, 700, 1, SCALE)
    check_output(O.cpu().numpy(), ref, "random sets")


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("k", [300, 600, 850])
def test_attn_cluster_combine_uneven_owners(cuda_dev, g, k):
    """4 units (2 sequences x 2 kv-heads) with k = 300, 600, 850 take ceil(k / 128)
    = 3, 5, 7 splits, one cluster a unit: the 32g output slots split unevenly
    among the owner CTAs (the last owns fewer).  The second sequence's 3 rows
    leave most of its CTAs without rows (they still send their empty partials)."""
    rng = np.random.default_rng(k * 10 + g)
    Hkv = 2
    lens = [2000, 5]
    L = layer(2, g * Hkv, Hkv, 2000, lens, seed=k + g, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    kb = [k, 3]
    idx = _rand_idx(rng, 2, Hkv, lens, k, kb)
    O, _ = G.run_attn(Q, K, V, ln, torch.from_numpy(idx).to(cuda_dev), kb, k, 1, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, kb, k, 1, SCALE)
    check_output(O.cpu().numpy(), ref, f"g={g}, k={k}")


def test_attn_stage_sliding_window_and_padding(cuda_dev):
    lens = [500, 64]
    L = layer(2, 8, 2, 512, lens, seed=9, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    idx = np.full((2, 2, 64), -1, dtype=np.int32)
    idx[0, :, :64] = np.arange(436, 500)  # the last 64 tokens (a sliding window)
    idx[1, :, :10] = np.arange(54, 64)
    idx[1, 1, 3] = -1  # a skipped entry inside the list
    kb = [64, 64]
    O, _ = G.run_attn(Q, K, V, ln, torch.from_numpy(idx).to(cuda_dev), kb, 64, 1, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, kb, 64, 1, SCALE)
    check_output(O.cpu().numpy(), ref, "window")


@pytest.mark.parametrize("lens", [[5000, 1], [128, 129], [0, 77]])
def test_attn_dense_mode(cuda_dev, lens):
    L = layer(len(lens), 32, 8, 5000, lens, seed=13, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    O, _ = G.run_attn(Q, K, V, ln, None, None, 0, 1, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE)
    check_output(O.cpu().numpy(), ref, "dense")


@pytest.mark.parametrize("Ncap", [1024, 1000])
def test_attn_block_mode_expansion(cuda_dev, Ncap):
    """128-token blocks; Ncap = 1000 puts the partial last block against the end of
    each unit's cache, so its 128-row tile reaches into the next unit's rows (or
    past the end of the cache for the last unit)."""
    lens = [1000, 130]
    L = layer(2, 8, 2, Ncap, lens, seed=17, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    idx = np.full((2, 2, 4), -1, dtype=np.int32)
    idx[0, 0, :3] = [0, 5, 7]  # block 7 is the partial last block (rows 896..999)
    idx[0, 1, :4] = [1, 2, 3, 4]
    idx[1, 0, :2] = [0, 1]  # block 1 holds 2 valid rows
    idx[1, 1, :1] = [1]
    kb = [4, 2]
    O, _ = G.run_attn(Q, K, V, ln, torch.from_numpy(idx).to(cuda_dev), kb, 4, 128, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, kb, 4, 128, SCALE)
    check_output(O.cpu().numpy(), ref, "block expansion")


# ------------------------------------------------------------------ block summaries

def test_block_summarize(cuda_dev):
    lens = [1000, 128, 5]
    L = layer(3, 8, 2, 1024, lens, seed=19, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    M = G.block_means(K, ln, 128).cpu().numpy()
    ref = oracle.block_means(L.K, L.seq_lens, 128)
    for b, n in enumerate(lens):
        nb = -(-n // 128)
        np.testing.assert_allclose(M[b, :, :nb], ref[b, :, :nb], rtol=0, atol=2e-6)


# ------------------------------------------------------------------ whole steps

def _select_and_check(dev, L, kreq, k_max, block=1, units=None):
    Q, K, V, ln = G.to_dev(L, dev)
    Kmean = G.block_means(K, ln, block) if block > 1 else None
    O, idx = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, block=block, kreq=kreq,
                    Kmean=Kmean)
    idx_np = idx.cpu().numpy()
    if block == 1:
        S = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
        nrows = L.seq_lens.numpy()
    else:
        nrows = oracle.nblocks_of(L.seq_lens, block)
        S = oracle.block_scores(L.Q, oracle.block_means(L.K, L.seq_lens, block), nrows, SCALE)
    counts = compare_idx(idx_np, S, nrows, kreq)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx_np, kreq, k_max, block, SCALE)
    check_output(O.cpu().numpy(), ref, "select step")
    return counts, idx, O, (Q, K, V, ln)


def test_tiny_workload_end_to_end(cuda_dev):
    """B=1, 8/2 heads, N=4096, k=128, 1% planted keys, seed 0: the small workload."""
    L = layer(1, 8, 2, 4096, seed=0, plant=0.01)
    counts, idx, O, _ = _select_and_check(cuda_dev, L, [128], 128)
    assert counts["exact"] + counts["near_tie"] == 2


@pytest.mark.parametrize("case", ["ragged", "k_gt_len", "k_eq_len", "k1", "equal_keys", "len_lt_128"])
def test_select_step_edge_cases(cuda_dev, case):
    if case == "ragged":
        L, kreq, k_max = layer(4, 32, 8, 3000, [3000, 1, 129, 0], seed=21, tail_fill=float("nan")), \
            [60, 60, 60, 60], 60
    elif case == "k_gt_len":
        L, kreq, k_max = layer(2, 8, 2, 256, [100, 256], seed=22), [150, 150], 150
    elif case == "k_eq_len":
        L, kreq, k_max = layer(1, 8, 2, 300, [300], seed=23), [300], 300
    elif case == "k1":
        L, kreq, k_max = layer(2, 16, 2, 2000, [2000, 1500], seed=24), [1, 1], 1
    elif case == "equal_keys":
        L = layer(1, 8, 2, 1000, seed=25)
        L.K[0, :, :] = L.K[0, :, :1]
        kreq, k_max = [40], 40
    else:
        L, kreq, k_max = layer(3, 8, 2, 127, [127, 100, 5], seed=26, tail_fill=float("nan")), \
            [12, 12, 12], 12
    counts, idx, O, _ = _select_and_check(cuda_dev, L, kreq, k_max)
    if case == "equal_keys":
        assert (idx[0, :, :40].cpu().numpy() == np.arange(40)).all()


def test_block_mode_step(cuda_dev):
    L = layer(2, 32, 8, 9000, [9000, 4100], seed=27, plant=0.01)
    counts, idx, O, _ = _select_and_check(cuda_dev, L, [32, 32], 32, block=128)
    assert counts["exact"] + counts["near_tie"] == 16


def test_reuse_and_full_steps(cuda_dev):
    L0 = layer(2, 32, 8, 6000, [6000, 3001], seed=29)
    counts, idx, O, _ = _select_and_check(cuda_dev, L0, [120, 120], 120)
    L1 = inputs.decode_layer(2, 32, 8, 6000, [6000, 3001], seed=30, Q=inputs.drift_query(L0.Q, 0.3, 31))
    Q, K, V, ln = G.to_dev(L1, cuda_dev)
    before = idx.clone()
    O1, _ = G.step(Q, K, V, ln, mode=tsa.REUSE, scale=SCALE, k_max=120, kreq=[120, 120], idx_in=idx)
    assert torch.equal(before, idx), "reuse must not touch the indices"
    ref = oracle.attn(L1.Q, L1.K, L1.V, L1.seq_lens, idx.cpu().numpy(), [120, 120], 120, 1, SCALE)
    check_output(O1.cpu().numpy(), ref, "reuse")
    O2, _ = G.step(Q, K, V, ln, mode=tsa.FULL, scale=SCALE)
    ref2 = oracle.attn(L1.Q, L1.K, L1.V, L1.seq_lens, None, None, 0, 1, SCALE)
    check_output(O2.cpu().numpy(), ref2, "full")


def test_select_is_deterministic(cuda_dev):
    L = layer(4, 32, 8, 20000, seed=33)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    a = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=400)
    b = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=400)
    assert torch.equal(a[1], b[1])
    assert torch.equal(a[0].view(torch.int32), b[0].view(torch.int32))


# ------------------------------------------------------------------ device-side errors

def test_device_bounds_flag_and_recovery(cuda_dev):
    L = layer(2, 8, 2, 512, seed=35)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    bad = torch.tensor([512, 600], dtype=torch.int32, device=cuda_dev)  # 600 > Ncap
    with pytest.raises(tsa.TsaError) as e:
        G.step(Q, K, V, bad, mode=tsa.SELECT, scale=SCALE, k_max=8)
    assert e.value.status == tsa.TSA_ERR_DEVICE_BOUNDS
    idx = torch.full((2, 2, 4), -1, dtype=torch.int32, device=cuda_dev)
    idx[0, 0, 0] = 700  # row past len_b
    O, ws = G.run_attn(Q, K, V, ln, idx, [4, 4], 4, 1, SCALE, check=False)
    with pytest.raises(tsa.TsaError) as e:
        tsa.check_device_status(ws)
    assert e.value.status == tsa.TSA_ERR_DEVICE_BOUNDS
    tsa.check_device_status(ws)  # the flag was cleared by the read
    O, _ = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=8)  # the context still works
    assert torch.isfinite(O).all()


@pytest.mark.parametrize("dense", [True, False])
def test_attn_many_splits_workspace_combine(cuda_dev, dense):
    """Few units with a long range: more than 16 splits per unit, so the splits
    combine through the workspace (last CTA to arrive) instead of a cluster."""
    N = 20000
    L = layer(1, 8, 2, N, [N - 3], seed=41, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    if dense:
        O, _ = G.run_attn(Q, K, V, ln, None, None, 0, 1, SCALE)
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE)
    else:
        rng = np.random.default_rng(3)
        idx = _rand_idx(rng, 1, 2, [N - 3], 3000, [3000])
        O, _ = G.run_attn(Q, K, V, ln, torch.from_numpy(idx).to(cuda_dev), [3000], 3000, 1, SCALE)
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, [3000], 3000, 1, SCALE)
    check_output(O.cpu().numpy(), ref, "many splits")


def test_read_probe_runs_clean(cuda_dev):
    """tsa_hbm_read streams a buffer and writes nothing: the workspace's flag and
    fold words stay zero, and the buffer is unchanged."""
    buf = torch.full((1 << 20,), 7, dtype=torch.uint8, device=cuda_dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_dev)
    tsa.hbm_read(buf, buf.numel(), ws)
    tsa.hbm_read(buf, 4096 + 16, ws)  # a size that leaves a ragged tail for the last loop
    torch.cuda.synchronize()
    assert int(ws[:8].sum()) == 0
    assert bool((buf == 7).all())
    tsa.check_device_status(ws)


def test_gather_probe_runs_and_flags_bad_rows(cuda_dev):
    base = torch.zeros(1 << 20, dtype=torch.uint8, device=cuda_dev)  # 4096 rows of 256 B
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_dev)
    rows = torch.randint(0, 4096, (1000,), dtype=torch.int32, device=cuda_dev)
    tsa.hbm_gather(base, rows, ws)
    tsa.check_device_status(ws)
    rows[7] = 4096  # one past the end: skipped and flagged, never read
    tsa.hbm_gather(base, rows, ws)
    with pytest.raises(tsa.TsaError) as e:
        tsa.check_device_status(ws)
    assert e.value.status == tsa.TSA_ERR_DEVICE_BOUNDS


def test_select_steps_share_one_workspace(cuda_dev):
    """The scorer leaves a first-pass histogram in the workspace that the top-k
    kernel consumes and clears: consecutive steps on one workspace (with units
    where every row is taken, which skip the select) must each match the oracle."""
    B, Hq, Hkv, N = 3, 16, 4, 3000
    lens, kreq, k_max = [3000, 40, 2999], [50, 60, 50], 60
    ws = G.ws_for(torch.empty(B, Hq, 128, device=cuda_dev, dtype=torch.bfloat16),
                  torch.empty(B, Hkv, N, 128, device=cuda_dev, dtype=torch.bfloat16), k_max, 1, tsa.SELECT)
    for seed in (51, 52, 53):
        L = layer(B, Hq, Hkv, N, lens, seed=seed)
        Q, K, V, ln = G.to_dev(L, cuda_dev)
        O, idx = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, kreq=kreq, ws=ws)
        S = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
        compare_idx(idx.cpu().numpy(), S, lens, kreq)
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx.cpu().numpy(), kreq, k_max, 1, SCALE)
        check_output(O.cpu().numpy(), ref, f"step with seed {seed}")


def test_block_select_steps_share_one_workspace(cuda_dev):
    """Block mode: the block-mean scorer also leaves the first-pass histogram for
    the top-k; consecutive block-mode steps on one workspace each match the oracle."""
    B, Hq, Hkv, N, k = 2, 16, 4, 6000, 8
    lens = [6000, 1000]
    ws = G.ws_for(torch.empty(B, Hq, 128, device=cuda_dev, dtype=torch.bfloat16),
                  torch.empty(B, Hkv, N, 128, device=cuda_dev, dtype=torch.bfloat16), k, 128, tsa.SELECT)
    for seed in (61, 62):
        L = layer(B, Hq, Hkv, N, lens, seed=seed)
        Q, K, V, ln = G.to_dev(L, cuda_dev)
        Km = G.block_means(K, ln, 128)
        O, idx = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k, block=128, kreq=[k, k],
                        Kmean=Km, ws=ws)
        nb = oracle.nblocks_of(L.seq_lens, 128)
        S = oracle.block_scores(L.Q, oracle.block_means(L.K, L.seq_lens, 128), nb, SCALE)
        compare_idx(idx.cpu().numpy(), S, nb, [k, k])
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx.cpu().numpy(), [k, k], k, 128, SCALE)
        check_output(O.cpu().numpy(), ref, f"block step with seed {seed}")


@pytest.mark.parametrize("case", ["plain", "tied_top", "k_near_len", "tie_cut", "tie_overflow"])
def test_decode_step_topk_from_the_scorers_histogram(cuda_dev, case):
    """Inside a decode step the top-k of long units starts from the scorer's
    first-digit histogram (a cluster per unit, lists in registers and shared
    memory).  Its paths: the plain one; 7000 identical top keys (exact ties at T:
    the lists overflow and every later pass runs over all keys); k one short of
    the length; the k-th row's key copied to 20 other rows (exact ties at the
    boundary, cut by the lowest rows across the cluster's CTAs: rank 0 ranks the
    few keys sharing the first two digits directly); the same with 300 copies
    (more than 64 keys share the first two digits: the last digit by a
    histogram pass).  Two steps on one workspace check that the histogram is
    zeroed."""
    B, Hq, Hkv, N = 2, 16, 4, 20000
    lens = [20000, 15000]
    L = layer(B, Hq, Hkv, N, lens, seed=71)
    if case in ("tie_cut", "tie_overflow"):
        kreq, k_max = [400, 300], 400
        S0 = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
        rng = np.random.default_rng(7)
        ncopy = 20 if case == "tie_cut" else 300
        for b in range(B):
            n = lens[b]
            for h in range(Hkv):
                order = np.lexsort((np.arange(n), -S0[b, h, :n]))
                r = int(order[kreq[b] - 1])  # the k-th row
                dst = rng.choice(n, size=ncopy, replace=False)
                L.K[b, h, dst] = L.K[b, h, r].clone()
    elif case == "tied_top":
        S0 = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
        for b in range(B):
            for h in range(Hkv):
                top = int(np.argmax(S0[b, h, :lens[b]]))
                L.K[b, h, 5000:12000] = L.K[b, h, top]
        kreq, k_max = [100, 6000], 6000
    elif case == "k_near_len":
        kreq, k_max = [19999, 14999], 19999
    else:
        kreq, k_max = [400, 300], 400
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    ws = G.ws_for(Q, K, k_max, 1, tsa.SELECT)
    S = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
    for rep in range(2):
        O, idx = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, kreq=kreq, ws=ws)
        compare_idx(idx.cpu().numpy(), S, lens, kreq)
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx.cpu().numpy(), kreq, k_max, 1, SCALE)
        check_output(O.cpu().numpy(), ref, f"{case} step {rep}")


@pytest.mark.parametrize("N,lens,kreq", [(12000, [12000, 9000], [150, 2]),
                                         (200000, [200000, 123457], [4000, 2469])])
def test_decode_step_topk_cluster_shapes(cuda_dev, N, lens, kreq):
    """The decode step's top-k on a cluster of one CTA (12000 rows) and on 32
    scores a thread in a cluster of 7 (200000 rows); both steps on one workspace."""
    B, Hq, Hkv = 2, 8, 2
    L = layer(B, Hq, Hkv, N, lens, seed=83)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    k_max = max(kreq)
    ws = G.ws_for(Q, K, k_max, 1, tsa.SELECT)
    S = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
    for rep in range(2):
        O, idx = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, kreq=kreq, ws=ws)
        compare_idx(idx.cpu().numpy(), S, lens, kreq)
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx.cpu().numpy(), kreq, k_max, 1, SCALE)
        check_output(O.cpu().numpy(), ref, f"N={N} step {rep}")


# ------------------------------------------------------------------ full layers that hand on their top-k

@pytest.mark.parametrize("case", ["ragged", "long", "k_gt_len", "g1"])
def test_full_step_emits_topk(cuda_dev, case):
    """A fully attended layer (HyLRA, sec. 2.3: a sensitive layer) also writes
    the top-k a SELECT step would choose: O is the dense attention, idx the
    exact top-k of the group-max scaled scores (formed inside the attention);
    a REUSE step then attends over it."""
    if case == "ragged":
        L, kreq = layer(4, 32, 8, 3000, [3000, 1, 129, 0], seed=91, tail_fill=float("nan")), [60] * 4
    elif case == "long":  # several splits per unit, the top-k from the one-CTA-per-unit kernel
        L, kreq = layer(2, 16, 4, 70000, [70000, 41234], seed=92), [1400, 800]
    elif case == "k_gt_len":
        L, kreq = layer(2, 8, 2, 256, [100, 256], seed=93), [150, 150]
    else:  # one query head per KV head
        L, kreq = layer(2, 8, 8, 5000, [5000, 4999], seed=94), [77, 1]
    k_max = max(kreq)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    ws = G.ws_for(Q, K, k_max, 1, tsa.FULL)
    assert ws.numel() > G.ws_for(Q, K, 0, 1, tsa.FULL).numel()
    S = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE)
    for rep in range(2):
        O, idx = G.step(Q, K, V, ln, mode=tsa.FULL, scale=SCALE, k_max=k_max, kreq=kreq, ws=ws, emit=True)
        check_output(O.cpu().numpy(), ref, f"{case} full step {rep}")
        compare_idx(idx.cpu().numpy(), S, L.seq_lens.numpy(), kreq)
    O1, _ = G.step(Q, K, V, ln, mode=tsa.REUSE, scale=SCALE, k_max=k_max, kreq=kreq, idx_in=idx)
    ref1 = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx.cpu().numpy(), kreq, k_max, 1, SCALE)
    check_output(O1.cpu().numpy(), ref1, f"{case} reuse of the full layer's top-k")


def test_full_step_emits_block_topk(cuda_dev):
    """Block mode: the full layer scores the block means (HyLRA, sec. 2.4) and
    hands on the top-k blocks; O is still the dense attention over every row."""
    L = layer(2, 32, 8, 9000, [9000, 4100], seed=95, plant=0.01)
    kreq, k_max, block = [32, 20], 32, 128
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    Kmean = G.block_means(K, ln, block)
    ws = G.ws_for(Q, K, k_max, block, tsa.FULL)
    nrows = oracle.nblocks_of(L.seq_lens, block)
    S = oracle.block_scores(L.Q, oracle.block_means(L.K, L.seq_lens, block), nrows, SCALE)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE)
    for rep in range(2):
        O, idx = G.step(Q, K, V, ln, mode=tsa.FULL, scale=SCALE, k_max=k_max, block=block, kreq=kreq,
                        Kmean=Kmean, ws=ws, emit=True)
        check_output(O.cpu().numpy(), ref, f"block full step {rep}")
        compare_idx(idx.cpu().numpy(), S, nrows, kreq)


# ------------------------------------------------------------------ layer overlap (HyLRA sec. 2.2)

def _overlap_gpu(idx_dev):
    L = idx_dev.shape[0]
    units = math.prod(idx_dev.shape[1:-1])
    counts = torch.full((L, L, units), -7, dtype=torch.int32, device=idx_dev.device)
    M = torch.full((L, L), float("nan"), dtype=torch.float64, device=idx_dev.device)
    ws = torch.zeros(256, dtype=torch.uint8, device=idx_dev.device)
    tsa.index_overlap(idx_dev, counts, M, ws)
    tsa.check_device_status(ws)
    torch.cuda.synchronize()
    return counts.cpu().numpy(), M.cpu().numpy()


def _check_overlap(idx):
    counts, M = _overlap_gpu(idx)
    c_ref, M_ref = oracle.index_overlap(idx.cpu().numpy())
    assert (counts == c_ref).all(), "overlap counts differ"
    assert np.allclose(M, M_ref, rtol=1e-12, atol=0), f"M differs: {np.abs(M - M_ref).max()}"
    return counts, M


@pytest.mark.parametrize("keep", [0.0, 0.7, 1.0])
def test_index_overlap_random_layers(cuda_dev, keep):
    """Exact counts for 6 layers x 32 units: ragged k, an empty unit, a full one."""
    rng = np.random.default_rng(7)
    n = rng.integers(1, 3000, 32).tolist()
    n[3] = 0
    k = [int(min(x, rng.integers(1, 700))) for x in n]
    k[5] = 700
    n[5] = max(n[5], 700)
    idx = inputs.layer_index_lists(6, n, k, 700, keep, seed=11).to(cuda_dev)
    counts, M = _check_overlap(idx)
    if keep == 1.0:
        assert (M[np.tril_indices(6)] == 1.0).all()


@pytest.mark.parametrize("k_max", [33, 256])
def test_index_overlap_short_lists_a_warp_a_unit(cuda_dev, k_max):
    """Lists of at most 256 entries take the warp-a-unit kernel: 150 units (three
    rounds of 64, the last partial), ragged lengths, empty and full units; counts
    exact and M against the oracle."""
    rng = np.random.default_rng(k_max)
    units = 150
    n = rng.integers(1, 2000, units).tolist()
    n[7] = 0
    k = [int(min(x, rng.integers(1, k_max + 1))) for x in n]
    k[9] = k_max
    n[9] = max(n[9], k_max)
    idx = inputs.layer_index_lists(5, n, k, k_max, 0.6, seed=21).to(cuda_dev)
    _check_overlap(idx)


def test_index_overlap_long_lists_and_degenerate_sizes(cuda_dev):
    """Lists longer than the shared-memory stage (13000 rows of 40000), one layer,
    no units, and k_max = 0."""
    idx = inputs.layer_index_lists(3, [40000, 30000], [13000, 12000], 13000, 0.5, seed=12).to(cuda_dev)
    _check_overlap(idx)
    _check_overlap(inputs.layer_index_lists(1, [50], [10], 10, 0.5, seed=13).to(cuda_dev))
    counts, M = _check_overlap(torch.empty(2, 0, 5, dtype=torch.int32, device=cuda_dev))
    assert (M == [[1.0, 0.0], [1.0, 1.0]]).all()
    counts, M = _check_overlap(torch.empty(2, 3, 0, dtype=torch.int32, device=cuda_dev))
    assert (counts == 0).all() and (M == [[1.0, 0.0], [1.0, 1.0]]).all()


def test_index_overlap_flags_malformed_lists(cuda_dev):
    """A list out of order, or with an entry after its -1, sets the bounds flag."""
    good = inputs.layer_index_lists(2, [100, 100], [10, 10], 12, 0.5, seed=14)
    for bad in ("order", "tail"):
        idx = good.clone()
        if bad == "order":
            idx[1, 0, 3], idx[1, 0, 4] = idx[1, 0, 4].item(), idx[1, 0, 3].item()
        else:
            idx[0, 1, 11] = 5
        ws = torch.zeros(256, dtype=torch.uint8, device=cuda_dev)
        counts = torch.zeros((2, 2, 2), dtype=torch.int32, device=cuda_dev)
        tsa.index_overlap(idx.to(cuda_dev), counts, None, ws)
        with pytest.raises(tsa.TsaError, match="BOUNDS"):
            tsa.check_device_status(ws)


def test_index_overlap_of_decode_steps(cuda_dev):
    """The similarity matrix of a chain of layers as the decode steps select
    them: a full layer that hands on its top-k, then SELECT layers whose queries
    drift; the lists go straight from the steps into one [L, B, Hkv, k] tensor."""
    B, Hq, Hkv, N, kreq, k_max = 2, 16, 4, 8000, [300, 200], 300
    lens = [8000, 5123]
    L0 = layer(B, Hq, Hkv, N, lens, seed=101)
    Q, K, V, ln = G.to_dev(L0, cuda_dev)
    nl = 5
    idx = torch.full((nl, B, Hkv, k_max), -7, dtype=torch.int32, device=cuda_dev)
    ws = G.ws_for(Q, K, k_max, 1, tsa.FULL)
    O = torch.empty(B, Hq, 128, dtype=torch.float32, device=cuda_dev)
    kr = torch.tensor(kreq, dtype=torch.int32, device=cuda_dev)
    q = L0.Q
    for l in range(nl):
        if l > 0:
            q = inputs.drift_query(q, 0.4, 200 + l)
        a = tsa.step_args(q.to(cuda_dev), K, V, ln, O, ws, mode=tsa.FULL if l == 0 else tsa.SELECT,
                          scale=SCALE, k_max=k_max, k_per_seq=kr, idx_out=idx[l])
        tsa.decode_step(a)
        tsa.check_device_status(ws)
        S = oracle.scores(q, L0.K, L0.seq_lens, SCALE)
        compare_idx(idx[l].cpu().numpy(), S, lens, kreq)
    counts, M = _check_overlap(idx)
    assert 0.0 < M[1, 0] < 1.0


# ------------------------------------------------------------------ index-guided offload (HyLRA sec. 2.4)

def _pinned(t):
    out = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    out.copy_(t)
    return out


def test_offloaded_cache_block_select_and_reuse(cuda_dev):
    """K and V in page-locked host memory, block means on the device: the SELECT
    step picks the same blocks as with the cache in HBM (same scorer, same
    top-k) and its attention, which fetches only those blocks across the host
    link, matches the oracle; then REUSE steps over those blocks, in block and
    in token mode, read from the host copy too."""
    L = layer(2, 32, 8, 5000, [5000, 2100], seed=111, plant=0.01, tail_fill=float("nan"))
    kreq, k_max, block = [12, 7], 12, 128
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    Kh, Vh = _pinned(L.K), _pinned(L.V)
    Kmean = G.block_means(K, ln, block)
    O_dev, idx_dev = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, block=block, kreq=kreq,
                            Kmean=Kmean)
    O_h, idx_h = G.step(Q, Kh, Vh, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, block=block, kreq=kreq,
                        Kmean=Kmean, flags=tsa.KV_HOST)
    assert torch.equal(idx_h, idx_dev)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx_h.cpu().numpy(), kreq, k_max, block, SCALE)
    check_output(O_h.cpu().numpy(), ref, "offloaded block select")
    O_r, _ = G.step(Q, Kh, Vh, ln, mode=tsa.REUSE, scale=SCALE, k_max=k_max, block=block, kreq=kreq,
                    idx_in=idx_h, flags=tsa.KV_HOST)
    check_output(O_r.cpu().numpy(), ref, "offloaded block reuse")
    # token mode reuse over a set of rows
    rows = np.full((2, 8, 200), -1, dtype=np.int32)
    rng = np.random.default_rng(5)
    for b, n in enumerate([5000, 2100]):
        for h in range(8):
            rows[b, h] = np.sort(rng.choice(n, 200, replace=False))
    O_t, _ = G.step(Q, Kh, Vh, ln, mode=tsa.REUSE, scale=SCALE, k_max=200, kreq=[200, 200],
                    idx_in=torch.from_numpy(rows).to(cuda_dev), flags=tsa.KV_HOST)
    ref_t = oracle.attn(L.Q, L.K, L.V, L.seq_lens, rows, [200, 200], 200, 1, SCALE)
    check_output(O_t.cpu().numpy(), ref_t, "offloaded token reuse")


def test_offloaded_cache_full_layers(cuda_dev):
    """A full layer over an offloaded cache reads every row across the link; in
    block mode it can still hand on its top-k (the means are on the device)."""
    L = layer(2, 16, 4, 3000, [3000, 1234], seed=112, tail_fill=float("nan"))
    kreq, k_max, block = [8, 5], 8, 128
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    Kh, Vh = _pinned(L.K), _pinned(L.V)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, None, None, 0, 1, SCALE)
    O, _ = G.step(Q, Kh, Vh, ln, mode=tsa.FULL, scale=SCALE, flags=tsa.KV_HOST)
    check_output(O.cpu().numpy(), ref, "offloaded full layer")
    Kmean = G.block_means(K, ln, block)
    ws = G.ws_for(Q, K, k_max, block, tsa.FULL)
    O2, idx = G.step(Q, Kh, Vh, ln, mode=tsa.FULL, scale=SCALE, k_max=k_max, block=block, kreq=kreq,
                     Kmean=Kmean, ws=ws, emit=True, flags=tsa.KV_HOST)
    check_output(O2.cpu().numpy(), ref, "offloaded full layer handing on its blocks")
    nrows = oracle.nblocks_of(L.seq_lens, block)
    S = oracle.block_scores(L.Q, oracle.block_means(L.K, L.seq_lens, block), nrows, SCALE)
    compare_idx(idx.cpu().numpy(), S, nrows, kreq)


def test_offload_refuses_memory_the_device_cannot_read(cuda_dev):
    """Pageable host memory is refused before anything is launched, and token-mode
    selection over an offloaded cache is unsupported."""
    L = layer(1, 8, 2, 512, seed=113)
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    idx = torch.zeros(1, 2, 4, dtype=torch.int32, device=cuda_dev)
    with pytest.raises(tsa.TsaError, match="page-locked"):
        G.step(Q, L.K, L.V, ln, mode=tsa.REUSE, scale=SCALE, k_max=4, idx_in=idx, flags=tsa.KV_HOST)
    with pytest.raises(tsa.TsaError, match="page-locked"):  # device memory is not host memory either
        G.step(Q, K, V, ln, mode=tsa.REUSE, scale=SCALE, k_max=4, idx_in=idx, flags=tsa.KV_HOST)
    with pytest.raises(tsa.TsaError, match="UNSUPPORTED"):
        G.step(Q, _pinned(L.K), _pinned(L.V), ln, mode=tsa.SELECT, scale=SCALE, k_max=4,
               flags=tsa.KV_HOST)


def test_hylra_calibrate_then_run_the_policy(cuda_dev):
    """HyLRA end to end (secs. 2.2-2.3): calibrate on a stack of layers whose
    queries drift (every layer full, handing on its top-k), measure M with
    tsa_index_overlap, derive the policy with tsa_reuse_policy, then run the stack
    by it -- resets as full layers that hand on their top-k, the others reusing
    their source's list -- and check every layer against the oracle."""
    B, Hq, Hkv, N, nl = 2, 16, 4, 6000, 6
    kreq, k_max = [240, 150], 240
    lens = [6000, 3777]
    L0 = layer(B, Hq, Hkv, N, lens, seed=121)
    Q0, K, V, ln = G.to_dev(L0, cuda_dev)
    qs = [L0.Q]
    for l in range(1, nl):  # layers 2 and 4 drift far, the others a little
        qs.append(inputs.drift_query(qs[-1], 1.5 if l in (2, 4) else 0.15, 300 + l))
    ws = G.ws_for(Q0, K, k_max, 1, tsa.FULL)
    kr = torch.tensor(kreq, dtype=torch.int32, device=cuda_dev)
    O = torch.empty(B, Hq, 128, dtype=torch.float32, device=cuda_dev)
    cal = torch.full((nl, B, Hkv, k_max), -7, dtype=torch.int32, device=cuda_dev)
    for l in range(nl):
        a = tsa.step_args(qs[l].to(cuda_dev), K, V, ln, O, ws, mode=tsa.FULL, scale=SCALE, k_max=k_max,
                          k_per_seq=kr, idx_out=cal[l])
        tsa.decode_step(a)
    tsa.check_device_status(ws)
    counts, M = _check_overlap(cal)
    # a threshold between the small-drift and the large-drift neighbours
    sub = np.sort(np.diagonal(M, -1))
    theta = float(sub[1] + sub[2]) / 2
    src, n_full, sim = tsa.reuse_policy(M, theta)
    want = oracle.reuse_policy(M, theta)
    assert src.tolist() == want[0].tolist() and n_full == want[1]
    assert 1 < n_full < nl, f"the drift should make some but not all layers reset: {src}"
    # run the stack by the policy
    lists = torch.full((nl, B, Hkv, k_max), -7, dtype=torch.int32, device=cuda_dev)
    for l in range(nl):
        q = qs[l].to(cuda_dev)
        if src[l] == l:
            O_l, idx_l = G.step(q, K, V, ln, mode=tsa.FULL, scale=SCALE, k_max=k_max, kreq=kreq, ws=ws,
                                emit=True)
            lists[l].copy_(idx_l)
            ref = oracle.attn(qs[l], L0.K, L0.V, L0.seq_lens, None, None, 0, 1, SCALE)
            compare_idx(lists[l].cpu().numpy(), oracle.scores(qs[l], L0.K, L0.seq_lens, SCALE), lens, kreq)
        else:
            O_l, _ = G.step(q, K, V, ln, mode=tsa.REUSE, scale=SCALE, k_max=k_max, kreq=kreq,
                            idx_in=lists[src[l]], ws=ws)
            ref = oracle.attn(qs[l], L0.K, L0.V, L0.seq_lens, lists[src[l]].cpu().numpy(), kreq, k_max, 1, SCALE)
        torch.cuda.synchronize()
        check_output(O_l.cpu().numpy(), ref, f"layer {l} ({'full' if src[l] == l else f'reuses {src[l]}'})")


# ------------------------------------------------------------------ sequence sharding (one GPU, shards in turn)

@pytest.mark.parametrize("case", ["two_uneven", "three_with_an_empty_shard", "four_k_eq_len", "ties_across_shards",
                                  "wide_fallback"])
def test_sequence_sharded_select_on_one_gpu(cuda_dev, case):
    """The sharded SELECT step with its R shards run one after another on one
    GPU and the all-gathers replaced by stacking: the same indices as the one-GPU
    SELECT step (exact top-k of the whole cache) and the same attention.  Up to
    24576 candidates a unit the merge is one kernel; "wide_fallback" (4 x 7000)
    takes the pack / top-k / map path."""
    if case == "two_uneven":
        B, Hq, Hkv, N, lens, kreq, bounds = 2, 32, 8, 7000, [7000, 3500], [200, 120], [0, 2900, 7000]
    elif case == "three_with_an_empty_shard":  # sequence 1 ends inside shard 0
        B, Hq, Hkv, N, lens, kreq, bounds = 2, 16, 4, 9000, [9000, 100], [300, 300], [0, 4000, 4100, 9000]
    elif case == "ties_across_shards":  # 21 equal scores around the k-th, either side of the shard boundary
        B, Hq, Hkv, N, lens, kreq, bounds = 1, 8, 2, 6000, [6000], [150], [0, 3000, 6000]
    elif case == "wide_fallback":
        B, Hq, Hkv, N, lens, kreq, bounds = 1, 8, 2, 28672, [28000], [7000], [0, 7168, 14336, 21504, 28672]
    else:  # k = len: every row, spread over four shards
        B, Hq, Hkv, N, lens, kreq, bounds = 1, 8, 2, 4096, [4000], [4000], [0, 1024, 2048, 3072, 4096]
    R, k_max = len(bounds) - 1, max(kreq)
    L = layer(B, Hq, Hkv, N, lens, seed=131, tail_fill=float("nan"))
    if case == "ties_across_shards":
        S0 = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
        for h in range(Hkv):
            src = int(np.argsort(-S0[0, h, :lens[0]], kind="stable")[kreq[0] - 6])  # rank k - 5
            for dst in list(range(2990, 3000)) + list(range(3000, 3010)):
                if dst != src:
                    L.K[0, h, dst] = L.K[0, h, src].clone()
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    kr = torch.tensor(kreq, dtype=torch.int32, device=cuda_dev)
    _, idx_one = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, kreq=kreq)
    shards = []
    for r in range(R):
        lo, hi = bounds[r], bounds[r + 1]
        K_r, V_r = K[:, :, lo:hi].contiguous(), V[:, :, lo:hi].contiguous()
        lens_r = (ln - lo).clamp(0, hi - lo).to(torch.int32)
        ws = torch.empty(tsa.shard_workspace_size(tsa.shape_of(Q, K_r), k_max, R), dtype=torch.uint8,
                         device=cuda_dev)
        tsa.workspace_init(ws)
        shards.append((lo, K_r, V_r, lens_r, ws))
    cs = torch.full((R, B, Hkv, k_max), float("nan"), dtype=torch.float32, device=cuda_dev)
    cr = torch.full((R, B, Hkv, k_max), -7, dtype=torch.int32, device=cuda_dev)
    for r, (lo, K_r, V_r, lens_r, ws) in enumerate(shards):
        tsa.shard_select(Q, K_r, lens_r, kr, k_max, SCALE, lo, cs[r], cr[r], ws)
        tsa.check_device_status(ws)
    idx = torch.full((B, Hkv, k_max), -7, dtype=torch.int32, device=cuda_dev)
    tsa.shard_merge(cs, cr, tsa.shape_of(Q, K), kr, k_max, idx, shards[0][4])
    tsa.check_device_status(shards[0][4])
    S = oracle.scores(L.Q, L.K, L.seq_lens, SCALE)
    compare_idx(idx.cpu().numpy(), S, lens, kreq)
    assert torch.equal(idx, idx_one), "the shards must select what one GPU selects"
    O_parts = torch.full((R, B, Hq, 128), float("nan"), dtype=torch.float32, device=cuda_dev)
    lse = torch.full((R, B, Hq), float("nan"), dtype=torch.float32, device=cuda_dev)
    for r, (lo, K_r, V_r, lens_r, ws) in enumerate(shards):
        tsa.shard_attend(Q, K_r, V_r, lens_r, idx, kr, k_max, lo, SCALE, O_parts[r], lse[r], ws)
        tsa.check_device_status(ws)
    O = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=cuda_dev)
    tsa.shard_combine(O_parts, lse, tsa.shape_of(Q, K), O)
    torch.cuda.synchronize()
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx.cpu().numpy(), kreq, k_max, 1, SCALE)
    check_output(O.cpu().numpy(), ref, f"sharded {case}")
    # each part alone is the attention over the rows its shard holds
    for r, (lo, K_r, V_r, lens_r, ws) in enumerate(shards):
        own = np.where((idx.cpu().numpy() >= lo) & (idx.cpu().numpy() < lo + K_r.shape[2]),
                       idx.cpu().numpy() - lo, -1).astype(np.int32)
        own = np.sort(np.where(own < 0, np.iinfo(np.int32).max, own), axis=-1)
        own = np.where(own == np.iinfo(np.int32).max, -1, own).astype(np.int32)
        ref_r = oracle.attn(L.Q, L.K[:, :, lo:lo + K_r.shape[2]].contiguous(), L.V[:, :, lo:lo + K_r.shape[2]].contiguous(),
                            lens_r.cpu(), own, kreq, k_max, 1, SCALE)
        check_output(O_parts[r].cpu().numpy(), ref_r, f"{case} shard {r} part")


@pytest.mark.parametrize("case", ["random", "all_equal", "heavy_ties", "k_edges", "one_shard", "past_cap"])
def test_shard_merge_against_the_oracle(cuda_dev, case):
    """tsa_shard_merge on candidate lists built here: the exact top-k of the
    union of the shards' valid prefixes (ties to the lower row), against the
    oracle's top-k over the union packed in row order.  Entries after a list's
    first -1 hold junk that must be ignored.  "all_equal" takes the kernel's
    no-pass branch (every key equal); "past_cap" (4 x 7000 candidates) the
    pack / top-k / map path."""
    rng = np.random.default_rng(len(case))
    B, Hkv = 2, 2
    R, k_max = {"one_shard": (1, 300), "past_cap": (4, 7000), "all_equal": (3, 200)}.get(case, (2, 300))
    cnt = rng.integers(0, k_max + 1, size=(R, B))
    cnt[0, 0] = k_max  # a full list (no -1 in it)
    kreq = {"k_edges": [0, int(cnt[:, 1].sum())]}.get(case, [int(rng.integers(1, k_max + 1)), k_max + 50])
    cs = np.full((R, B, Hkv, k_max), np.nan, dtype=np.float32)
    cr = rng.integers(-50, 100000, size=(R, B, Hkv, k_max)).astype(np.int32)  # junk past the prefix
    for r in range(R):
        for b in range(B):
            c = int(cnt[r, b])
            for h in range(Hkv):
                cr[r, b, h, :c] = np.sort(rng.choice(20000, size=c, replace=False)) + 20000 * r
                if c < k_max:
                    cr[r, b, h, c] = -1
                if case == "all_equal":
                    cs[r, b, h, :c] = 1.25
                elif case == "heavy_ties":
                    cs[r, b, h, :c] = rng.integers(-2, 3, size=c) * 0.5
                else:
                    cs[r, b, h, :c] = rng.standard_normal(c).astype(np.float32) + 2.0
    # the oracle: top-k over the packed union, positions -> rows
    n = cnt.sum(axis=0)
    width = R * k_max
    S_pack = np.zeros((B, Hkv, width))
    rows_pack = np.full((B, Hkv, width), -1, dtype=np.int64)
    for b in range(B):
        for h in range(Hkv):
            sc = np.concatenate([cs[r, b, h, :cnt[r, b]] for r in range(R)])
            rw = np.concatenate([cr[r, b, h, :cnt[r, b]] for r in range(R)])
            S_pack[b, h, :len(sc)] = sc.astype(np.float64)
            rows_pack[b, h, :len(rw)] = rw
    # k_b = min(k, n): above k_max the library takes k_max and raises the bounds flag
    k_eff = [min(max(kreq[b], 0), int(n[b])) for b in range(B)]
    flagged = any(k > k_max for k in k_eff)
    pos = oracle.topk(S_pack, n.tolist(), [min(k, k_max) for k in k_eff], k_max)
    want = np.where(pos >= 0, np.take_along_axis(rows_pack, np.maximum(pos, 0).astype(np.int64), axis=-1), -1)
    shape = tsa.tsa_shape(B, Hkv * 4, Hkv, 20000 * R, 128)
    ws = torch.zeros(tsa.shard_workspace_size(tsa.tsa_shape(B, Hkv * 4, Hkv, 20000, 128), k_max, R),
                     dtype=torch.uint8, device=cuda_dev)
    idx = torch.full((B, Hkv, k_max), -7, dtype=torch.int32, device=cuda_dev)
    kr = torch.tensor(kreq, dtype=torch.int32, device=cuda_dev)
    tsa.shard_merge(torch.from_numpy(cs).to(cuda_dev), torch.from_numpy(cr).to(cuda_dev), shape, kr, k_max, idx, ws)
    got = idx.cpu().numpy()
    np.testing.assert_array_equal(got, want.astype(np.int32))
    if flagged:
        with pytest.raises(tsa.TsaError):
            tsa.check_device_status(ws)
    else:
        tsa.check_device_status(ws)


def test_sequence_sharded_step_through_nccl(cuda_dev):
    """shard.sharded_select_step on a real NCCL process group (one rank on this
    GPU: every all-gather is a device NCCL collective, nothing waits on another
    rank), against the one-GPU SELECT step and the oracle."""
    import os
    import socket

    import torch.distributed as dist

    from top_sparse_attention_02_b200 import shard

    B, Hq, Hkv, N, lens, kreq = 2, 32, 8, 9000, [9000, 5000], [300, 200]
    k_max = max(kreq)
    L = layer(B, Hq, Hkv, N, lens, seed=141, tail_fill=float("nan"))
    Q, K, V, ln = G.to_dev(L, cuda_dev)
    kr = torch.tensor(kreq, dtype=torch.int32, device=cuda_dev)
    _, idx_one = G.step(Q, K, V, ln, mode=tsa.SELECT, scale=SCALE, k_max=k_max, kreq=kreq)
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=cuda_dev)
    try:
        ws = torch.empty(tsa.shard_workspace_size(tsa.shape_of(Q, K), k_max, 1), dtype=torch.uint8,
                         device=cuda_dev)
        tsa.workspace_init(ws)
        O = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=cuda_dev)
        idx = torch.full((B, Hkv, k_max), -7, dtype=torch.int32, device=cuda_dev)
        stream = torch.cuda.Stream(device=cuda_dev)
        shard.sharded_select_step(Q, K, V, ln, kr, k_max, SCALE, 0, O, idx, ws, stream=stream)
        stream.synchronize()
        tsa.check_device_status(ws)
    finally:
        dist.destroy_process_group()
    assert torch.equal(idx, idx_one)
    ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx.cpu().numpy(), kreq, k_max, 1, SCALE)
    check_output(O.cpu().numpy(), ref, "sharded step over NCCL")
