"""Pins that tie the fp64 oracle to facts other than itself (CPU only).

Each test checks the oracle against a closed form, a brute-force enumeration on
tiny inputs, a library routine in a special case (torch fp64 SDPA), or a worked
example printed on the pages, so that a dropped term, a wrong sign or index, or
a transposed operand in oracle.c fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from top_sparse_attention_02_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_layer(B=2, Hq=8, Hkv=2, N=96, lens=None, seed=1, plant=0.0):
    lens = lens if lens is not None else [N] * B
    return inputs.decode_layer(B, Hq, Hkv, N, lens, plant_frac=plant, seed=seed)


def _sdpa_fp64(Q, K, V, lens, scale, rows=None):
    """torch's own scaled_dot_product_attention in float64 on CPU (GQA by repeat_interleave)."""
    B, Hq, d = Q.shape
    out = torch.empty(B, Hq, d, dtype=torch.float64)
    for b in range(B):
        sel = torch.arange(int(lens[b])) if rows is None else torch.as_tensor(rows[b])
        q = Q[b:b + 1].double().unsqueeze(2)
        k = K[b:b + 1, :, sel].double()
        v = V[b:b + 1, :, sel].double()
        out[b] = F.scaled_dot_product_attention(q, k, v, scale=scale, enable_gqa=True)[0, :, 0]
    return out.numpy()


def _brute_topk(S_row: np.ndarray, n: int, k: int) -> np.ndarray:
    """Full lexicographic sort on (-score, index): the definition, enumerated."""
    j = np.arange(n)
    order = np.lexsort((j, -S_row[:n]))
    return np.sort(order[:min(k, n)])


# ---------------------------------------------------------------- scores

def test_scores_basis_keys_closed_form():
    """K rows = e_c (unit basis vectors): s_j = scale * max_h q_h[c_j]."""
    B, Hq, Hkv, d, N = 1, 6, 2, 128, 40
    g = torch.Generator().manual_seed(3)
    Q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    cols = torch.randint(0, d, (Hkv, N), generator=g)
    K = torch.zeros(B, Hkv, N, d, dtype=torch.bfloat16)
    for kvh in range(Hkv):
        K[0, kvh, torch.arange(N), cols[kvh]] = 1.0
    scale = 0.37
    S = oracle.scores(Q, K, [N], scale)
    grp = Hq // Hkv
    for kvh in range(Hkv):
        for j in range(N):
            qcol = Q[0, kvh * grp:(kvh + 1) * grp, cols[kvh, j]].double()
            assert S[0, kvh, j] == pytest.approx(scale * float(qcol.max()), rel=0, abs=1e-15)


def test_scores_group_uses_only_own_heads():
    """A query head outside the group never changes that group's scores."""
    L = _rand_layer(B=1, Hq=8, Hkv=2, N=50, seed=5)
    S0 = oracle.scores(L.Q, L.K, L.seq_lens, 0.1)
    Q2 = L.Q.clone()
    Q2[0, 4:8] = 100.0  # heads of kv-head 1 only
    S1 = oracle.scores(Q2, L.K, L.seq_lens, 0.1)
    np.testing.assert_array_equal(S0[0, 0], S1[0, 0])
    assert not np.allclose(S0[0, 1], S1[0, 1])


def test_scores_ragged_tail_untouched():
    L = _rand_layer(B=2, N=64, lens=[64, 17], seed=7)
    S = oracle.scores(L.Q, L.K, L.seq_lens, 0.2)
    assert np.isfinite(S[0]).all()
    assert np.isfinite(S[1, :, :17]).all() and np.isnan(S[1, :, 17:]).all()


# ---------------------------------------------------------------- top-k

@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_full_sort_with_forced_ties(seed):
    """Brute force on tiny inputs with duplicated keys (exact ties)."""
    B, Hq, Hkv, N = 2, 4, 2, 48
    L = _rand_layer(B=B, Hq=Hq, Hkv=Hkv, N=N, lens=[48, 31], seed=seed)
    g = torch.Generator().manual_seed(100 + seed)
    # duplicate some rows so that equal scores occur at different indices
    for b in range(B):
        src = torch.randint(0, 31, (12,), generator=g)
        dst = torch.randint(0, 31, (12,), generator=g)
        L.K[b, :, dst] = L.K[b, :, src]
    S = oracle.scores(L.Q, L.K, L.seq_lens, 1 / math.sqrt(128))
    for k in (1, 5, 16, 31, 40):
        idx = oracle.topk(S, L.seq_lens, [k, k], k_max=40)
        for b in range(B):
            n = int(L.seq_lens[b])
            for kvh in range(Hkv):
                want = _brute_topk(S[b, kvh], n, k)
                got = idx[b, kvh]
                np.testing.assert_array_equal(got[:len(want)], want)
                assert (got[len(want):] == -1).all()


def test_topk_all_equal_scores_lowest_indices():
    S = np.zeros((1, 1, 30))
    idx = oracle.topk(S, [30], [7], 8)
    np.testing.assert_array_equal(idx[0, 0], [0, 1, 2, 3, 4, 5, 6, -1])


def test_topk_signed_zero_and_negative_scores():
    S = np.array([[[-0.0, 0.0, -1.5, -0.25, 0.0, -0.0, -3.0]]])
    idx = oracle.topk(S, [7], [3], 3)
    np.testing.assert_array_equal(idx[0, 0], [0, 1, 4])  # all four zeros tie; lowest three win
    idx = oracle.topk(S, [7], [6], 6)
    np.testing.assert_array_equal(idx[0, 0], [0, 1, 2, 3, 4, 5])


def test_topk_scale_invariant_and_permutation_equivariant():
    L = _rand_layer(B=1, Hq=8, Hkv=2, N=80, seed=11)
    S1 = oracle.scores(L.Q, L.K, L.seq_lens, 0.05)
    S2 = oracle.scores(L.Q, L.K, L.seq_lens, 3.0)
    i1 = oracle.topk(S1, L.seq_lens, [9], 9)
    i2 = oracle.topk(S2, L.seq_lens, [9], 9)
    np.testing.assert_array_equal(i1, i2)
    perm = torch.randperm(80, generator=torch.Generator().manual_seed(2))
    Kp = L.K[:, :, perm]
    Sp = oracle.scores(L.Q, Kp, L.seq_lens, 0.05)
    ip = oracle.topk(Sp, L.seq_lens, [9], 9)
    for kvh in range(2):
        mapped = np.sort(perm.numpy()[ip[0, kvh]])
        np.testing.assert_array_equal(mapped, i1[0, kvh])


def test_topk_k_clamped_to_length():
    S = np.random.default_rng(0).standard_normal((2, 1, 10))
    idx = oracle.topk(S, [10, 4], [6, 6], 6)
    assert (idx[1, 0, :4] == np.arange(4)).all() and (idx[1, 0, 4:] == -1).all()
    with pytest.raises(ValueError):
        oracle.topk(S, [10, 10], [6, 6], 5)


def test_planted_key_is_selected():
    """A key equal to 20 * unit(q_h) dominates every N(0,1) key: it must be the top-1."""
    L = _rand_layer(B=1, Hq=8, Hkv=2, N=200, seed=13)
    q = L.Q[0, 5].float()
    L.K[0, 1, 123] = (20 * q / q.norm()).to(torch.bfloat16)
    S = oracle.scores(L.Q, L.K, L.seq_lens, 1 / math.sqrt(128))
    idx = oracle.topk(S, L.seq_lens, [1], 1)
    assert idx[0, 1, 0] == 123


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (8, 1)])
def test_k_equals_len_is_dense_sdpa(Hq, Hkv):
    """k = len selects everything: equals torch's fp64 SDPA (GQA) over all valid rows."""
    L = _rand_layer(B=2, Hq=Hq, Hkv=Hkv, N=70, lens=[70, 23], seed=17)
    scale = 1 / math.sqrt(128)
    O, idx, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [70, 70], 70, scale, mode=1)
    ref = _sdpa_fp64(L.Q, L.K, L.V, L.seq_lens, scale)
    np.testing.assert_allclose(O, ref, rtol=0, atol=1e-12)
    Ofull, _, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, None, 0, scale, mode=0)
    np.testing.assert_allclose(Ofull, ref, rtol=0, atol=1e-12)


def test_sparse_equals_sdpa_over_selected_rows():
    L = _rand_layer(B=2, Hq=8, Hkv=2, N=90, lens=[90, 61], seed=19, plant=0.05)
    scale = 1 / math.sqrt(128)
    O, idx, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [12, 12], 12, scale)
    for b in range(2):
        for kvh in range(2):
            rows = idx[b, kvh]
            Kb = L.K[b:b + 1, kvh:kvh + 1, rows]
            Vb = L.V[b:b + 1, kvh:kvh + 1, rows]
            q = L.Q[b:b + 1, kvh * 4:(kvh + 1) * 4].double().unsqueeze(2)
            ref = F.scaled_dot_product_attention(q, Kb.double(), Vb.double(), scale=scale,
                                                 enable_gqa=True)[0, :, 0]
            np.testing.assert_allclose(O[b, kvh * 4:(kvh + 1) * 4], ref.numpy(), atol=1e-12, rtol=0)


def test_k1_returns_v_row_of_argmax_exactly():
    L = _rand_layer(B=1, Hq=8, Hkv=2, N=64, seed=23)
    q = L.Q[0, 2].float()
    L.K[0, 0, 40] = (30 * q / q.norm()).to(torch.bfloat16)
    O, idx, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [1], 1, 1 / math.sqrt(128))
    assert idx[0, 0, 0] == 40
    for h in range(4):  # every head of the group sees one row: weight exactly 1
        np.testing.assert_array_equal(O[0, h], L.V[0, 0, 40].double().numpy())


def test_identical_keys_give_mean_of_v():
    B, Hq, Hkv, N, d = 1, 4, 1, 33, 128
    L = _rand_layer(B=B, Hq=Hq, Hkv=Hkv, N=N, seed=29)
    L.K[0, 0, :] = L.K[0, 0, 0]
    k = 9
    O, idx, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [k], k, 0.1)
    np.testing.assert_array_equal(idx[0, 0], np.arange(k))
    mean = L.V[0, 0, :k].double().mean(0).numpy()
    for h in range(Hq):
        np.testing.assert_allclose(O[0, h], mean, atol=1e-14, rtol=0)


def test_reuse_passes_indices_through_bit_identical():
    L = _rand_layer(B=2, N=64, seed=31)
    L2 = _rand_layer(B=2, N=64, seed=32)
    O0, idx0, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [8, 8], 8, 0.1)
    O1, idx1, _ = oracle.decode_step(L2.Q, L2.K, L2.V, L2.seq_lens, [8, 8], 8, 0.1, mode=2,
                                     idx_in=idx0)
    assert idx1 is idx0
    direct = oracle.attn(L2.Q, L2.K, L2.V, L2.seq_lens, idx0, [8, 8], 8, 1, 0.1)
    np.testing.assert_array_equal(O1, direct)


def test_sliding_window_worked_example():
    """The pages' sliding-window picture (W=4 at token 8) as an index set: equals SDPA
    over rows 4..7, and differs from full attention over rows 0..7."""
    vals = {}
    with open(os.path.join(GOLDEN, "sliding_window_w4.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, *rest = line.split()
            vals[key] = [int(x) for x in rest]
    n = vals["context_len"][0]
    rows = vals["attended_rows"]
    assert len(rows) == vals["window"][0]
    L = _rand_layer(B=1, Hq=4, Hkv=1, N=n, seed=37)
    idx = np.array(rows, dtype=np.int32).reshape(1, 1, -1)
    O = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, [len(rows)], len(rows), 1, 0.3)
    ref = _sdpa_fp64(L.Q, L.K, L.V, L.seq_lens, 0.3, rows=[rows])
    np.testing.assert_allclose(O, ref, atol=1e-12, rtol=0)
    full = _sdpa_fp64(L.Q, L.K, L.V, L.seq_lens, 0.3, rows=[vals["full_rows"]])
    assert not np.allclose(O, full)


def test_attention_is_order_independent():
    L = _rand_layer(B=1, Hq=4, Hkv=1, N=40, seed=41)
    a = np.array([[[3, 9, 17, 22, 35]]], dtype=np.int32)
    b = np.array([[[35, 3, 22, 17, 9]]], dtype=np.int32)
    Oa = oracle.attn(L.Q, L.K, L.V, L.seq_lens, a, [5], 5, 1, 0.2)
    Ob = oracle.attn(L.Q, L.K, L.V, L.seq_lens, b, [5], 5, 1, 0.2)
    np.testing.assert_allclose(Oa, Ob, atol=1e-15, rtol=0)


def test_attention_rejects_out_of_range_index():
    L = _rand_layer(B=1, Hq=4, Hkv=1, N=40, lens=[20], seed=43)
    bad = np.array([[[3, 25]]], dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.attn(L.Q, L.K, L.V, L.seq_lens, bad, [2], 2, 1, 0.2)


# ---------------------------------------------------------------- block mode

def test_block_means_closed_form_constant_blocks():
    B, Hkv, N, d, blk = 1, 2, 20, 128, 8
    K = torch.zeros(B, Hkv, N, d, dtype=torch.bfloat16)
    for t in range(N):
        K[0, :, t] = float(t // blk) + 0.5 * (t % 2)  # block beta: values beta and beta+0.5
    M = oracle.block_means(K, [19], blk)
    # blocks 0,1 have 4 rows of each value -> beta + 0.25; block 2 holds rows 16,17,18
    np.testing.assert_allclose(M[0, :, 0], 0.25)
    np.testing.assert_allclose(M[0, :, 1], 1.25)
    np.testing.assert_allclose(M[0, :, 2], 2.0 + 0.5 / 3)


def test_block_size_one_equals_token_mode():
    """Blocks of one token: the means are the rows, block scores are token scores, and the
    block path's selection and attention equal the token path's."""
    L = _rand_layer(B=2, N=50, lens=[50, 37], seed=47, plant=0.05)
    scale = 1 / math.sqrt(128)
    Ot, it, St = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [7, 7], 7, scale, block=1)
    M = oracle.block_means(L.K, L.seq_lens, 1)
    valid = np.arange(50)[None, None, :, None] < L.seq_lens.numpy()[:, None, None, None]
    np.testing.assert_array_equal(M, np.where(valid, L.K.double().numpy(), np.nan))
    nb = oracle.nblocks_of(L.seq_lens, 1)
    Sb = oracle.block_scores(L.Q, M, nb, scale)
    np.testing.assert_allclose(Sb, St, atol=1e-15, rtol=0, equal_nan=True)
    ib = oracle.topk(Sb, nb, [7, 7], 7)
    np.testing.assert_array_equal(ib, it)
    Ob = oracle.attn(L.Q, L.K, L.V, L.seq_lens, ib, [7, 7], 7, 1, scale)
    np.testing.assert_array_equal(Ob, Ot)


def test_block_mode_all_blocks_is_dense():
    L = _rand_layer(B=2, N=300, lens=[300, 129], seed=53)
    scale = 1 / math.sqrt(128)
    nb = oracle.nblocks_of(L.seq_lens, 128)
    O, idx, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [3, 3], 3, scale, block=128)
    assert (idx[0, :, :3] == [0, 1, 2]).all() and (idx[1, :, :2] == [0, 1]).all()
    assert (idx[1, :, 2] == -1).all() and list(nb) == [3, 2]
    np.testing.assert_allclose(O, _sdpa_fp64(L.Q, L.K, L.V, L.seq_lens, scale), atol=1e-12, rtol=0)


def test_block_mode_selects_planted_block_and_expands_partial_tail():
    L = _rand_layer(B=1, Hq=4, Hkv=1, N=400, lens=[390], seed=59)
    q = L.Q[0, 1].float()
    L.K[0, 0, 384:390] = (8 * q / q.norm()).to(torch.bfloat16)  # partial last block 3
    scale = 1 / math.sqrt(128)
    O, idx, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [1], 1, scale, block=128)
    assert idx[0, 0, 0] == 3
    ref = _sdpa_fp64(L.Q, L.K, L.V, L.seq_lens, scale, rows=[list(range(384, 390))])
    np.testing.assert_allclose(O, ref, atol=1e-12, rtol=0)


def test_empty_sequence_gives_zero_output_and_no_indices():
    L = _rand_layer(B=2, Hq=4, Hkv=1, N=16, lens=[16, 0], seed=61)
    O, idx, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, [4, 4], 4, 0.2)
    assert (idx[1] == -1).all() and (O[1] == 0).all()
    Of, _, _ = oracle.decode_step(L.Q, L.K, L.V, L.seq_lens, None, 0, 0.2, mode=0)
    assert (Of[1] == 0).all()
    np.testing.assert_allclose(Of[0], _sdpa_fp64(L.Q[:1], L.K[:1], L.V[:1], [16], 0.2)[0], atol=1e-12)


# ------------------------------------------------------------------ layer overlap (HyLRA sec. 2.2)

def _lists(sets, k_max):
    """Index lists in the library's form: ascending, then -1."""
    out = np.full((len(sets), len(sets[0]), k_max), -1, dtype=np.int32)
    for l, per_unit in enumerate(sets):
        for u, s in enumerate(per_unit):
            v = sorted(s)
            out[l, u, :len(v)] = v
    return out


def test_overlap_identical_and_disjoint_layers():
    """Layers 0 and 1 hold the same sets (ratio 1); layer 2 the odd rows where they
    hold even ones (ratio 0); the diagonal counts are the set sizes."""
    even = [set(range(0, 64, 2)), set(range(10, 40, 2))]
    odd = [set(range(1, 64, 2)), set(range(11, 41, 2))]
    counts, M = oracle.index_overlap(_lists([even, even, odd], 40))
    assert (counts[0, 1] == [32, 15]).all() and (counts[0, 2] == 0).all() and (counts[1, 2] == 0).all()
    assert (np.diagonal(counts, axis1=0, axis2=1).T == [[32, 15], [32, 15], [32, 15]]).all()
    assert np.allclose(np.diag(M), 1.0) and M[1, 0] == 1.0 and M[2, 0] == 0.0 and M[2, 1] == 0.0
    assert (M[np.triu_indices(3, 1)] == 0).all()


def test_overlap_shifted_window_closed_form():
    """I_0 = [0, k), I_1 = [s, s + k): |I_0 ∩ I_1| = k - s for 0 <= s <= k."""
    k = 50
    for s in (0, 1, 17, 49, 50, 80):
        counts, M = oracle.index_overlap(_lists([[set(range(k))], [set(range(s, s + k))]], k))
        assert counts[0, 1, 0] == counts[1, 0, 0] == max(k - s, 0)
        assert M[1, 0] == max(k - s, 0) / k


def test_overlap_normalises_by_the_target_set_and_orients_rows_as_targets():
    """Source layer 0 holds 4 rows, target layer 1 holds 2 of which 1 is shared:
    reusing layer 0's indices keeps 1 of the target's 2 (0.5), not 1 of 4 (0.25).
    With the roles swapped (layer 1 is the source of nothing, as it comes later)
    M[0, 1] stays 0: the matrix is lower triangular, rows are targets."""
    counts, M = oracle.index_overlap(_lists([[{3, 5, 7, 9}], [{5, 100}]], 4))
    assert counts[0, 1, 0] == 1
    assert M[1, 0] == 0.5 and M[0, 1] == 0.0


def test_overlap_mean_over_units_skips_empty_targets():
    """Units with an empty target list leave the mean; with none left M is 1."""
    src = [{1, 2, 3, 4}, {1, 2}, {7}]
    tgt = [{1, 2, 9, 10}, set(), {7}]  # ratios 0.5, (skipped), 1.0
    counts, M = oracle.index_overlap(_lists([src, tgt], 4))
    assert M[1, 0] == 0.75
    _, M0 = oracle.index_overlap(_lists([[set(), set()], [set(), set()]], 3))
    assert (M0[np.tril_indices(2)] == 1.0).all()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_overlap_brute_force_tiny(seed):
    """Random small sets of rows in [0, 30): every count equals the size of the
    Python set intersection and every M entry the plain mean of the ratios."""
    rng = np.random.default_rng(seed)
    L, units, k_max = 4, 5, 9
    sets = [[set(rng.choice(30, size=int(rng.integers(0, k_max + 1)), replace=False).tolist())
             for _ in range(units)] for _ in range(L)]
    counts, M = oracle.index_overlap(_lists(sets, k_max))
    for i in range(L):
        for j in range(L):
            for u in range(units):
                assert counts[i, j, u] == len(sets[i][u] & sets[j][u])
            if i <= j:
                r = [len(sets[i][u] & sets[j][u]) / len(sets[j][u]) for u in range(units) if sets[j][u]]
                want = sum(r) / len(r) if r else 1.0
                assert abs(M[j, i] - want) < 1e-15
            else:  # above the diagonal: a later layer is no source for an earlier one
                assert M[j, i] == 0.0


def test_layer_index_lists_form_and_drift():
    """The generator's lists have the library's form, and keep = 1 / 0 give
    identical / (for n >= 2k) disjoint consecutive layers."""
    lists = inputs.layer_index_lists(3, [100, 7, 0], [20, 20, 5], 24, 1.0, seed=3)
    a = lists.numpy()
    for l in range(3):
        for u, (n, k) in enumerate([(100, 20), (7, 7), (0, 0)]):
            v = a[l, u]
            assert (np.diff(v[:k]) > 0).all() and (v[:k] >= 0).all() and (v[:k] < max(n, 1)).all()
            assert (v[k:] == -1).all()
    counts, M = oracle.index_overlap(a)
    assert (M[np.tril_indices(3)] == 1.0).all()
    _, M0 = oracle.index_overlap(inputs.layer_index_lists(2, [100], [20], 20, 0.0, seed=4).numpy())
    assert M0[1, 0] == 0.0


def test_overlap_degenerate_shapes():
    """No units, or lists of width 0: every count is 0 and M is 1 on and below
    the diagonal (no unit has a non-empty target)."""
    for shape in ((2, 0, 5), (2, 3, 0), (1, 1, 1)):
        counts, M = oracle.index_overlap(np.full(shape, -1, dtype=np.int32))
        assert counts.shape == (shape[0], shape[0], shape[1]) and (counts == 0).all()
        assert (M == np.tril(np.ones((shape[0], shape[0])))).all()


# ------------------------------------------------------------------ reuse policy (HyLRA sec. 2.2)

def _sim(L, entries, fill=0.0):
    """Lower-triangular M [L, L] (row = target) from {(target, source): value}."""
    M = np.full((L, L), fill)
    for (j, i), v in entries.items():
        M[j, i] = v
    return M


def test_policy_everything_similar_or_nothing_similar():
    """All similarities 1 > theta: one full layer, every other reuses layer 0;
    all 0: every layer is full."""
    src, n, sim = oracle.reuse_policy(np.ones((6, 6)), 0.5)
    assert src.tolist() == [0] * 6 and n == 1 and sim == 5.0
    src, n, sim = oracle.reuse_policy(np.zeros((6, 6)), 0.5)
    assert src.tolist() == list(range(6)) and n == 6 and sim == 0.0


def test_policy_beats_resetting_as_late_as_possible():
    """Layer 0 reaches layers 1-2, layer 1 reaches 2-4, layers 3 and 4 nothing
    useful: resetting only when forced (0, 3, 4) takes 3 full layers, resetting
    early at 1 covers the rest with 2."""
    M = _sim(5, {(1, 0): 0.9, (2, 0): 0.9, (2, 1): 0.8, (3, 1): 0.8, (4, 1): 0.8})
    src, n, sim = oracle.reuse_policy(M, 0.5)
    assert src.tolist() == [0, 1, 1, 1, 1] and n == 2 and sim == 0.8 + 0.8 + 0.8


def test_policy_prefers_more_similarity_at_equal_full_count():
    """Two 2-full policies: layer 1 reusing layer 0 (0.6) or layer 2 reusing
    layer 1 (0.9); the second keeps more."""
    M = _sim(3, {(1, 0): 0.6, (2, 1): 0.9})
    src, n, sim = oracle.reuse_policy(M, 0.5)
    assert src.tolist() == [0, 1, 1] and n == 2 and sim == 0.9
    # and the other way round, where the tie rule alone would pick the other policy
    M = _sim(3, {(1, 0): 0.9, (2, 1): 0.6})
    src, n, sim = oracle.reuse_policy(M, 0.5)
    assert src.tolist() == [0, 0, 2] and n == 2 and sim == 0.9


def test_policy_threshold_is_strict_and_forced_layers_are_full():
    M = _sim(3, {(1, 0): 0.5, (2, 0): 0.75, (2, 1): 0.75})
    assert oracle.reuse_policy(M, 0.5)[0].tolist() == [0, 1, 1]  # 0.5 does not exceed 0.5
    assert oracle.reuse_policy(M, 0.49)[0].tolist() == [0, 0, 0]
    src, n, _ = oracle.reuse_policy(M, 0.49, force_full=[0, 0, 1])
    assert src.tolist() == [0, 0, 2] and n == 2


def test_policy_ties_go_to_the_smaller_source_from_the_end():
    """[0, 0, 2] and [0, 1, 1] both have 2 full layers and similarity 0.5; read
    from the last layer, 1 < 2."""
    M = _sim(3, {(1, 0): 0.5, (2, 1): 0.5})
    assert oracle.reuse_policy(M, 0.25)[0].tolist() == [0, 1, 1]
