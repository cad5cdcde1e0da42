"""The N > 1 host path of bench.py on CPU: world size 2 over gloo.  Each rank runs
its own replica; the only collectives are a barrier and a max of the timings."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        bench.barrier(world)
        mine = 1.0 + rank * 0.5  # rank 1 is the slower one
        slowest = bench.max_over_ranks(mine, world, torch.device("cpu"))
        q.put((rank, slowest, bench.whole_job_value(10**12, 2.0, world)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [1.5, 1.5]  # both ranks report the max
    assert got[0][2] == pytest.approx(2 * 10**12 / 2e-3 / 1e12)  # work of both replicas


# ------------------------------------------------------------------ sequence-sharded SELECT step

class OracleShardOps:
    """The four libtsa sharding calls restated with the fp64 oracle on CPU tensors,
    so that the exchange in shard.sharded_select_step can run over gloo."""

    @staticmethod
    def shape_of(Q, K):
        return (Q.shape[0], Q.shape[1], K.shape[1], K.shape[2], Q.shape[2])

    @staticmethod
    def shard_select(Q, K_r, lens_r, kreq, k_max, scale, row0, cand_scores, cand_rows, ws, stream):
        import numpy as np

        import oracle

        S = oracle.scores(Q, K_r, lens_r, scale)
        idx = oracle.topk(S, lens_r.numpy(), kreq.numpy(), k_max)
        B, Hkv, _ = idx.shape
        cs = np.full(idx.shape, -np.inf, dtype=np.float32)
        cr = np.full(idx.shape, -1, dtype=np.int32)
        for b in range(B):
            for h in range(Hkv):
                for t, r in enumerate(idx[b, h]):
                    if r >= 0:
                        cs[b, h, t], cr[b, h, t] = S[b, h, r], row0 + r
        cand_scores.copy_(torch.from_numpy(cs))
        cand_rows.copy_(torch.from_numpy(cr))

    @staticmethod
    def shard_merge(all_s, all_r, shape, kreq, k_max, idx, ws, stream):
        R, B, Hkv, _ = all_s.shape
        idx.fill_(-1)
        for b in range(B):
            for h in range(Hkv):
                pairs = [(float(all_s[r, b, h, t]), int(all_r[r, b, h, t])) for r in range(R) for t in range(k_max)
                         if all_r[r, b, h, t] >= 0]
                kb = min(int(kreq[b]), len(pairs))
                rows = sorted(row for _, row in sorted(pairs, key=lambda p: (-p[0], p[1]))[:kb])
                idx[b, h, :kb] = torch.tensor(rows, dtype=torch.int32)

    @staticmethod
    def shard_attend(Q, K_r, V_r, lens_r, idx, kreq, k_max, row0, scale, O_part, lse_part, ws, stream):
        import numpy as np

        import oracle

        B, Hkv, ncap = K_r.shape[:3]
        g = Q.shape[1] // Hkv
        local = np.full((B, Hkv, k_max), -1, dtype=np.int32)
        lse = np.full((B, Q.shape[1]), -np.inf)
        q, k = Q.double().numpy(), K_r.double().numpy()
        for b in range(B):
            for h in range(Hkv):
                own = [int(x) - row0 for x in idx[b, h] if row0 <= x < row0 + ncap]
                local[b, h, :len(own)] = own
                for hh in range(g):
                    if own:
                        z = scale * (k[b, h, own] @ q[b, h * g + hh])
                        lse[b, h * g + hh] = (z.max() + np.log(np.exp(z - z.max()).sum())) / np.log(2.0)
        O_part.copy_(torch.from_numpy(oracle.attn(Q, K_r, V_r, lens_r, local, kreq.numpy(), k_max, 1, scale)))
        lse_part.copy_(torch.from_numpy(lse))

    @staticmethod
    def shard_combine(O_all, lse_all, shape, O, stream):
        M = lse_all.max(dim=0).values
        w = torch.where(torch.isinf(lse_all), torch.zeros_like(lse_all), torch.exp2(lse_all - M))
        den = w.sum(dim=0)
        num = (w.unsqueeze(-1) * O_all).sum(dim=0)
        O.copy_(torch.where(den.unsqueeze(-1) > 0, num / den.clamp_min(1e-300).unsqueeze(-1), torch.zeros_like(num)))


SHARD_CASES = {
    # the second sequence lies wholly in rank 0's part
    "two": dict(B=2, Hq=8, Hkv=2, N=3000, lens=[3000, 1100], kreq=[90, 90], bounds=[0, 1300, 3000]),
    # three ranks, the middle one narrow; k above a sequence's length; g = 4
    "three": dict(B=2, Hq=16, Hkv=4, N=2000, lens=[2000, 700], kreq=[60, 900], bounds=[0, 650, 720, 2000]),
}


def _shard_rank_main(rank, world, port, q, name):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import sys

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
        from top_sparse_attention_02_b200 import inputs, shard

        c = SHARD_CASES[name]
        L = inputs.decode_layer(c["B"], c["Hq"], c["Hkv"], c["N"], c["lens"], plant_frac=0.01, seed=41)
        lo, hi = c["bounds"][rank], c["bounds"][rank + 1]
        K_r, V_r = L.K[:, :, lo:hi].contiguous(), L.V[:, :, lo:hi].contiguous()
        lens_r = (L.seq_lens - lo).clamp(0, hi - lo).to(torch.int32)
        kreq = torch.tensor(c["kreq"], dtype=torch.int32)
        k_max = max(c["kreq"])
        O = torch.empty(c["B"], c["Hq"], 128, dtype=torch.float64)
        idx = torch.empty(c["B"], c["Hkv"], k_max, dtype=torch.int32)
        shard.sharded_select_step(L.Q, K_r, V_r, lens_r, kreq, k_max, 1 / 128 ** 0.5, lo, O, idx, None,
                                  ops=OracleShardOps)
        q.put((rank, idx.numpy(), O.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(SHARD_CASES))
def test_sequence_sharded_step_exchange(name):
    """Ranks each holding a contiguous part of every sequence's rows: after the
    candidate and the partial exchanges every rank holds the unsharded top-k and
    attention."""
    import sys

    import numpy as np

    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import oracle
    from parity import check_output, compare_idx
    from top_sparse_attention_02_b200 import inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    c = SHARD_CASES[name]
    world = len(c["bounds"]) - 1
    procs = [ctx.Process(target=_shard_rank_main, args=(r, world, port, q, name)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    L = inputs.decode_layer(c["B"], c["Hq"], c["Hkv"], c["N"], c["lens"], plant_frac=0.01, seed=41)
    S = oracle.scores(L.Q, L.K, L.seq_lens, 1 / 128 ** 0.5)
    k_max = max(c["kreq"])
    for rank, idx, O in got:
        compare_idx(idx, S, c["lens"], c["kreq"])
        ref = oracle.attn(L.Q, L.K, L.V, L.seq_lens, idx, c["kreq"], k_max, 1, 1 / 128 ** 0.5)
        check_output(O, ref, f"rank {rank}")
    for _, idx, O in got[1:]:
        assert np.array_equal(got[0][1], idx) and np.array_equal(got[0][2], O)


def test_bench_gpus_n_starts_n_ranks():
    """`bench.py --gpus 2` started by hand (no WORLD_SIZE) starts two ranks of
    itself; they rendezvous, take the slower rank's time and rank 0 alone prints
    one line with n_gpus = 2 (the rank plumbing only, on the CPU over gloo)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--dry-run",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300,
                         env=env, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    res = json.loads(lines[0])
    assert res["n_gpus"] == 2 and res["dry_run"]
    assert res["ms_per_step"] == 1.25  # rank 1's stand-in time, the slower one


def test_bench_refuses_a_world_size_that_disagrees_with_gpus():
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--dry-run"],
                         capture_output=True, text=True, timeout=120, env=env, cwd=root)
    assert out.returncode != 0 and "WORLD_SIZE=3" in out.stderr
