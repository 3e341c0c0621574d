"""Multi-rank host paths on CPU (gloo, world size 2).

The layer shards by (batch, head): every (b, h) sequence is an independent
problem, so N GPUs run N replicas with no data-path collective and the only
cross-rank step is the max of the timed region.  These tests run that
reduction and the reference arm's rank handling on gloo ranks, and check on
the oracle that a head partition across ranks reproduces the single-process
result exactly.
"""
import json
import os
import socket
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank: int, world: int, port: int):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _max_worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, world, port)
    try:
        ms_local = 3.0 + 4.0 * rank          # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local, torch.device("cpu"))
        val = bench.job_value(world, 1000, 5, ms)
        with open(os.path.join(outdir, f"r{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": val}, f)
    finally:
        dist.destroy_process_group()


def test_timed_region_takes_the_slowest_rank():
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_max_worker, args=(2, _free_port(), d), nprocs=2, join=True, start_method="spawn")
        res = [json.load(open(os.path.join(d, f"r{r}.json"))) for r in range(2)]
    for r in res:
        assert r["ms"] == 7.0                       # max over ranks, on every rank
        assert r["value"] == pytest.approx(2 * 1000 * 5 / 7e-3)   # all ranks' tokens / slowest time


def test_one_rank_reduces_to_itself():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, torch.device("cpu")) == 2.5
    assert bench.job_value(1, 10, 2, 4.0) == pytest.approx(5000.0)


def _partition_worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    from lact_inputs import WORKLOADS, make_inputs
    import oracle
    _init(rank, world, port)
    try:
        w = WORKLOADS[1]
        inp = make_inputs(w, seed=0)
        heads = [(b, h) for b in range(w.B) for h in range(w.H)][rank::world]
        out, w1o, w2o, w3o = oracle.ttt_layer(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"],
                                              inp["w2"], inp["w3"], w.chunk, w.order, w.rule, heads=heads)
        # each rank fills its heads; NaN elsewhere -> gather and merge on rank 0
        parts = [torch.from_numpy(np.nan_to_num(x, nan=0.0)) for x in (out, w1o, w2o, w3o)]
        for t in parts:
            dist.all_reduce(t)                      # disjoint supports: the sum is the merge
        if rank == 0:
            np.savez(os.path.join(outdir, "merged.npz"), *[t.numpy() for t in parts])
    finally:
        dist.destroy_process_group()


def test_head_partition_across_ranks_equals_the_whole_layer():
    sys.path.insert(0, ROOT)
    from lact_inputs import WORKLOADS, make_inputs
    import oracle
    w = WORKLOADS[1]
    inp = make_inputs(w, seed=0)
    full = oracle.ttt_layer(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"], inp["w2"],
                            inp["w3"], w.chunk, w.order, w.rule)
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_partition_worker, args=(2, _free_port(), d), nprocs=2, join=True,
                           start_method="spawn")
        merged = np.load(os.path.join(d, "merged.npz"))
        merged = [merged[f"arr_{i}"] for i in range(4)]
    for a, b in zip(full, merged):
        np.testing.assert_array_equal(a, b)       # (b, h) problems are independent: exact


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--workload", "1"]
    outs = []
    for rank in (0, 1):
        e = dict(env, RANK=str(rank), LOCAL_RANK=str(rank))
        r = subprocess.run(cmd, env=e, capture_output=True, text=True, timeout=600, cwd=ROOT)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    assert outs[1] == ""                            # the other ranks exit 0 without work
    line = json.loads(outs[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


# ---------------------------------------------------------------- context parallelism
def _cp_hook_worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    import chunk_test_b200 as ct
    _init(rank, world, port)
    try:
        fn = ct.torch_distributed_allreduce()
        a = torch.arange(6, dtype=torch.float32) + 10.0 * rank
        fn(a, ct.REDUCE_SUM)
        # a per-chunk mean over ranks that hold unequal shares: the library
        # sums the (sum, count) pairs and divides on the device
        sums = torch.tensor([3.0 * (rank + 1), 5.0, 2.0 * (rank + 1), 1.0 + rank])
        fn(sums, ct.REDUCE_SUM)
        try:
            fn(torch.ones(2), ct.REDUCE_MEAN)
            rejected = False
        except ValueError:
            rejected = True
        with open(os.path.join(outdir, f"cp{rank}.json"), "w") as f:
            json.dump({"sum": a.tolist(), "pairs": sums.tolist(), "mean_rejected": rejected}, f)
    finally:
        dist.destroy_process_group()


def test_context_parallel_hook_sums_over_ranks():
    """The torch.distributed hook that the layer calls between a chunk's
    gradient and its rule: a sum over the ranks in place (the gradient
    planes, and the per-chunk beta sums and token counts whose quotient the
    library forms on the device).  The hook performs no other arithmetic and
    refuses any other op."""
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_cp_hook_worker, args=(2, _free_port(), d), nprocs=2, join=True,
                           start_method="spawn")
        res = [json.load(open(os.path.join(d, f"cp{r}.json"))) for r in range(2)]
    for r in res:
        assert r["sum"] == [10.0 + 2 * i for i in range(6)]
        # rank r held [3 (r + 1), 5, 2 (r + 1), 1 + r]: the sums add element-wise
        assert r["pairs"] == [9.0, 10.0, 6.0, 3.0]
        assert r["mean_rejected"]
    # the mean of beta over a chunk split 1 : 2 between the ranks is the
    # quotient of the summed pair, not the mean of the two ranks' means
    total_sum, total_count = res[0]["pairs"][2], res[0]["pairs"][3]
    assert total_sum / total_count == (2.0 + 4.0) / (1.0 + 2.0)


@pytest.mark.parametrize("rule", [0, 1, 2])
def test_context_parallel_shards_reproduce_the_layer(rule):
    """Context parallelism ("大块测试时训练（LaCT）技术解析" §2.2.2): every
    rank takes the gradient of its share of the chunk, the gradients are
    summed over the ranks, and every rank applies the same update.  Emulated
    here on the oracle's own steps for 2 ranks: the per-rank gradients of the
    shares sum to the whole chunk's gradient (the chunk gradient is a sum
    over tokens), and the beta mean of the chunk is the mean of the shares'
    means, so the sharded loop gives the layer's weights and outputs."""
    sys.path.insert(0, ROOT)
    import oracle
    rng = np.random.default_rng(7)
    H, T, d, dh, chunk, world = 2, 24, 6, 8, 8, 2
    q, k, v = (rng.standard_normal((1, H, T, d)) for _ in range(3))
    lr = np.log1p(np.exp(rng.standard_normal((1, H, T, 3)) - 1.0))
    beta = 1 / (1 + np.exp(-(2 + 0.5 * rng.standard_normal((1, H, T)))))
    w1 = rng.standard_normal((H, dh, d)) / d ** 0.5
    w2 = rng.standard_normal((H, d, dh)) / dh ** 0.5
    w3 = rng.standard_normal((H, dh, d)) / d ** 0.5
    want = oracle.ttt_layer(q, k, v, lr, beta if rule == 1 else None, w1, w2, w3, chunk, 0, rule)
    for h in range(H):
        W = (w1[h].copy(), w2[h].copy(), w3[h].copy())
        M = tuple(np.zeros_like(x) for x in W)
        out = np.zeros((T, d))
        kh, qh = oracle.qk_prologue(k[0, h]), oracle.qk_prologue(q[0, h])
        for c0 in range(0, T, chunk):
            rows = slice(c0, c0 + chunk)
            out[rows] = oracle.fast_net(*W, qh[rows])
            parts, means = [], []
            for r in range(world):
                sl = slice(c0 + r * chunk // world, c0 + (r + 1) * chunk // world)
                parts.append(oracle.chunk_gradient(*W, kh[sl], v[0, h, sl], lr[0, h, sl]))
                means.append(beta[0, h, sl].mean())
            G = tuple(sum(p[j] for p in parts) for j in range(3))
            if rule == 1:
                bbar = float(np.mean(means))
                M = tuple(bbar * m + g for m, g in zip(M, G))
                U = M
            else:
                U, _ = oracle.rule_step(rule, G, M, None)
            W = tuple(oracle.renorm_rows(w - u, w) for w, u in zip(W, U))
        np.testing.assert_allclose(out, want[0][0, h], rtol=1e-10, atol=1e-12)
        for j in range(3):
            np.testing.assert_allclose(W[j], want[1 + j][h], rtol=1e-10, atol=1e-12)
