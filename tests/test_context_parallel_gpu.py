"""Context parallelism through the C ABI on one GPU, against the oracle.

Context parallelism ("大块测试时训练（LaCT）技术解析" §2.2.2): each rank holds
an equal share of every chunk's tokens, takes the gradient of its share, the
gradients are summed over the ranks and every rank applies the same update.
The library calls the caller's all-reduce hook between a chunk's gradient and
its rule (and once for the per-chunk beta means).

Here two ranks run as two host threads on one GPU, each on its own stream,
and the hook is an emulated all-reduce: events and host barriers order it,
and the sum is taken with torch on each rank's stream.  No kernel waits on
another; every barrier has a timeout, so a rank that fails ends the test
instead of hanging it.  Checked: the ranks' outputs, put back in token
order, and the final weights match the unsharded oracle within the usual
tolerances, and both ranks end with bit-identical weights.
"""
import threading

import numpy as np
import pytest
import torch

import chunk_test_b200 as ct
import oracle
from lact_inputs import (APPLY_THEN_UPDATE, BF16, F32, RULE_GD, RULE_MOMENTUM, RULE_MUON,
                         UPDATE_THEN_APPLY, Workload, make_inputs)

pytestmark = pytest.mark.gpu

TOL = {F32: 1e-4, BF16: 2e-2}


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


class EmulatedGroup:
    """An in-process all-reduce over `n` ranks (threads) sharing one GPU."""

    def __init__(self, n):
        self.n = n
        self.barrier = threading.Barrier(n, timeout=120)
        self.bufs = [None] * n
        self.ready = [None] * n
        self.done = [None] * n
        self.calls = [0] * n

    def hook(self, rank):
        def fn(buf, op, stream):
            self.calls[rank] += 1
            ev = torch.cuda.Event()
            ev.record(stream)
            self.bufs[rank], self.ready[rank] = buf, ev
            self.barrier.wait()                       # every rank's buffer is enqueued
            with torch.cuda.stream(stream):
                for e in self.ready:
                    stream.wait_event(e)
                total = self.bufs[0].clone()
                for b in self.bufs[1:]:
                    total += b                        # the same order on every rank
                assert op == ct.REDUCE_SUM            # the library asks only for sums
                done = torch.cuda.Event()
                done.record(stream)
            self.done[rank] = done
            self.barrier.wait()                       # every rank has read every buffer
            with torch.cuda.stream(stream):
                for e in self.done:
                    stream.wait_event(e)
                buf.copy_(total)
            self.barrier.wait()                       # slots free for the next call
        return fn


def shard_index(n, chunk, world, rank):
    part = chunk // world
    return np.concatenate([np.arange(c0 + rank * part, c0 + (rank + 1) * part)
                           for c0 in range(0, n, chunk)])


CASES = [
    # one chunk of keys, separate queries (the view-synthesis form; fused key + gradient kernel)
    Workload("cp-bf16-d64-set", 1, 3, 2048, 512, 64, 128, 2048, UPDATE_THEN_APPLY, RULE_GD, BF16),
    # causal, several chunks: the side-stream apply and two shadow sets
    Workload("cp-bf16-d256-causal", 1, 2, 2048, 2048, 256, 512, 512, APPLY_THEN_UPDATE, RULE_GD, BF16),
    # momentum: the beta means are averaged over the ranks
    Workload("cp-bf16-d128-momentum", 2, 2, 1536, 1536, 128, 256, 512, UPDATE_THEN_APPLY,
             RULE_MOMENTUM, BF16),
    Workload("cp-bf16-d128-muon", 1, 2, 1024, 1024, 128, 256, 512, APPLY_THEN_UPDATE, RULE_MUON, BF16),
    Workload("cp-f32-momentum", 1, 2, 1024, 1024, 64, 128, 256, APPLY_THEN_UPDATE, RULE_MOMENTUM, F32),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_two_ranks_match_the_unsharded_layer(w):
    world = 2
    inp = make_inputs(w, seed=21)
    want = oracle.ttt_layer(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"],
                            inp["w2"], inp["w3"], w.chunk, w.order, w.rule)
    single = w.chunk >= w.T
    kidx = [shard_index(w.T, w.chunk, world, r) for r in range(world)]
    qidx = ([np.arange(r * w.Tq // world, (r + 1) * w.Tq // world) for r in range(world)] if single
            else kidx)
    group = EmulatedGroup(world)
    results, errors = [None] * world, []

    def rank_main(r):
        try:
            torch.cuda.set_device(0)
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                dev = {}
                for name in ("k", "v", "lr", "beta"):
                    t = inp[name]
                    dev[name] = None if t is None else t[:, :, kidx[r]].contiguous().cuda()
                dev["q"] = inp["q"][:, :, qidx[r]].contiguous().cuda()
                for name in ("w1", "w2", "w3"):
                    dev[name] = inp[name].cuda()
                res = ct.ttt_fwd(dev["q"], dev["k"], dev["v"], dev["lr"], dev["beta"], dev["w1"],
                                 dev["w2"], dev["w3"], w.chunk // world, w.order, w.rule, stream=st,
                                 allreduce=group.hook(r))
                assert ct.status(st) == ct.LACT_OK
                results[r] = [x.float().cpu() for x in res]
        except BaseException as e:  # noqa: BLE001
            errors.append(e)
            group.barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=600)
    assert not errors, errors
    n_updates = w.n_chunks
    assert group.calls == [n_updates + (1 if w.rule == RULE_MOMENTUM else 0)] * world
    out = torch.zeros(w.B, w.H, w.Tq, w.d)
    for r in range(world):
        out[:, :, qidx[r]] = results[r][0]
    for j in range(1, 4):
        assert torch.equal(results[0][j], results[1][j])      # every rank holds the same state
    errs = {"out": rel_l2(out.numpy(), want[0])}
    for j, name in enumerate(("w1", "w2", "w3")):
        errs[name] = rel_l2(results[0][1 + j].numpy(), want[1 + j])
    assert max(errs.values()) <= TOL[w.dtype], errs
