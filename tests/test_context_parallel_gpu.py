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

The backward under the same sharding: each rank's loss is its queries'
<out, dout> plus its share of <w_out, dw> and <m_out, dm>; the ranks'
gradients of their own tokens, put back in token order, and their gradients
of the shared initial state (both ranks alike, bit for bit) match the
unsharded autograd oracle.
"""
import threading

import numpy as np
import pytest
import torch

import chunk_test_b200 as ct
import oracle
from oracle import lact_oracle_bwd as ob
from lact_inputs import (APPLY_THEN_UPDATE, BF16, F32, RULE_GD, RULE_MOMENTUM, RULE_MUON,
                         UPDATE_THEN_APPLY, Workload, make_inputs, make_momentum, make_output_grads)

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


BWD_CASES = [
    (Workload("cp-bwd-f32-gd-causal", 1, 2, 1024, 1024, 64, 128, 256, APPLY_THEN_UPDATE, RULE_GD, F32), {}),
    (Workload("cp-bwd-f32-momentum-uta", 2, 1, 768, 768, 32, 64, 256, UPDATE_THEN_APPLY, RULE_MOMENTUM, F32),
     dict(mask=[1, 0, 1], mom_io=True)),
    (Workload("cp-bwd-f32-muon", 1, 2, 768, 768, 64, 128, 256, APPLY_THEN_UPDATE, RULE_MUON, F32), {}),
    (Workload("cp-bwd-bf16-d256-causal", 1, 2, 2048, 2048, 256, 512, 512, APPLY_THEN_UPDATE, RULE_GD, BF16),
     {}),
    (Workload("cp-bwd-bf16-d128-momentum", 1, 2, 1536, 1536, 128, 256, 512, APPLY_THEN_UPDATE,
              RULE_MOMENTUM, BF16), dict(mom_io=True)),
    (Workload("cp-bwd-bf16-d64-set", 1, 2, 2048, 512, 64, 128, 2048, UPDATE_THEN_APPLY, RULE_GD, BF16), {}),
]


@pytest.mark.parametrize("w,kw", BWD_CASES, ids=lambda x: x.name if hasattr(x, "name") else "")
def test_two_ranks_backward_matches_the_unsharded_gradients(w, kw):
    world = 2
    mask, mom_io = kw.get("mask"), kw.get("mom_io", False)
    inp = make_inputs(w, seed=23)
    dout, dws = make_output_grads(w, seed=23, with_weights=True)
    m_in = make_momentum(w, seed=23) if mom_io else None
    dm = make_momentum(w, seed=24) if mom_io else None
    want = ob.ttt_layer_bwd(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"], inp["w2"],
                            inp["w3"], w.chunk, w.order, w.rule, dout, dw=dws, update_mask=mask,
                            m_in=m_in, dm=dm)
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
                half = lambda xs: None if xs is None else tuple((0.5 * x).cuda() for x in xs)  # noqa: E731
                res = ct.ttt_bwd(dev["q"], dev["k"], dev["v"], dev["lr"], dev["beta"], dev["w1"], dev["w2"],
                                 dev["w3"], w.chunk // world, w.order, w.rule,
                                 dout[:, :, qidx[r]].contiguous().cuda(), dw_out=half(dws), update_mask=mask,
                                 m_in=None if m_in is None else tuple(x.cuda() for x in m_in),
                                 dm_out=half(dm), stream=st, allreduce=group.hook(r))
                assert ct.status(st) == ct.LACT_OK
                st.synchronize()
                results[r] = {k_: (None if v_ is None else v_.cpu()) for k_, v_ in res.items()}
        except BaseException as e:  # noqa: BLE001
            errors.append(e)
            group.barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=600)
    assert not errors, errors
    n_upd = w.n_chunks if mask is None else sum(mask)
    mom = w.rule == RULE_MOMENTUM
    # recompute: each chunk's gradient (+ the beta sums); reverse loop: the own
    # contributions before each renorm and once at the end (+ dL/dM_final)
    assert group.calls == [2 * n_upd + 1 + (1 if mom else 0) + (1 if mom_io else 0)] * world
    tol = TOL[w.dtype]
    errs = {}
    for name, idx, full in (("dq", qidx, want["dq"]), ("dk", kidx, want["dk"]), ("dv", kidx, want["dv"]),
                            ("dlr", kidx, want["dlr"]), ("dbeta", kidx, want["dbeta"])):
        if full is None:
            continue
        got = np.zeros_like(full)
        for r in range(world):
            got[:, :, idx[r]] = results[r][name].numpy()
        errs[name] = rel_l2(got, full)
    shared = ["dw1", "dw2", "dw3"] + (["dm1", "dm2", "dm3"] if mom_io else [])
    for name in shared:
        errs[name] = rel_l2(results[0][name].numpy(), want[name])
        assert torch.equal(results[0][name], results[1][name]), f"{name} differs between the ranks"
    assert max(errs.values()) <= tol, f"{w.name}: {errs}"
    print(w.name, {k_: f"{v_:.1e}" for k_, v_ in errs.items()})
