"""Data-parallel exchange step on CPU ranks (gloo, world size 2).

The layer shards by tokens: each rank routes and computes its own batch
against replicated weights, and the only exchange is the sum of the weight
gradients.  These tests check that the sum of per-shard oracle gradients is
the full-batch gradient, and that a rank that fails before the collective is
detected by the others as an error instead of a hang."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as orc


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _layer(seed=3, T=96, d=16, E=6, n=8):
    rs = np.random.RandomState(seed)
    return (rs.randn(T, d), rs.randn(E, d, 2 * n) * 0.3, rs.randn(E, n, d) * 0.3, rs.randn(d, E) * 0.5,
            rs.randn(E) * 0.5, rs.randn(T, d))


def _shard_worker(rank, world, port, K, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    X, W1, W2, Wr, b, dO = _layer()
    T = X.shape[0]
    sl = slice(rank * T // world, (rank + 1) * T // world)
    fw = orc.forward(X[sl], Wr, b, W1, W2, K)
    bw = orc.backward(fw, dO[sl], X[sl], Wr, W1, W2)
    grads = [torch.from_numpy(bw[k].copy()) for k in ("dW1", "dW2", "dWr")]
    for g in grads:
        dist.all_reduce(g)
    if rank == 0:
        out_q.put([g.numpy() for g in grads] + [bw["dX"]])
    dist.barrier()
    dist.destroy_process_group()


def test_sum_of_shard_gradients_is_full_batch_gradient():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, K = 2, 2
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, K, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W1, W2, Wr, b, dO = _layer()
    fw = orc.forward(X, Wr, b, W1, W2, K)
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    for mine, k in zip(got[:3], ("dW1", "dW2", "dWr")):
        np.testing.assert_allclose(mine, bw[k], rtol=1e-10, atol=1e-12)
    # dX of a shard is that shard's rows of the full-batch dX: no exchange needed
    np.testing.assert_allclose(got[3], bw["dX"][:X.shape[0] // 2], rtol=1e-10, atol=1e-12)


def _failing_worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        # this rank fails between steps, before joining the gradient exchange
        os._exit(3)
    g = torch.ones(8)
    try:
        dist.all_reduce(g)
        out_q.put("no error")
    except Exception as e:  # the surviving rank learns of the failure
        out_q.put(type(e).__name__)


def test_rank_failing_before_exchange_is_reported_not_hung():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert res != "no error"
    assert procs[1].exitcode == 3


# ----------------------------------------------------------------------------
# Expert parallelism: experts split over the ranks, routed rows exchanged by
# all-to-all.  The plan and the exchanges are the product's
# (fine_grained_mixture_top_b200.ep); the arithmetic is the oracle's.
# ----------------------------------------------------------------------------
def _ep_worker(rank, world, port, K, T, E, out_q, round_mode=0):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from fine_grained_mixture_top_b200.ep import ExpertParallelMoE
    from ep_oracle_engine import OracleEngine
    X, W1, W2, Wr, b, dO = _layer(seed=5, T=T * world, E=E)
    sl = slice(rank * T, (rank + 1) * T)
    E_loc = E // world
    es = slice(rank * E_loc, (rank + 1) * E_loc)
    ep = ExpertParallelMoE(T, X.shape[1], E, W2.shape[1], K,
                           OracleEngine(E, K, world, round_mode=round_mode, seed=11, tile=8))
    t = torch.from_numpy
    O = ep.forward(t(X[sl].copy()), t(Wr), t(b), t(W1[es].copy()), t(W2[es].copy()))
    dX, dW1, dW2, dWr = ep.backward(t(dO[sl].copy()), t(X[sl].copy()), t(Wr), t(W1[es].copy()), t(W2[es].copy()))
    out_q.put((rank, O.numpy(), dX.numpy(), dW1.numpy(), dW2.numpy(), dWr.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,E,K", [(2, 6, 2), (3, 6, 3), (2, 8, 1)])
def test_expert_parallel_equals_full_batch(world, E, K):
    """Each rank holds E/world experts and its own tokens; O, dX, its experts'
    dW1/dW2 and the all-reduced dWr equal the single-process full batch."""
    T = 40
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, K, T, E, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r[0], r[1:]) for r in (q.get(timeout=180) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W1, W2, Wr, b, dO = _layer(seed=5, T=T * world, E=E)
    fw = orc.forward(X, Wr, b, W1, W2, K)
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    E_loc = E // world
    for r in range(world):
        O, dX, dW1, dW2, dWr = got[r]
        sl = slice(r * T, (r + 1) * T)
        es = slice(r * E_loc, (r + 1) * E_loc)
        np.testing.assert_allclose(O, fw["O"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dX, bw["dX"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dW1, bw["dW1"][es], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dW2, bw["dW2"][es], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dWr, bw["dWr"], rtol=1e-10, atol=1e-12)


def test_exchange_plan_orders_rows_by_source_then_expert():
    from fine_grained_mixture_top_b200.ep import exchange_plan
    send = np.array([[3, 0], [1, 2], [0, 0]])        # this rank's rows for experts (g, l)
    recv = np.array([[2, 1], [0, 4], [1, 0]])        # rows rank g sends for local expert l
    ss, rs, le = exchange_plan(send, recv)
    assert ss == [3, 3, 0] and rs == [3, 4, 1]
    np.testing.assert_array_equal(le, [0, 0, 1, 1, 1, 1, 1, 0])


def test_expert_parallel_with_token_rounding():
    """Each rank rounds its own batch's expert counts (tile 8 here) before the
    exchange; the layer equals the single-process oracle run on the
    concatenation of the ranks' rounded routings."""
    world, E, K, T = 2, 6, 2, 40
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, K, T, E, q, 2)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r[0], r[1:]) for r in (q.get(timeout=180) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W1, W2, Wr, b, dO = _layer(seed=5, T=T * world, E=E)
    ptrs, exps, gates = [np.zeros(1, np.int64)], [], []
    for r in range(world):
        sl = slice(r * T, (r + 1) * T)
        rt = orc.route(X[sl], Wr, b, K)
        tr = orc.token_round(rt["probs"], rt["tok_ptr"], rt["pair_expert"], 2, 11, 8)
        assert np.all(tr["counts"] % 8 == 0)
        ptrs.append(tr["tok_ptr"][1:] + ptrs[-1][-1])
        exps.append(tr["pair_expert"])
        gates.append(tr["pair_gate"])
    routing = {"tok_ptr": np.concatenate(ptrs), "pair_expert": np.concatenate(exps),
               "pair_gate": np.concatenate(gates)}
    fw = orc.forward(X, Wr, b, W1, W2, K, routing=routing)
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    E_loc = E // world
    for r in range(world):
        O, dX, dW1, dW2, dWr = got[r]
        sl = slice(r * T, (r + 1) * T)
        es = slice(r * E_loc, (r + 1) * E_loc)
        np.testing.assert_allclose(O, fw["O"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dX, bw["dX"][sl], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dW1, bw["dW1"][es], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dW2, bw["dW2"][es], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dWr, bw["dWr"], rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------
# The product's overlapped data-parallel reduction (moe.OverlappedGradReduce)
# on gloo ranks: host stand-ins replace the CUDA streams and events, and a
# layer whose step is the oracle's stands in for the kernels.  Checks the
# order the reductions are issued in (each after its gradient's event, dW2
# then dW1 then dWr), that the stream join comes last, and that the reduced
# gradients are the full-batch ones.
# ----------------------------------------------------------------------------
class _HostHooks:
    def __init__(self, log):
        import contextlib
        self.log = log
        self.events = ["dW2 ready", "dW1 ready", "dWr ready"]
        self._ctx = contextlib.nullcontext

    def on_comm(self):
        self.log.append("comm stream")
        return self._ctx()

    def wait(self, ev):
        assert ev in self.log, f"waited on {ev} before the backward recorded it"
        self.log.append("wait " + ev)

    def join(self):
        self.log.append("join")


class _OracleLayer:
    """Stand-in for MoELayer: its step is the oracle's on this rank's shard,
    and it 'records' the gradient events in the backward's order."""

    def __init__(self, K, log, router_grad=1):
        import types
        self.K = K
        self.log = log
        self.opts = types.SimpleNamespace(router_grad=router_grad)

    def step(self, X, Wr, bias, W1, W2, dO, grad_events=None):
        fw = orc.forward(X, Wr, bias, W1, W2, self.K)
        bw = orc.backward(fw, dO, X, Wr, W1, W2, router_grad=bool(self.opts.router_grad))
        self.dW2 = torch.from_numpy(bw["dW2"].copy())
        self.log.append(grad_events[0])
        self.dW1 = torch.from_numpy(bw["dW1"].copy())
        self.log.append(grad_events[1])
        self.dWr = torch.from_numpy(bw["dWr"].copy()) if self.opts.router_grad else None
        self.log.append(grad_events[2])
        self.dX = bw["dX"]


def _overlap_worker(rank, world, port, K, router_grad, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from fine_grained_mixture_top_b200 import moe
    X, W1, W2, Wr, b, dO = _layer()
    T = X.shape[0]
    sl = slice(rank * T // world, (rank + 1) * T // world)
    log = []
    layer = _OracleLayer(K, log, router_grad)
    red = moe.OverlappedGradReduce(layer, hooks=_HostHooks(log))
    # all_reduce is logged by wrapping the collective the class calls
    real = dist.all_reduce

    def logged(g, group=None):
        log.append("all_reduce " + ("dW2" if g is layer.dW2 else "dW1" if g is layer.dW1 else "dWr"))
        return real(g, group=group)

    dist.all_reduce = logged
    try:
        dX, dW1, dW2, dWr = red.step(X[sl], Wr, b, W1, W2, dO[sl])
    finally:
        dist.all_reduce = real
    out_q.put((rank, log, dW1.numpy(), dW2.numpy(), None if dWr is None else dWr.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("router_grad", [1, 0])
def test_overlapped_reduce_orders_and_sums_on_two_ranks(router_grad):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, K = 2, 2
    port = _free_port()
    procs = [ctx.Process(target=_overlap_worker, args=(r, world, port, K, router_grad, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W1, W2, Wr, b, dO = _layer()
    fw = orc.forward(X, Wr, b, W1, W2, K)
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    want = ["dW2 ready", "dW1 ready", "dWr ready", "comm stream", "wait dW2 ready", "all_reduce dW2",
            "wait dW1 ready", "all_reduce dW1"]
    if router_grad:
        want += ["wait dWr ready", "all_reduce dWr"]
    want += ["join"]
    for rank, log, dW1, dW2, dWr in got:
        assert log == want, (rank, log)
        np.testing.assert_allclose(dW1, bw["dW1"], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dW2, bw["dW2"], rtol=1e-10, atol=1e-12)
        if router_grad:
            np.testing.assert_allclose(dWr, bw["dWr"], rtol=1e-10, atol=1e-12)
        else:
            assert dWr is None
