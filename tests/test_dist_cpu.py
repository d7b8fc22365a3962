"""The multi-process path of bench.py on CPU: two gloo ranks run the same
setup, barrier and max-over-ranks code that the GPU runs use with NCCL, and a
rank that fails before a collective makes the other rank's collective end with
an error (short process-group timeout) instead of hanging."""
from __future__ import annotations

import multiprocessing as mp
import os
import socket
import time

import pytest
from hypothesis import given, settings, strategies as st

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, ws, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))


def _worker_max(rank, ws, port, q):
    _env(rank, ws, port)
    import torch.distributed as dist

    try:
        w, r, local = bench.dist_setup(backend="gloo", timeout_s=30)
        bench.barrier(w)
        step_ms = 10.0 + 5.0 * r  # rank 1 is the slower one
        slowest = bench.allreduce_max(step_ms, w)
        value = bench.whole_job_value(w, 1000.0, slowest)
        bench.barrier(w)
        q.put((r, w, local, slowest, value))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _worker_fail(rank, ws, port, q):
    _env(rank, ws, port)
    import torch.distributed as dist

    w, r, _ = bench.dist_setup(backend="gloo", timeout_s=5)
    bench.barrier(w)
    if r == 1:
        os._exit(3)  # leaves between steps, with no collective in flight
    t0 = time.time()
    try:
        bench.allreduce_max(1.0, w)
        q.put(("no error", time.time() - t0))
    except Exception as e:  # noqa: BLE001 - any backend error is the expected outcome
        q.put((type(e).__name__, time.time() - t0))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:  # noqa: BLE001
            pass


def _run(target, ws=2, join_s=90):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=target, args=(r, ws, port, q)) for r in range(ws)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(join_s)
    for p in ps:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
    out = []
    while not q.empty():
        out.append(q.get())
    return ps, out


def test_two_ranks_max_over_ranks_and_whole_job_value():
    ps, out = _run(_worker_max)
    assert all(p.exitcode == 0 for p in ps)
    assert sorted(o[0] for o in out) == [0, 1]
    for r, w, local, slowest, value in out:
        assert w == 2 and local == r
        assert slowest == 15.0  # the max over ranks, seen by every rank
        assert value == pytest.approx(2 * 1000.0 / 0.015)


def test_failed_rank_ends_the_others_collective_with_an_error():
    ps, out = _run(_worker_fail)
    assert ps[1].exitcode == 3
    assert len(out) == 1
    name, dt = out[0]
    assert name != "no error"
    assert dt < 60.0


def test_reference_arm_prints_on_rank_zero_only(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        schedule, steps, warmup = "one_reference", 1, 0

    bench.run_reference(A(), bench.workloads.WORKLOADS["small512"])
    assert capsys.readouterr().out == ""


def _worker_halo(rank, ws, port, q):
    """One rank of a sequence-sharded vector: own entries filled with their
    global values, halos empty; after the exchange the local vector must equal
    the global one over [lo, hi), and the row padding must be untouched."""
    _env(rank, ws, port)
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import banded_log_domain_b200 as sa

    try:
        dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=timedelta(seconds=30))
        Lt, W, rows = 23, 3, 4
        own_lo, own_hi, lo, hi = sa.shard_bounds(Lt, W, rank, ws)
        glob = torch.arange(Lt, dtype=torch.float32)[None, :] * 10 + torch.arange(rows)[:, None]
        buf = torch.full((rows, hi - lo + 5), -1.0)  # rows wider than L, like the state's
        view = buf[:, :hi - lo]
        view[:, own_lo - lo:own_hi - lo] = glob[:, own_lo:own_hi]
        ex = sa.HaloExchange(own_lo - lo, hi - own_hi)
        ex(view)
        ok = torch.equal(view, glob[:, lo:hi]) and bool((buf[:, hi - lo:] == -1).all())
        # a second exchange (the next sweep) with new values
        view[:, own_lo - lo:own_hi - lo] += 1000.0
        ex(view)
        ok = ok and torch.equal(view, glob[:, lo:hi] + 1000.0)
        q.put((rank, ok, (own_lo, own_hi, lo, hi)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 3])
def test_halo_exchange_fills_every_halo(ws):
    ps, out = _run(_worker_halo, ws=ws)
    assert all(p.exitcode == 0 for p in ps)
    assert sorted(o[0] for o in out) == list(range(ws))
    assert all(o[1] for o in out), out
    bounds = sorted(o[2] for o in out)
    assert bounds[0][0] == 0 and bounds[-1][1] == 23           # shards cover the sequence
    assert all(a[1] == b[0] for a, b in zip(bounds, bounds[1:]))  # contiguously


def test_shard_bounds():
    import banded_log_domain_b200 as sa

    assert sa.shard_bounds(10, 2, 0, 1) == (0, 10, 0, 10)
    assert sa.shard_bounds(10, 2, 0, 3) == (0, 4, 0, 6)
    assert sa.shard_bounds(10, 2, 1, 3) == (4, 7, 2, 9)
    assert sa.shard_bounds(10, 2, 2, 3) == (7, 10, 5, 10)
    with pytest.raises(ValueError):
        sa.shard_bounds(10, 4, 0, 3)  # 3 own tokens < W


@settings(max_examples=200, deadline=None, derandomize=True)
@given(L=st.integers(1, 5000), W=st.integers(0, 64), world=st.integers(1, 8))
def test_shard_bounds_partition_the_sequence(L, W, world):
    """Own ranges tile [0, L) in rank order with sizes differing by at most one;
    each local range is the own range widened by W on each side (clipped to the
    sequence), so a boundary's two halos both hold W tokens."""
    import banded_log_domain_b200 as sa

    if world > 1 and L // world < max(W, 1):
        with pytest.raises(ValueError):
            sa.shard_bounds(L, W, 0, world)
        return
    b = [sa.shard_bounds(L, W, r, world) for r in range(world)]
    assert b[0][0] == 0 and b[-1][1] == L
    assert all(x[1] == y[0] for x, y in zip(b, b[1:]))
    sizes = [hi - lo for lo, hi, _, _ in b]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= (max(W, 1) if world > 1 else 0)
    for own_lo, own_hi, lo, hi in b:
        assert (lo, hi) == (max(0, own_lo - W), min(L, own_hi + W))
