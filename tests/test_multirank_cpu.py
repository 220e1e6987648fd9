"""The multi-process path's host logic on CPU: two gloo ranks split a variable-length batch
by tokens, each runs the oracle on its share, and rank 0 checks the gathered outputs and
states against one single-process run; the max-over-ranks timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_deltanet_03_b200.sharding import balance_sequences, max_over_ranks, pack, shard_range


def test_balance_and_ranges():
    lens = [5000, 100, 3000, 2900, 50, 7000]
    parts = balance_sequences(lens, 2)
    assert sorted(sum(parts, [])) == list(range(6))
    loads = [sum(lens[i] for i in p) for p in parts]
    assert max(loads) - min(loads) <= max(lens)
    assert [shard_range(10, 3, r) for r in range(3)] == [(0, 3), (3, 6), (6, 10)]
    cu, sl = pack(lens, [0, 2])
    assert list(cu) == [0, 5000, 8000] and sl[1] == slice(5100, 8100)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        w = workloads.custom("mr", (70, 5, 33, 128, 1), 1, 2, 16, io="f32", s0_std=0.1, seed=31)
        x = workloads.generate(w)
        parts = balance_sequences(w.seqlens, world)
        mine = parts[rank]
        cu, slices = pack(w.seqlens, mine)
        take = lambda a: np.concatenate([a[s] for s in slices]) if slices else a[:0]  # noqa: E731
        o, S = oracle.gdn_scan(take(x["q"]), take(x["k"]), take(x["v"]), take(x["a"]), take(x["b"]),
                               x["A_log"], x["dt_bias"], cu_seqlens=cu,
                               initial_state=x["initial_state"][mine], threads=1)
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, o, S))
        t = max_over_ranks(1.0 + rank)
        if rank == 0:
            o_ref, S_ref = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                                           cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])
            full_cu = x["cu_seqlens"]
            for idx, o_r, S_r in gathered:
                off = 0
                for j, i in enumerate(idx):
                    L = int(full_cu[i + 1] - full_cu[i])
                    np.testing.assert_array_equal(o_r[off:off + L], o_ref[full_cu[i]:full_cu[i + 1]])
                    np.testing.assert_array_equal(S_r[j], S_ref[i])
                    off += L
            out.put(("ok", t))
    except Exception as e:  # pragma: no cover - reported to the parent
        out.put(("error %d: %r" % (rank, e), None))
        raise
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_the_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    status, t = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert status == "ok", status
    assert t == 2.0
    assert all(p.exitcode == 0 for p in procs)
