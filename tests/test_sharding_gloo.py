"""The multi-process path on CPU: two gloo ranks (127.0.0.1). Head ranges
partition the heads, the timing reductions take the max and the work the sum
over ranks, and a forward pass sharded over heads (here the oracle stands in
for the per-rank library call) reassembles to the unsharded result."""

import datetime
import os
import socket

import numpy as np
import pytest

from block_sparse_video_geometry_b200 import sharding, workloads as W


def test_head_range_partitions():
    for H in range(0, 30):
        for world in range(1, 9):
            got = [sharding.head_range(r, world, H) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [h1 - h0 for h0, h1 in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sharding.head_range(2, 2, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from oracle import vsa_oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # timing and work reductions
        res["max"] = sharding.max_over_ranks([rank + 1.0, 10.0 - rank], dist)
        res["sum"] = sharding.sum_over_ranks([rank + 1.0], dist)
        # a head-sharded forward pass: each rank takes its heads
        wl = W.WORKLOADS["tiny"].with_(H=3)
        lay = O.build_layout([O.Segment(k, s, n, g) for (k, s, n, g) in wl.segments()], wl.seq_len)
        q, k, v, g = (O.bf16_bits_to_f64(x) for x in W.make_inputs(wl, lay.inv // O.TILE))
        h0, h1 = sharding.head_range(rank, world, wl.H)
        qs, ks, vs, gs = (sharding.head_slice(x, h0, h1) for x in (q, k, v, g))
        mine = {h0 + j: O.vsa_forward_head(qs[0, :, j], ks[0, :, j], vs[0, :, j], gs[0, :, j], lay,
                                           O.Params(keep=wl.keep)).out
                for j in range(h1 - h0)}
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        if rank == 0:
            full = {}
            for part in gathered:
                full.update(part)
            assert sorted(full) == list(range(wl.H))
            for h in range(wl.H):
                ref = O.vsa_forward_head(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], lay,
                                         O.Params(keep=wl.keep)).out
                res["head%d" % h] = bool(np.array_equal(full[h], ref))
        out.put((rank, res))
    except Exception as e:       # reported to the parent
        out.put((rank, {"error": repr(e)}))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in procs:
        rank, res = out.get(timeout=240)
        results[rank] = res
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        assert "error" not in results[r], results[r]
        assert results[r]["max"] == [2.0, 10.0]
        assert results[r]["sum"] == [3.0]
    assert all(results[0]["head%d" % h] for h in range(3))
