"""The multi-rank host logic of bench.py on CPU: gloo, world size 2.

Each rank is an independent replica (its own seed, its own batch); the only
collectives are the barrier and the max over ranks of the timings, and the
reported value is the whole job's bytes over the slowest rank's time."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    from w4a8_codebook_quantized_b200 import inputs
    try:
        w, r, local = bench.dist_setup("gloo")
        assert (w, r, local) == (world, rank, rank)
        # per-rank replica: its own layer and batch, computed independently
        seed = bench.rank_seed(3, r)
        layer = inputs.layer(64, 512, seed)
        x = inputs.activations(4, 512, seed)
        y = oracle.linear(x, layer.qdata, layer.srel, layer.codebook, layer.s_channel)["y"]
        digest = torch.tensor([int(y.astype(np.int64).sum())], dtype=torch.int64)
        gathered = [torch.zeros_like(digest) for _ in range(w)]
        dist.all_gather(gathered, digest)
        # the max over ranks of a per-rank "time"
        t = bench.max_over_ranks(1.0 + r, w)
        bench.barrier(w)
        v = bench.aggregate_value(1e9, 10, w, t)
        # reference arm: only rank 0 prints, the other ranks exit without work
        buf = io.StringIO()
        sys.argv = ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                    "--workload", "c1_decode_m1_1k"]
        with redirect_stdout(buf):
            bench.main()
        q.put((r, [int(g.item()) for g in gathered], t, v, buf.getvalue()))
        dist.destroy_process_group()
    except Exception as e:  # surface the failure to the parent
        q.put((rank, "error", repr(e), None, None))
        raise


def test_two_rank_replicas_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        r, digests, t, v, out = q.get(timeout=300)
        assert digests != "error", t
        results[r] = (digests, t, v, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d0, t0, v0, out0 = results[0]
    d1, t1, v1, out1 = results[1]
    assert d0 == d1 and d0[0] != d0[1]       # both ranks see both replicas; replicas differ
    assert t0 == t1 == 2.0                   # the slowest rank's time everywhere
    assert v0 == v1 == pytest.approx(2 * 1e9 * 10 / 2.0 / 1e9)
    line = json.loads(out0.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["n_gpus"] == 2
    assert out1.strip() == ""
