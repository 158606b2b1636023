"""Host-side logic of the multi-GPU bench on CPU: two `gloo` ranks.

The decode step shards by problem (every rank runs its own batch of heads,
no data-path collective), so what N > 1 adds is plumbing: process-group
setup from the torchrun environment, the barrier around the timed region,
the max over ranks of the step time, per-rank seeds that give each rank its
own workload, and a reference arm that only rank 0 runs and prints.  All of
it is exercised here with world_size 2 on the CPU.
"""
import contextlib
import io
import json
import os
import socket
import sys
from argparse import Namespace

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench
    from hash_aware_top_hata_b200 import workloads as wl
    out = {}
    try:
        args = Namespace(impl="hata")
        w, r, local = bench.dist_setup(args)
        out["world"], out["rank"], out["backend"] = w, r, dist.get_backend()
        bench.barrier(w)
        out["max"] = bench.max_over_ranks(w, 1.5 * (rank + 1))
        # per-rank workloads: the bench seeds rank r with SEED_BASE + config + 1000 r
        cfg = wl.CONFIGS["tiny_mha_4k"]
        seed = wl.SEED_BASE + wl.CONFIG_ORDER.index(cfg.name) + 1000 * rank
        q0 = wl.make_workload(cfg, seed, steps=1).q[0].reshape(-1)[:8]
        gathered = [torch.zeros(8) for _ in range(w)]
        dist.all_gather(gathered, q0.float())
        out["q_differ"] = not torch.equal(gathered[0], gathered[1])
        # reference arm: rank 0 alone runs the oracle and prints one line
        buf = io.StringIO()
        rargs = Namespace(impl="reference", config="tiny_mha_4k", steps=1, warmup=1,
                          context=0, batch=0)
        with contextlib.redirect_stdout(buf):
            bench.run_reference(rargs, w, r)
        out["ref_lines"] = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        out["error"] = repr(e)
    q.put(out)


@pytest.mark.timeout(300)
def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    res.sort(key=lambda d: d.get("rank", -1))
    for d in res:
        assert "error" not in d, d
        assert d["world"] == 2 and d["backend"] == "gloo"
        assert d["max"] == 3.0          # max over ranks of 1.5 and 3.0
        assert d["q_differ"]            # each rank has its own problem
    assert len(res[0]["ref_lines"]) == 1 and res[1]["ref_lines"] == []
    line = json.loads(res[0]["ref_lines"][0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
