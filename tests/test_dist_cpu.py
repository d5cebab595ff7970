"""Multi-process host logic on CPU (gloo, world size 2): the max/sum-over-ranks
reductions and barrier bench.py uses for the timing; the reference arm under
torchrun (rank 0 runs and prints one line; the other rank exits 0 without
work); and the context-parallel exchange (ar_decoding_b200.cp): each rank
shards the same cache, computes its slice's attention with the oracle, the
ranks all-gather and merge, and every rank ends with the whole-cache
attention."""
import json
import os
import socket
import subprocess
import sys

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_setup(None)
    assert (r, w) == (rank, world)
    bench.barrier(w)
    mx = bench.reduce_max(10.0 + rank, w)
    sm = bench.reduce_sum(1.5 * (rank + 1), w)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((rank, mx, sm))


def test_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, sm in res:
        assert mx == 11.0
        assert sm == pytest.approx(1.5 + 3.0)


def test_reference_arm_under_torchrun_cpu():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--k", "4",
           "--prefix", "512", "--no-cpu-sweep"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _cp_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from ar_decoding_b200 import cp, synth
    dist.init_process_group("gloo")
    cfg = synth.StepConfig("cp-dist", B=2, Hq=4, Hkv=2, D=64, k=3, prefix=(257, 40), dtype="f32",
                           seed=21)
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    n = synth.to_np
    args = (n(step["q"]), n(step["k_blk"]), n(step["v_blk"]))
    loc = cp.shard_cache(cache, world, rank, cfg.k)
    o, l = oracle.step_attn(*args, n(loc["k_pages"]), n(loc["v_pages"]), n(loc["page_table"]),
                            n(loc["seq_lens"]), cfg.k, step_keys=rank == world - 1)

    def merge(po, pl):
        out, lse = oracle.merge(po.numpy(), pl.numpy())
        return torch.from_numpy(out), torch.from_numpy(lse)

    got, got_lse = cp.gather_merge(torch.from_numpy(o), torch.from_numpy(l), merge)
    want, want_lse = oracle.step_attn(*args, n(cache["k_pages"]), n(cache["v_pages"]),
                                      n(cache["page_table"]), n(cache["seq_lens"]), cfg.k)
    err = max(float(np.abs(got.numpy() - want).max()), float(np.abs(got_lse.numpy() - want_lse).max()))
    dist.destroy_process_group()
    q.put((rank, err))


def test_context_parallel_exchange_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, err in res:
        assert err < 1e-12, (rank, err)
