"""Benchmark of one TiDAR decode step on B200: step attention (three zones over a
paged bf16 GQA KV cache, plus the draft-row append), greedy verification with
block selection, and the KV commit -- all through the C ABI of libtidar.so.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: 8B-class heads (32 q / 8 kv, head_dim 128, bf16), prefix 8192, k = 16
(16 draft rows + 16 blocks of 16 mask slots = 272 query rows), verification over
vocab 32768 logits N(0,3) with each draft equal to the row argmax w.p. 0.7.
Inputs are seeded synthetic tensors generated on the device.  One rank per GPU
(torchrun); every rank runs its own independent sequence (weak scaling, no
collective on the data path).

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and
cudaDeviceSynchronize.  The steps (step attention, then verification and
commit, captured from the public API calls) run back to back as a serving loop
issues them: replays of CUDA graphs that each hold the steps of up to n
independent input/cache copies in a row, timed on the device with CUDA events
on the launching stream, one event pair per replay.  The copies are enough
that each step's working set is evicted from L2 (126 MB) before it is reused;
after each replay (outside the events) a second graph restores those copies'
prefix lengths and page tables, so every step does identical work.
ms_per_step / value is the mean step time, max over ranks.  For reference the
line also carries step_call_us: each step alone, its own one-step graph between
two events (adding the device-side cost of one graph launch per step).

Also in the line: the attention kernel's roofline (algorithmic bytes or flops
over its launch duration, against the measured peaks), the k sweep, the other
workloads (extra_configs: the serving batch, long-context corners, 1.5B-class
and tiny, each with its own roofline fractions), the same step end to end with
host buffers (e2e, rotating the same cold copies), the chained decode loops
(decode_loop: reserve -> attention -> verify -> commit for 8 steps of 10
interleaved sequences in one CUDA graph, greedy and rejection with q read
from the previous step's mask blocks), and the CPU oracle on the host cores.

--impl reference times the plain CPU oracle instead (the only reference this
path has): one whole step of the same workload per timed step on every
allowed host core, plus the oracle's whole-step time on each timed workload
single-threaded and on all cores (cpu_sweep).

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
METRIC = "TiDAR step latency (µs) and achieved HBM GB/s vs draft length k"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--k", type=int, default=16)
    ap.add_argument("--prefix", type=int, default=8192)
    ap.add_argument("--no-sweep", action="store_true", help="skip the k sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc05", "dec", "pair"])
    ap.add_argument("--no-loop", action="store_true", help="skip the chained decode-loop timing")
    ap.add_argument("--loop-chain", type=int, default=8,
                    help="steps chained per sequence in the decode-loop graph")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (serving batch, long-context corners, "
                         "1.5B-class, tiny) reported under extra_configs")
    ap.add_argument("--no-layer", action="store_true",
                    help="skip the layer-level k sweep (projections + attention)")
    ap.add_argument("--no-cpu-sweep", action="store_true",
                    help="reference arm: skip the per-workload oracle timings (cpu_sweep)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- setup
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


PATH_NAMES = {1: "simt", 2: "tc05", 3: "dec", 4: "pair"}


def workload(k: int, prefix: int, rank: int = 0):
    from ar_decoding_b200 import synth
    return synth.class_8b(seed=synth.SEED_BASE + 2 + 1000 * rank, k=k, prefix=prefix)


def step_key_counts(k: int) -> int:
    """Visible step keys summed over the rows of one sequence: draft row r sees r
    drafts; a slot of block j sees j drafts and the k slots of its block."""
    if k == 0:
        return 1
    return k * (k + 1) // 2 + k * sum(j + k for j in range(1, k + 1))


def algorithmic(cfg):
    """Bytes that must move and flops of one step attention: KV prefix read, Q read
    and O write, step K/V read, draft-row append write; flops 4*D per (row, head,
    visible key) for QK^T and PV."""
    e = cfg.elem_bytes
    P = sum(cfg.prefix)
    kv = P * cfg.Hkv * cfg.D * 2 * e
    qo = 2 * cfg.B * cfg.R * cfg.Hq * cfg.D * e
    stepkv = cfg.B * cfg.R * cfg.Hkv * cfg.D * 2 * e
    append = cfg.B * cfg.n * cfg.Hkv * cfg.D * 2 * e
    vis = sum(cfg.R * p + step_key_counts(cfg.k) for p in cfg.prefix)
    flops = 4 * cfg.D * cfg.Hq * vis
    return kv + qo + stepkv + append, flops


class Step:
    """Device-resident inputs for `copies` independent instances of the workload,
    and one decode step (attention, verify, commit) on a chosen copy."""

    def __init__(self, cfg, copies, path="auto"):
        import ar_decoding_b200 as tidar
        from ar_decoding_b200 import synth
        self.tidar, self.cfg, self.path = tidar, cfg, path
        dev = torch.device("cuda")
        self.copies = []
        for c in range(copies):
            cc = synth.StepConfig(**{**cfg.__dict__, "seed": cfg.seed + 17 * c})
            cache = synth.make_cache(cc, device=dev)
            step = synth.make_step(cc, device=dev)
            vin = synth.make_verify(cc, "greedy")
            self.copies.append(dict(
                cache=cache, step=step,
                logits=vin["logits"].to(dev), drafts=vin["drafts"].to(dev),
                guesses=vin["block_guesses"].to(dev),
                seq0=cache["seq_lens"].clone(), pt0=cache["page_table"].clone()))
        self.max_prefix = max(cfg.prefix)
        c0 = self.copies[0]
        self.desc = tidar.make_desc(c0["step"]["q"], c0["step"]["k_blk"], c0["cache"], cfg.k,
                                    self.max_prefix, path=path)
        self.path_id, self.splits = tidar.plan(self.desc)
        need = tidar.step_attn_workspace_bytes(self.desc)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(c0["step"]["q"])
        self.lse = torch.empty(c0["step"]["q"].shape[:3], dtype=torch.float32, device=dev)
        B, n, V = c0["logits"].shape
        self.vws = torch.empty(max(tidar.verify_workspace_bytes(B, cfg.k, V, 0), 256),
                               dtype=torch.uint8, device=dev)
        self.vout = dict(accept_count=torch.empty(B, dtype=torch.int32, device=dev),
                         out_tokens=torch.empty((B, n), dtype=torch.int32, device=dev),
                         next_drafts=torch.empty((B, max(cfg.k, 1)), dtype=torch.int32, device=dev),
                         selected_block=torch.empty(B, dtype=torch.int32, device=dev))
        cap = cfg.B * ((cfg.n + cfg.page_size - 1) // cfg.page_size + 1)
        self.rel = torch.empty(cap, dtype=torch.int32, device=dev)
        self.nrel = torch.empty(1, dtype=torch.int32, device=dev)
        # attention: one launch when the kernel merges its splits itself on the
        # tensor-core or decode path, else kernel + finalize; then greedy
        # verification and commit (tidar_verify_commit: the chunk statistics,
        # then acceptance + commit in one cluster kernel)
        self.merge = tidar.plan_full(self.desc)[2]
        self.attn_launches = 2 if (self.merge == 2 or self.path_id == 1) else 1
        self.launches_per_step = self.attn_launches + 2

    def attn(self, i):
        c = self.copies[i]
        self.tidar.step_attn(c["step"]["q"], c["step"]["k_blk"], c["step"]["v_blk"], c["cache"],
                             self.cfg.k, max_prefix_len=self.max_prefix, path=self.path,
                             out=self.out, lse=self.lse, workspace=self.ws)

    def verify_commit(self, i):
        c = self.copies[i]
        self.tidar.verify_commit(c["logits"], c["drafts"], c["cache"], self.cfg.k, "greedy",
                                 max_prefix_len=self.max_prefix, block_guesses=c["guesses"],
                                 outputs=self.vout, released=self.rel, num_released=self.nrel,
                                 workspace=self.vws)

    def restore(self, i):
        c = self.copies[i]
        c["cache"]["seq_lens"].copy_(c["seq0"], non_blocking=True)
        c["cache"]["page_table"].copy_(c["pt0"], non_blocking=True)

    def round_graph(self, m):
        """(graph of the steps of copies 0..m-1 back to back, graph restoring
        those copies), captured once per m."""
        rg = self.__dict__.setdefault("_rounds", {})
        if m not in rg:
            gs, gr = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(gs):
                for i in range(m):
                    self.attn(i)
                    self.verify_commit(i)
            with torch.cuda.graph(gr):
                for i in range(m):
                    self.restore(i)
            torch.cuda.synchronize()
            gr.replay()
            torch.cuda.synchronize()
            rg[m] = (gs, gr)
        return rg[m]

    def capture(self):
        """Per copy, one CUDA graph of the whole step (attention, verify, commit),
        one of the attention call alone, and one that restores the copy's
        prefix length and page table.  Replaying them keeps the host out of the
        timed device work."""
        n = len(self.copies)
        for i in range(n):          # first calls outside capture (module load, attributes)
            self.attn(i); self.verify_commit(i); self.restore(i)
        torch.cuda.synchronize()
        self.graphs = []
        for i in range(n):
            gs, ga, gr = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(gs):
                self.attn(i)
                self.verify_commit(i)
            with torch.cuda.graph(ga):
                self.attn(i)
            with torch.cuda.graph(gr):
                self.restore(i)
            self.graphs.append((gs, ga, gr))
        torch.cuda.synchronize()


class Loop:
    """The decode loop on the device: `chain` steps of reserve -> step attention
    -> verify -> commit per sequence, each step's drafts, lengths and pages
    coming from the step before (no host round-trip), for `copies` independent
    sequences interleaved step by step (each copy's KV is cold in L2 when its
    turn comes).  One CUDA graph holds the whole loop; a second restores every
    copy's lengths, page table and free-page stack."""

    def __init__(self, cfg, copies, chain, path="auto", mode="greedy"):
        import ar_decoding_b200 as tidar
        from ar_decoding_b200 import synth
        self.tidar, self.cfg, self.chain, self.path, self.mode = tidar, cfg, chain, path, mode
        dev = torch.device("cuda")
        n = cfg.n
        self.max_prefix = max(cfg.prefix) + chain * n
        width = -(-(self.max_prefix + n) // cfg.page_size)
        self.copies = []
        for c in range(copies):
            cc = synth.StepConfig(**{**cfg.__dict__, "seed": cfg.seed + 31 * c + 5})
            cache = synth.make_cache(cc, device=dev, extra_pages=chain * n // cfg.page_size + 2,
                                     draft_pages=False, max_pages=width)
            pool = {k: v.to(dev) for k, v in synth.make_pool(cc, cache).items()}
            attn, ver = synth.make_loop(cc, chain, mode)
            rej = mode != "greedy"
            self.copies.append(dict(
                cache=cache, pool=pool,
                attn=[{k: v.to(dev) for k, v in a.items()} for a in attn],
                logits=[v["logits"].to(dev) for v in ver],
                guesses=[v["block_guesses"].to(dev) for v in ver],
                uniforms=[v["uniforms"].to(dev) for v in ver] if rej else None,
                q0=ver[0]["draft_logits"].to(dev) if rej and cfg.k > 1 else None,
                blocks=[v["block_logits"].to(dev) for v in ver] if mode == "blockq" else None,
                sel=[torch.empty(cfg.B, dtype=torch.int32, device=dev) for _ in range(2)],
                drafts0=ver[0]["drafts"].to(dev),
                saved={k: t.clone() for k, t in (("seq_lens", cache["seq_lens"]),
                                                  ("page_table", cache["page_table"]))},
                saved_pool={k: t.clone() for k, t in pool.items()},
                drafts=[torch.empty((cfg.B, max(cfg.k, 1)), dtype=torch.int32, device=dev)
                        for _ in range(2)],
                rel=[torch.empty(cfg.B * (-(-n // cfg.page_size) + 1), dtype=torch.int32,
                                 device=dev) for _ in range(2)],
                nrel=[torch.empty(1, dtype=torch.int32, device=dev) for _ in range(2)]))
        c0 = self.copies[0]
        q0 = c0["attn"][0]["q"]
        self.desc = tidar.make_desc(q0, c0["attn"][0]["k_blk"], c0["cache"], cfg.k,
                                    self.max_prefix, path=path)
        self.path_id, self.splits = tidar.plan(self.desc)
        need = tidar.step_attn_workspace_bytes(self.desc)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        self.out = torch.empty_like(q0)
        self.lse = torch.empty(q0.shape[:3], dtype=torch.float32, device=dev)
        V = c0["logits"][0].shape[2]
        vmode = tidar.GREEDY if mode == "greedy" else tidar.REJECTION
        self.vws = torch.empty(max(tidar.verify_workspace_bytes(cfg.B, cfg.k, V, vmode), 256),
                               dtype=torch.uint8, device=dev)
        self.vout = dict(accept_count=torch.empty(cfg.B, dtype=torch.int32, device=dev),
                         out_tokens=torch.empty((cfg.B, n), dtype=torch.int32, device=dev))
        # reserve, attention (+ finalize), verify + commit (greedy: chunk
        # statistics, then acceptance + commit in one launch; rejection: chunk
        # statistics, residual sums + inverse CDF in one cluster when the
        # vocabulary's 4096-wide chunks fit a portable cluster of 8, else two
        # launches, then the commit)
        nchunk = -(-V // 4096)
        merge = tidar.plan_full(self.desc)[2]
        self.launches_per_step = (1 + (2 if (merge == 2 or self.path_id == 1) else 1) +
                                  (1 if mode == "greedy" else (2 if nchunk <= 8 else 3)) + 1)

    def step(self, c, s):
        """Step s of copy c: pages, attention (with the draft-row append),
        verification (next drafts into a ping-pong buffer), commit."""
        t, k = self.tidar, self.cfg.k
        cp = self.copies[c]
        prev = (s + 1) % 2
        t.reserve(cp["cache"], cp["pool"], k, max_prefix_len=self.max_prefix,
                  returned=cp["rel"][prev] if s else None, num_returned=cp["nrel"][prev] if s else None)
        a = cp["attn"][s]
        t.step_attn(a["q"], a["k_blk"], a["v_blk"], cp["cache"], k, max_prefix_len=self.max_prefix,
                    path=self.path, out=self.out, lse=self.lse, workspace=self.ws)
        drafts = cp["drafts0"] if s == 0 else cp["drafts"][prev]
        vout = dict(self.vout, next_drafts=cp["drafts"][s % 2], selected_block=cp["sel"][s % 2])
        g = cp["guesses"][s] if k else None
        if self.mode == "greedy":
            # verification and commit as one call (acceptance inside the commit's launch)
            t.verify_commit(cp["logits"][s], drafts if k else None, cp["cache"], k, "greedy",
                            max_prefix_len=self.max_prefix, block_guesses=g, outputs=vout,
                            released=cp["rel"][s % 2], num_released=cp["nrel"][s % 2],
                            workspace=self.vws)
            return
        elif self.mode == "blockq" and s > 0:
            # q from the previous step's mask blocks, through its selected block
            t.verify_blockq(cp["logits"][s], drafts, k, cp["blocks"][s - 1], cp["sel"][prev],
                            cp["uniforms"][s], block_guesses=g, outputs=vout, workspace=self.vws)
        else:
            t.verify(cp["logits"][s], drafts if k else None, k, "rejection", draft_logits=cp["q0"],
                     uniforms=cp["uniforms"][s], block_guesses=g, outputs=vout, workspace=self.vws)
        t.commit(cp["cache"], self.vout["accept_count"], k, max_prefix_len=self.max_prefix,
                 released=cp["rel"][s % 2], num_released=cp["nrel"][s % 2])

    def run(self):
        for s in range(self.chain):
            for c in range(len(self.copies)):
                self.step(c, s)

    def restore(self):
        for cp in self.copies:
            for k, v in cp["saved"].items():
                cp["cache"][k].copy_(v, non_blocking=True)
            for k, v in cp["saved_pool"].items():
                cp["pool"][k].copy_(v, non_blocking=True)

    def grown(self) -> int:
        """Tokens the loop committed (sum of accept counts) since the last restore."""
        return int(sum(int((cp["cache"]["seq_lens"] - cp["saved"]["seq_lens"]).sum())
                       for cp in self.copies))

    def time(self, reps: int):
        """Returns (µs per step, committed tokens per loop) over `reps` replays."""
        self.run(); self.restore()                 # first calls outside capture
        torch.cuda.synchronize()
        status, bits = self.tidar.device_status()
        if status != self.tidar.OK:
            raise RuntimeError(f"decode loop: device status {status} bits {bits:#x}")
        gl, gr = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gl):
            self.run()
        with torch.cuda.graph(gr):
            self.restore()
        stream = torch.cuda.current_stream()
        gl.replay(); gr.replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        tokens = None
        hold_stream(reps)
        for i in range(reps):
            ev[i][0].record(stream)
            gl.replay()
            ev[i][1].record(stream)
            if i == reps - 1:
                torch.cuda.synchronize()
                tokens = self.grown()
            gr.replay()
        torch.cuda.synchronize()
        status, bits = self.tidar.device_status()
        if status != self.tidar.OK:
            raise RuntimeError(f"decode loop: device status {status} bits {bits:#x}")
        steps = self.chain * len(self.copies)
        us = statistics.mean(a.elapsed_time(b) * 1e3 for a, b in ev) / steps
        del gl, gr
        return us, tokens


class LayerStep:
    """The layer-level step (query/key/value projection with the rotary
    embedding, step attention with the draft append, output projection) on
    `copies` independent instances, each with its own random weights and
    cache, so neither the weights (84 MB at 8B-class sizes) nor the KV cache of
    a copy are in L2 when its turn comes."""

    def __init__(self, cfg, copies):
        import ar_decoding_b200 as tidar
        from ar_decoding_b200 import synth
        self.tidar, self.cfg = tidar, cfg
        dev = torch.device("cuda")
        self.copies = []
        for c in range(copies):
            cc = synth.StepConfig(**{**cfg.__dict__, "seed": cfg.seed + 23 * c})
            lay = synth.make_layer(cc, device=dev)
            self.copies.append(dict(cache=synth.make_cache(cc, device=dev), **lay))
        c0 = self.copies[0]
        self.dm = c0["d_model"]
        self.max_prefix = max(cfg.prefix)
        self.desc = tidar._layer_desc(c0["x"], cfg.k, cfg.Hq, cfg.Hkv, self.max_prefix)
        need = tidar.layer_step_workspace_bytes(self.desc, self.dm)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        B, R = cfg.B, cfg.R
        self.y = torch.empty((B, R, self.dm), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, R, cfg.Hq), dtype=torch.float32, device=dev)
        self.qkv_out = (torch.empty((B, R, cfg.Hq, 128), dtype=torch.bfloat16, device=dev),
                        torch.empty((B, R, cfg.Hkv, 128), dtype=torch.bfloat16, device=dev),
                        torch.empty((B, R, cfg.Hkv, 128), dtype=torch.bfloat16, device=dev))
        self.attn_out = torch.empty((B, R, cfg.Hq, 128), dtype=torch.bfloat16, device=dev)

    def layer(self, i):
        c, cfg = self.copies[i], self.cfg
        self.tidar.layer_step(c["x"], c["w_qkv"], c["w_o"], c["cache"], cfg.k, cfg.Hq, cfg.Hkv,
                              max_prefix_len=self.max_prefix, out=self.y, lse=self.lse,
                              workspace=self.ws)

    def qkv(self, i):
        c, cfg = self.copies[i], self.cfg
        self.tidar.qkv_rope(c["x"], c["w_qkv"], c["cache"]["seq_lens"], cfg.k, cfg.Hq, cfg.Hkv,
                            max_prefix_len=self.max_prefix, out=self.qkv_out, workspace=self.ws)

    def oproj(self, i):
        self.tidar.linear(self.attn_out, self.copies[i]["w_o"], out=self.y, workspace=self.ws)

    def time(self, fn, reps):
        """Average device µs of fn over all copies back to back in one graph."""
        n = len(self.copies)
        for i in range(n):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                fn(i)
        stream = torch.cuda.current_stream()
        g.replay(); g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold_stream(reps)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / (reps * n)


def layer_sweep(hbm_peak, tc_peak, world, ks=(0, 4, 8, 16), reps=5):
    """Layer-level step at 8B-class sizes (d_model 4096, 32 q / 8 kv heads,
    prefix 8192) for each k: the whole layer and its projections, with the
    projections' algorithmic bytes (weights + activations) and flops."""
    from ar_decoding_b200 import synth
    out = []
    for k in ks:
        cfg = synth.class_8b(k=k)
        dm = synth.D_MODEL["8B-class"]
        T = cfg.B * cfg.R
        nqkv, no = (cfg.Hq + 2 * cfg.Hkv) * 128, dm
        w_bytes = (nqkv * dm + no * cfg.Hq * 128) * 2
        per_copy = w_bytes + algorithmic(cfg)[0]
        ls = LayerStep(cfg, max(3, math.ceil(3 * L2_BYTES / per_copy)))
        lay_us = reduce_max(ls.time(ls.layer, reps), world)
        qkv_us = reduce_max(ls.time(ls.qkv, reps), world)
        o_us = reduce_max(ls.time(ls.oproj, reps), world)
        qkv_b = nqkv * dm * 2 + T * dm * 2 + T * nqkv * 2
        o_b = no * cfg.Hq * 128 * 2 + T * cfg.Hq * 128 * 2 + T * no * 2
        qkv_f, o_f = 2 * T * nqkv * dm, 2 * T * no * cfg.Hq * 128
        a_b, a_f = algorithmic(cfg)

        def frac(b, f, us):
            return max(b / (hbm_peak * 1e9), f / (tc_peak * 1e12)) / (us * 1e-6)
        out.append({"k": k, "rows": T, "d_model": dm, "copies": len(ls.copies),
                    "layer_us": lay_us, "qkv_rope_us": qkv_us, "o_proj_us": o_us,
                    "weight_bytes": w_bytes,
                    "qkv_rope_gbs": qkv_b / (qkv_us * 1e-6) / 1e9,
                    "qkv_rope_tflops": qkv_f / (qkv_us * 1e-6) / 1e12,
                    "qkv_rope_roofline_frac": frac(qkv_b, qkv_f, qkv_us),
                    "o_proj_gbs": o_b / (o_us * 1e-6) / 1e9,
                    "o_proj_tflops": o_f / (o_us * 1e-6) / 1e12,
                    "o_proj_roofline_frac": frac(o_b, o_f, o_us),
                    "layer_roofline_us": (max((qkv_b) / (hbm_peak * 1e9), qkv_f / (tc_peak * 1e12)) +
                                          max(a_b / (hbm_peak * 1e9), a_f / (tc_peak * 1e12)) +
                                          max(o_b / (hbm_peak * 1e9), o_f / (tc_peak * 1e12))) * 1e6})
        del ls
        torch.cuda.empty_cache()
    base = out[0]["layer_us"] if out else None
    for r in out:
        r["layer_vs_k0"] = r["layer_us"] / base if base else None
    return out


KERNEL_SRC = {2: "attn_tc05.cu", 3: "attn_dec.cu", 4: "attn_pair.cu"}
KERNEL_HEADERS = ("tc05.cuh", "sm100.cuh", "common.cuh", "kernels.h")


def kernel_source_hash(path_id: int) -> str:
    """sha256 prefix of an attention kernel's source and the headers it
    includes (the key of profiles/traffic.txt)."""
    import hashlib
    h = hashlib.sha256()
    for name in (KERNEL_SRC[path_id],) + KERNEL_HEADERS:
        with open(os.path.join(ROOT, "ar_decoding_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(k: int, path_id: int):
    """DRAM bytes of one attention launch from the committed ncu record, if the
    kernel source is unchanged since the capture; else None."""
    if path_id not in KERNEL_SRC:
        return None
    rec = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        sha = kernel_source_hash(path_id)
        for line in open(rec):
            parts = line.split()
            if len(parts) == 3 and not line.startswith("#") and parts[0] == sha and int(parts[1]) == k:
                return int(parts[2])
    except OSError:
        pass
    return None


MAX_COPIES = 64


def copies_for(cfg):
    """Independent input copies to rotate over: enough that 3x L2 of other
    copies' data passes between two uses of one copy, at most MAX_COPIES (small
    workloads then flush L2 between timed steps instead, see l2_policy)."""
    per = algorithmic(cfg)[0] + cfg.B * cfg.n * cfg.vocab * cfg.elem_bytes
    return min(MAX_COPIES, max(3, math.ceil(3 * L2_BYTES / per)))


def needs_flush(cfg) -> bool:
    per = algorithmic(cfg)[0] + cfg.B * cfg.n * cfg.vocab * cfg.elem_bytes
    return copies_for(cfg) * per < 3 * L2_BYTES


def l2_policy(cfg) -> str:
    if needs_flush(cfg):
        return (f"rotating {copies_for(cfg)} input copies and reading a {2 * L2_BYTES >> 20} MiB "
                "buffer (> L2) between timed steps")
    return f"rotating {copies_for(cfg)} independent input copies (> 3x L2) between timed steps"


_FLUSH = {}


def flush_l2():
    """Read a buffer twice the size of L2 (evicts every earlier line).  A read,
    not a write: a flush that leaves L2 full of dirty lines makes the next
    kernel wait for their write-back (~100 µs), which is not the workload's."""
    buf = _FLUSH.get("buf")
    if buf is None:
        buf = _FLUSH["buf"] = torch.zeros(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        _FLUSH["sink"] = torch.empty((), dtype=torch.uint8, device="cuda")
    torch.amax(buf, dim=0, out=_FLUSH["sink"])


def hold_stream(items: int, us_per_item: float = 40.0) -> None:
    """Queue a GPU-side wait (a spin of about 0.2 ms + `us_per_item` per timed
    item) ahead of the timed launches, so that the host has enqueued all of
    them before the first one runs: the events then bracket device work only,
    never a gap in which the device waits for the host to submit the next
    graph.  The work between the events is unchanged."""
    torch.cuda._sleep(int((200.0 + items * us_per_item) * 2000))   # clock cycles, ~2 GHz


def bench_config(cfg, prefix: int, k: int) -> dict:
    """The `config` object of the JSON line: the workload, identical for the GPU
    arm and the oracle (reference) arm."""
    return {"workload": "8B-class TiDAR step", "B_per_gpu": cfg.B, "Hq": cfg.Hq,
            "Hkv": cfg.Hkv, "head_dim": cfg.D, "prefix": prefix, "k": k, "rows": cfg.R,
            "vocab": cfg.vocab, "page": cfg.page_size, "l2": l2_policy(cfg)}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.proc = None
        self.index = index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- timing
def time_steps(st: Step, K: int, W: int, world: int):
    """Returns (per-step device µs, per-call step_attn µs, per-step µs of a
    one-step graph) as lists.  The step: graphs of consecutive steps of
    different copies, back to back as a serving loop issues them (the
    attention's own figure is taken the same way), each replay between two
    events on the launching stream, the restore graphs outside the events.
    For reference each step is also timed alone, its copy's one-step graph
    between two events (that adds the device-side cost of launching a graph
    to every step), and the attention call likewise."""
    n = len(st.copies)
    st.capture()
    stream = torch.cuda.current_stream()
    flush = needs_flush(st.cfg)

    def run(which, count, warm):
        for i in range(warm):
            g = st.graphs[i % n]
            g[which].replay(); g[2].replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(count)]
        barrier(world)
        torch.cuda.synchronize()
        hold_stream(count, 60.0 if flush else 40.0)
        for i in range(count):
            g = st.graphs[(warm + i) % n]
            ev[i][0].record(stream)
            g[which].replay()
            ev[i][1].record(stream)
            g[2].replay()
            if flush:
                flush_l2()
        torch.cuda.synchronize()
        barrier(world)
        return [a.elapsed_time(b) * 1e3 for a, b in ev]

    def run_rounds(count, warm):
        """Steps back to back: one graph holds the steps of m <= n copies in
        a row (each copy once, so every step does the same work), replayed
        between two events; the restore of those copies runs after the second
        event.  Each timed step gets its round's mean."""
        for i in range(warm):
            st.round_graph(n)[0].replay(); st.round_graph(n)[1].replay()
        torch.cuda.synchronize()
        sizes = [n] * (count // n) + ([count % n] if count % n else [])
        graphs = [st.round_graph(m) for m in sizes]
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in sizes]
        barrier(world)
        torch.cuda.synchronize()
        hold_stream(count)
        for (gs, gr), (e0, e1) in zip(graphs, ev):
            e0.record(stream)
            gs.replay()
            e1.record(stream)
            gr.replay()
        torch.cuda.synchronize()
        barrier(world)
        out = []
        for m, (e0, e1) in zip(sizes, ev):
            out += [e0.elapsed_time(e1) * 1e3 / m] * m
        return out

    step_call_us = run(0, K, W)
    attn_us = run(1, K, W)
    # small workloads flush L2 between steps: there every step keeps its own graph
    step_us = step_call_us if flush else run_rounds(K, W)
    return step_us, attn_us, step_call_us


def time_attention_launches(st: Step, reps: int, attn_call_us=None):
    """Average device time of one tidar_step_attn call: a CUDA graph of one call
    per input copy, back to back (each copy's KV is cold in L2 when its turn
    comes), replayed `reps` times between two events on the launching stream.
    A workload too small for that (it flushes L2 between steps instead) reports
    the per-call time measured between flushes (attn_call_us)."""
    if needs_flush(st.cfg) and attn_call_us is not None:
        return attn_call_us
    n = len(st.copies)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            st.attn(i)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold_stream(reps)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * n)
    del g
    return us


def time_e2e(st: Step, K: int, W: int):
    """Same step through the public API with host buffers: the step's inputs are
    copied from pinned host memory and the verification results read back, inside
    the timed region.  The copies and calls of one step are one CUDA graph (as a
    serving loop would issue them): Q and the step K/V are copied first on the
    launching stream; then the verification inputs (logits, drafts, guesses)
    are copied on a second stream while the attention runs (the two sets of
    copies would otherwise share the host link and delay the attention), joined
    before verify.  Timed steps rotate over the same independent copies as the
    device-resident timing, so each step's KV cache is cold in L2, exactly as
    for `value`.  Freshly pinned buffers copy slowly the first few times, so
    the warm-up is longer than W.  Returns (µs per step, h2d bytes, d2h
    bytes)."""
    n = len(st.copies)
    names = (("q", "step", "q"), ("k_blk", "step", "k_blk"), ("v_blk", "step", "v_blk"))
    host_in = []
    for c in st.copies:
        h = {k: c[a][b].cpu().pin_memory() for k, a, b in names}
        h.update({k: c[k].cpu().pin_memory() for k in ("logits", "drafts", "guesses")})
        host_in.append(h)
    host_out = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in st.vout.items()}
    h2d = sum(v.numel() * v.element_size() for v in host_in[0].values())
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    side = torch.cuda.Stream()

    def one(i):
        c, h = st.copies[i], host_in[i]
        main = torch.cuda.current_stream()
        c["step"]["q"].copy_(h["q"], non_blocking=True)
        c["step"]["k_blk"].copy_(h["k_blk"], non_blocking=True)
        c["step"]["v_blk"].copy_(h["v_blk"], non_blocking=True)
        side.wait_stream(main)
        with torch.cuda.stream(side):
            c["logits"].copy_(h["logits"], non_blocking=True)
            c["drafts"].copy_(h["drafts"], non_blocking=True)
            c["guesses"].copy_(h["guesses"], non_blocking=True)
        st.attn(i)
        main.wait_stream(side)
        st.verify_commit(i)
        for k2 in host_out:
            host_out[k2].copy_(st.vout[k2], non_blocking=True)

    for j in range(max(W, 10)):              # eager warm-up
        one(j % n); st.restore(j % n)
    torch.cuda.synchronize()
    graphs = []
    for i in range(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one(i)
        graphs.append(g)
    stream = torch.cuda.current_stream()
    for j in range(max(W, 10)):
        graphs[j % n].replay(); st.graphs[j % n][2].replay()
    torch.cuda.synchronize()
    ts = []
    for j in range(K):
        i = j % n
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graphs[i].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
        if j == K - 1:                       # the results did come back
            for k2 in host_out:
                if not torch.equal(host_out[k2], st.vout[k2].cpu()):
                    raise RuntimeError(f"e2e: host copy of {k2} differs from the device result")
        st.graphs[i][2].replay()             # restore the copy's lengths and table (untimed)
    torch.cuda.synchronize()
    del graphs
    return statistics.mean(ts), h2d, d2h


# ----------------------------------------------------------------------------- CPU oracle
def oracle_step_seconds(cfg, threads=0):
    """Wall time of the oracle doing one whole step of `cfg`: attention over every
    (b, row, head), the draft-row append, greedy verification and the commit.
    `threads` = 0 uses every allowed core (OpenMP), else that many."""
    import oracle
    from ar_decoding_b200 import synth
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    vin = synth.make_verify(cfg, "greedy")
    n = synth.to_np
    npc = {k: n(v) for k, v in cache.items()}
    nps = {k: n(v) for k, v in step.items()}
    t0 = time.perf_counter()
    oracle.step_attn(nps["q"], nps["k_blk"], nps["v_blk"], npc["k_pages"], npc["v_pages"],
                     npc["page_table"], npc["seq_lens"], cfg.k, num_threads=threads)
    kp, vp = oracle.append(npc["k_pages"], npc["v_pages"], npc["page_table"], npc["seq_lens"],
                           nps["k_blk"], nps["v_blk"], cfg.k)
    res = oracle.verify(n(vin["logits"]), n(vin["drafts"]), cfg.k, oracle.GREEDY,
                        block_guesses=n(vin["block_guesses"]))
    oracle.commit(kp, vp, npc["page_table"], npc["seq_lens"], res["accept_count"], cfg.k)
    return time.perf_counter() - t0


def oracle_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- main
def cpu_sweep(cores: int):
    """The oracle's whole-step time on the workloads it is timed on (tiny,
    1.5B-class, 8B-class at k = 0, 4, 8, 16, one long-context point), single
    threaded and on every allowed core."""
    from ar_decoding_b200 import synth
    out = []
    for cfg in (synth.tiny(), synth.class_1p5b(), synth.class_8b(k=0), synth.class_8b(k=4),
                synth.class_8b(k=8), synth.class_8b(k=16), synth.long_context(1, 32768, 4)):
        row = {"workload": cfg.name, "B": cfg.B, "prefix": max(cfg.prefix), "k": cfg.k,
               "rows": cfg.R, "dtype": cfg.dtype}
        for threads, key in ((1, "us_1_thread"), (cores, f"us_{cores}_threads")):
            row[key] = oracle_step_seconds(cfg, threads) * 1e6
        out.append(row)
    return out


def run_reference(args, rank, world):
    """The oracle arm: the plain CPU oracle timed on the host cores, one whole
    step of the same workload per timed step (nothing sampled or scaled)."""
    if rank != 0:
        return
    cfg = workload(args.k, args.prefix)
    cores = oracle_threads()
    times = []
    for i in range(args.warmup + args.steps):
        t = oracle_step_seconds(cfg, cores)
        if i >= args.warmup:
            times.append(t)
    us = statistics.mean(times) * 1e6
    sample = (f"one whole step per timed step: all {cfg.B * cfg.R * cfg.Hq} (b, row, head) "
              f"attention rows, the draft-row append, greedy verify and commit; {cores} "
              "OpenMP threads")
    sweep = None if args.no_cpu_sweep else cpu_sweep(cores)
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": "us", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": bench_config(cfg, args.prefix, args.k),
            "cpu_baseline": {"value": us, "unit": "us", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "cpu_sweep": sweep,
            "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local):
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    tc_peak = peaks.get("bf16_tflops", 1590.0)
    peak_src = "measured" if peaks else "fallback"

    cfg = workload(args.k, args.prefix, rank)
    st = Step(cfg, copies_for(cfg), path=args.path)
    clocks = ClockSampler(local)
    clocks.start()
    step_us, attn_us, step_call_us = time_steps(st, args.steps, args.warmup, world)
    kern_us = reduce_max(time_attention_launches(st, max(3, args.steps // 3)), world)
    clk = clocks.stop()
    mean_step = reduce_max(statistics.mean(step_us), world)
    mean_attn = reduce_max(statistics.mean(attn_us), world)
    bytes_, flops = algorithmic(cfg)
    t_mem = bytes_ / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    attn_s = kern_us * 1e-6
    bound = "tensor" if t_tc > t_mem else "hbm"
    if bound == "tensor":
        achieved, peak, unit = flops / attn_s / 1e12, tc_peak, "TFLOP/s"
    else:
        achieved, peak, unit = bytes_ / attn_s / 1e9, hbm_peak, "GB/s"
    e2e_us, h2d, d2h = time_e2e(st, max(5, args.steps // 2), 3)
    e2e_us = reduce_max(e2e_us, world)

    sweep = []
    if not args.no_sweep:
        for kk in (0, 4, 8, 16):
            c2 = workload(kk, args.prefix, rank)
            s2 = Step(c2, copies_for(c2), path=args.path)
            su, au, sc = time_steps(s2, max(10, args.steps // 2), 3, world)
            b2, f2 = algorithmic(c2)
            a2 = reduce_max(time_attention_launches(s2, 3), world) * 1e-6
            sweep.append({"k": kk, "rows": c2.R, "step_us": reduce_max(statistics.mean(su), world),
                          "step_call_us": reduce_max(statistics.mean(sc), world),
                          "attn_call_us": reduce_max(statistics.mean(au), world),
                          "attn_us": a2 * 1e6, "attn_hbm_gbs": b2 / a2 / 1e9,
                          "hbm_frac": (b2 / a2 / 1e9) / hbm_peak,
                          "tc_frac": (f2 / a2 / 1e12) / tc_peak,
                          "roofline_frac": max(b2 / (hbm_peak * 1e9), f2 / (tc_peak * 1e12)) / a2,
                          "path": PATH_NAMES[s2.path_id], "splits": s2.splits})
            del s2
            torch.cuda.empty_cache()

    extra = []
    if not args.no_configs:
        from ar_decoding_b200 import synth
        for c2 in (synth.serving(), synth.long_context(1, 32768, 0), synth.long_context(1, 32768, 16),
                   synth.long_context(4, 65536, 4), synth.long_context(4, 65536, 8),
                   synth.long_context(8, 131072, 0), synth.long_context(8, 131072, 16),
                   synth.class_1p5b(), synth.tiny()):
            s2 = Step(c2, copies_for(c2), path=args.path)
            su, au, _ = time_steps(s2, max(5, args.steps // 4), 3, world)
            a2 = reduce_max(time_attention_launches(s2, 2, statistics.mean(au)), world) * 1e-6
            b2, f2 = algorithmic(c2)
            extra.append({"workload": c2.name, "B": c2.B, "prefix_total": sum(c2.prefix),
                          "prefix_range": [min(c2.prefix), max(c2.prefix)], "k": c2.k,
                          "Hq": c2.Hq, "Hkv": c2.Hkv, "head_dim": c2.D, "dtype": c2.dtype,
                          "path": PATH_NAMES[s2.path_id], "splits": s2.splits,
                          "copies": len(s2.copies), "l2": l2_policy(c2),
                          "step_us": reduce_max(statistics.mean(su), world), "attn_us": a2 * 1e6,
                          "attn_hbm_gbs": b2 / a2 / 1e9, "attn_tflops": f2 / a2 / 1e12,
                          "hbm_frac": (b2 / a2 / 1e9) / hbm_peak, "tc_frac": (f2 / a2 / 1e12) / tc_peak,
                          "roofline_frac": max(b2 / (hbm_peak * 1e9), f2 / (tc_peak * 1e12)) / a2,
                          "bound": "tensor" if f2 / (tc_peak * 1e12) > b2 / (hbm_peak * 1e9) else "hbm"})
            del s2
            torch.cuda.empty_cache()

    layer = None
    if not args.no_layer:
        layer = layer_sweep(hbm_peak, tc_peak, world)

    loop = None
    if not args.no_loop:
        loop = {}
        for mode in ("greedy", "blockq"):
            lp = Loop(cfg, copies_for(cfg), args.loop_chain, path=args.path, mode=mode)
            lus, ltok = lp.time(max(3, args.steps // 6))
            lus = reduce_max(lus, world)
            nsteps = lp.chain * len(lp.copies)
            loop[mode] = {
                "workload": f"{cfg.name} decode loop",
                "verify": ("greedy" if mode == "greedy" else
                           "rejection, q read from the previous step's selected mask block"),
                "chained_steps": lp.chain, "interleaved_sequences": len(lp.copies),
                "us_per_step": lus, "launches_per_step": lp.launches_per_step,
                "committed_tokens_per_step": ltok / nsteps,
                "tokens_per_s_per_sequence": ltok / nsteps / (lus * 1e-6),
                "acceptance": ("planted: drafts match the next step's argmax up to a depth "
                               "uniform on 1..k" if mode == "greedy" else
                               "planted: q_i = p_i below a depth uniform on 1..k") +
                              " (synthetic, not a model's acceptance)",
                "path": PATH_NAMES[lp.path_id], "splits": lp.splits}
            del lp
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = oracle_threads()
        t = oracle_step_seconds(cfg, cores)
        cpu = {"value": t * 1e6, "unit": "us", "cores": cores, "kind": "oracle",
               "sample": f"one whole step of the same workload ({cfg.B * cfg.R * cfg.Hq} attention "
                         f"rows, append, verify, commit) on {cores} OpenMP threads"}

    agg_gbs = reduce_sum(bytes_ / attn_s / 1e9, world)
    if rank == 0:
        line = {
            "metric": METRIC, "value": mean_step, "unit": "us", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_step / 1e3,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, generated on device)",
            "config": bench_config(cfg, args.prefix, args.k),
            "attn_plan": {"path": PATH_NAMES[st.path_id], "splits": st.splits},
            "step_call_us": reduce_max(statistics.mean(step_call_us), world),
            "attn_call_us": mean_attn, "attn_us": kern_us, "attn_launches": st.attn_launches,
            "hbm_gbs_attn": bytes_ / attn_s / 1e9,
            "hbm_gbs_all_gpus": agg_gbs,
            "roofline": {"kernel": {2: "attn_tc05_kernel", 3: "attn_dec_kernel",
                                    4: "attn_pair_kernel"}.get(st.path_id, "tidar_step_attn"),
                         "bound": bound, "achieved": achieved,
                         "peak": peak, "unit": unit, "frac": achieved / peak,
                         "peak_source": peak_src, "peak_kind": "burst",
                         "traffic": measured_traffic(args.k, st.path_id),
                         "algorithmic_bytes": bytes_, "algorithmic_flops": flops,
                         "roofline_frac_max_of_both": max(t_mem, t_tc) / attn_s},
            "k_sweep": sweep,
            "extra_configs": extra,
            "layer_sweep": layer,
            "decode_loop": loop,
            "e2e": {"value": e2e_us, "unit": "us", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": st.launches_per_step * args.steps,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
