"""Seeded synthetic inputs for the TiDAR decode step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no attention, no softmax-based decision, no commit).  Both
the CUDA path's tests/benchmark and the CPU oracle's tests take their inputs
from here, so the two sides see identical bytes.

Workloads (sizes from the model classes the pages evaluate, 1.5B and 8B, and
from the serving / long-context settings of the hot path):

  tiny         B=1, 2 heads MHA, D=64, prefix 256, k=4, fp32 N(0,1); vocab 512 N(0,2)
  1.5B-class   B=1, 12 q / 2 kv heads, D=128, prefix 4096, k=8, bf16 N(0,1);
               vocab 32768 N(0,3)
  8B-class     B=1, 32 q / 8 kv heads, D=128, prefix 8192, k=16, bf16; vocab 32768
               N(0,3), each draft equal to the row argmax with probability 0.7
  serving      B=32, 8B-class heads, prefixes uniform on 512..16384, k=8, shuffled
               page ids, previous-step accept counts uniform on 0..k
  long         B in {1,4,8}, 8B-class heads, prefix in {32768,65536,131072},
               k in {0,4,8,16}

Every floating-point tensor is drawn in fp32 from a seeded torch.Generator and
rounded to the storage dtype; bf16 tensors are handed to the oracle as their
uint16 bit patterns.  Seeds are 0xD1A0 + workload index unless given.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SEED_BASE = 0xD1A0


@dataclass
class StepConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    k: int
    prefix: tuple            # P_b per sequence
    dtype: str = "bf16"      # "f32" or "bf16"
    page_size: int = 64
    vocab: int = 32768
    logit_std: float = 3.0
    mode: str = "greedy"     # "greedy" or "rejection"
    plant: float | None = None   # probability that a draft equals the row argmax
    shuffle_pages: bool = True
    seed: int = SEED_BASE
    q_scale: float = 1.0     # 8.0 gives the "peaked" variant (|O| of order 1)
    extra: dict = field(default_factory=dict)

    @property
    def R(self) -> int:
        return 1 if self.k == 0 else self.k + self.k * self.k

    @property
    def n(self) -> int:
        return max(self.k, 1)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


def tiny(seed: int = SEED_BASE + 0, mode: str = "greedy") -> StepConfig:
    return StepConfig("tiny", B=1, Hq=2, Hkv=2, D=64, k=4, prefix=(256,), dtype="f32",
                      vocab=512, logit_std=2.0, mode=mode, seed=seed)


def class_1p5b(seed: int = SEED_BASE + 1, k: int = 8) -> StepConfig:
    return StepConfig("1.5B-class", B=1, Hq=12, Hkv=2, D=128, k=k, prefix=(4096,),
                      vocab=32768, logit_std=3.0, seed=seed)


def class_8b(seed: int = SEED_BASE + 2, k: int = 16, prefix: int = 8192) -> StepConfig:
    return StepConfig("8B-class", B=1, Hq=32, Hkv=8, D=128, k=k, prefix=(prefix,),
                      vocab=32768, logit_std=3.0, plant=0.7, seed=seed)


def serving(seed: int = SEED_BASE + 3, B: int = 32, k: int = 8, lo: int = 512,
            hi: int = 16384) -> StepConfig:
    g = torch.Generator().manual_seed(seed)
    prefix = tuple(int(x) for x in torch.randint(lo, hi + 1, (B,), generator=g))
    return StepConfig("serving", B=B, Hq=32, Hkv=8, D=128, k=k, prefix=prefix, vocab=32768,
                      logit_std=3.0, seed=seed)


def long_context(B: int, P: int, k: int, seed: int = SEED_BASE + 4) -> StepConfig:
    return StepConfig(f"long-B{B}-P{P}-k{k}", B=B, Hq=32, Hkv=8, D=128, k=k,
                      prefix=tuple([P] * B), vocab=32768, logit_std=3.0, seed=seed)


def _randn(shape, gen, dtype, device="cpu", std=1.0):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def make_cache(cfg: StepConfig, device="cpu", extra_pages: int = 0, draft_pages: bool = True,
               max_pages: int | None = None):
    """Paged KV cache holding each prefix, with pages reserved for the n draft rows.

    Returns dict(k_pages, v_pages [num_pages][Hkv][page][D], page_table
    [B][max_pages] int32 (-1 = none), seq_lens [B] int32).  Page ids are a
    seeded permutation when cfg.shuffle_pages.  Rows past P_b inside reserved
    pages hold random values too (they are not part of the prefix).  With
    draft_pages=False only the pages holding prefix rows are mapped (the draft
    pages stay unmapped and their ids unused); max_pages widens the table.
    """
    gen = torch.Generator(device=device).manual_seed(cfg.seed * 7 + 1)
    ps = cfg.page_size
    need = [-(-(p + cfg.n) // ps) for p in cfg.prefix]
    num_pages = sum(need) + extra_pages
    width = max(need) + 1 if max_pages is None else max(max_pages, max(need))
    cpu_gen = torch.Generator().manual_seed(cfg.seed * 7 + 2)
    ids = (torch.randperm(num_pages, generator=cpu_gen) if cfg.shuffle_pages
           else torch.arange(num_pages)).to(torch.int32)
    table = torch.full((cfg.B, width), -1, dtype=torch.int32)
    pos = 0
    for b, cnt in enumerate(need):
        mapped = cnt if draft_pages else -(-cfg.prefix[b] // ps)
        table[b, :mapped] = ids[pos:pos + mapped]
        pos += cnt
    shape = (num_pages, cfg.Hkv, ps, cfg.D)
    k_pages = _randn(shape, gen, cfg.torch_dtype, device)
    v_pages = _randn(shape, gen, cfg.torch_dtype, device)
    return dict(k_pages=k_pages, v_pages=v_pages, page_table=table.to(device),
                seq_lens=torch.tensor(cfg.prefix, dtype=torch.int32, device=device))


def make_step(cfg: StepConfig, device="cpu"):
    """Query block and step K/V: q [B][R][Hq][D], k_blk/v_blk [B][R][Hkv][D]."""
    gen = torch.Generator(device=device).manual_seed(cfg.seed * 7 + 3)
    q = _randn((cfg.B, cfg.R, cfg.Hq, cfg.D), gen, cfg.torch_dtype, device, std=cfg.q_scale)
    k_blk = _randn((cfg.B, cfg.R, cfg.Hkv, cfg.D), gen, cfg.torch_dtype, device)
    v_blk = _randn((cfg.B, cfg.R, cfg.Hkv, cfg.D), gen, cfg.torch_dtype, device)
    return dict(q=q, k_blk=k_blk, v_blk=v_blk)


def make_verify(cfg: StepConfig, mode: str | None = None, seed_offset: int = 0):
    """Verification inputs on the CPU.

    logits [B][n][V] (dtype of cfg), drafts [B][k] int32, draft_logits
    [B][k-1][V] and uniforms [B][n] fp32 (rejection), block_guesses [B][k][k].
    Greedy drafts are uniform tokens, or (cfg.plant) the row's first maximal
    index with probability cfg.plant and otherwise a uniform other token.
    Rejection drafts d_{i+1} are drawn from the categorical distribution of
    draft_logits row i (as the acceptance rule assumes).
    """
    mode = mode or cfg.mode
    gen = torch.Generator().manual_seed(cfg.seed * 7 + 4 + 1000 * seed_offset)
    B, n, k, V = cfg.B, cfg.n, cfg.k, cfg.vocab
    logits = _randn((B, n, V), gen, cfg.torch_dtype, std=cfg.logit_std)
    drafts = torch.randint(0, V, (B, k), generator=gen, dtype=torch.int64)
    draft_logits = None
    uniforms = torch.rand((B, n), generator=gen, dtype=torch.float32)
    if mode == "rejection" and k > 1:
        draft_logits = _randn((B, k - 1, V), gen, cfg.torch_dtype, std=cfg.logit_std)
        probs = torch.softmax(draft_logits.float().double(), dim=-1)
        for i in range(k - 1):
            drafts[:, i + 1] = torch.multinomial(probs[:, i, :], 1, generator=gen)[:, 0]
    elif cfg.plant is not None and k > 1:
        top = torch.argmax(logits[:, : k - 1, :].float(), dim=-1)   # first maximal index
        hit = torch.rand((B, k - 1), generator=gen) < cfg.plant
        other = torch.randint(0, V - 1, (B, k - 1), generator=gen)
        other = other + (other >= top).long()                      # uniform over the rest
        drafts[:, 1:] = torch.where(hit, top, other)
    block_guesses = torch.randint(0, V, (B, k, k), generator=gen, dtype=torch.int64)
    return dict(logits=logits, drafts=drafts.to(torch.int32),
                draft_logits=draft_logits, uniforms=uniforms,
                block_guesses=block_guesses.to(torch.int32), mode=mode)


def make_pool(cfg: StepConfig, cache, capacity: int | None = None):
    """Stack of free pages: the ids the cache's page table does not use, in a
    seeded order.  Returns dict(free_pages [capacity] int32 (-1 past the
    count), free_count [1] int32); capacity defaults to the number of pages."""
    num_pages = cache["k_pages"].shape[0]
    pt = cache["page_table"].cpu()
    used = set(int(x) for x in pt[pt >= 0])
    free = torch.tensor([p for p in range(num_pages) if p not in used], dtype=torch.int32)
    perm = torch.randperm(free.numel(), generator=torch.Generator().manual_seed(cfg.seed * 7 + 6))
    cap = num_pages if capacity is None else capacity
    arr = torch.full((cap,), -1, dtype=torch.int32)
    arr[:free.numel()] = free[perm]
    return dict(free_pages=arr, free_count=torch.tensor([free.numel()], dtype=torch.int32))


def random_pool_state(seed: int):
    """A random page-reservation problem (numpy): returns dict(table [B][cols],
    lens [B], free [capacity], count, returned (or None), k, ps, num_pages,
    max_prefix).  Prefix pages are mapped, some draft pages already are, the
    stack may be short, and with probability 0.3 one sequence is made invalid
    (length past max_prefix, or its prefix page unmapped / out of range)."""
    rng = np.random.default_rng(seed)
    k = int(rng.choice([0, 1, 3, 8, 16]))
    ps = int(rng.choice([16, 32, 64, 128]))
    B = int(rng.integers(1, 12))
    max_prefix = int(rng.integers(0, 400))
    n = max(k, 1)
    cols = -(-(max_prefix + n) // ps) + int(rng.integers(0, 3))
    num_pages = B * cols + 8
    lens = rng.integers(0, max_prefix + 1, B).astype(np.int32)
    ids = rng.permutation(num_pages).astype(np.int32)
    table = np.full((B, cols), -1, np.int32)
    pos = 0
    for b in range(B):
        for i in range(-(-(int(lens[b]) + n) // ps)):
            if i * ps < lens[b] or rng.random() < 0.3:       # prefix pages, some draft pages
                table[b, i] = ids[pos]
                pos += 1
    cap = int(rng.integers(0, 3 * B + 4))
    count = int(rng.integers(0, cap + 1))
    free = np.full(cap, -1, np.int32)
    free[:count] = rng.integers(0, num_pages, count)
    returned = None
    if rng.random() < 0.6:
        returned = rng.integers(0, num_pages, int(rng.integers(0, 2 * B + 2))).astype(np.int32)
    if rng.random() < 0.3:
        b = int(rng.integers(B))
        if rng.random() < 0.5:
            lens[b] = max_prefix + 1 + int(rng.integers(3))
        elif lens[b] % ps:
            table[b, int(lens[b]) // ps] = -1
        else:
            table[b, int(lens[b]) // ps] = num_pages + 5
    return dict(table=table, lens=lens, free=free, count=count, returned=returned, k=k, ps=ps,
                num_pages=num_pages, max_prefix=max_prefix)


def make_block_logits(cfg: StepConfig, seed_offset: int = 0, plant_from=None):
    """Mask-block logits of a step, [B][k][k][V] (block j-1, slot s-1), N(0,
    logit_std) in cfg's dtype, and draft_block [B] int32 uniform on 1..k.

    With plant_from (the logits [B][k][V] of the step that will read these
    blocks as its q), rows (any block, slot i+1) for i below a seeded depth in
    1..k are copies of plant_from row i-1, so q_i = p_i there and those drafts
    are accepted whatever they are."""
    gen = torch.Generator().manual_seed(cfg.seed * 7 + 8 + 1000 * seed_offset)
    B, k, V = cfg.B, cfg.k, cfg.vocab
    bl = _randn((B, k, k, V), gen, cfg.torch_dtype, std=cfg.logit_std)
    blk = torch.randint(1, k + 1, (B,), generator=gen, dtype=torch.int32) if k else \
        torch.zeros(B, dtype=torch.int32)
    if plant_from is not None and k > 1:
        depth = torch.randint(1, k + 1, (B,), generator=gen)
        for b in range(B):
            for i in range(1, int(depth[b])):
                bl[b, :, i] = plant_from[b, i - 1]
    return bl, blk


def make_loop(cfg: StepConfig, steps: int, mode: str = "greedy"):
    """Inputs of `steps` chained steps (CPU tensors).

    Returns (attn, ver): attn[s] = make_step of a per-step seed; ver[s] =
    make_verify(mode, seed_offset=s+1), whose drafts matter only at s = 0
    (later steps inherit t*, g_{j,2..k} from the step before).  Greedy: the
    block guesses of step s are set so that the drafts step s+1 inherits equal
    the row argmaxes (first maximal index) of step s+1's logits up to a seeded
    depth in 1..k.  Rejection: the draft-logit rows of step s below a seeded
    depth are copies of the matching logit rows (q_i = p_i, so those drafts are
    accepted whatever they are).  Either way accept counts spread over 1..k.
    "blockq": rejection where step s+1 draws its q from step s's mask-block
    logits (ver[s]["block_logits"], planted from step s+1's logits as in
    make_block_logits) through step s's selected block; step 0 uses
    ver[0]["draft_logits"].
    """
    attn = [make_step(StepConfig(**{**cfg.__dict__, "seed": cfg.seed + 101 * (s + 1)}))
            for s in range(steps)]
    vmode = "rejection" if mode == "blockq" else mode
    ver = [make_verify(cfg, vmode, seed_offset=s + 1) for s in range(steps)]
    gen = torch.Generator().manual_seed(cfg.seed * 7 + 7)
    k = cfg.k
    if mode == "blockq":
        for s in range(steps):
            nxt = ver[s + 1]["logits"] if s + 1 < steps else None
            ver[s]["block_logits"] = make_block_logits(cfg, seed_offset=s + 1, plant_from=nxt)[0]
        mode = "rejection"
    if mode == "rejection":
        for s in range(steps):
            if k < 2:
                break
            depth = torch.randint(1, k + 1, (cfg.B,), generator=gen)
            dl = ver[s]["draft_logits"].clone()
            for b in range(cfg.B):
                for i in range(1, int(depth[b])):
                    dl[b, i - 1] = ver[s]["logits"][b, i - 1]
            ver[s]["draft_logits"] = dl
        return attn, ver
    for s in range(steps - 1):
        if k < 2:
            break
        top = torch.argmax(ver[s + 1]["logits"][:, : k - 1, :].float(), dim=-1)   # [B][k-1]
        depth = torch.randint(1, k + 1, (cfg.B,), generator=gen)
        g = ver[s]["block_guesses"].clone()
        for b in range(cfg.B):
            for m in range(1, int(depth[b])):
                g[b, :, m] = top[b, m - 1]
        ver[s]["block_guesses"] = g
    return attn, ver


D_MODEL = {"tiny": 128, "1.5B-class": 1536, "8B-class": 4096}


def make_layer(cfg: StepConfig, d_model: int | None = None, device="cpu"):
    """Inputs of the layer-level step: the step rows' hidden states x
    [B][R][d_model] ~ N(0,1), the projection weights w_qkv [(Hq + 2 Hkv) D]
    [d_model] ~ N(0, 1/d_model) (queries, then keys, then values; unit-variance
    q, k, v) and w_o [d_model][Hq D] ~ N(0, 1/(Hq D)); bf16, random (no
    trained weights).  d_model defaults to the model class's hidden size
    (4096 for 8B-class heads, 1536 for 1.5B-class)."""
    dm = d_model if d_model is not None else D_MODEL.get(cfg.name, 4096)
    gen = torch.Generator(device=device).manual_seed(cfg.seed * 7 + 11)
    N = (cfg.Hq + 2 * cfg.Hkv) * cfg.D
    x = _randn((cfg.B, cfg.R, dm), gen, torch.bfloat16, device)
    w_qkv = _randn((N, dm), gen, torch.bfloat16, device, std=dm ** -0.5)
    w_o = _randn((dm, cfg.Hq * cfg.D), gen, torch.bfloat16, device, std=(cfg.Hq * cfg.D) ** -0.5)
    return dict(x=x, w_qkv=w_qkv, w_o=w_o, d_model=dm)


def prev_accept_counts(cfg: StepConfig) -> torch.Tensor:
    """Previous-step accept counts, uniform on 0..k (serving workload)."""
    gen = torch.Generator().manual_seed(cfg.seed * 7 + 5)
    return torch.randint(0, cfg.k + 1, (cfg.B,), generator=gen, dtype=torch.int32)


def to_np(t: torch.Tensor | None):
    """CPU numpy view for the oracle: bf16 -> uint16 bit patterns."""
    if t is None:
        return None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
