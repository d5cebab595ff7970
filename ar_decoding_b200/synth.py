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


def make_cache(cfg: StepConfig, device="cpu", extra_pages: int = 0):
    """Paged KV cache holding each prefix, with pages reserved for the n draft rows.

    Returns dict(k_pages, v_pages [num_pages][Hkv][page][D], page_table
    [B][max_pages] int32 (-1 = none), seq_lens [B] int32).  Page ids are a
    seeded permutation when cfg.shuffle_pages.  Rows past P_b inside reserved
    pages hold random values too (they are not part of the prefix).
    """
    gen = torch.Generator(device=device).manual_seed(cfg.seed * 7 + 1)
    ps = cfg.page_size
    need = [-(-(p + cfg.n) // ps) for p in cfg.prefix]
    num_pages = sum(need) + extra_pages
    max_pages = max(need) + 1
    cpu_gen = torch.Generator().manual_seed(cfg.seed * 7 + 2)
    ids = (torch.randperm(num_pages, generator=cpu_gen) if cfg.shuffle_pages
           else torch.arange(num_pages)).to(torch.int32)
    table = torch.full((cfg.B, max_pages), -1, dtype=torch.int32)
    pos = 0
    for b, cnt in enumerate(need):
        table[b, :cnt] = ids[pos:pos + cnt]
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
