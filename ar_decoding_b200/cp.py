"""Context parallelism: one long sequence's step attention over several GPUs.

The settled prefix of each sequence is split by pages into `world` contiguous
slices, one per rank.  Softmax attention over a union of disjoint key sets is
the log-sum-exp mixture of the attention over each set, so every rank attends
its slice, the last rank -- which holds the sequence's tail pages and the
pages reserved for the draft rows -- also attends the step keys (the zone
mask) and appends the drafts' K/V, and the ranks exchange their (out, lse)
and merge them.  The exchange is one all-gather per step of
world x [B][R][Hq][D] outputs and [B][R][Hq] lse (about 2.2 MB at the
8B-class k = 16 step), over NCCL on GPUs.

The pages do not describe this split (they describe one standalone model on
one device); it is this library's way of running the same step when one
sequence's cache outgrows a GPU.

  local = shard_cache(cache, world, rank, k)          # host-side bookkeeping
  out, lse = step_attn(q, k_blk, v_blk, local, k, world=world, rank=rank,
                       max_prefix_len=..., group=group)

Argument marshalling and plumbing only: the attention and the merge run in the
library's kernels (tidar_step_attn_part, tidar_merge_attn).
"""
from __future__ import annotations

import torch

import ar_decoding_b200 as tidar


def slice_rows(P: int, world: int, rank: int, page_size: int) -> tuple[int, int]:
    """Rows [lo, hi) of a prefix of P rows held by `rank`: the prefix's pages
    split into `world` contiguous runs as evenly as possible (rank r takes pages
    [r p / world, (r+1) p / world), rounded down).  The last rank's run always
    ends at the last prefix page, so it holds the page of row P when P is not
    page-aligned; ranks may hold no rows when there are fewer pages than ranks."""
    pages = -(-P // page_size)
    lo = min(P, (rank * pages // world) * page_size)
    hi = min(P, ((rank + 1) * pages // world) * page_size)
    return lo, hi


def shard_cache(cache: dict, world: int, rank: int, k: int) -> dict:
    """This rank's local cache: the pages of its slice of every sequence's
    prefix (and, on the last rank, the pages reserved for the draft rows),
    renumbered locally.  seq_lens of the local cache = the slice lengths."""
    kp, vp = cache["k_pages"], cache["v_pages"]
    table, lens = cache["page_table"].cpu(), cache["seq_lens"].cpu()
    B = lens.shape[0]
    ps = kp.shape[2]
    n = max(k, 1)
    last = rank == world - 1
    ids, rows, width = [], [], 1
    for b in range(B):
        P = int(lens[b])
        lo, hi = slice_rows(P, world, rank, ps)
        p0 = (rank * (-(-P // ps)) // world)               # first page of the run
        p1 = -(-(P + n) // ps) if last else -(-hi // ps)    # the last rank also holds the draft pages
        pages = [int(x) for x in table[b, p0:p1]] if p1 > p0 else []
        ids.append(pages)
        rows.append(hi - lo)
        width = max(width, len(pages) + 1)
    flat = [p for pages in ids for p in pages]
    sel = torch.tensor(flat if flat else [0], dtype=torch.long, device=kp.device)
    lk, lv = kp.index_select(0, sel).contiguous(), vp.index_select(0, sel).contiguous()
    lt = torch.full((B, width), -1, dtype=torch.int32)
    pos = 0
    for b, pages in enumerate(ids):
        lt[b, : len(pages)] = torch.arange(pos, pos + len(pages), dtype=torch.int32)
        pos += len(pages)
    return dict(k_pages=lk, v_pages=lv, page_table=lt.to(kp.device),
                seq_lens=torch.tensor(rows, dtype=torch.int32, device=kp.device))


def gather_merge(out: torch.Tensor, lse: torch.Tensor, merge_fn, group=None):
    """All-gather every rank's (out, lse) in rank order and merge them with
    merge_fn(parts_out [world][...], parts_lse [world][...])."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    po = [torch.empty_like(out) for _ in range(world)]
    pl = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(po, out.contiguous(), group=group)
    dist.all_gather(pl, lse.contiguous(), group=group)
    return merge_fn(torch.stack(po), torch.stack(pl))


def step_attn(q, k_blk, v_blk, local_cache, k, *, world, rank, max_prefix_len, group=None,
              path="auto"):
    """The step attention of sequences whose prefixes are sharded over `world`
    ranks (this rank holds `local_cache` = shard_cache(..., rank)).  Returns
    the merged (out, lse), identical on every rank.  max_prefix_len bounds the
    local slice lengths."""
    last = rank == world - 1
    flags = (tidar.PART_STEP_KEYS | tidar.PART_APPEND) if last else 0
    out, lse = tidar.step_attn_part(q, k_blk, v_blk, local_cache, k, flags,
                                    max_prefix_len=max_prefix_len, path=path)
    return gather_merge(out, lse, tidar.merge_attn, group=group)
