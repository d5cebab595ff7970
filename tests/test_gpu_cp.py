"""GPU parity of context-parallel step attention, through the C ABI: the
ranks of a context-parallel group are emulated one after another on one GPU
(no rank waits on another).  Each rank's slice of the cache
(ar_decoding_b200.cp.shard_cache) goes through tidar_step_attn_part -- the
last rank with the step keys and the draft-row append -- and the results are
merged by tidar_merge_attn; the merged output must match the oracle's
attention over the whole cache within the bf16 / fp32 attention tolerances,
and the draft rows must land in the last rank's slice exactly where the
oracle's append puts them in the whole cache.
"""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import cp, synth
from gpu_harness import compare_attention, oracle_attention, to_dev

pytestmark = pytest.mark.gpu


def _run(cfg, world, path="auto"):
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    ds = to_dev(step)
    outs, lses, locs = [], [], []
    for rank in range(world):
        loc = to_dev(cp.shard_cache(cache, world, rank, cfg.k))
        last = rank == world - 1
        flags = (tidar.PART_STEP_KEYS | tidar.PART_APPEND) if last else 0
        mp = max(1, int(loc["seq_lens"].max()))
        o, l = tidar.step_attn_part(ds["q"], ds["k_blk"], ds["v_blk"], loc, cfg.k, flags,
                                    max_prefix_len=mp, path=path)
        outs.append(o)
        lses.append(l)
        locs.append(loc)
    out, lse = tidar.merge_attn(torch.stack(outs), torch.stack(lses))
    st, bits = tidar.device_status()
    assert st == tidar.OK, f"device status {st} bits {bits:#x}"
    return cache, step, out.cpu(), lse.cpu(), locs[-1]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("path,cfg", [
    ("auto", synth.class_8b(k=16, prefix=8192)),
    ("auto", synth.class_8b(k=0, prefix=8192)),
    ("pair", synth.class_8b(k=8, prefix=4096)),
    ("auto", synth.StepConfig("cp-ragged", B=3, Hq=8, Hkv=2, D=128, k=4, prefix=(3000, 70, 1),
                              dtype="bf16", seed=71)),
    ("simt", synth.StepConfig("cp-f32", B=2, Hq=4, Hkv=2, D=64, k=4, prefix=(513, 64), dtype="f32",
                              seed=72)),
], ids=lambda x: x if isinstance(x, str) else x.name + f"-k{x.k}")
def test_context_parallel_matches_whole_cache(oracle_mod, world, path, cfg):
    cache, step, out, lse, last = _run(cfg, world, path)
    want, want_lse = oracle_attention(oracle_mod, cfg, cache, step)
    compare_attention(cfg, out, want, lse, want_lse)
    # the draft rows went into the last rank's slice at its rows P_local ..
    n = synth.to_np
    kp, vp = oracle_mod.append(n(cache["k_pages"]), n(cache["v_pages"]), n(cache["page_table"]),
                               n(cache["seq_lens"]), n(step["k_blk"]), n(step["v_blk"]), cfg.k)
    lk = n(last["k_pages"].cpu())
    for b, P in enumerate(cfg.prefix):
        Pl = int(last["seq_lens"][b])
        for r in range(cfg.n):
            gpage = int(cache["page_table"][b, (P + r) // cfg.page_size])
            lpage = int(last["page_table"][b, (Pl + r) // cfg.page_size].cpu())
            np.testing.assert_array_equal(lk[lpage, :, (Pl + r) % cfg.page_size],
                                          kp[gpage, :, (P + r) % cfg.page_size])


def test_prefix_only_on_an_empty_slice_gives_no_weight():
    cfg = synth.StepConfig("empty", B=1, Hq=8, Hkv=2, D=128, k=4, prefix=(0,), dtype="bf16", seed=73)
    cache, step = to_dev(synth.make_cache(cfg)), to_dev(synth.make_step(cfg))
    for path in ("tc05", "pair", "simt"):
        o, l = tidar.step_attn_part(step["q"], step["k_blk"], step["v_blk"], cache, cfg.k, 0,
                                    max_prefix_len=64, path=path)
        assert tidar.device_status() == (tidar.OK, 0)
        assert torch.isneginf(l).all() and (o.float() == 0).all(), path


def test_merge_attn_closed_forms():
    g = torch.Generator().manual_seed(4)
    o = torch.randn(3, 5, 128, generator=g).to(torch.bfloat16).cuda()
    l = torch.full((3, 5), 0.25).cuda()
    out, lse = tidar.merge_attn(o, l)
    want = o.float().mean(0)
    assert (out.float() - want).abs().max() <= 2e-2
    assert torch.allclose(lse, torch.full_like(lse, 0.25 + float(np.log(3.0))), atol=1e-6)
    l2 = torch.tensor([[-float("inf")] * 5, [1.0] * 5, [-float("inf")] * 5]).cuda()
    out2, _ = tidar.merge_attn(o, l2)
    assert torch.equal(out2, o[1])
