"""Pins for the oracle's context-parallel pieces (CPU only): attention over a
slice of the prefix without the step keys, and the log-sum-exp merge.

  * the merge against closed forms: one part is returned as is; two parts with
    equal lse average, with lse + log 2; a part with lse -inf is ignored; all
    -inf gives 0 and -inf;
  * prefix-only attention against dense attention over the prefix rows
    (numpy, fp64); an empty prefix gives 0 and -inf;
  * the partition property: the prefix of every sequence split by
    ar_decoding_b200.cp.shard_cache into 2..5 slices (the last with the step
    keys), each slice's attention merged, equals the oracle's attention over
    the whole cache -- so the slicing rule, the step keys' placement and the
    merge must all be right.
"""
import numpy as np
import pytest
import torch

from ar_decoding_b200 import cp, synth


def test_merge_closed_forms(oracle_mod):
    rng = np.random.default_rng(1)
    o = rng.standard_normal((1, 3, 8))
    l = rng.standard_normal((1, 3))
    out, lse = oracle_mod.merge(o, l)
    np.testing.assert_allclose(out, o[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, l[0], rtol=0, atol=1e-15)
    o2 = rng.standard_normal((2, 4, 8))
    l2 = np.full((2, 4), 0.7)
    out, lse = oracle_mod.merge(o2, l2)
    np.testing.assert_allclose(out, o2.mean(axis=0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, 0.7 + np.log(2.0), rtol=0, atol=1e-15)
    l3 = np.array([[-np.inf] * 4, [0.3] * 4])
    out, lse = oracle_mod.merge(o2, l3)
    np.testing.assert_allclose(out, o2[1], rtol=0, atol=1e-15)
    out, lse = oracle_mod.merge(o2, np.full((2, 4), -np.inf))
    assert (out == 0).all() and np.isneginf(lse).all()


def test_prefix_only_is_dense_attention_over_the_prefix(oracle_mod):
    cfg = synth.StepConfig("pfx", B=2, Hq=4, Hkv=2, D=64, k=3, prefix=(70, 0), dtype="f32", seed=3)
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    n = synth.to_np
    out, lse = oracle_mod.step_attn(n(step["q"]), n(step["k_blk"]), n(step["v_blk"]), n(cache["k_pages"]),
                                    n(cache["v_pages"]), n(cache["page_table"]), n(cache["seq_lens"]), cfg.k,
                                    step_keys=False)
    kp, vp, pt = n(cache["k_pages"]), n(cache["v_pages"]), n(cache["page_table"])
    q = n(step["q"]).astype(np.float64)
    P = 70
    K = np.stack([kp[pt[0, i // 64], :, i % 64] for i in range(P)]).astype(np.float64)   # [P][Hkv][D]
    V = np.stack([vp[pt[0, i // 64], :, i % 64] for i in range(P)]).astype(np.float64)
    for rho in range(cfg.R):
        for h in range(cfg.Hq):
            s = K[:, h // 2] @ q[0, rho, h] / np.sqrt(cfg.D)
            w = np.exp(s - s.max())
            np.testing.assert_allclose(out[0, rho, h], (w / w.sum()) @ V[:, h // 2], rtol=0, atol=1e-12)
            assert abs(lse[0, rho, h] - (s.max() + np.log(w.sum()))) < 1e-12
    assert (out[1] == 0).all() and np.isneginf(lse[1]).all()      # empty prefix


@pytest.mark.parametrize("world", [2, 3, 5])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_slices_merge_to_the_whole_attention(oracle_mod, world, dtype):
    cfg = synth.StepConfig("cp", B=3, Hq=4, Hkv=2, D=64 if dtype == "f32" else 128, k=4,
                           prefix=(300, 64, 5), dtype=dtype, seed=11 + world)
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    n = synth.to_np
    args = (n(step["q"]), n(step["k_blk"]), n(step["v_blk"]))
    want, want_lse = oracle_mod.step_attn(*args, n(cache["k_pages"]), n(cache["v_pages"]),
                                          n(cache["page_table"]), n(cache["seq_lens"]), cfg.k)
    parts, lses = [], []
    for rank in range(world):
        loc = cp.shard_cache(cache, world, rank, cfg.k)
        o, l = oracle_mod.step_attn(*args, n(loc["k_pages"]), n(loc["v_pages"]), n(loc["page_table"]),
                                    n(loc["seq_lens"]), cfg.k, step_keys=rank == world - 1)
        parts.append(o)
        lses.append(l)
    got, got_lse = oracle_mod.merge(np.stack(parts), np.stack(lses))
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_lse, want_lse, rtol=0, atol=1e-12)


def test_shard_cache_covers_the_prefix_once():
    cfg = synth.StepConfig("cov", B=4, Hq=2, Hkv=1, D=64, k=2, prefix=(0, 1, 130, 4096), dtype="f32", seed=5)
    cache = synth.make_cache(cfg)
    for world in (1, 2, 3, 8):
        lens = [cp.shard_cache(cache, world, r, cfg.k)["seq_lens"] for r in range(world)]
        np.testing.assert_array_equal(torch.stack(lens).sum(0).numpy(), np.array(cfg.prefix))
        last = cp.shard_cache(cache, world, world - 1, cfg.k)
        # the last rank holds the pages of the draft rows P_b .. P_b + n - 1
        for b, P in enumerate(cfg.prefix):
            Pl = int(last["seq_lens"][b])
            for r in range(cfg.n):
                assert int(last["page_table"][b, (Pl + r) // 64]) >= 0
