"""GPU parity of tidar_step_attn against the oracle, through the C ABI.

Full element-by-element comparison wherever the oracle finishes in seconds --
which includes the full 8B-class workload at every k of the sweep and the
32-sequence serving batch (one oracle run per workload, shared by the kernel
paths); only the long-context prefixes (32768 and up) compare a seeded sample
of (b, row, head) triples covering every zone and head.  The draft-row append is compared
bit-exactly on the whole cache.
"""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth
from gpu_harness import (compare_attention, oracle_attention, run_attention, sample_rows, to_dev)

pytestmark = pytest.mark.gpu

PATHS = ["simt", "tc05", "dec", "pair"]


def _tc05_ok(cfg):
    return cfg.dtype == "bf16" and cfg.D == 128 and cfg.page_size == 64


def _dec_ok(cfg):
    return _tc05_ok(cfg) and cfg.R * (cfg.Hq // cfg.Hkv) <= 16


def _supported(cfg, path):
    # the tensor-core kernel takes bf16, head_dim 128, page 64; the warp-MMA
    # decode kernel in addition at most 16 packed query rows per KV head
    return {"tc05": _tc05_ok, "pair": _tc05_ok, "dec": _dec_ok}.get(path, lambda c: True)(cfg)


def _check_full(oracle_mod, cfg, path):
    if not _supported(cfg, path):
        return
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    out, lse, cache_after = run_attention(cfg, path, cache, step)
    want, want_lse = oracle_attention(oracle_mod, cfg, cache, step)
    compare_attention(cfg, out, want, lse, want_lse)
    # the draft rows' K/V land in cache rows P_b .. P_b+n-1, nothing else changes
    n = synth.to_np
    kp, vp = oracle_mod.append(n(cache["k_pages"]), n(cache["v_pages"]), n(cache["page_table"]),
                               n(cache["seq_lens"]), n(step["k_blk"]), n(step["v_blk"]), cfg.k)
    np.testing.assert_array_equal(n(cache_after["k_pages"]), kp)
    np.testing.assert_array_equal(n(cache_after["v_pages"]), vp)


def test_tiny_fp32(oracle_mod):
    _check_full(oracle_mod, synth.tiny(), "simt")
    _check_full(oracle_mod, synth.tiny(), "auto")


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("P", [0, 1, 63, 64, 65, 130, 257])
@pytest.mark.parametrize("k", [0, 1, 2, 4])
def test_edges_prefix_and_k(oracle_mod, path, P, k):
    for dtype, D in (("f32", 64), ("bf16", 128)):
        cfg = synth.StepConfig("edge", B=2, Hq=4, Hkv=2, D=D, k=k, prefix=(P, max(P - 7, 0)),
                               dtype=dtype, seed=100 + P + 10 * k)
        _check_full(oracle_mod, cfg, path)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("k", [3, 8, 16])
@pytest.mark.parametrize("heads", [(1, 1), (4, 1), (6, 1), (8, 2), (32, 8)])
def test_heads_and_k(oracle_mod, path, k, heads):
    Hq, Hkv = heads
    cfg = synth.StepConfig("heads", B=1, Hq=Hq, Hkv=Hkv, D=128, k=k, prefix=(200,),
                           dtype="bf16", seed=7 + k + Hq)
    _check_full(oracle_mod, cfg, path)


@pytest.mark.parametrize("path", PATHS)
def test_peaked_queries(oracle_mod, path):
    # |O| of order one: q scaled by 8 concentrates each softmax on few keys
    cfg = synth.StepConfig("peaked", B=2, Hq=8, Hkv=2, D=128, k=4, prefix=(300, 77),
                           dtype="bf16", q_scale=8.0, seed=31)
    _check_full(oracle_mod, cfg, path)
    cfg32 = synth.StepConfig("peaked32", B=1, Hq=2, Hkv=2, D=64, k=4, prefix=(256,),
                             dtype="f32", q_scale=8.0, seed=32)
    _check_full(oracle_mod, cfg32, path)


@pytest.mark.parametrize("path", PATHS)
def test_1p5b_class_full(oracle_mod, path):
    _check_full(oracle_mod, synth.class_1p5b(), path)


def _check_sampled(oracle_mod, cfg, path, count, max_prefix=None):
    if not _supported(cfg, path):
        return
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    out, lse, _ = run_attention(cfg, path, cache, step, max_prefix=max_prefix)
    sel = sample_rows(cfg, count)
    want, want_lse = oracle_attention(oracle_mod, cfg, cache, step, sel=sel)
    got = torch.stack([out[b, r, h] for b, r, h in sel])
    got_lse = torch.stack([lse[b, r, h] for b, r, h in sel])
    compare_attention(cfg, got, want, got_lse, want_lse)


# The oracle's answer for a full-size workload, computed once per session and
# shared by the kernel paths that are compared against it.
_FULL_ORACLE = {}


def _full_oracle(oracle_mod, cfg):
    key = (cfg.name, cfg.seed, cfg.k, cfg.B, tuple(cfg.prefix))
    if key not in _FULL_ORACLE:
        cache, step = synth.make_cache(cfg), synth.make_step(cfg)
        want, want_lse = oracle_attention(oracle_mod, cfg, cache, step)
        n = synth.to_np
        kp, vp = oracle_mod.append(n(cache["k_pages"]), n(cache["v_pages"]), n(cache["page_table"]),
                                   n(cache["seq_lens"]), n(step["k_blk"]), n(step["v_blk"]), cfg.k)
        _FULL_ORACLE.clear()                # one full-size answer held at a time
        _FULL_ORACLE[key] = (cache, step, want, want_lse, kp, vp)
    return _FULL_ORACLE[key]


def _check_full_cached(oracle_mod, cfg, path, max_prefix=None):
    """Every output row, every lse and the whole cache after the append, at the
    full size of the workload, against one oracle run shared by the paths."""
    if not _supported(cfg, path):
        return
    cache, step, want, want_lse, kp, vp = _full_oracle(oracle_mod, cfg)
    out, lse, cache_after = run_attention(cfg, path, cache, step, max_prefix=max_prefix)
    compare_attention(cfg, out, want, lse, want_lse)
    n = synth.to_np
    np.testing.assert_array_equal(n(cache_after["k_pages"]), kp)
    np.testing.assert_array_equal(n(cache_after["v_pages"]), vp)


@pytest.mark.parametrize("path", PATHS + ["auto"])
@pytest.mark.parametrize("k", [4, 8, 16])
def test_8b_class_k_sweep_full(oracle_mod, k, path):
    # the headline workload (32 q / 8 kv heads, prefix 8192) at every k of the
    # sweep: all B*R*Hq output rows, lse and the appended cache rows
    _check_full_cached(oracle_mod, synth.class_8b(k=k), path)


class _ForcedPartials:
    """Tensor-core key splits merged through workspace partials (second launch)."""
    def __enter__(self):
        tidar.debug_set(tidar.DEBUG_FORCE_SPLIT_PARTIALS, 1)

    def __exit__(self, *exc):
        tidar.debug_set(tidar.DEBUG_FORCE_SPLIT_PARTIALS, 0)


@pytest.mark.parametrize("path", ["tc05", "dec", "pair"])
@pytest.mark.parametrize("merge", ["auto", "partials"])
def test_8b_class_k0_full_every_split_merged(oracle_mod, merge, path):
    # k = 0: one query row per head, the prefix cut into many splits; every
    # output row and the appended cache row are compared
    cfg = synth.class_8b(k=0)
    d = tidar.make_desc(torch.empty(1, 1, 32, 128, dtype=torch.bfloat16, device="cuda"),
                        torch.empty(1, 1, 8, 128, dtype=torch.bfloat16, device="cuda"),
                        to_dev(synth.make_cache(cfg)), 0, max(cfg.prefix), path=path)
    if merge == "partials":
        with _ForcedPartials():
            assert tidar.plan(d)[1] > 8 and tidar.step_attn_workspace_bytes(d) > 0
            _check_full(oracle_mod, cfg, path)
    else:
        assert tidar.plan(d)[1] > 1
        _check_full(oracle_mod, cfg, path)


@pytest.mark.parametrize("path", PATHS + ["dec-partials"])
def test_decode_splits_past_a_short_sequence(oracle_mod, path):
    # plain decode (k = 0), sequence 1 far shorter than sequence 0: most of its
    # splits hold no prefix key; unaligned prefix ends inside a page
    cfg = synth.StepConfig("ragged-decode", B=3, Hq=8, Hkv=2, D=128, k=0, prefix=(5000, 130, 1),
                           dtype="bf16", seed=58)
    if path == "dec-partials":
        with _ForcedPartials():
            _check_full(oracle_mod, cfg, "dec")
    else:
        _check_full(oracle_mod, cfg, path)


def test_auto_picks_the_decode_kernel_for_thin_blocks():
    q = lambda R, Hq: torch.empty(1, R, Hq, 128, dtype=torch.bfloat16, device="cuda")
    kb = lambda R, Hkv: torch.empty(1, R, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    cache = to_dev(synth.make_cache(synth.class_8b(k=0)))
    assert tidar.plan(tidar.make_desc(q(1, 32), kb(1, 8), cache, 0, 8192))[0] == tidar.PATH_DEC
    cache16 = to_dev(synth.make_cache(synth.class_8b(k=16)))
    assert tidar.plan(tidar.make_desc(q(272, 32), kb(272, 8), cache16, 16, 8192))[0] == tidar.PATH_TC05


@pytest.mark.parametrize("path", PATHS + ["tc05-partials", "pair-partials"])
def test_splits_past_a_short_sequence(oracle_mod, path):
    # sequence 1 is far shorter than sequence 0: most of its key splits hold no
    # prefix key and contribute an empty partial to the merge
    cfg = synth.StepConfig("ragged-splits", B=2, Hq=8, Hkv=2, D=128, k=4, prefix=(4096, 300),
                           dtype="bf16", seed=57)
    if path.endswith("-partials"):
        with _ForcedPartials():
            _check_full(oracle_mod, cfg, path.split("-")[0])
    else:
        _check_full(oracle_mod, cfg, path)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("B,P,k", [(1, 32768, 16), (4, 32768, 4), (1, 131072, 0)])
def test_long_context_sampled(oracle_mod, path, B, P, k):
    _check_sampled(oracle_mod, synth.long_context(B, P, k), path, 120)


@pytest.mark.parametrize("path", PATHS + ["auto"])
def test_serving_full(oracle_mod, path):
    # 32 sequences with ragged prefixes 512..16384 on shuffled pages, k = 8:
    # every output row, lse and the appended cache rows
    cfg = synth.serving()
    _check_full_cached(oracle_mod, cfg, path, max_prefix=max(cfg.prefix))


def test_step_attn_reports_bad_page_without_fault(oracle_mod):
    cfg = synth.StepConfig("bad", B=1, Hq=2, Hkv=2, D=64, k=2, prefix=(100,), dtype="f32")
    cache, step = to_dev(synth.make_cache(cfg)), to_dev(synth.make_step(cfg))
    cache["page_table"][0, 0] = -1
    tidar.step_attn(step["q"], step["k_blk"], step["v_blk"], cache, cfg.k, max_prefix_len=100)
    st, bits = tidar.device_status()
    assert st == tidar.ERR_DEVICE and bits & tidar.DEVERR_BAD_PAGE
    assert tidar.device_status() == (tidar.OK, 0)      # the word was cleared


def test_step_attn_reports_bad_length():
    cfg = synth.StepConfig("len", B=1, Hq=2, Hkv=2, D=64, k=2, prefix=(100,), dtype="f32")
    cache, step = to_dev(synth.make_cache(cfg)), to_dev(synth.make_step(cfg))
    tidar.step_attn(step["q"], step["k_blk"], step["v_blk"], cache, cfg.k, max_prefix_len=50)
    st, bits = tidar.device_status()
    assert st == tidar.ERR_DEVICE and bits & tidar.DEVERR_BAD_LEN


def test_attention_wait_timeout_is_reported_and_recovered(oracle_mod):
    # failure injected on the host: the producer issues no copies, so the
    # kernel's bounded waits run out (~1 s); the call must report a timeout,
    # and the same context must then compute a correct step
    cfg = synth.StepConfig("starve", B=1, Hq=4, Hkv=1, D=128, k=2, prefix=(256,), dtype="bf16",
                           seed=61)
    cache, step = to_dev(synth.make_cache(cfg)), to_dev(synth.make_step(cfg))
    tidar.debug_set(tidar.DEBUG_STARVE_ATTENTION_LOADS, 1)
    try:
        tidar.step_attn(step["q"], step["k_blk"], step["v_blk"], cache, cfg.k, max_prefix_len=256,
                        path="tc05")
    finally:
        tidar.debug_set(tidar.DEBUG_STARVE_ATTENTION_LOADS, 0)
    st, bits = tidar.device_status()
    assert st == tidar.ERR_TIMEOUT and bits & tidar.DEVERR_TIMEOUT
    _check_full(oracle_mod, cfg, "tc05")
