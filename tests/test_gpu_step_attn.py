"""GPU parity of tidar_step_attn against the oracle, through the C ABI.

Full element-by-element comparison where the oracle finishes in seconds; at the
full 8B-class / serving / long-context sizes, a seeded sample of (b, row, head)
triples covering every zone and head.  The draft-row append is compared
bit-exactly on the whole cache.
"""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth
from gpu_harness import (compare_attention, oracle_attention, run_attention, sample_rows, to_dev)

pytestmark = pytest.mark.gpu

PATHS = ["simt", "tc05"]


def _tc05_ok(cfg):
    return cfg.dtype == "bf16" and cfg.D == 128 and cfg.page_size == 64


def _check_full(oracle_mod, cfg, path):
    if path == "tc05" and not _tc05_ok(cfg):
        return                      # the tensor-core kernel takes bf16, head_dim 128 only
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
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    out, lse, _ = run_attention(cfg, path, cache, step, max_prefix=max_prefix)
    sel = sample_rows(cfg, count)
    want, want_lse = oracle_attention(oracle_mod, cfg, cache, step, sel=sel)
    got = torch.stack([out[b, r, h] for b, r, h in sel])
    got_lse = torch.stack([lse[b, r, h] for b, r, h in sel])
    compare_attention(cfg, got, want, got_lse, want_lse)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("k", [0, 4, 8, 16])
def test_8b_class_k_sweep_sampled(oracle_mod, path, k):
    _check_sampled(oracle_mod, synth.class_8b(k=k), path, 160)


@pytest.mark.parametrize("path", PATHS)
def test_serving_ragged_sampled(oracle_mod, path):
    cfg = synth.serving()
    _check_sampled(oracle_mod, cfg, path, 200, max_prefix=max(cfg.prefix))


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
