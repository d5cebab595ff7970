"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, then compare.

Tolerances (written in each test as these constants):
  fp32 attention:  max |delta| <= 1e-5 (and lse within 1e-5)
  bf16 attention:  max |delta| <= 2e-2, per-row relative L2 <= 1e-2, lse within 2e-3
Integer outputs (accept counts, tokens, selected blocks, committed cache bytes,
page tables, released ids) must match exactly.
"""
from __future__ import annotations

import numpy as np
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth

TOL_F32 = 1e-5
TOL_BF16_ABS = 2e-2
TOL_BF16_REL = 1e-2
TOL_LSE_F32 = 1e-5
TOL_LSE_BF16 = 2e-3


def to_dev(d: dict, dev="cuda"):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def run_attention(cfg: synth.StepConfig, path="auto", cache=None, step=None, max_prefix=None):
    """Returns (out, lse, cache_after) from the GPU (all moved to CPU)."""
    cache = cache if cache is not None else synth.make_cache(cfg)
    step = step if step is not None else synth.make_step(cfg)
    dc, ds = to_dev(cache), to_dev(step)
    mp = max_prefix if max_prefix is not None else max(cfg.prefix)
    out, lse = tidar.step_attn(ds["q"], ds["k_blk"], ds["v_blk"], dc, cfg.k, max_prefix_len=mp,
                               path=path)
    st, bits = tidar.device_status()
    assert st == tidar.OK, f"device status {st} bits {bits:#x}"
    return out.cpu(), lse.cpu(), {k: v.cpu() for k, v in dc.items()}


def oracle_attention(oracle_mod, cfg, cache, step, sel=None, threads=0):
    n = synth.to_np
    return oracle_mod.step_attn(n(step["q"]), n(step["k_blk"]), n(step["v_blk"]),
                                n(cache["k_pages"]), n(cache["v_pages"]), n(cache["page_table"]),
                                n(cache["seq_lens"]), cfg.k, sel=sel, num_threads=threads)


def compare_attention(cfg, got, want, got_lse, want_lse):
    """got [N][D] (torch, any float dtype), want [N][D] fp64 numpy."""
    g = got.double().numpy().reshape(-1, cfg.D)
    w = np.asarray(want).reshape(-1, cfg.D)
    gl = got_lse.double().numpy().reshape(-1)
    wl = np.asarray(want_lse).reshape(-1)
    err = np.abs(g - w)
    if cfg.dtype == "f32":
        assert err.max() <= TOL_F32, f"max |delta| {err.max():.3g} > {TOL_F32}"
        assert np.abs(gl - wl).max() <= TOL_LSE_F32, f"lse {np.abs(gl - wl).max():.3g}"
    else:
        assert err.max() <= TOL_BF16_ABS, f"max |delta| {err.max():.3g} > {TOL_BF16_ABS}"
        rel = np.linalg.norm(g - w, axis=1) / np.maximum(np.linalg.norm(w, axis=1), 1e-30)
        assert rel.max() <= TOL_BF16_REL, f"row rel L2 {rel.max():.3g} > {TOL_BF16_REL}"
        assert np.abs(gl - wl).max() <= TOL_LSE_BF16, f"lse {np.abs(gl - wl).max():.3g}"
    return float(err.max())


def sample_rows(cfg, count, seed=0):
    """(b, rho, h) triples covering draft rows, first/last slots of blocks, every head."""
    rng = np.random.default_rng(seed)
    R = cfg.R
    count = min(count, cfg.B * R * cfg.Hq)
    special = {0, R - 1, min(cfg.k, R - 1), max(cfg.k - 1, 0)}
    if cfg.k:
        for j in (1, 2, cfg.k):
            special |= {cfg.k + (j - 1) * cfg.k, min(cfg.k + j * cfg.k - 1, R - 1)}
    out = set()
    for b in range(cfg.B):
        for rho in special:
            out.add((b, rho, int(rng.integers(cfg.Hq))))
    for h in range(cfg.Hq):
        out.add((int(rng.integers(cfg.B)), int(rng.integers(R)), h))
    while len(out) < count:
        out.add((int(rng.integers(cfg.B)), int(rng.integers(R)), int(rng.integers(cfg.Hq))))
    return sorted(out)
