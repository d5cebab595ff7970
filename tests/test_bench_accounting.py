"""The benchmark's roofline arithmetic, pinned on CPU against definitions that
do not come from bench.py:

  * the visible step keys summed over a sequence's rows (the per-unit flop
    count behind roofline.achieved) against the oracle's mask predicate,
    counted key by key for every k;
  * the algorithmic bytes and flops of small configurations against a
    brute-force count from the workload's shapes.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ar_decoding_b200 import synth  # noqa: E402


@pytest.mark.parametrize("k", list(range(0, 17)))
def test_step_key_count_matches_mask_predicate(oracle_mod, k):
    R = synth.StepConfig("c", B=1, Hq=1, Hkv=1, D=64, k=k, prefix=(0,)).R
    brute = sum(oracle_mod.step_key_visible(k, row, key) for row in range(R) for key in range(R))
    assert bench.step_key_counts(k) == brute


@pytest.mark.parametrize("k,prefix,dtype", [(0, (5,), "f32"), (3, (7, 0, 64), "bf16"),
                                            (16, (8192,), "bf16")])
def test_algorithmic_bytes_and_flops(oracle_mod, k, prefix, dtype):
    cfg = synth.StepConfig("c", B=len(prefix), Hq=8, Hkv=2, D=128, k=k, prefix=prefix, dtype=dtype)
    e = 4 if dtype == "f32" else 2
    R, n = cfg.R, cfg.n
    # bytes: every cached prefix key of every KV head (K and V) once, Q in and
    # O out, the step K/V in, the appended draft rows out
    want_bytes = 0
    for P in prefix:
        want_bytes += P * cfg.Hkv * cfg.D * 2 * e
        want_bytes += 2 * R * cfg.Hq * cfg.D * e
        want_bytes += R * cfg.Hkv * cfg.D * 2 * e
        want_bytes += n * cfg.Hkv * cfg.D * 2 * e
    # flops: 2*D for q.k and 2*D for p*v per (row, head, visible key)
    want_flops = 0
    for P in prefix:
        for row in range(R):
            vis = P + sum(oracle_mod.step_key_visible(k, row, key) for key in range(R))
            want_flops += 4 * cfg.D * cfg.Hq * vis
    got_bytes, got_flops = bench.algorithmic(cfg)
    assert got_bytes == want_bytes
    assert got_flops == want_flops
