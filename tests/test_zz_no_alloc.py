"""tidar_verify_noalloc: verification for callers that cannot allocate device
memory when they verify (for example while a decode loop is being captured into
a CUDA graph, or from a runtime that can only pass tensors it already owns).

The entry point uses the library's fixed device scratch instead of a caller
workspace.  These tests call it through the C ABI and check, on two calls in a
row, that it returns exactly what tidar_verify (with a workspace) returns on
the same inputs -- accept counts, tokens, selected blocks and next drafts are
integers, so the comparison is exact -- and that a call needing more scratch
than the fixed array is refused before any launch.  The file is named so that
pytest collects it after every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(cfg, mode, seed_offset):
    vin = synth.make_verify(cfg, mode, seed_offset=seed_offset)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in vin.items()}
    return d


def _call_both(cfg, mode, vin):
    kw = dict(draft_logits=vin["draft_logits"], uniforms=vin["uniforms"],
              block_guesses=vin["block_guesses"] if cfg.k else None)
    drafts = vin["drafts"] if cfg.k else None
    ref = tidar.verify(vin["logits"], drafts, cfg.k, mode, **kw)
    got = tidar.verify_noalloc(vin["logits"], drafts, cfg.k, mode, **kw)
    torch.cuda.synchronize()
    return ({k: v.cpu().numpy() for k, v in ref.items()},
            {k: v.cpu().numpy() for k, v in got.items()})


@pytest.mark.parametrize("mode", ["greedy", "rejection"])
@pytest.mark.parametrize("cfg", [synth.tiny(), synth.class_8b(),
                                 synth.StepConfig("b32", B=32, Hq=8, Hkv=8, D=64, k=8,
                                                  prefix=(0,) * 32, dtype="bf16", vocab=32768,
                                                  seed=41),
                                 synth.StepConfig("k0", B=4, Hq=2, Hkv=2, D=64, k=0,
                                                  prefix=(0,) * 4, dtype="f32", vocab=1000,
                                                  seed=42)],
                         ids=lambda c: c.name)
def test_noalloc_matches_verify_twice(cfg, mode):
    for call in range(2):                      # the second call sees the first call's scratch
        vin = _inputs(cfg, mode, seed_offset=call)
        ref, got = _call_both(cfg, mode, vin)
        np.testing.assert_array_equal(got["accept_count"], ref["accept_count"])
        np.testing.assert_array_equal(got["out_tokens"], ref["out_tokens"])
        np.testing.assert_array_equal(got["selected_block"], ref["selected_block"])
        if cfg.k:
            np.testing.assert_array_equal(got["next_drafts"][:, :cfg.k], ref["next_drafts"][:, :cfg.k])
    assert tidar.device_status() == (tidar.OK, 0)


def test_noalloc_refuses_oversized_calls():
    # 4096 sequences x 31 rows x 64 chunks of statistics do not fit the fixed scratch
    B, k, V = 4096, 16, 262144
    need = tidar.verify_workspace_bytes(B, k, V, tidar.REJECTION)
    assert need > tidar.VERIFY_NOALLOC_MAX_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)       # never dereferenced: refused before any launch
    st = tidar.lib().tidar_verify_noalloc(B, k, V, tidar.BF16, tidar.REJECTION, fake, fake, fake,
                                          fake, None, fake, fake, None, None, None)
    assert st == tidar.ERR_UNSUPPORTED
