"""GPU parity of tidar_verify_commit (verification and the commit of its accept
counts in one call; greedy computes the acceptance inside the commit's launch)
against the oracle's verify then commit: verification outputs, cache bytes,
page tables, lengths, released ids and count, all exact.  Batches below and
above the commit cluster's CTA count take its two bookkeeping paths."""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth
from gpu_harness import to_dev

pytestmark = pytest.mark.gpu


def _run(oracle_mod, cfg, mode, seed):
    n = synth.to_np
    cache = synth.make_cache(cfg)
    vin = synth.make_verify(cfg, mode)
    m = oracle_mod.GREEDY if mode == "greedy" else oracle_mod.REJECTION
    want = oracle_mod.verify(n(vin["logits"]), n(vin["drafts"]) if cfg.k else None, cfg.k, m,
                             draft_logits=n(vin["draft_logits"]), uniforms=n(vin["uniforms"]),
                             block_guesses=n(vin["block_guesses"]) if cfg.k else None, with_margins=True)
    kp, vp, pt, sl, wrel, wn, _ = oracle_mod.commit(n(cache["k_pages"]), n(cache["v_pages"]),
                                                    n(cache["page_table"]), n(cache["seq_lens"]),
                                                    want["accept_count"], cfg.k)
    dc = to_dev(cache)
    d = lambda t: None if t is None else t.cuda()
    out, rel, nrel = tidar.verify_commit(d(vin["logits"]), d(vin["drafts"]), dc, cfg.k, mode,
                                         max_prefix_len=max(cfg.prefix), draft_logits=d(vin["draft_logits"]),
                                         uniforms=d(vin["uniforms"]), block_guesses=d(vin["block_guesses"]))
    st, bits = tidar.device_status()
    assert st == tidar.OK, bits
    skip = want["margins"].min(axis=1) < 1e-9 if mode == "rejection" else np.zeros(cfg.B, bool)
    assert skip.sum() == 0
    for key in ("accept_count", "out_tokens", "selected_block"):
        np.testing.assert_array_equal(out[key].cpu().numpy(), want[key], err_msg=key)
    if cfg.k:
        np.testing.assert_array_equal(out["next_drafts"].cpu().numpy()[:, :cfg.k], want["next_drafts"])
    np.testing.assert_array_equal(n(dc["k_pages"].cpu()), kp)
    np.testing.assert_array_equal(n(dc["v_pages"].cpu()), vp)
    np.testing.assert_array_equal(n(dc["page_table"].cpu()), pt)
    np.testing.assert_array_equal(n(dc["seq_lens"].cpu()), sl)
    assert int(nrel.cpu()[0]) == wn
    np.testing.assert_array_equal(rel.cpu().numpy(), wrel)


@pytest.mark.parametrize("mode", ["greedy", "rejection"])
@pytest.mark.parametrize("B,k", [(1, 16), (1, 0), (3, 4), (12, 8), (40, 2), (20, 16)])
def test_verify_commit_matches_oracle(oracle_mod, mode, B, k):
    g = torch.Generator().manual_seed(B * 31 + k)
    prefix = tuple(int(x) for x in torch.randint(0, 400, (B,), generator=g))
    cfg = synth.StepConfig("vc", B=B, Hq=8, Hkv=2, D=128, k=k, prefix=prefix, dtype="bf16",
                           vocab=4099 if B == 3 else 32768, seed=B + 7 * k)
    _run(oracle_mod, cfg, mode, B + k)


def test_verify_commit_8b_class_step(oracle_mod):
    # the headline step's verification and commit (B = 1, k = 16, vocab 32768)
    cfg = synth.class_8b(k=16)
    _run(oracle_mod, cfg, "greedy", 1)


def test_verify_commit_checks_before_launching():
    cfg = synth.StepConfig("vcbad", B=2, Hq=2, Hkv=2, D=64, k=4, prefix=(10, 20), dtype="f32",
                           vocab=64, seed=3)
    dc = to_dev(synth.make_cache(cfg))
    vin = synth.make_verify(cfg, "greedy")
    sl0 = dc["seq_lens"].clone()
    with pytest.raises((ValueError, tidar.TidarError)):   # logits of the wrong batch
        tidar.verify_commit(vin["logits"][:1].cuda(), vin["drafts"][:1].cuda(), dc, 4, "greedy",
                            max_prefix_len=20)
    with pytest.raises((ValueError, tidar.TidarError)):   # rejection without uniforms: nothing queued
        tidar.verify_commit(vin["logits"].cuda(), vin["drafts"].cuda(), dc, 4, "rejection",
                            max_prefix_len=20, draft_logits=vin["logits"][:, :3].contiguous().cuda())
    torch.cuda.synchronize()
    assert torch.equal(dc["seq_lens"], sl0)
