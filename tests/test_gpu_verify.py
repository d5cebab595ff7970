"""GPU parity of tidar_verify (greedy and rejection) against the oracle: accept
counts, emitted tokens, selected blocks and next drafts must match exactly.

Rejection decisions are taken in fp64 on both sides; a decision whose oracle
margin (relative distance to its threshold) is below 1e-9 could differ by
summation order alone and is excluded -- the tests assert that this happens at
most once per 1e5 decisions (it is expected never to happen).
"""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth

pytestmark = pytest.mark.gpu

MARGIN = 1e-9


def _gpu_verify(cfg, vin, mode):
    d = lambda t: None if t is None else t.cuda()
    res = tidar.verify(d(vin["logits"]), d(vin["drafts"]) if cfg.k else None, cfg.k, mode,
                       draft_logits=d(vin["draft_logits"]), uniforms=d(vin["uniforms"]),
                       block_guesses=d(vin["block_guesses"]) if cfg.k else None)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in res.items()}


def _oracle_verify(oracle_mod, cfg, vin, mode):
    n = synth.to_np
    return oracle_mod.verify(n(vin["logits"]), n(vin["drafts"]) if cfg.k else None, cfg.k,
                             oracle_mod.GREEDY if mode == "greedy" else oracle_mod.REJECTION,
                             draft_logits=n(vin["draft_logits"]), uniforms=n(vin["uniforms"]),
                             block_guesses=n(vin["block_guesses"]) if cfg.k else None,
                             with_margins=True)


def _compare(cfg, got, want, mode):
    keep = np.ones(cfg.B, bool)
    if mode == "rejection":
        keep = (want["margins"] > MARGIN).all(axis=1)
        assert (~keep).sum() <= max(1, cfg.B * cfg.n // 100_000)
    np.testing.assert_array_equal(got["accept_count"][keep], want["accept_count"][keep])
    np.testing.assert_array_equal(got["out_tokens"][keep], want["out_tokens"][keep])
    np.testing.assert_array_equal(got["selected_block"][keep], want["selected_block"][keep])
    if cfg.k:
        np.testing.assert_array_equal(got["next_drafts"][keep][:, :cfg.k], want["next_drafts"][keep])


@pytest.mark.parametrize("mode", ["greedy", "rejection"])
@pytest.mark.parametrize("k", [0, 1, 2, 4, 8, 16])
@pytest.mark.parametrize("dtype,V", [("f32", 512), ("bf16", 32768), ("f32", 1000), ("bf16", 333)])
def test_verify_matches_oracle(oracle_mod, mode, k, dtype, V):
    cfg = synth.StepConfig("v", B=48, Hq=1, Hkv=1, D=64, k=k, prefix=(0,) * 48, dtype=dtype,
                           vocab=V, logit_std=2.0 if dtype == "f32" else 3.0,
                           plant=0.7 if mode == "greedy" else None, seed=500 + k + V)
    vin = synth.make_verify(cfg, mode)
    _compare(cfg, _gpu_verify(cfg, vin, mode), _oracle_verify(oracle_mod, cfg, vin, mode), mode)


@pytest.mark.parametrize("mode", ["greedy", "rejection"])
def test_verify_tiny_config(oracle_mod, mode):
    cfg = synth.tiny(mode=mode)
    for off in range(20):
        vin = synth.make_verify(cfg, mode, seed_offset=off)
        _compare(cfg, _gpu_verify(cfg, vin, mode), _oracle_verify(oracle_mod, cfg, vin, mode), mode)


def test_verify_8b_planted(oracle_mod):
    cfg = synth.class_8b()
    vin = synth.make_verify(cfg, "greedy")
    _compare(cfg, _gpu_verify(cfg, vin, "greedy"), _oracle_verify(oracle_mod, cfg, vin, "greedy"),
             "greedy")


def test_verify_argmax_ties_lowest_index(oracle_mod):
    # logits quantised to 4 levels: every row has many exact ties at its maximum
    cfg = synth.StepConfig("ties", B=32, Hq=1, Hkv=1, D=64, k=8, prefix=(0,) * 32, dtype="bf16",
                           vocab=32768, seed=77)
    vin = synth.make_verify(cfg, "greedy")
    vin["logits"] = torch.round(vin["logits"].float().clamp(-1.5, 1.5)).to(torch.bfloat16)
    first = torch.argmax(vin["logits"].float(), dim=-1)          # first maximal index
    hit = torch.rand(cfg.B, cfg.k - 1, generator=torch.Generator().manual_seed(1)) < 0.8
    vin["drafts"][:, 1:] = torch.where(hit, first[:, :-1], first[:, :-1] + 1).to(torch.int32)
    _compare(cfg, _gpu_verify(cfg, vin, "greedy"), _oracle_verify(oracle_mod, cfg, vin, "greedy"),
             "greedy")


def test_verify_rejection_large_batch_margins(oracle_mod):
    cfg = synth.StepConfig("rej", B=512, Hq=1, Hkv=1, D=64, k=4, prefix=(0,) * 512, dtype="f32",
                           vocab=512, logit_std=1.0, seed=91)
    vin = synth.make_verify(cfg, "rejection")
    _compare(cfg, _gpu_verify(cfg, vin, "rejection"),
             _oracle_verify(oracle_mod, cfg, vin, "rejection"), "rejection")


def test_verify_out_of_range_drafts_rejected(oracle_mod):
    cfg = synth.StepConfig("oor", B=8, Hq=1, Hkv=1, D=64, k=4, prefix=(0,) * 8, dtype="f32",
                           vocab=512, seed=3)
    for mode in ("greedy", "rejection"):
        vin = synth.make_verify(cfg, mode)
        vin["drafts"][:, 2] = torch.tensor([-1, 512, 10**6, -5, 0, 511, 3, 9], dtype=torch.int32)
        _compare(cfg, _gpu_verify(cfg, vin, mode), _oracle_verify(oracle_mod, cfg, vin, mode), mode)


@pytest.mark.parametrize("k", [1, 2, 4, 16])
@pytest.mark.parametrize("dtype,V", [("f32", 512), ("bf16", 32768), ("bf16", 333)])
def test_verify_blockq_matches_oracle(oracle_mod, k, dtype, V):
    """q read in place from the previous step's mask blocks through draft_block."""
    cfg = synth.StepConfig("vbq", B=40, Hq=1, Hkv=1, D=64, k=k, prefix=(0,) * 40, dtype=dtype,
                           vocab=V, logit_std=2.0 if dtype == "f32" else 3.0, seed=700 + k + V)
    vin = synth.make_verify(cfg, "rejection")
    bl, blk = synth.make_block_logits(cfg, plant_from=vin["logits"])
    d = lambda t: t.cuda()
    res = tidar.verify_blockq(d(vin["logits"]), d(vin["drafts"]) if k else None, k,
                              d(bl) if k > 1 else None, d(blk) if k > 1 else None,
                              d(vin["uniforms"]), block_guesses=d(vin["block_guesses"]) if k else None)
    st, bits = tidar.device_status()
    assert st == tidar.OK, bits
    got = {key: v.cpu().numpy() for key, v in res.items()}
    n = synth.to_np
    dl = oracle_mod.gather_block_q(n(bl), n(blk), k)[0] if k > 1 else None
    want = oracle_mod.verify(n(vin["logits"]), n(vin["drafts"]) if k else None, k,
                             oracle_mod.REJECTION, draft_logits=dl, uniforms=n(vin["uniforms"]),
                             block_guesses=n(vin["block_guesses"]) if k else None,
                             with_margins=True)
    _compare(cfg, got, want, "rejection")
    if k > 1:
        assert len(set(int(x) for x in want["accept_count"])) >= 2


def test_verify_blockq_bad_block_reads_block_one(oracle_mod):
    k, V = 4, 512
    cfg = synth.StepConfig("vbq-bad", B=6, Hq=1, Hkv=1, D=64, k=k, prefix=(0,) * 6, dtype="f32",
                           vocab=V, logit_std=2.0, seed=733)
    vin = synth.make_verify(cfg, "rejection")
    bl, blk = synth.make_block_logits(cfg, plant_from=vin["logits"])
    blk[1], blk[4] = 0, k + 1
    res = tidar.verify_blockq(vin["logits"].cuda(), vin["drafts"].cuda(), k, bl.cuda(), blk.cuda(),
                              vin["uniforms"].cuda(), block_guesses=vin["block_guesses"].cuda())
    st, bits = tidar.device_status()
    assert st == tidar.ERR_DEVICE and bits == tidar.DEVERR_BAD_COUNT
    n = synth.to_np
    dl, flags = oracle_mod.gather_block_q(n(bl), n(blk), k)
    assert flags == oracle_mod.GATHER_FLAG_BLOCK
    want = oracle_mod.verify(n(vin["logits"]), n(vin["drafts"]), k, oracle_mod.REJECTION,
                             draft_logits=dl, uniforms=n(vin["uniforms"]),
                             block_guesses=n(vin["block_guesses"]), with_margins=True)
    _compare(cfg, {key: v.cpu().numpy() for key, v in res.items()}, want, "rejection")


@pytest.mark.parametrize("V,dtype", [(69632, "bf16"), (70001, "f32")])
def test_verify_rejection_vocab_past_one_cluster(oracle_mod, V, dtype):
    """More 4096-wide chunks than a cluster holds: the residual sums and the
    inverse CDF take two launches through the workspace instead of the cluster."""
    cfg = synth.StepConfig("vwide", B=6, Hq=1, Hkv=1, D=64, k=4, prefix=(0,) * 6, dtype=dtype,
                           vocab=V, logit_std=3.0, seed=900 + V)
    vin = synth.make_verify(cfg, "rejection")
    _compare(cfg, _gpu_verify(cfg, vin, "rejection"),
             _oracle_verify(oracle_mod, cfg, vin, "rejection"), "rejection")
