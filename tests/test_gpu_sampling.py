"""GPU parity of verification under the sampling transform (temperature,
nucleus top_p) and of the draft sampling from the selected mask block
(tidar_verify_sampled, tidar_sample_drafts), through the C ABI, against the
oracle (oracle.verify_sampled, oracle.sample_drafts).

Every output is an integer (accept counts, tokens, selected blocks, next
drafts), so the comparison is exact.  Floating point decides those integers;
both sides decide in fp64 but sum in different orders, so decisions closer to a
boundary than 1e-9 (relative) -- which summation order alone could flip -- are
excluded, counted, and required to be rare (none expected with these seeds).
"""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth

pytestmark = pytest.mark.gpu

MARGIN = 1e-9


def _bits(x, dtype):
    if dtype == "bf16":
        t = torch.from_numpy(x).to(torch.bfloat16)
        return t, synth.to_np(t)
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32))
    return t, t.numpy()


def _inputs(seed, B, k, V, dtype, std=2.0):
    rng = np.random.default_rng(seed)
    n = max(k, 1)
    lg = (rng.standard_normal((B, n, V)) * std).astype(np.float32)
    # draft rows near the AR rows so that truncated supports overlap
    dl = (lg[:, : max(k - 1, 0)] + 0.7 * rng.standard_normal((B, max(k - 1, 0), V))).astype(np.float32)
    drafts = rng.integers(0, V, (B, max(k, 1))).astype(np.int32)[:, :k]
    if k > 1:
        top = np.argmax(dl, axis=-1)                     # always kept by any truncation
        hit = rng.random((B, k - 1)) < 0.6
        drafts[:, 1:] = np.where(hit, top, drafts[:, 1:])
    u = rng.random((B, n), dtype=np.float32)
    g = rng.integers(0, V, (B, k, k)).astype(np.int32)
    return lg, dl, drafts, u, g


def _compare(got, want, k, skip):
    for key in ("accept_count", "out_tokens", "selected_block"):
        g = got[key].cpu().numpy()
        np.testing.assert_array_equal(g[~skip], want[key][~skip], err_msg=key)
    if k:
        g = got["next_drafts"].cpu().numpy()[:, :k]
        np.testing.assert_array_equal(g[~skip], want["next_drafts"][~skip])


def _skip_mask(want):
    return (want["margins"].min(axis=1) < MARGIN) | (want["cut_margins"] < MARGIN)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("B,k,V", [(64, 4, 512), (16, 8, 32768), (4, 16, 32768), (32, 0, 1000),
                                   (32, 1, 1000), (8, 3, 70001)])
@pytest.mark.parametrize("T,top_p", [(0.7, 0.9), (1.3, 1.0), (1.0, 0.5), (0.4, 0.97)])
def test_verify_sampled_matches_oracle(oracle_mod, dtype, B, k, V, T, top_p):
    lg, dl, drafts, u, g = _inputs(1000 * k + V + int(T * 10), B, k, V, dtype)
    tl, nl = _bits(lg, dtype)
    tdl, ndl = _bits(dl, dtype)
    want = oracle_mod.verify_sampled(nl, drafts if k else None, k, oracle_mod.REJECTION,
                                     temperature=T, top_p=top_p, draft_logits=ndl if k > 1 else None,
                                     uniforms=u, block_guesses=g if k else None)
    got = tidar.verify_sampled(tl.cuda(), torch.from_numpy(drafts).cuda() if k else None, k,
                               "rejection", temperature=T, top_p=top_p,
                               draft_logits=tdl.cuda() if k > 1 else None,
                               uniforms=torch.from_numpy(u).cuda(),
                               block_guesses=torch.from_numpy(g).cuda() if k else None)
    assert tidar.device_status() == (tidar.OK, 0)
    skip = _skip_mask(want)
    assert skip.sum() <= max(1, B // 100_000)
    _compare(got, want, k, skip)


@pytest.mark.parametrize("k,V,dtype", [(4, 4096, "f32"), (16, 32768, "bf16")])
def test_verify_sampled_blockq_matches_oracle(oracle_mod, k, V, dtype):
    # q read in place from the previous step's mask blocks through draft_block
    rng = np.random.default_rng(k + V)
    B, T, tp = 6, 0.8, 0.92
    lg, _, drafts, u, g = _inputs(7 + k, B, k, V, dtype)
    bl = (rng.standard_normal((B, k, k, V)) * 2).astype(np.float32)
    blk = rng.integers(1, k + 1, B).astype(np.int32)
    for b in range(B):                                   # plant agreement in the block read
        bl[b, blk[b] - 1, 1:] = lg[b, : k - 1] + 0.5 * rng.standard_normal((k - 1, V))
        drafts[b, 1:] = np.argmax(bl[b, blk[b] - 1, 1:], axis=-1)
    tl, nl = _bits(lg, dtype)
    tbl, nbl = _bits(bl, dtype)
    ndl, flags = oracle_mod.gather_block_q(nbl, blk, k)
    assert flags == 0
    want = oracle_mod.verify_sampled(nl, drafts, k, oracle_mod.REJECTION, temperature=T, top_p=tp,
                                     draft_logits=ndl, uniforms=u, block_guesses=g)
    got = tidar.verify_sampled(tl.cuda(), torch.from_numpy(drafts).cuda(), k, "rejection",
                               temperature=T, top_p=tp, prev_block_logits=tbl.cuda(),
                               draft_block=torch.from_numpy(blk).cuda(),
                               uniforms=torch.from_numpy(u).cuda(), block_guesses=torch.from_numpy(g).cuda())
    assert tidar.device_status() == (tidar.OK, 0)
    _compare(got, want, k, _skip_mask(want))


def test_verify_sampled_greedy_is_verify(oracle_mod):
    cfg = synth.class_8b(k=16)
    vin = synth.make_verify(cfg, "greedy")
    d = {k2: v.cuda() for k2, v in vin.items() if isinstance(v, torch.Tensor)}
    a = tidar.verify(d["logits"], d["drafts"], 16, "greedy", block_guesses=d["block_guesses"])
    b = tidar.verify_sampled(d["logits"], d["drafts"], 16, "greedy", temperature=0.3, top_p=0.2,
                             block_guesses=d["block_guesses"])
    for key in a:
        assert torch.equal(a[key], b[key]), key


def test_untransformed_sampled_path_equals_tidar_verify():
    # T = 1, top_p = 1 through the sampled kernels vs the rejection kernels of
    # tidar_verify on the same inputs: two independent GPU paths, one rule
    cfg = synth.StepConfig("rej", B=24, Hq=8, Hkv=8, D=64, k=8, prefix=(0,) * 24, dtype="bf16",
                           vocab=32768, seed=55)
    vin = synth.make_verify(cfg, "rejection")
    d = {k2: v.cuda() for k2, v in vin.items() if isinstance(v, torch.Tensor)}
    a = tidar.verify(d["logits"], d["drafts"], 8, "rejection", draft_logits=d["draft_logits"],
                     uniforms=d["uniforms"], block_guesses=d["block_guesses"])
    b = tidar.verify_sampled(d["logits"], d["drafts"], 8, "rejection", draft_logits=d["draft_logits"],
                             uniforms=d["uniforms"], block_guesses=d["block_guesses"])
    for key in a:
        assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("mode", ["greedy", "rejection"])
@pytest.mark.parametrize("B,k,V,dtype", [(5, 4, 1000, "f32"), (3, 16, 32768, "bf16"), (64, 2, 512, "bf16")])
@pytest.mark.parametrize("T,top_p", [(1.0, 1.0), (0.6, 0.8)])
def test_sample_drafts_matches_oracle(oracle_mod, mode, B, k, V, dtype, T, top_p):
    rng = np.random.default_rng(B * k + V)
    bl = (rng.standard_normal((B, k, k, V)) * 2).astype(np.float32)
    sel = rng.integers(1, k + 1, B).astype(np.int32)
    u = rng.random((B, k), dtype=np.float32)
    prev = rng.integers(0, V, (B, k)).astype(np.int32)
    tbl, nbl = _bits(bl, dtype)
    m = oracle_mod.GREEDY if mode == "greedy" else oracle_mod.REJECTION
    want, marg, st = oracle_mod.sample_drafts(nbl, sel, k, m, temperature=T, top_p=top_p, uniforms=u,
                                              next_drafts=prev)
    assert st == 0
    nd = torch.from_numpy(prev.copy()).cuda()
    tidar.sample_drafts(tbl.cuda(), torch.from_numpy(sel).cuda(), k, mode, temperature=T, top_p=top_p,
                        uniforms=torch.from_numpy(u).cuda(), next_drafts=nd)
    assert tidar.device_status() == (tidar.OK, 0)
    got = nd.cpu().numpy()
    ok = marg >= MARGIN
    assert (~ok).sum() <= 1
    np.testing.assert_array_equal(got[ok], want[ok])
    np.testing.assert_array_equal(got[:, 0], prev[:, 0])        # t* untouched


def test_sample_drafts_bad_block_reads_block_one_and_reports(oracle_mod):
    rng = np.random.default_rng(3)
    B, k, V = 3, 4, 300
    bl = (rng.standard_normal((B, k, k, V)) * 2).astype(np.float32)
    sel = np.array([0, 2, 9], np.int32)
    want, _, st = oracle_mod.sample_drafts(bl, sel, k, oracle_mod.GREEDY)
    assert st == 3
    nd = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    tidar.sample_drafts(torch.from_numpy(bl).cuda(), torch.from_numpy(sel).cuda(), k, "greedy",
                        next_drafts=nd)
    st2, bits = tidar.device_status()
    assert st2 == tidar.ERR_DEVICE and bits & tidar.DEVERR_BAD_COUNT
    np.testing.assert_array_equal(nd.cpu().numpy()[:, 1:], want[:, 1:])


def test_sampling_arguments_are_checked():
    x = torch.zeros(1, 2, 64, device="cuda")
    with pytest.raises(tidar.TidarError):
        tidar.verify_sampled(x, torch.zeros(1, 2, dtype=torch.int32, device="cuda"), 2, "rejection",
                             temperature=0.0, draft_logits=x[:, :1].contiguous(),
                             uniforms=torch.zeros(1, 2, device="cuda"))
    with pytest.raises(tidar.TidarError):
        tidar.sample_drafts(torch.zeros(1, 2, 2, 64, device="cuda"),
                            torch.ones(1, dtype=torch.int32, device="cuda"), 2, "rejection",
                            top_p=0.0, uniforms=torch.zeros(1, 2, device="cuda"))
