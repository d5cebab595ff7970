"""GPU parity of tidar_commit against the oracle (bit-exact cache bytes, page
tables, lengths, released ids and count), plus the serving-batch flow:
commit of the previous step's counts -> step attention -> verify -> commit."""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth
from gpu_harness import compare_attention, oracle_attention, sample_rows, to_dev

pytestmark = pytest.mark.gpu


def _gpu_commit(cache, acc, k, max_prefix):
    dc = to_dev(cache)
    rel, nrel = tidar.commit(dc, acc.cuda(), k, max_prefix_len=max_prefix)
    st, bits = tidar.device_status()
    return {k: v.cpu() for k, v in dc.items()}, rel.cpu().numpy(), int(nrel.cpu()[0]), st, bits


def _oracle_commit(oracle_mod, cache, acc, k):
    n = synth.to_np
    return oracle_mod.commit(n(cache["k_pages"]), n(cache["v_pages"]), n(cache["page_table"]),
                             n(cache["seq_lens"]), n(acc), k)


def _assert_same(got, rel, nrel, want):
    kp, vp, pt, sl, wrel, wn, _ = want
    n = synth.to_np
    np.testing.assert_array_equal(n(got["k_pages"]), kp)
    np.testing.assert_array_equal(n(got["v_pages"]), vp)
    np.testing.assert_array_equal(n(got["page_table"]), pt)
    np.testing.assert_array_equal(n(got["seq_lens"]), sl)
    assert nrel == wn
    np.testing.assert_array_equal(rel, wrel)


@pytest.mark.parametrize("k,ps,dtype", [(0, 64, "bf16"), (1, 16, "f32"), (4, 16, "bf16"),
                                        (8, 64, "bf16"), (16, 64, "bf16"), (16, 32, "f32")])
def test_commit_matches_oracle(oracle_mod, k, ps, dtype):
    B = 24
    g = torch.Generator().manual_seed(k * 10 + ps)
    prefix = tuple(int(x) for x in torch.randint(0, 300, (B,), generator=g))
    prefix = (ps - 1, 2 * ps, 0) + prefix[3:]            # boundary cases
    cfg = synth.StepConfig("c", B=B, Hq=8, Hkv=4, D=128 if dtype == "bf16" else 64, k=k,
                           prefix=prefix, dtype=dtype, page_size=ps, seed=k + ps)
    cache = synth.make_cache(cfg)
    acc = torch.randint(0, cfg.n + 1, (B,), generator=g, dtype=torch.int32)
    acc[0], acc[1], acc[2] = 0, cfg.n, 1
    got, rel, nrel, st, bits = _gpu_commit(cache, acc, k, max(prefix))
    assert st == tidar.OK, bits
    _assert_same(got, rel, nrel, _oracle_commit(oracle_mod, cache, acc, k))


@pytest.mark.parametrize("B,k,Hkv", [(1, 16, 3), (2, 8, 6), (5, 4, 3), (1, 2, 8), (1, 16, 5)])
def test_commit_zeroing_shapes(oracle_mod, B, k, Hkv):
    # rows of 2 * Hkv * 16 sixteen-byte pieces that do (Hkv 8) and do not
    # (Hkv 3, 6) divide the CTA's threads, with one CTA (up to 32 KB of rows
    # to zero) or a cluster sharing them
    g = torch.Generator().manual_seed(100 * B + 10 * k + Hkv)
    prefix = tuple(int(x) for x in torch.randint(0, 700, (B,), generator=g))
    cfg = synth.StepConfig("cz", B=B, Hq=2 * Hkv, Hkv=Hkv, D=128, k=k, prefix=prefix, dtype="bf16",
                           page_size=64, seed=B + k + Hkv)
    cache = synth.make_cache(cfg)
    acc = torch.randint(0, cfg.n + 1, (B,), generator=g, dtype=torch.int32)
    acc[0] = 0                                            # every draft row rejected
    got, rel, nrel, st, bits = _gpu_commit(cache, acc, k, max(prefix))
    assert st == tidar.OK, bits
    _assert_same(got, rel, nrel, _oracle_commit(oracle_mod, cache, acc, k))


def test_commit_bad_count_and_page_leave_sequence_untouched(oracle_mod):
    cfg = synth.StepConfig("cbad", B=4, Hq=2, Hkv=2, D=64, k=4, prefix=(10, 70, 5, 64),
                           dtype="f32", page_size=16, seed=4)
    cache = synth.make_cache(cfg)
    acc = torch.tensor([1, 9, 2, -1], dtype=torch.int32)
    got, rel, nrel, st, bits = _gpu_commit(cache, acc, cfg.k, 70)
    assert st == tidar.ERR_DEVICE and bits & tidar.DEVERR_BAD_COUNT
    want = _oracle_commit(oracle_mod, cache, acc, cfg.k)
    assert want[6] != 0
    _assert_same(got, rel, nrel, want)


def test_serving_flow(oracle_mod):
    """Serving batch: ragged prefixes, shuffled pages; the previous step's accept
    counts (uniform on 0..k) are committed first, then one full step."""
    cfg = synth.serving()
    cache = synth.make_cache(cfg, extra_pages=cfg.B)      # spare pages for the next step
    prev = synth.prev_accept_counts(cfg)
    max_prefix = max(cfg.prefix) + cfg.n                  # lengths grow by at most n
    # 1) commit the previous step's counts (its draft rows sit at P..P+n-1)
    got, rel, nrel, st, _ = _gpu_commit(cache, prev, cfg.k, max_prefix)
    assert st == tidar.OK
    want = _oracle_commit(oracle_mod, cache, prev, cfg.k)
    _assert_same(got, rel, nrel, want)
    # 2) reserve pages for this step's drafts (host allocator: the released ids first)
    pt = got["page_table"].clone()
    free = [int(x) for x in rel[:nrel]]
    used = set(int(x) for x in pt[pt >= 0])
    spare = [p for p in range(got["k_pages"].shape[0]) if p not in used and p not in free]
    pool = free + spare
    for b in range(cfg.B):
        P = int(got["seq_lens"][b])
        for i in range((P + cfg.page_size - 1) // cfg.page_size,
                       (P + cfg.n + cfg.page_size - 1) // cfg.page_size):
            if pt[b, i] < 0:
                pt[b, i] = pool.pop(0)
    cache2 = dict(got, page_table=pt)
    # 3) step attention on the committed state
    step = synth.make_step(cfg)
    dc, ds = to_dev(cache2), to_dev(step)
    out, lse = tidar.step_attn(ds["q"], ds["k_blk"], ds["v_blk"], dc, cfg.k, max_prefix_len=max_prefix)
    assert tidar.device_status()[0] == tidar.OK
    sel = sample_rows(cfg, 160, seed=5)
    w, wl = oracle_attention(oracle_mod, cfg, cache2, step, sel=sel)
    out, lse = out.cpu(), lse.cpu()
    compare_attention(cfg, torch.stack([out[b, r, h] for b, r, h in sel]), w,
                      torch.stack([lse[b, r, h] for b, r, h in sel]), wl)
    # 4) verify (greedy) and commit this step
    vin = synth.make_verify(cfg, "greedy")
    res = tidar.verify(vin["logits"].cuda(), vin["drafts"].cuda(), cfg.k, "greedy",
                       block_guesses=vin["block_guesses"].cuda())
    n = synth.to_np
    wv = oracle_mod.verify(n(vin["logits"]), n(vin["drafts"]), cfg.k, oracle_mod.GREEDY,
                           block_guesses=n(vin["block_guesses"]))
    np.testing.assert_array_equal(res["accept_count"].cpu().numpy(), wv["accept_count"])
    after_attn = {k2: v.cpu() for k2, v in dc.items()}
    kp_app, vp_app = oracle_mod.append(n(cache2["k_pages"]), n(cache2["v_pages"]),
                                       n(cache2["page_table"]), n(cache2["seq_lens"]),
                                       n(step["k_blk"]), n(step["v_blk"]), cfg.k)
    np.testing.assert_array_equal(n(after_attn["k_pages"]), kp_app)
    rel2, nrel2 = tidar.commit(dc, res["accept_count"], cfg.k, max_prefix_len=max_prefix)
    assert tidar.device_status()[0] == tidar.OK
    want2 = oracle_mod.commit(kp_app, vp_app, n(cache2["page_table"]), n(cache2["seq_lens"]),
                              wv["accept_count"], cfg.k)
    _assert_same({k2: v.cpu() for k2, v in dc.items()}, rel2.cpu().numpy(), int(nrel2.cpu()[0]),
                 want2)
