"""Pins for the oracle's step attention (CPU only).

Each test checks the oracle against something other than itself:
  * the hand-written mask tables in tests/golden (from the pages' zone text);
  * k = 0 against torch's scaled_dot_product_attention in fp64 (a library
    routine) -- the step is ordinary decode attention;
  * every draft row against dense causal attention over the explicitly
    concatenated keys [prefix, D_1..D_r] (numpy, fp64);
  * every mask-slot block against a separate dense, unmasked attention over
    [prefix, D_1..D_j, M_{j,1..k}];
  * closed forms (one visible key, equal scores), invariances (page order, GQA
    head mapping) and the exact bf16 widening.
"""
import numpy as np
import pytest
import torch

from conftest import read_golden
from ar_decoding_b200 import synth


def _golden_masks():
    lines = read_golden("mask_k3.txt") + read_golden("mask_k1_k0.txt")
    tables, cur, k = {}, None, None
    for ln in lines:
        if ln.startswith("k "):
            k = int(ln.split()[1])
            cur = tables.setdefault(k, [])
        else:
            cur.append([int(x) for x in ln.split()])
    return {k: np.array(v, dtype=bool) for k, v in tables.items()}


def test_mask_matches_hand_tables(oracle_mod):
    for k, table in _golden_masks().items():
        R = oracle_mod.rows_per_seq(k)
        assert table.shape == (R, R)
        got = np.array([[oracle_mod.step_key_visible(k, r, c) for c in range(R)] for r in range(R)])
        np.testing.assert_array_equal(got, table, err_msg=f"k={k}")


def _zone_sets(k):
    """Visible step keys per row, built from zone membership as sets."""
    drafts = list(range(k))
    blocks = [list(range(k + j * k, k + (j + 1) * k)) for j in range(k)]
    rows = []
    for r in range(k):
        rows.append(set(drafts[: r + 1]))            # causal over the carried drafts
    for j in range(k):
        for _ in range(k):
            rows.append(set(drafts[: j + 1]) | set(blocks[j]))   # future j+1 survives
    return rows if k else [{0}]


@pytest.mark.parametrize("k", [0, 1, 2, 3, 4, 5, 8, 16])
def test_mask_zone_sets(oracle_mod, k):
    sets = _zone_sets(k)
    R = oracle_mod.rows_per_seq(k)
    for r in range(R):
        got = {c for c in range(R) if oracle_mod.step_key_visible(k, r, c)}
        assert got == sets[r], (k, r)


def _gather_prefix(kp, vp, table, b, g, P, ps):
    """Prefix keys/values of sequence b, KV head g, in position order (fp64)."""
    K = np.stack([kp[table[b, i // ps], g, i % ps] for i in range(P)]).astype(np.float64) if P else np.zeros((0, kp.shape[-1]))
    V = np.stack([vp[table[b, i // ps], g, i % ps] for i in range(P)]).astype(np.float64) if P else np.zeros((0, kp.shape[-1]))
    return K, V


def _dense_attention(qv, K, V, scale):
    s = (K @ qv) * scale
    w = np.exp(s - s.max())
    return (w[:, None] * V).sum(0) / w.sum()


def _small_cfg(k, P=(70,), Hq=4, Hkv=2, D=16, dtype="f32", seed=5):
    return synth.StepConfig("t", B=len(P), Hq=Hq, Hkv=Hkv, D=D, k=k, prefix=tuple(P),
                            dtype=dtype, page_size=16, seed=seed)


def _inputs(cfg):
    c = synth.make_cache(cfg)
    s = synth.make_step(cfg)
    return {key: synth.to_np(v) for key, v in {**c, **s}.items()}


@pytest.mark.parametrize("k,P", [(1, (0, 33)), (2, (17,)), (3, (64, 5)), (4, (100,))])
def test_rows_equal_dense_attention_over_zone_keys(oracle_mod, k, P):
    cfg = _small_cfg(k, P)
    x = _inputs(cfg)
    out, lse = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                    x["page_table"], x["seq_lens"], k)
    scale = 1.0 / np.sqrt(cfg.D)
    G = cfg.G
    for b in range(cfg.B):
        for h in range(cfg.Hq):
            g = h // G
            Kp, Vp = _gather_prefix(x["k_pages"], x["v_pages"], x["page_table"], b, g, P[b], 16)
            Ks = x["k_blk"][b, :, g].astype(np.float64)
            Vs = x["v_blk"][b, :, g].astype(np.float64)
            for r in range(k):                               # draft row r+1: [prefix, D_1..D_{r+1}]
                K = np.concatenate([Kp, Ks[: r + 1]])
                V = np.concatenate([Vp, Vs[: r + 1]])
                ref = _dense_attention(x["q"][b, r, h].astype(np.float64), K, V, scale)
                np.testing.assert_allclose(out[b, r, h], ref, rtol=1e-12, atol=1e-12)
            for j in range(1, k + 1):                        # block j: [prefix, D_1..D_j, M_j*]
                blk = slice(k + (j - 1) * k, k + j * k)
                K = np.concatenate([Kp, Ks[:j], Ks[blk]])
                V = np.concatenate([Vp, Vs[:j], Vs[blk]])
                for s in range(k):
                    row = k + (j - 1) * k + s
                    qv = x["q"][b, row, h].astype(np.float64)
                    ref = _dense_attention(qv, K, V, scale)
                    np.testing.assert_allclose(out[b, row, h], ref, rtol=1e-12, atol=1e-12)
                    sc = (K @ qv) * scale
                    ref_lse = sc.max() + np.log(np.exp(sc - sc.max()).sum())
                    assert abs(lse[b, row, h] - ref_lse) < 1e-10


@pytest.mark.parametrize("P", [0, 1, 63, 64, 65])
def test_k0_is_plain_decode_attention_sdpa(oracle_mod, P):
    cfg = _small_cfg(0, (P,), Hq=6, Hkv=2, D=32, dtype="bf16")
    x = _inputs(cfg)
    out, _ = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                  x["page_table"], x["seq_lens"], 0)
    def f64(a):
        return torch.from_numpy(a.astype(np.uint32) << 16).view(torch.float32).double()
    for h in range(cfg.Hq):
        g = h // cfg.G
        keys = [x["k_pages"][x["page_table"][0, i // 16], g, i % 16] for i in range(P)]
        vals = [x["v_pages"][x["page_table"][0, i // 16], g, i % 16] for i in range(P)]
        K = f64(np.stack(keys + [x["k_blk"][0, 0, g]]))
        V = f64(np.stack(vals + [x["v_blk"][0, 0, g]]))
        qv = f64(x["q"][0, 0, h][None])
        ref = torch.nn.functional.scaled_dot_product_attention(qv[None], K[None], V[None])[0, 0]
        np.testing.assert_allclose(out[0, 0, h], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_single_visible_key_returns_its_value(oracle_mod):
    # k = 0, empty prefix: the row sees only D_1, so softmax weight 1 on it.
    cfg = _small_cfg(0, (0,))
    x = _inputs(cfg)
    out, lse = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                    x["page_table"], x["seq_lens"], 0)
    for h in range(cfg.Hq):
        np.testing.assert_array_equal(out[0, 0, h], x["v_blk"][0, 0, h // cfg.G].astype(np.float64))
        s = float(x["q"][0, 0, h].astype(np.float64) @ x["k_blk"][0, 0, h // cfg.G]) / np.sqrt(cfg.D)
        assert abs(lse[0, 0, h] - s) < 1e-12


def test_equal_scores_give_mean_of_visible_values(oracle_mod):
    # q = 0 makes every score 0: the output is the mean of the visible values and
    # lse = log(#visible).
    k, P = 3, 40
    cfg = _small_cfg(k, (P,))
    x = _inputs(cfg)
    x["q"][:] = 0
    out, lse = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                    x["page_table"], x["seq_lens"], k)
    sets = _zone_sets(k)
    for h in range(cfg.Hq):
        g = h // cfg.G
        _, Vp = _gather_prefix(x["k_pages"], x["v_pages"], x["page_table"], 0, g, P, 16)
        for r in range(cfg.R):
            vis = sorted(sets[r])
            V = np.concatenate([Vp, x["v_blk"][0, vis, g].astype(np.float64)])
            np.testing.assert_allclose(out[0, r, h], V.mean(0), rtol=1e-12, atol=1e-13)
            assert abs(lse[0, r, h] - np.log(P + len(vis))) < 1e-12


def test_gqa_reads_only_its_kv_head(oracle_mod):
    # Poison every KV head except g with NaN: query heads of group g stay finite.
    k = 2
    cfg = _small_cfg(k, (37,), Hq=6, Hkv=3)
    x = _inputs(cfg)
    for g in range(cfg.Hkv):
        kp, vp = x["k_pages"].copy(), x["v_pages"].copy()
        kb, vb = x["k_blk"].copy(), x["v_blk"].copy()
        others = [o for o in range(cfg.Hkv) if o != g]
        kp[:, others] = np.nan; vp[:, others] = np.nan
        kb[:, :, others] = np.nan; vb[:, :, others] = np.nan
        out, _ = oracle_mod.step_attn(x["q"], kb, vb, kp, vp, x["page_table"], x["seq_lens"], k)
        for h in range(cfg.Hq):
            assert np.isfinite(out[0, :, h]).all() == (h // cfg.G == g)


def test_page_order_does_not_matter(oracle_mod):
    # Moving the prefix to other physical pages (same logical order) changes nothing.
    k = 2
    cfg = _small_cfg(k, (50, 20))
    x = _inputs(cfg)
    out1, lse1 = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                      x["page_table"], x["seq_lens"], k)
    rng = np.random.default_rng(3)
    perm = rng.permutation(x["k_pages"].shape[0])        # new physical slot of page p: perm[p]
    kp = np.empty_like(x["k_pages"]); vp = np.empty_like(x["v_pages"])
    kp[perm] = x["k_pages"]; vp[perm] = x["v_pages"]
    table = np.where(x["page_table"] >= 0, perm[np.maximum(x["page_table"], 0)], -1).astype(np.int32)
    out2, lse2 = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], kp, vp, table, x["seq_lens"], k)
    np.testing.assert_array_equal(out1, out2)
    np.testing.assert_array_equal(lse1, lse2)


def test_bf16_inputs_widen_exactly(oracle_mod):
    # bf16 inputs must give the same fp64 result as the same values stored in fp32.
    k = 2
    cfg = _small_cfg(k, (45,), dtype="bf16")
    x = _inputs(cfg)
    def as_f32(a):
        return (a.astype(np.uint32) << 16).view(np.float32)
    names = ["q", "k_blk", "v_blk", "k_pages", "v_pages"]
    y = {n: as_f32(x[n]) for n in names}
    o1, l1 = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                  x["page_table"], x["seq_lens"], k)
    o2, l2 = oracle_mod.step_attn(y["q"], y["k_blk"], y["v_blk"], y["k_pages"], y["v_pages"],
                                  x["page_table"], x["seq_lens"], k)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_selected_rows_match_full_run(oracle_mod):
    k = 3
    cfg = _small_cfg(k, (30, 61))
    x = _inputs(cfg)
    full, lfull = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                       x["page_table"], x["seq_lens"], k)
    sel = [(1, 5, 3), (0, 0, 0), (1, 11, 2)]
    part, lpart = oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                                       x["page_table"], x["seq_lens"], k, sel=sel)
    for i, (b, r, h) in enumerate(sel):
        np.testing.assert_array_equal(part[i], full[b, r, h])
        assert lpart[i] == lfull[b, r, h]


def test_unmapped_prefix_page_is_an_error(oracle_mod):
    cfg = _small_cfg(1, (40,))
    x = _inputs(cfg)
    x["page_table"][0, 1] = -1
    with pytest.raises(ValueError):
        oracle_mod.step_attn(x["q"], x["k_blk"], x["v_blk"], x["k_pages"], x["v_pages"],
                             x["page_table"], x["seq_lens"], 1)


def test_append_places_draft_rows(oracle_mod):
    k = 3
    cfg = _small_cfg(k, (14, 16))
    x = _inputs(cfg)
    kp, vp = oracle_mod.append(x["k_pages"], x["v_pages"], x["page_table"], x["seq_lens"],
                               x["k_blk"], x["v_blk"], k)
    ps = 16
    changed = np.zeros(kp.shape[:3], bool)
    for b, P in enumerate(cfg.prefix):
        for r in range(k):
            pos = P + r
            page = x["page_table"][b, pos // ps]
            np.testing.assert_array_equal(kp[page, :, pos % ps], x["k_blk"][b, r])
            np.testing.assert_array_equal(vp[page, :, pos % ps], x["v_blk"][b, r])
            changed[page, :, pos % ps] = True
    np.testing.assert_array_equal(kp[~changed], x["k_pages"][~changed])
    np.testing.assert_array_equal(vp[~changed], x["v_pages"][~changed])
