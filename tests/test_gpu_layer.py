"""GPU parity of the layer-level step (tidar_linear, tidar_qkv_rope,
tidar_layer_step) against the oracle, through the C ABI.

The oracle chain is the plain definition: y = x w^T in fp64 (oracle.linear),
the rotate-half rotary embedding at the zone positions in fp64
(oracle.zone_positions, oracle.rope), the three-zone step attention in fp64
(oracle.step_attn) and the output projection.  The GPU computes in fp32 and
stores bf16.

Tolerances (derived from the arithmetic, written here):
  projections: each output is one fp32 dot product rounded once to bf16, so
    |got - want| <= 2^-8 |want| (round to nearest, 8 significant bits) plus
    fp32 accumulation error, covered by 1e-3 * rms(want) absolute;
  layer output: the attention's bf16 tolerance (per-row relative L2 <= 1e-2)
    composed with one more bf16 rounding of q/k/v and of the projection:
    per-row relative L2 <= 1.5e-2.
"""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth
from gpu_harness import to_dev

pytestmark = pytest.mark.gpu

RTOL_PROJ = 2.0 ** -8
ATOL_PROJ_RMS = 1e-3
TOL_LAYER_REL = 1.5e-2


def _bf16_np(t):
    return synth.to_np(t)


def _check_proj(got, want):
    got = got.double().cpu().numpy().reshape(want.shape)
    rms = float(np.sqrt(np.mean(want ** 2))) if want.size else 1.0
    err = np.abs(got - want)
    bound = RTOL_PROJ * np.abs(want) + ATOL_PROJ_RMS * rms
    worst = float((err - bound).max()) if want.size else 0.0
    assert worst <= 0, f"max |delta| {err.max():.3g} exceeds the bound by {worst:.3g}"


@pytest.mark.parametrize("T,K,N", [(1, 64, 128), (16, 256, 384), (17, 128, 256), (272, 4096, 256),
                                   (289, 192, 128), (600, 128, 640), (2304, 64, 128)])
def test_linear_matches_oracle(oracle_mod, T, K, N):
    # token tiles of one MMA (<= 256), two MMAs (257..288), several tiles
    # (> 288, ragged last tile); one to many K splits
    g = torch.Generator().manual_seed(1000 + T + K + N)
    x = torch.randn(T, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * K ** -0.5).to(torch.bfloat16)
    y = tidar.linear(x.cuda(), w.cuda())
    assert tidar.device_status() == (tidar.OK, 0)
    _check_proj(y, oracle_mod.linear(_bf16_np(x), _bf16_np(w)))


def test_linear_8b_class_o_projection_sampled_features(oracle_mod):
    # the full-size output projection (272 rows x 4096 in -> 4096 out): every
    # row, a seeded sample of 256 output features computed by the oracle
    cfg = synth.class_8b(k=16)
    lay = synth.make_layer(cfg)
    x = torch.randn(cfg.R, cfg.Hq * 128, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    y = tidar.linear(x.cuda(), lay["w_o"].cuda())
    feats = np.sort(np.random.default_rng(3).choice(lay["w_o"].shape[0], 256, replace=False))
    want = oracle_mod.linear(_bf16_np(x), _bf16_np(lay["w_o"][feats]))
    _check_proj(y.cpu()[:, feats], want)


def _oracle_qkv(oracle_mod, cfg, lay, heads=None, base=10000.0):
    """Oracle q, k_blk, v_blk (fp64) for the (kind, head) pairs in `heads`
    (all when None): linear over the head's weight rows, then the rotary
    embedding at each row's zone position."""
    x = _bf16_np(lay["x"]).reshape(cfg.B * cfg.R, -1)
    w = lay["w_qkv"]
    out = {}
    pos = np.concatenate([oracle_mod.zone_positions(cfg.k, P) for P in cfg.prefix])
    kinds = [("q", h) for h in range(cfg.Hq)] + [("k", h) for h in range(cfg.Hkv)] + \
            [("v", h) for h in range(cfg.Hkv)] if heads is None else heads
    for kind, h in kinds:
        r0 = {"q": h, "k": cfg.Hq + h, "v": cfg.Hq + cfg.Hkv + h}[kind] * 128
        y = oracle_mod.linear(x, _bf16_np(w[r0:r0 + 128]))          # [B R][128]
        if kind != "v":
            y = _rope_f64(oracle_mod, y, pos, base)
        out[(kind, h)] = y
    return out


def _rope_f64(oracle_mod, y, pos, base):
    # the oracle's rotary embedding takes fp32/bf16 storage: hand it the fp64
    # projection split into an fp32 head and an fp32 remainder, rotate both
    # (the rotation is linear) and add -- so nothing is lost to fp32 rounding
    hi = y.astype(np.float32)
    lo = (y - hi.astype(np.float64)).astype(np.float32)
    r_hi = oracle_mod.rope(hi[:, None, :], pos, base)[:, 0, :]
    r_lo = oracle_mod.rope(lo[:, None, :], pos, base)[:, 0, :]
    return r_hi + r_lo


def _gpu_qkv(cfg, lay, base=10000.0):
    seq = torch.tensor(cfg.prefix, dtype=torch.int32, device="cuda")
    q, kb, vb = tidar.qkv_rope(lay["x"].cuda(), lay["w_qkv"].cuda(), seq, cfg.k, cfg.Hq, cfg.Hkv,
                               max_prefix_len=max(cfg.prefix), rope_base=base)
    assert tidar.device_status() == (tidar.OK, 0)
    return q.cpu(), kb.cpu(), vb.cpu()


def _compare_qkv(cfg, got, want):
    q, kb, vb = got
    for (kind, h), w in want.items():
        t = {"q": q, "k": kb, "v": vb}[kind]
        _check_proj(t[:, :, h, :].reshape(cfg.B * cfg.R, 128), w)


@pytest.mark.parametrize("k,prefix,heads", [(0, (5, 1000), (4, 2)), (1, (0,), (2, 1)),
                                            (3, (7, 64, 300), (4, 2)), (4, (8191, 12), (8, 2)),
                                            (8, (100,) * 5, (6, 1))])
def test_qkv_rope_full(oracle_mod, k, prefix, heads):
    Hq, Hkv = heads
    cfg = synth.StepConfig("qkv", B=len(prefix), Hq=Hq, Hkv=Hkv, D=128, k=k, prefix=prefix,
                           dtype="bf16", seed=77 + k)
    lay = synth.make_layer(cfg, d_model=256)
    _compare_qkv(cfg, _gpu_qkv(cfg, lay), _oracle_qkv(oracle_mod, cfg, lay))


def test_qkv_rope_other_base_and_long_positions(oracle_mod):
    # positions past 10^5 (angles of ~10^5 rad reduced in fp64) and base 5e5
    cfg = synth.StepConfig("qkv-long", B=2, Hq=2, Hkv=1, D=128, k=2, prefix=(131072, 99999),
                           dtype="bf16", seed=81)
    lay = synth.make_layer(cfg, d_model=128)
    _compare_qkv(cfg, _gpu_qkv(cfg, lay, base=500000.0),
                 _oracle_qkv(oracle_mod, cfg, lay, base=500000.0))


@pytest.mark.parametrize("k", [0, 4, 16])
def test_qkv_rope_8b_class_sampled_heads(oracle_mod, k):
    # full 8B-class projection (4096 -> 6144 features); every row of the
    # queries of heads 0, 13, 31, the keys of heads 0, 7 and the values of head 3
    cfg = synth.class_8b(k=k)
    lay = synth.make_layer(cfg)
    want = _oracle_qkv(oracle_mod, cfg, lay,
                       heads=[("q", 0), ("q", 13), ("q", 31), ("k", 0), ("k", 7), ("v", 3)])
    _compare_qkv(cfg, _gpu_qkv(cfg, lay), want)


def _oracle_layer(oracle_mod, cfg, lay, cache, base=10000.0):
    """fp64 chain: projection + rotary embedding, step attention on those q/k/v
    (handed to the oracle as fp32), output projection."""
    qkv = _oracle_qkv(oracle_mod, cfg, lay, base=base)
    B, R = cfg.B, cfg.R
    q = np.stack([qkv[("q", h)] for h in range(cfg.Hq)], axis=1).reshape(B, R, cfg.Hq, 128)
    kb = np.stack([qkv[("k", h)] for h in range(cfg.Hkv)], axis=1).reshape(B, R, cfg.Hkv, 128)
    vb = np.stack([qkv[("v", h)] for h in range(cfg.Hkv)], axis=1).reshape(B, R, cfg.Hkv, 128)
    n = synth.to_np
    f32 = lambda a: np.asarray(a, np.float32)
    kp = n(cache["k_pages"].float()) if cache["k_pages"].dtype == torch.bfloat16 else n(cache["k_pages"])
    vp = n(cache["v_pages"].float()) if cache["v_pages"].dtype == torch.bfloat16 else n(cache["v_pages"])
    o, lse = oracle_mod.step_attn(f32(q), f32(kb), f32(vb), kp, vp, n(cache["page_table"]),
                                  n(cache["seq_lens"]), cfg.k)
    y = oracle_mod.linear(f32(o).reshape(B * R, cfg.Hq * 128), _bf16_np(lay["w_o"]))
    return y.reshape(B, R, -1), lse, (q, kb, vb)


@pytest.mark.parametrize("cfg", [
    synth.StepConfig("layer-small", B=2, Hq=8, Hkv=2, D=128, k=4, prefix=(300, 77), dtype="bf16", seed=91),
    synth.StepConfig("layer-k0", B=3, Hq=4, Hkv=4, D=128, k=0, prefix=(5000, 130, 1), dtype="bf16", seed=92),
    synth.class_8b(k=16)], ids=lambda c: c.name)
def test_layer_step_matches_oracle_chain(oracle_mod, cfg):
    dm = 256 if cfg.name != "8B-class" else None
    lay = synth.make_layer(cfg, d_model=dm)
    cache = synth.make_cache(cfg)
    want_y, want_lse, (q, kb, vb) = _oracle_layer(oracle_mod, cfg, lay, cache)
    dc = to_dev(cache)
    y, lse = tidar.layer_step(lay["x"].cuda(), lay["w_qkv"].cuda(), lay["w_o"].cuda(), dc, cfg.k,
                              cfg.Hq, cfg.Hkv, max_prefix_len=max(cfg.prefix))
    st, bits = tidar.device_status()
    assert st == tidar.OK, f"device status {st} bits {bits:#x}"
    got = y.double().cpu().numpy().reshape(cfg.B * cfg.R, -1)
    want = want_y.reshape(cfg.B * cfg.R, -1)
    rel = np.linalg.norm(got - want, axis=1) / np.maximum(np.linalg.norm(want, axis=1), 1e-30)
    assert rel.max() <= TOL_LAYER_REL, f"row rel L2 {rel.max():.3g}"
    assert np.abs(lse.double().cpu().numpy() - want_lse).max() <= 2e-2
    # the drafts' rotated K/V went into cache rows P_b .. P_b + n - 1
    kp = dc["k_pages"].cpu()
    for b, P in enumerate(cfg.prefix):
        for r in range(cfg.n):
            page = int(cache["page_table"][b, (P + r) // 64])
            _check_proj(kp[page, :, (P + r) % 64, :], kb[b, r])
