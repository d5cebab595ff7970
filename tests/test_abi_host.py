"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
function include/tidar.h declares, and rejects bad arguments before launching
anything.  Device pointers here are fake aligned addresses; every call below
fails validation before any pointer could be used."""
import ctypes

import pytest

import ar_decoding_b200 as tidar
from ar_decoding_b200 import build

FAKE = 0x10000          # aligned, never dereferenced
MISALIGNED = 0x10008


@pytest.fixture(scope="module")
def L():
    build.build()
    return tidar.lib()


def test_exports_every_declared_symbol(L):
    names = tidar.header_functions()
    assert {"tidar_step_attn", "tidar_verify", "tidar_commit", "tidar_reserve",
            "tidar_get_device_status"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def _desc(**kw):
    d = dict(batch=1, num_q_heads=4, num_kv_heads=2, head_dim=128, k=4, page_size=64,
             max_prefix_len=100, dtype=tidar.BF16, softmax_scale=0.0, path=tidar.PATH_AUTO)
    d.update(kw)
    return tidar.StepDesc(**d)


def _cache(**kw):
    c = dict(k_pages=FAKE, v_pages=FAKE, page_table=FAKE, seq_lens=FAKE, num_pages=8,
             max_pages_per_seq=2)
    c.update(kw)
    return tidar.KVCacheDesc(**c)


def _attn(L, desc, cache, q=FAKE, out=FAKE, ws=None, wsb=0):
    return L.tidar_step_attn(ctypes.byref(desc) if desc is not None else None,
                             ctypes.byref(cache) if cache is not None else None,
                             q, FAKE, FAKE, out, None, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_heads=3), tidar.ERR_INVALID_ARG),          # Hq not a multiple of Hkv
    (dict(head_dim=96), tidar.ERR_UNSUPPORTED),
    (dict(k=17), tidar.ERR_UNSUPPORTED),
    (dict(k=-1), tidar.ERR_INVALID_ARG),
    (dict(page_size=48), tidar.ERR_UNSUPPORTED),
    (dict(dtype=7), tidar.ERR_UNSUPPORTED),
    (dict(path=9), tidar.ERR_INVALID_ARG),
    (dict(max_prefix_len=-5), tidar.ERR_INVALID_ARG),
    (dict(max_prefix_len=1000), tidar.ERR_INVALID_ARG),    # table too short for it
])
def test_step_attn_rejects_bad_desc(L, kw, status):
    assert _attn(L, _desc(**kw), _cache()) == status


def test_step_attn_rejects_null_and_misaligned(L):
    assert _attn(L, None, _cache()) == tidar.ERR_INVALID_ARG
    assert _attn(L, _desc(), None) == tidar.ERR_INVALID_ARG
    assert _attn(L, _desc(), _cache(), q=None) == tidar.ERR_INVALID_ARG
    assert _attn(L, _desc(), _cache(), q=MISALIGNED) == tidar.ERR_INVALID_ARG
    assert _attn(L, _desc(), _cache(k_pages=MISALIGNED)) == tidar.ERR_INVALID_ARG
    assert _attn(L, _desc(), _cache(num_pages=0)) == tidar.ERR_INVALID_ARG


def test_step_attn_rejects_small_workspace(L):
    # CUDA-core path: split partials go through the workspace
    d = _desc(max_prefix_len=8192, batch=1, num_q_heads=32, num_kv_heads=8, k=0,
              path=tidar.PATH_SIMT)
    c = _cache(max_pages_per_seq=129)
    need = L.tidar_step_attn_workspace_bytes(ctypes.byref(d))
    assert need > 0
    assert _attn(L, d, c, ws=FAKE, wsb=need - 1) == tidar.ERR_INVALID_ARG
    assert _attn(L, d, c, ws=FAKE + 16, wsb=need) == tidar.ERR_INVALID_ARG   # not 256-aligned


def test_last_split_may_hold_only_the_step_windows(L):
    # 8B-class k = 4 (one query tile of 20 rows x 4 heads): 64 prefix blocks of
    # 128 keys plus the tile's one step-key window are dealt out 4 per split,
    # so 16 splits take the prefix and a 17th only the window
    d = _desc(max_prefix_len=8192, batch=1, num_q_heads=32, num_kv_heads=8, k=4,
              path=tidar.PATH_TC05)
    assert tidar.plan_full(d)[:2] == (tidar.PATH_TC05, 17)


def test_tensor_core_plan_splits_long_prefixes(L):
    # one query row per head: the 8192-key prefix is split to fill the SMs; the
    # workspace holds split partials unless the kernel merges them itself
    d = _desc(max_prefix_len=8192, batch=1, num_q_heads=32, num_kv_heads=8, k=0,
              path=tidar.PATH_TC05)
    path, splits, merge = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    assert L.tidar_step_attn_plan(ctypes.byref(d), ctypes.byref(path), ctypes.byref(splits),
                                  ctypes.byref(merge)) == tidar.OK
    assert path.value == 2 and splits.value > 1 and merge.value in (1, 2)
    assert L.tidar_step_attn_plan(ctypes.byref(d), None, None, None) == tidar.OK
    ws = L.tidar_step_attn_workspace_bytes(ctypes.byref(d))
    rows = 32                                  # B * R * Hq
    assert ws == (0 if merge.value == 1 else ((splits.value * rows * 128 * 4 + 255) // 256 * 256) +
                  ((splits.value * rows * 4 + 255) // 256 * 256))
    assert tidar.plan_full(d) == (path.value, splits.value, merge.value)


def test_batch_zero_is_a_noop(L):
    assert _attn(L, _desc(batch=0), None) == tidar.OK


def test_verify_rejects_bad_args(L):
    V = L.tidar_verify
    ws = L.tidar_verify_workspace_bytes(2, 4, 512, tidar.REJECTION)
    args = lambda **kw: dict(dict(B=2, k=4, V=512, dt=tidar.F32, mode=tidar.REJECTION, logits=FAKE,
                                  drafts=FAKE, dl=FAKE, u=FAKE, acc=FAKE, toks=FAKE, ws=FAKE,
                                  wsb=ws), **kw)
    def call(a):
        return V(a["B"], a["k"], a["V"], a["dt"], a["mode"], a["logits"], a["drafts"], a["dl"],
                 a["u"], None, a["acc"], a["toks"], None, None, a["ws"], a["wsb"], None)
    assert call(args(k=17)) == tidar.ERR_UNSUPPORTED
    assert call(args(V=0)) == tidar.ERR_INVALID_ARG
    assert call(args(dl=None)) == tidar.ERR_INVALID_ARG
    assert call(args(u=None)) == tidar.ERR_INVALID_ARG
    assert call(args(drafts=None)) == tidar.ERR_INVALID_ARG
    assert call(args(wsb=ws - 1)) == tidar.ERR_INVALID_ARG
    assert call(args(ws=FAKE + 8)) == tidar.ERR_INVALID_ARG
    assert call(args(mode=5)) == tidar.ERR_INVALID_ARG
    assert call(args(B=0)) == tidar.OK


def test_commit_rejects_bad_args(L):
    d, c = _desc(), _cache()
    assert L.tidar_commit(ctypes.byref(d), ctypes.byref(c), None, FAKE, FAKE, None) == tidar.ERR_INVALID_ARG
    assert L.tidar_commit(ctypes.byref(_desc(k=20)), ctypes.byref(c), FAKE, FAKE, FAKE, None) == tidar.ERR_UNSUPPORTED
    assert L.tidar_commit(ctypes.byref(d), None, FAKE, FAKE, FAKE, None) == tidar.ERR_INVALID_ARG


def test_verify_blockq_rejects_bad_args(L):
    Q = L.tidar_verify_blockq
    ws = L.tidar_verify_workspace_bytes(2, 4, 512, tidar.REJECTION)
    def call(B=2, k=4, bl=FAKE, db=FAKE, u=FAKE, wsb=ws):
        return Q(B, k, 512, tidar.F32, FAKE, FAKE, bl, db, u, None, FAKE, FAKE, None, None, FAKE,
                 wsb, None)
    assert call(bl=None) == tidar.ERR_INVALID_ARG
    assert call(db=None) == tidar.ERR_INVALID_ARG
    assert call(u=None) == tidar.ERR_INVALID_ARG
    assert call(wsb=ws - 1) == tidar.ERR_INVALID_ARG
    assert call(k=17) == tidar.ERR_UNSUPPORTED
    assert call(B=0) == tidar.OK


def test_reserve_rejects_bad_args(L):
    d, c = _desc(), _cache()
    R = L.tidar_reserve
    pool = lambda **kw: ctypes.byref(tidar.PagePool(**dict(dict(free_pages=FAKE, free_count=FAKE,
                                                                 capacity=4), **kw)))
    assert R(ctypes.byref(d), ctypes.byref(c), None, None, None, None) == tidar.ERR_INVALID_ARG
    assert R(ctypes.byref(d), ctypes.byref(c), pool(free_count=None), None, None, None) == tidar.ERR_INVALID_ARG
    assert R(ctypes.byref(d), ctypes.byref(c), pool(capacity=-1), None, None, None) == tidar.ERR_INVALID_ARG
    assert R(ctypes.byref(d), ctypes.byref(c), pool(free_pages=None), None, None, None) == tidar.ERR_INVALID_ARG
    assert R(ctypes.byref(d), ctypes.byref(c), pool(), FAKE, None, None) == tidar.ERR_INVALID_ARG
    assert R(ctypes.byref(d), ctypes.byref(c), pool(), None, FAKE, None) == tidar.ERR_INVALID_ARG
    assert R(ctypes.byref(_desc(k=20)), ctypes.byref(c), pool(), None, None, None) == tidar.ERR_UNSUPPORTED
    assert R(ctypes.byref(_desc(batch=65537)), ctypes.byref(c), pool(), None, None, None) == tidar.ERR_UNSUPPORTED
    assert R(ctypes.byref(d), None, pool(), None, None, None) == tidar.ERR_INVALID_ARG
    assert R(ctypes.byref(_desc(max_prefix_len=1000)), ctypes.byref(c), pool(), None, None,
             None) == tidar.ERR_INVALID_ARG                  # table too short for it
    assert R(ctypes.byref(_desc(batch=0)), None, None, None, None, None) == tidar.OK


def test_plan_covers_workloads(L):
    # host-only planning: the 8B-class step fills the machine, small prefixes use one split
    d = _desc(batch=1, num_q_heads=32, num_kv_heads=8, k=16, max_prefix_len=8192)
    path, splits = tidar.plan(d)
    assert path in (1, 2) and splits >= 1
    d = _desc(max_prefix_len=64)
    assert tidar.plan(d)[1] == 1
    d = _desc(dtype=tidar.F32, head_dim=64, path=tidar.PATH_AUTO)
    assert tidar.plan(d)[0] == 1                        # fp32 -> CUDA-core kernel


def test_status_strings(L):
    for s in range(6):
        assert L.tidar_status_string(s)


def test_binding_refuses_host_tensors(L):
    """No CPU fallback: host tensors are refused before anything reaches the library."""
    import torch
    from ar_decoding_b200 import synth
    cfg = synth.StepConfig("host", B=1, Hq=2, Hkv=2, D=64, k=2, prefix=(10,), dtype="f32",
                           vocab=64)
    cache, step = synth.make_cache(cfg), synth.make_step(cfg)
    vin = synth.make_verify(cfg, "rejection")
    with pytest.raises(ValueError):
        tidar.step_attn(step["q"], step["k_blk"], step["v_blk"], cache, cfg.k, max_prefix_len=10)
    with pytest.raises(ValueError):
        tidar.verify(vin["logits"], vin["drafts"], cfg.k, "greedy")
    with pytest.raises(ValueError):
        tidar.verify_noalloc(vin["logits"], vin["drafts"], cfg.k, "rejection",
                             draft_logits=vin["draft_logits"], uniforms=vin["uniforms"])
    bl, blk = synth.make_block_logits(cfg)
    with pytest.raises(ValueError):
        tidar.verify_blockq(vin["logits"], vin["drafts"], cfg.k, bl, blk, vin["uniforms"])
    with pytest.raises(ValueError):
        tidar.commit(cache, torch.ones(1, dtype=torch.int32), cfg.k, max_prefix_len=10)
    pool = synth.make_pool(cfg, cache)
    with pytest.raises(ValueError):
        tidar.reserve(cache, pool, cfg.k, max_prefix_len=10)


def test_projection_workspace_is_checked(L):
    # split-K partials pass through the caller's workspace: an 8B-class query /
    # key / value projection of a 272-row step splits its reduction, a single
    # 64-wide reduction cannot split (no workspace)
    need = L.tidar_linear_workspace_bytes(272, 6144, 4096)
    assert need > 0 and need % 256 == 0
    assert L.tidar_linear_workspace_bytes(16, 128, 64) == 0
    assert L.tidar_linear_workspace_bytes(0, 128, 64) == 0
    lin = lambda ws, wsb: L.tidar_linear(272, 6144, 4096, tidar.BF16, FAKE, FAKE, FAKE, ws, wsb, None)
    assert lin(None, 0) == tidar.ERR_INVALID_ARG
    assert lin(FAKE, need - 1) == tidar.ERR_INVALID_ARG
    assert lin(FAKE + 16, need) == tidar.ERR_INVALID_ARG               # not 256-aligned
    assert L.tidar_linear(272, 6144, 4000, tidar.BF16, FAKE, FAKE, FAKE, None, 0, None) == \
        tidar.ERR_UNSUPPORTED                                             # in_features % 64
    d = _desc(batch=1, num_q_heads=32, num_kv_heads=8, k=16, max_prefix_len=8192, head_dim=128,
              dtype=tidar.BF16)
    assert L.tidar_qkv_rope_workspace_bytes(ctypes.byref(d), 4096) == need
    assert L.tidar_qkv_rope(ctypes.byref(d), 4096, FAKE, FAKE, FAKE, ctypes.c_float(10000.0), FAKE, FAKE,
                            FAKE, None, 0, None) == tidar.ERR_INVALID_ARG
    assert L.tidar_layer_step_workspace_bytes(ctypes.byref(d), 4096) > need
