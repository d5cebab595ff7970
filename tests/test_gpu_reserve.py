"""GPU parity of tidar_reserve against the oracle (bit-exact page tables, free
stacks, counts and error bits), and a decode loop -- reserve -> step attention
-> verify -> commit, several steps chained on the device -- captured as ONE
CUDA graph and compared step by step with the same loop run by the oracle."""
import numpy as np
import pytest
import torch

import ar_decoding_b200 as tidar
from ar_decoding_b200 import synth
from gpu_harness import compare_attention, to_dev

pytestmark = pytest.mark.gpu


def _bits(oracle_mod, flags):
    out = 0
    if flags & oracle_mod.RESERVE_FLAG_PAGE:
        out |= tidar.DEVERR_BAD_PAGE
    if flags & oracle_mod.RESERVE_FLAG_LEN:
        out |= tidar.DEVERR_BAD_LEN
    if flags & oracle_mod.RESERVE_FLAG_POOL:
        out |= tidar.DEVERR_POOL
    return out


def _gpu_reserve(st, dtype=torch.bfloat16):
    """Runs tidar_reserve on the state of synth.random_pool_state."""
    B, cols = st["table"].shape
    cache = dict(k_pages=torch.zeros((st["num_pages"], 1, st["ps"], 64), dtype=dtype, device="cuda"),
                 page_table=torch.from_numpy(st["table"].copy()).cuda(),
                 seq_lens=torch.from_numpy(st["lens"].copy()).cuda())
    cache["v_pages"] = cache["k_pages"]
    pool = dict(free_pages=torch.from_numpy(st["free"].copy()).cuda(),
                free_count=torch.tensor([st["count"]], dtype=torch.int32, device="cuda"))
    ret = nret = None
    if st["returned"] is not None:
        ret = torch.from_numpy(st["returned"].copy()).cuda()
        if ret.numel() == 0:
            ret = torch.full((1,), -7, dtype=torch.int32, device="cuda")
        nret = torch.tensor([st["returned"].shape[0]], dtype=torch.int32, device="cuda")
    tidar.reserve(cache, pool, st["k"], max_prefix_len=st["max_prefix"], returned=ret,
                  num_returned=nret)
    status, bits = tidar.device_status()
    return (cache["page_table"].cpu().numpy(), pool["free_pages"].cpu().numpy(),
            int(pool["free_count"].cpu()[0]), status, bits)


def _oracle_reserve(oracle_mod, st):
    return oracle_mod.reserve(st["table"], st["lens"], st["free"], st["count"], st["k"], st["ps"],
                              st["num_pages"], max_prefix=st["max_prefix"],
                              returned=st["returned"])


def _check(oracle_mod, st):
    pt, fp, cnt, status, bits = _gpu_reserve(st)
    wpt, wfp, wcnt, flags = _oracle_reserve(oracle_mod, st)
    np.testing.assert_array_equal(pt, wpt)
    np.testing.assert_array_equal(fp, wfp)
    assert cnt == wcnt
    assert bits == _bits(oracle_mod, flags)
    assert (status == tidar.OK) == (flags == 0)
    return flags


@pytest.mark.parametrize("seed", range(60))
def test_reserve_matches_oracle(oracle_mod, seed):
    _check(oracle_mod, synth.random_pool_state(seed))


def test_reserve_flags_are_all_reached(oracle_mod):
    seen = 0
    for seed in range(60):
        seen |= _oracle_reserve(oracle_mod, synth.random_pool_state(seed))[3]
    assert seen == (oracle_mod.RESERVE_FLAG_PAGE | oracle_mod.RESERVE_FLAG_LEN |
                    oracle_mod.RESERVE_FLAG_POOL)


@pytest.mark.parametrize("B,k,ps", [(1, 0, 64), (1023, 16, 16), (1025, 8, 64), (5000, 4, 16)])
def test_reserve_large_batches(oracle_mod, B, k, ps):
    # more sequences than threads: the count and the pops run chunk by chunk
    rng = np.random.default_rng(B + k)
    n = max(k, 1)
    max_prefix = 3 * ps
    cols = -(-(max_prefix + n) // ps)
    lens = rng.integers(0, max_prefix + 1, B).astype(np.int32)
    table = np.full((B, cols), -1, np.int32)
    nxt = 0
    for b in range(B):
        for i in range(-(-int(lens[b]) // ps)):
            table[b, i] = nxt
            nxt += 1
    num_pages = nxt + 2 * B
    free = np.arange(nxt, num_pages, dtype=np.int32)[::-1].copy()
    ret = rng.permutation(np.arange(nxt, nxt + 5, dtype=np.int32))    # pushed again on top
    st = dict(table=table, lens=lens, free=np.concatenate([free, np.full(8, -1, np.int32)]),
              count=free.shape[0], returned=ret, k=k, ps=ps, num_pages=num_pages,
              max_prefix=max_prefix)
    assert _check(oracle_mod, st) == 0


def test_reserve_pool_exhausted_and_overflow(oracle_mod):
    # too few free pages: nothing is reserved, the push stands
    lens = np.zeros(4, np.int32)
    base = dict(table=np.full((4, 2), -1, np.int32), lens=lens, k=4, ps=16, num_pages=64,
                max_prefix=16)
    s1 = dict(base, free=np.array([5, 6, -1, -1], np.int32), count=2,
              returned=np.array([9], np.int32))
    assert _check(oracle_mod, s1) == oracle_mod.RESERVE_FLAG_POOL
    # no room for the returned ids: nothing at all changes
    s2 = dict(base, free=np.array([5, 6, 7, 8], np.int32), count=4,
              returned=np.array([9], np.int32))
    assert _check(oracle_mod, s2) == oracle_mod.RESERVE_FLAG_POOL
    # exactly enough
    s3 = dict(base, free=np.array([5, 6, 7, -1, -1], np.int32), count=3,
              returned=np.array([9], np.int32))
    assert _check(oracle_mod, s3) == 0


# --- the chained decode loop ---------------------------------------------------

LOOPS = [
    # (name, cfg kwargs, steps, verify mode, use tidar_verify_noalloc):
    # M = R*G decides the attention kernel
    ("tc05", dict(B=4, Hq=8, Hkv=2, D=128, k=4, prefix=(62, 63, 64, 190), dtype="bf16",
                  page_size=64), 6, "greedy", False),
    ("tc05-rejection", dict(B=3, Hq=8, Hkv=2, D=128, k=4, prefix=(60, 127, 5), dtype="bf16",
                            page_size=64), 6, "rejection", False),
    ("dec", dict(B=3, Hq=4, Hkv=2, D=128, k=2, prefix=(61, 127, 300), dtype="bf16",
                 page_size=64), 6, "greedy", False),
    ("dec-noalloc-rejection", dict(B=3, Hq=4, Hkv=2, D=128, k=2, prefix=(62, 1, 255),
                                   dtype="bf16", page_size=64), 6, "rejection", True),
    ("dec-k0", dict(B=3, Hq=8, Hkv=2, D=128, k=0, prefix=(62, 63, 129), dtype="bf16",
                    page_size=64), 5, "greedy", False),
    # rejection with q read from the previous step's mask blocks through its
    # selected block (tidar_verify_blockq), chained on the device
    ("tc05-blockq", dict(B=3, Hq=8, Hkv=2, D=128, k=4, prefix=(63, 64, 200), dtype="bf16",
                         page_size=64), 6, "blockq", False),
    ("simt", dict(B=3, Hq=4, Hkv=2, D=64, k=3, prefix=(14, 15, 40), dtype="f32",
                  page_size=16), 6, "greedy", True),
]


def _oracle_loop(oracle_mod, cfg, cache, pool, attn, ver, steps, max_prefix, mode):
    n = synth.to_np
    kp, vp = n(cache["k_pages"]), n(cache["v_pages"])
    pt, sl = n(cache["page_table"]), n(cache["seq_lens"])
    free, cnt = n(pool["free_pages"]), int(pool["free_count"][0])
    ret, drafts, per = None, n(ver[0]["drafts"]), []
    for s in range(steps):
        pt, free, cnt, flags = oracle_mod.reserve(pt, sl, free, cnt, cfg.k, cfg.page_size,
                                                  kp.shape[0], max_prefix=max_prefix, returned=ret)
        assert flags == 0
        a = attn[s]
        kp, vp = oracle_mod.append(kp, vp, pt, sl, n(a["k_blk"]), n(a["v_blk"]), cfg.k)
        out, lse = oracle_mod.step_attn(n(a["q"]), n(a["k_blk"]), n(a["v_blk"]), kp, vp, pt, sl,
                                        cfg.k)
        dl = n(ver[s]["draft_logits"])
        if mode == "blockq" and s > 0:
            dl, fl = oracle_mod.gather_block_q(n(ver[s - 1]["block_logits"]),
                                               per[-1]["verify"]["selected_block"], cfg.k)
            assert fl == 0
        v = oracle_mod.verify(n(ver[s]["logits"]), drafts if cfg.k else None, cfg.k,
                              oracle_mod.GREEDY if mode == "greedy" else oracle_mod.REJECTION,
                              draft_logits=dl,
                              uniforms=n(ver[s]["uniforms"]),
                              block_guesses=n(ver[s]["block_guesses"]))
        kp, vp, pt, sl, rel, nrel, st = oracle_mod.commit(kp, vp, pt, sl, v["accept_count"], cfg.k)
        assert st == 0
        ret = rel[:nrel]
        drafts = v["next_drafts"]
        per.append(dict(out=out, lse=lse, verify=v, released=rel, num_released=nrel))
    return per, dict(k_pages=kp, v_pages=vp, page_table=pt, seq_lens=sl, free_pages=free,
                     free_count=cnt)


def _clone(d):
    return {k: v.clone() for k, v in d.items()}


def _enqueue_loop(cfg, dc, dpool, dattn, dver, outs, steps, max_prefix, drafts0, mode, noalloc):
    """Queues `steps` chained steps on the current stream (graph-capturable)."""
    ret = nret = None
    drafts = drafts0
    for s in range(steps):
        o = outs[s]
        tidar.reserve(dc, dpool, cfg.k, max_prefix_len=max_prefix, returned=ret, num_returned=nret)
        tidar.step_attn(dattn[s]["q"], dattn[s]["k_blk"], dattn[s]["v_blk"], dc, cfg.k,
                        max_prefix_len=max_prefix, out=o["out"], lse=o["lse"],
                        workspace=o["ws"])
        vkw = dict(draft_logits=dver[s].get("draft_logits") if cfg.k > 1 else None,
                   uniforms=dver[s]["uniforms"] if mode != "greedy" else None,
                   block_guesses=dver[s]["block_guesses"] if cfg.k else None,
                   outputs=o["verify"])
        if mode == "blockq" and s > 0:
            tidar.verify_blockq(dver[s]["logits"], drafts, cfg.k, dver[s - 1]["block_logits"],
                                outs[s - 1]["verify"]["selected_block"], vkw["uniforms"],
                                block_guesses=vkw["block_guesses"], outputs=o["verify"],
                                workspace=o["vws"])
        elif noalloc:
            tidar.verify_noalloc(dver[s]["logits"], drafts if cfg.k else None, cfg.k,
                                 "greedy" if mode == "greedy" else "rejection", **vkw)
        else:
            tidar.verify(dver[s]["logits"], drafts if cfg.k else None, cfg.k,
                         "greedy" if mode == "greedy" else "rejection", workspace=o["vws"], **vkw)
        tidar.commit(dc, o["verify"]["accept_count"], cfg.k, max_prefix_len=max_prefix,
                     num_q_heads=cfg.Hq, released=o["released"], num_released=o["num_released"])
        ret, nret = o["released"], o["num_released"]
        drafts = o["verify"]["next_drafts"]


@pytest.mark.parametrize("name,kw,steps,mode,noalloc", LOOPS, ids=[x[0] for x in LOOPS])
def test_decode_loop_in_one_cuda_graph(oracle_mod, name, kw, steps, mode, noalloc):
    cfg = synth.StepConfig(f"loop-{name}", vocab=4096, seed=0x10F + len(name), **kw)
    n = cfg.n
    max_prefix = max(cfg.prefix) + steps * n
    width = -(-(max_prefix + n) // cfg.page_size)
    cache = synth.make_cache(cfg, extra_pages=cfg.B * (steps * n // cfg.page_size + 2),
                             draft_pages=False, max_pages=width)
    pool = synth.make_pool(cfg, cache)
    attn, ver = synth.make_loop(cfg, steps, mode)
    per, final = _oracle_loop(oracle_mod, cfg, cache, pool, attn, ver, steps, max_prefix, mode)

    dc, dpool = to_dev(cache), to_dev(pool)
    dattn = [to_dev(a) for a in attn]
    dver = [to_dev({k: v for k, v in x.items() if isinstance(v, torch.Tensor)}) for x in ver]
    drafts0 = dver[0]["drafts"]
    desc = tidar.make_desc(dattn[0]["q"], dattn[0]["k_blk"], dc, cfg.k, max_prefix)
    wsb = tidar.step_attn_workspace_bytes(desc)
    vwsb = tidar.verify_workspace_bytes(cfg.B, cfg.k, cfg.vocab,
                                        tidar.GREEDY if mode == "greedy" else tidar.REJECTION)
    cap = cfg.B * (-(-n // cfg.page_size) + 1)
    outs = []
    for s in range(steps):
        outs.append(dict(
            out=torch.empty_like(dattn[s]["q"]),
            lse=torch.empty(dattn[s]["q"].shape[:3], dtype=torch.float32, device="cuda"),
            ws=torch.empty(max(wsb, 256), dtype=torch.uint8, device="cuda") if wsb else None,
            vws=torch.empty(max(vwsb, 256), dtype=torch.uint8, device="cuda"),
            verify=dict(accept_count=torch.empty(cfg.B, dtype=torch.int32, device="cuda"),
                        out_tokens=torch.empty((cfg.B, n), dtype=torch.int32, device="cuda"),
                        next_drafts=torch.empty((cfg.B, max(cfg.k, 1)), dtype=torch.int32,
                                                device="cuda"),
                        selected_block=torch.empty(cfg.B, dtype=torch.int32, device="cuda")),
            released=torch.empty(cap, dtype=torch.int32, device="cuda"),
            num_released=torch.empty(1, dtype=torch.int32, device="cuda")))

    # eager warm-up on copies (first calls look up symbols and set attributes)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _enqueue_loop(cfg, _clone(dc), _clone(dpool), dattn, dver, outs, steps, max_prefix, drafts0,
                      mode, noalloc)
    torch.cuda.current_stream().wait_stream(side)
    assert tidar.device_status()[0] == tidar.OK

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _enqueue_loop(cfg, dc, dpool, dattn, dver, outs, steps, max_prefix, drafts0, mode, noalloc)
    graph.replay()
    status, bits = tidar.device_status()
    assert status == tidar.OK, f"bits {bits:#x}"

    accepts = []
    for s in range(steps):
        o, w = outs[s], per[s]
        compare_attention(cfg, o["out"].cpu().reshape(-1, cfg.D), w["out"].reshape(-1, cfg.D),
                          o["lse"].cpu().reshape(-1), w["lse"].reshape(-1))
        for key in ("accept_count", "out_tokens", "selected_block"):
            np.testing.assert_array_equal(o["verify"][key].cpu().numpy(), w["verify"][key],
                                          err_msg=f"step {s} {key}")
        if cfg.k:
            np.testing.assert_array_equal(o["verify"]["next_drafts"].cpu().numpy(),
                                          w["verify"]["next_drafts"], err_msg=f"step {s}")
        assert int(o["num_released"].cpu()[0]) == w["num_released"]
        np.testing.assert_array_equal(o["released"].cpu().numpy(), w["released"])
        accepts += list(w["verify"]["accept_count"])
    for key in ("k_pages", "v_pages", "page_table", "seq_lens"):
        np.testing.assert_array_equal(synth.to_np(dc[key]), final[key], err_msg=key)
    np.testing.assert_array_equal(dpool["free_pages"].cpu().numpy(), final["free_pages"])
    assert int(dpool["free_count"].cpu()[0]) == final["free_count"]
    if cfg.k >= 2:
        assert len(set(int(a) for a in accepts)) >= 2       # the accept counts vary
    # the sequences grew, and crossed page boundaries along the way
    assert (final["seq_lens"] > np.array(cfg.prefix)).all()
    graph.reset()
