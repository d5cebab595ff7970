"""CPU oracle for the TiDAR decode step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  It wraps
``tidar_oracle.c`` (plain C, fp64 arithmetic, unfused loops) through ctypes and
shares no code with the CUDA library in ``ar_decoding_b200``.

Functions take numpy arrays (fp32 or bf16-as-uint16 for the floating-point
inputs, int32 for indices) and return numpy arrays.  See ``tidar_oracle.c`` for
the method each one restates and the pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tidar_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16 = 0, 1
GREEDY, REJECTION = 0, 1
RESERVE_FLAG_PAGE, RESERVE_FLAG_LEN, RESERVE_FLAG_POOL = 1, 2, 4
GATHER_FLAG_BLOCK = 1


def build(force: bool = False) -> str:
    """Compile tidar_oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.tidar_oracle_step_key_visible.argtypes = [i, i, i]
        lib.tidar_oracle_step_key_visible.restype = i
        lib.tidar_oracle_step_attn.argtypes = [i, i, i, i, i, i, i, ctypes.c_double, P, P, P, i, i,
                                               P, P, P, P, i, P, P, P, i]
        lib.tidar_oracle_step_attn.restype = i
        lib.tidar_oracle_step_attn_keys.argtypes = [i, i, i, i, i, i, i, ctypes.c_double, P, P, P, i, i,
                                                    P, P, P, P, i, i, P, P, P, i]
        lib.tidar_oracle_step_attn_keys.restype = i
        lib.tidar_oracle_merge.argtypes = [i, ctypes.c_int64, i, P, P, P, P]
        lib.tidar_oracle_merge.restype = i
        lib.tidar_oracle_append.argtypes = [i, i, i, i, i, i, P, P, P, i, i, P, P, P]
        lib.tidar_oracle_append.restype = i
        lib.tidar_oracle_verify.argtypes = [i, i, i, i, i, P, P, P, P, P, P, P, P, P, P]
        lib.tidar_oracle_verify.restype = i
        lib.tidar_oracle_commit.argtypes = [i, i, i, i, i, i, P, P, P, i, i, P, P, P, P]
        lib.tidar_oracle_commit.restype = i
        lib.tidar_oracle_reserve.argtypes = [i, i, i, i, P, i, i, P, P, P, i, P, i]
        lib.tidar_oracle_reserve.restype = i
        lib.tidar_oracle_gather_block_q.argtypes = [i, i, i, i, P, P, P]
        lib.tidar_oracle_gather_block_q.restype = i
        lib.tidar_oracle_zone_positions.argtypes = [i, ctypes.c_int64, P]
        lib.tidar_oracle_zone_positions.restype = i
        lib.tidar_oracle_rope.argtypes = [i, i, i, ctypes.c_double, P, P, i, P]
        lib.tidar_oracle_rope.restype = i
        lib.tidar_oracle_linear.argtypes = [i, i, i, P, i, P, i, P]
        lib.tidar_oracle_linear.restype = i
        d = ctypes.c_double
        lib.tidar_oracle_verify_sampled.argtypes = [i, i, i, i, i, d, d, P, P, P, P, P, P, P, P, P,
                                                    P, P]
        lib.tidar_oracle_verify_sampled.restype = i
        lib.tidar_oracle_sample_drafts.argtypes = [i, i, i, i, i, d, d, P, P, P, P, P]
        lib.tidar_oracle_sample_drafts.restype = i
        lib.tidar_oracle_dist_row.argtypes = [i, i, d, d, P, P, P]
        lib.tidar_oracle_dist_row.restype = i
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle inputs are float32 or bf16 stored as uint16, got {a.dtype}")


def rows_per_seq(k: int) -> int:
    """Query rows of one sequence in one step: k drafts + k blocks of k slots (1 if k = 0)."""
    return 1 if k == 0 else k + k * k


def step_key_visible(k: int, row: int, key: int) -> bool:
    return bool(_load().tidar_oracle_step_key_visible(k, row, key))


def step_attn(q, k_blk, v_blk, k_pages, v_pages, page_table, seq_lens, k, *, scale=0.0,
              sel=None, num_threads=0, step_keys=True):
    """Three-zone step attention in fp64.

    q [B][R][Hq][D], k_blk/v_blk [B][R][Hkv][D], k_pages/v_pages
    [num_pages][Hkv][page][D] (fp32 or uint16 bf16 bits), page_table
    [B][max_pages] int32, seq_lens [B] int32.  Returns (out, lse): out
    [B][R][Hq][D] and lse [B][R][Hq] (natural log), or [n][D] / [n] for the
    (b, rho, h) triples in ``sel``.  step_keys=False: every row sees only the
    cache's prefix rows (one slice of a longer sequence; no key: 0 and -inf).
    """
    lib = _load()
    q = np.ascontiguousarray(q)
    dt = _dtype_code(q)
    B, R, Hq, D = q.shape
    Hkv = k_blk.shape[2]
    num_pages, _, page_size, _ = k_pages.shape
    assert R == rows_per_seq(k)
    k_blk, v_blk = np.ascontiguousarray(k_blk), np.ascontiguousarray(v_blk)
    k_pages, v_pages = np.ascontiguousarray(k_pages), np.ascontiguousarray(v_pages)
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    for a in (k_blk, v_blk, k_pages, v_pages):
        assert a.dtype == q.dtype
    if sel is None:
        n_sel, sel_arr = -1, None
        out = np.zeros((B, R, Hq, D), np.float64)
        lse = np.zeros((B, R, Hq), np.float64)
    else:
        sel_arr = np.ascontiguousarray(np.asarray(sel, dtype=np.int32).reshape(-1, 3))
        n_sel = sel_arr.shape[0]
        out = np.zeros((n_sel, D), np.float64)
        lse = np.zeros((n_sel,), np.float64)
    st = lib.tidar_oracle_step_attn_keys(B, Hq, Hkv, D, k, page_size, dt, float(scale),
                                         _ptr(k_pages), _ptr(v_pages), _ptr(page_table),
                                         page_table.shape[1], num_pages, _ptr(seq_lens), _ptr(q),
                                         _ptr(k_blk), _ptr(v_blk), 1 if step_keys else 0, n_sel,
                                         _ptr(sel_arr), _ptr(out), _ptr(lse), int(num_threads))
    if st != 0:
        raise ValueError(f"oracle step_attn failed with status {st}")
    return out, lse


def merge(parts_o, parts_lse):
    """Attention over a union of disjoint key sets from the per-set results:
    parts_o [nparts][...][D], parts_lse [nparts][...] -> (out [...][D], lse
    [...]) in fp64 (the log-sum-exp merge)."""
    po = np.ascontiguousarray(parts_o, dtype=np.float64)
    pl = np.ascontiguousarray(parts_lse, dtype=np.float64)
    nparts, D = po.shape[0], po.shape[-1]
    rows = int(np.prod(pl.shape[1:]))
    assert po.shape[:-1] == pl.shape
    out = np.zeros(pl.shape[1:] + (D,), np.float64)
    lse = np.zeros(pl.shape[1:], np.float64)
    st = _load().tidar_oracle_merge(nparts, rows, D, _ptr(po), _ptr(pl), _ptr(out), _ptr(lse))
    if st != 0:
        raise ValueError(f"oracle merge failed with status {st}")
    return out, lse


def dist_row(row, temperature=1.0, top_p=1.0):
    """The sampling transform of one logit row (fp32 or bf16 bits): returns
    (p [V] fp64, cut margin)."""
    row = np.ascontiguousarray(row)
    V = row.shape[0]
    p = np.zeros(V, np.float64)
    cm = np.zeros(1, np.float64)
    st = _load().tidar_oracle_dist_row(V, _dtype_code(row), float(temperature), float(top_p),
                                       _ptr(row), _ptr(p), _ptr(cm))
    if st != 0:
        raise ValueError(f"oracle dist_row failed with status {st}")
    return p, float(cm[0])


def verify_sampled(logits, drafts, k, mode, *, temperature=1.0, top_p=1.0, draft_logits=None,
                   uniforms=None, block_guesses=None):
    """tidar_oracle_verify with the sampling transform (temperature, nucleus
    top_p) applied to p and q.  Returns verify's dict plus margins [B][n] and
    cut_margins [B] (the smallest nucleus-cut margin the sequence's decisions
    read; +inf without truncation)."""
    lib = _load()
    logits = np.ascontiguousarray(logits)
    dt = _dtype_code(logits)
    B, n, V = logits.shape
    assert n == max(k, 1)
    drafts = None if drafts is None else np.ascontiguousarray(drafts, dtype=np.int32)
    if draft_logits is not None:
        draft_logits = np.ascontiguousarray(draft_logits)
        assert draft_logits.dtype == logits.dtype
    if uniforms is not None:
        uniforms = np.ascontiguousarray(uniforms, dtype=np.float32)
    if block_guesses is not None:
        block_guesses = np.ascontiguousarray(block_guesses, dtype=np.int32)
    acc = np.zeros(B, np.int32)
    toks = np.zeros((B, n), np.int32)
    nxt = np.zeros((B, max(k, 1)), np.int32)
    selb = np.zeros(B, np.int32)
    marg = np.zeros((B, n), np.float64)
    cut = np.zeros(B, np.float64)
    st = lib.tidar_oracle_verify_sampled(B, k, V, dt, mode, float(temperature), float(top_p),
                                         _ptr(logits), _ptr(drafts), _ptr(draft_logits),
                                         _ptr(uniforms), _ptr(block_guesses), _ptr(acc), _ptr(toks),
                                         _ptr(nxt), _ptr(selb), _ptr(marg), _ptr(cut))
    if st != 0:
        raise ValueError(f"oracle verify_sampled failed with status {st}")
    return dict(accept_count=acc, out_tokens=toks, next_drafts=nxt[:, :k], selected_block=selb,
                margins=marg, cut_margins=cut)


def sample_drafts(block_logits, selected_block, k, mode, *, temperature=1.0, top_p=1.0,
                  uniforms=None, next_drafts=None):
    """The next drafts from the selected mask block: slot s = 2..k of block
    selected_block[b] gives next_drafts[b][s-1] (argmax in mode GREEDY, inverse
    CDF of the transformed slot distribution with uniforms[b][s-1] in mode
    REJECTION).  Returns (next_drafts [B][k] int32, margins [B][k], status);
    entry 0 keeps next_drafts' value (or -1)."""
    lib = _load()
    bl = np.ascontiguousarray(block_logits)
    dt = _dtype_code(bl)
    B, kk, k2, V = bl.shape
    assert kk == k and k2 == k
    sb = np.ascontiguousarray(selected_block, dtype=np.int32)
    u = None if uniforms is None else np.ascontiguousarray(uniforms, dtype=np.float32)
    out = (np.full((B, k), -1, np.int32) if next_drafts is None
           else np.array(next_drafts, dtype=np.int32, copy=True))
    marg = np.zeros((B, k), np.float64)
    st = lib.tidar_oracle_sample_drafts(B, k, V, dt, mode, float(temperature), float(top_p),
                                        _ptr(bl), _ptr(sb), _ptr(u), _ptr(out), _ptr(marg))
    return out, marg, int(st)


def append(k_pages, v_pages, page_table, seq_lens, k_blk, v_blk, k):
    """Return copies of the caches with the draft rows' K/V written at P_b.. P_b+n-1."""
    lib = _load()
    kp, vp = np.array(k_pages, copy=True), np.array(v_pages, copy=True)
    num_pages, Hkv, page_size, D = kp.shape
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    k_blk, v_blk = np.ascontiguousarray(k_blk), np.ascontiguousarray(v_blk)
    B = seq_lens.shape[0]
    st = lib.tidar_oracle_append(B, Hkv, D, k, page_size, kp.dtype.itemsize, _ptr(kp), _ptr(vp),
                                 _ptr(page_table), page_table.shape[1], num_pages, _ptr(seq_lens),
                                 _ptr(k_blk), _ptr(v_blk))
    if st != 0:
        raise ValueError(f"oracle append failed with status {st}")
    return kp, vp


def verify(logits, drafts, k, mode, *, draft_logits=None, uniforms=None, block_guesses=None,
           with_margins=False):
    """Left-to-right verification, acceptance and selection (fp64).

    Returns dict(accept_count [B], out_tokens [B][n], next_drafts [B][k],
    selected_block [B], margins [B][n] if requested).
    """
    lib = _load()
    logits = np.ascontiguousarray(logits)
    dt = _dtype_code(logits)
    B, n, V = logits.shape
    assert n == max(k, 1)
    drafts = None if drafts is None else np.ascontiguousarray(drafts, dtype=np.int32)
    if draft_logits is not None:
        draft_logits = np.ascontiguousarray(draft_logits)
        assert draft_logits.dtype == logits.dtype
    if uniforms is not None:
        uniforms = np.ascontiguousarray(uniforms, dtype=np.float32)
    if block_guesses is not None:
        block_guesses = np.ascontiguousarray(block_guesses, dtype=np.int32)
    acc = np.zeros(B, np.int32)
    toks = np.zeros((B, n), np.int32)
    nxt = np.zeros((B, max(k, 1)), np.int32)
    selb = np.zeros(B, np.int32)
    marg = np.zeros((B, n), np.float64) if with_margins else None
    st = lib.tidar_oracle_verify(B, k, V, dt, mode, _ptr(logits), _ptr(drafts), _ptr(draft_logits),
                                 _ptr(uniforms), _ptr(block_guesses), _ptr(acc), _ptr(toks),
                                 _ptr(nxt), _ptr(selb), _ptr(marg))
    if st != 0:
        raise ValueError(f"oracle verify failed with status {st}")
    res = dict(accept_count=acc, out_tokens=toks, next_drafts=nxt[:, :k], selected_block=selb)
    if with_margins:
        res["margins"] = marg
    return res


def commit(k_pages, v_pages, page_table, seq_lens, accept_count, k):
    """KV commit/evict on copies.  Returns (k_pages, v_pages, page_table, seq_lens,
    released, num_released, status)."""
    lib = _load()
    kp, vp = np.array(k_pages, copy=True), np.array(v_pages, copy=True)
    pt = np.array(page_table, dtype=np.int32, copy=True)
    sl = np.array(seq_lens, dtype=np.int32, copy=True)
    acc = np.ascontiguousarray(accept_count, dtype=np.int32)
    num_pages, Hkv, page_size, D = kp.shape
    B = sl.shape[0]
    n = max(k, 1)
    cap = B * ((n + page_size - 1) // page_size + 1)
    rel = np.zeros(cap, np.int32)
    nrel = np.zeros(1, np.int32)
    st = lib.tidar_oracle_commit(B, Hkv, D, k, page_size, kp.dtype.itemsize, _ptr(kp), _ptr(vp),
                                 _ptr(pt), pt.shape[1], num_pages, _ptr(sl), _ptr(acc), _ptr(rel),
                                 _ptr(nrel))
    return kp, vp, pt, sl, rel, int(nrel[0]), st


def reserve(page_table, seq_lens, free_pages, free_count, k, page_size, num_pages, *,
            max_prefix, returned=None):
    """Page reservation from a free-page stack, on copies.

    page_table [B][max_pages] int32, seq_lens [B] int32, free_pages [capacity]
    int32 with free_count valid entries, returned: the ids to push first (or
    None).  Returns (page_table, free_pages, free_count, flags), flags a
    combination of RESERVE_FLAG_PAGE / _LEN / _POOL (0 = success).
    """
    lib = _load()
    pt = np.array(page_table, dtype=np.int32, copy=True)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    fp = np.array(free_pages, dtype=np.int32, copy=True)
    fc = np.array([free_count], dtype=np.int32)
    ret = None if returned is None else np.ascontiguousarray(returned, dtype=np.int32)
    nret = 0 if ret is None else int(ret.shape[0])
    flags = lib.tidar_oracle_reserve(sl.shape[0], k, page_size, int(max_prefix), _ptr(pt),
                                     pt.shape[1], num_pages, _ptr(sl), _ptr(fp), _ptr(fc),
                                     fp.shape[0], _ptr(ret), nret)
    return pt, fp, int(fc[0]), int(flags)


def gather_block_q(block_logits, draft_block, k):
    """Draft distributions from the previous step's mask blocks.

    block_logits [B][k][k][V] (fp32 or bf16 bits), draft_block [B] int32 (1..k).
    Returns (draft_logits [B][k-1][V], flags): row i-1 is block
    draft_block[b], slot i+1; a block outside 1..k reads block 1 and sets
    GATHER_FLAG_BLOCK.
    """
    lib = _load()
    bl = np.ascontiguousarray(block_logits)
    db = np.ascontiguousarray(draft_block, dtype=np.int32)
    B, kk, k2, V = bl.shape
    assert kk == k and k2 == k
    out = np.zeros((B, max(k - 1, 0), V), bl.dtype)
    flags = lib.tidar_oracle_gather_block_q(B, k, V, bl.dtype.itemsize, _ptr(bl), _ptr(db), _ptr(out))
    return out, int(flags)


def zone_positions(k, P):
    """Positions of a step's R query rows (drafts at P + r - 1, slot s of block
    j at P + j + s - 1, the single row of k = 0 at P), int64 [R]."""
    out = np.zeros(rows_per_seq(k), np.int64)
    st = _load().tidar_oracle_zone_positions(k, int(P), _ptr(out))
    if st != 0:
        raise ValueError(f"oracle zone_positions failed with status {st}")
    return out


def rope(x, pos, base=10000.0):
    """Rotate-half rotary embedding of x [rows][H][D] (fp32 or bf16 bits) at
    pos [rows], fp64 [rows][H][D]."""
    x = np.ascontiguousarray(x)
    rows, H, D = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    out = np.zeros((rows, H, D), np.float64)
    st = _load().tidar_oracle_rope(rows, H, D, float(base), _ptr(pos), _ptr(x), _dtype_code(x),
                                   _ptr(out))
    if st != 0:
        raise ValueError(f"oracle rope failed with status {st}")
    return out


def linear(x, w):
    """y = x w^T for x [M][K], w [N][K] (fp32 or bf16 bits), fp64 [M][N]."""
    x, w = np.ascontiguousarray(x), np.ascontiguousarray(w)
    M, K = x.shape
    N = w.shape[0]
    assert w.shape[1] == K
    y = np.zeros((M, N), np.float64)
    st = _load().tidar_oracle_linear(M, N, K, _ptr(x), _dtype_code(x), _ptr(w), _dtype_code(w),
                                     _ptr(y))
    if st != 0:
        raise ValueError(f"oracle linear failed with status {st}")
    return y
