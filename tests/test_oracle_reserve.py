"""Pins for the oracle's page reservation (CPU only).

  * the hand-worked case in tests/golden/reserve_ps4.txt, and the same state
    with too few free pages (nothing changes) or too little room for the
    returned ids (nothing at all changes);
  * a sequential model written differently (a Python list used as the stack,
    pages found as the set of row // page_size, prefix pages as i*ps < P) on
    random states, the failure flags included;
  * conservation over reserve -> commit cycles with the oracle's commit: the
    page-table entries, the stack and the released ids always hold every page
    exactly once, and after each reserve every draft row has a page.
"""
import numpy as np
import pytest

from ar_decoding_b200 import synth
from conftest import read_golden


def _golden():
    hdr, seqs = {}, []
    for ln in read_golden("reserve_ps4.txt"):
        key, rest = ln.split(None, 1)
        if key == "seq":
            seqs.append([[int(v) for v in p.split()] for p in rest.split("|")])
        elif key in ("free", "returned", "free_after"):
            hdr[key] = [int(v) for v in rest.split()]
        else:
            hdr[key] = int(rest)
    return hdr, seqs


def _golden_state():
    hdr, seqs = _golden()
    table = np.array([s[1] for s in seqs], np.int32)
    lens = np.array([s[0][0] for s in seqs], np.int32)
    return hdr, seqs, table, lens


def test_golden_reserve(oracle_mod):
    hdr, seqs, table, lens = _golden_state()
    pt, fp, cnt, flags = oracle_mod.reserve(table, lens, np.array(hdr["free"], np.int32),
                                            hdr["count"], hdr["k"], hdr["ps"], hdr["num_pages"],
                                            max_prefix=hdr["max_prefix"],
                                            returned=hdr["returned"])
    assert flags == 0
    np.testing.assert_array_equal(pt, np.array([s[2] for s in seqs], np.int32))
    np.testing.assert_array_equal(fp, np.array(hdr["free_after"], np.int32))
    assert cnt == hdr["count_after"]


def test_golden_pool_too_small_changes_no_entry(oracle_mod):
    # without the two returned ids the stack holds 3 pages and 4 are needed
    hdr, seqs, table, lens = _golden_state()
    free = np.array(hdr["free"], np.int32)
    pt, fp, cnt, flags = oracle_mod.reserve(table, lens, free, hdr["count"], hdr["k"], hdr["ps"],
                                            hdr["num_pages"], max_prefix=hdr["max_prefix"])
    assert flags == oracle_mod.RESERVE_FLAG_POOL
    np.testing.assert_array_equal(pt, table)
    np.testing.assert_array_equal(fp, free)
    assert cnt == hdr["count"]


def test_golden_push_overflow_changes_nothing(oracle_mod):
    hdr, seqs, table, lens = _golden_state()
    free = np.array(hdr["free"], np.int32)
    pt, fp, cnt, flags = oracle_mod.reserve(table, lens, free, hdr["count"], hdr["k"], hdr["ps"],
                                            hdr["num_pages"], max_prefix=hdr["max_prefix"],
                                            returned=[20, 21, 22, 23])      # 3 + 4 > 6
    assert flags == oracle_mod.RESERVE_FLAG_POOL
    np.testing.assert_array_equal(pt, table)
    np.testing.assert_array_equal(fp, free)
    assert cnt == hdr["count"]


def test_golden_bad_sequences_are_skipped(oracle_mod):
    hdr, seqs, table, lens = _golden_state()
    table = table.copy()
    lens = lens.copy()
    table[1, 1] = -1          # seq1's page holding prefix row 4 is unmapped
    lens[4] = 13              # seq4 past max_prefix
    want = np.array([s[2] for s in seqs], np.int32)
    want[1] = table[1]
    want[4] = table[4]
    pt, fp, cnt, flags = oracle_mod.reserve(table, lens, np.array(hdr["free"], np.int32),
                                            hdr["count"], hdr["k"], hdr["ps"], hdr["num_pages"],
                                            max_prefix=hdr["max_prefix"],
                                            returned=hdr["returned"])
    assert flags == oracle_mod.RESERVE_FLAG_PAGE | oracle_mod.RESERVE_FLAG_LEN
    np.testing.assert_array_equal(pt, want)
    assert cnt == hdr["count_after"]


def _model(table, lens, free, count, k, ps, num_pages, max_prefix, returned, flags_mod):
    """The reservation restated as a list-based stack, one pop per page."""
    n = max(k, 1)
    table, free = table.copy(), free.copy()
    stack = [int(x) for x in free[:count]]
    if returned is not None:
        if count + len(returned) > len(free):
            return table, free, count, flags_mod.RESERVE_FLAG_POOL
        free[count:count + len(returned)] = returned
        stack += [int(x) for x in returned]
    flags, wants = 0, []
    for b, P in enumerate(int(x) for x in lens):
        if P < 0 or P > max_prefix or -(-(P + n) // ps) > table.shape[1]:
            flags |= flags_mod.RESERVE_FLAG_LEN
            continue
        pages = sorted({r // ps for r in range(P, P + n)})
        mine, ok = [], True
        for i in pages:
            e = int(table[b, i])
            if 0 <= e < num_pages:
                continue
            if e == -1 and not i * ps < P:
                mine.append((b, i))
            else:
                ok = False
        if not ok:
            flags |= flags_mod.RESERVE_FLAG_PAGE
            continue
        wants += mine
    if len(wants) > len(stack):
        return table, free, len(stack), flags | flags_mod.RESERVE_FLAG_POOL
    for b, i in wants:
        table[b, i] = stack.pop()
    return table, free, len(stack), flags


@pytest.mark.parametrize("seed", range(40))
def test_reserve_matches_stack_model(oracle_mod, seed):
    st = synth.random_pool_state(seed)
    args = (st["table"], st["lens"], st["free"], st["count"], st["k"], st["ps"], st["num_pages"])
    got = oracle_mod.reserve(*args, max_prefix=st["max_prefix"], returned=st["returned"])
    want = _model(*args, st["max_prefix"], st["returned"], oracle_mod)
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])
    assert got[2] == want[2] and got[3] == want[3]


@pytest.mark.parametrize("k,ps", [(0, 4), (3, 4), (8, 16), (16, 16), (16, 64)])
def test_pages_conserved_over_reserve_commit_cycles(oracle_mod, k, ps):
    rng = np.random.default_rng(k * 100 + ps)
    n = max(k, 1)
    B, steps = 6, 12
    lens = rng.integers(0, 3 * ps, B).astype(np.int32)
    max_prefix = int(lens.max()) + steps * n
    cols = -(-(max_prefix + n) // ps)
    num_pages = B * cols
    ids = list(rng.permutation(num_pages).astype(np.int32))
    table = np.full((B, cols), -1, np.int32)
    for b in range(B):
        for i in range(-(-int(lens[b]) // ps)):
            table[b, i] = ids.pop()
    free = np.full(num_pages, -1, np.int32)
    free[:len(ids)] = ids
    count, returned = len(ids), None
    kp = np.zeros((num_pages, 1, ps, 2), np.float32)
    every = list(range(num_pages))
    for _ in range(steps):
        table, free, count, flags = oracle_mod.reserve(table, lens, free, count, k, ps, num_pages,
                                                       max_prefix=max_prefix, returned=returned)
        assert flags == 0
        held = sorted([int(x) for x in table[table >= 0]] + [int(x) for x in free[:count]])
        assert held == every
        for b in range(B):
            P = int(lens[b])
            assert (table[b, P // ps: -(-(P + n) // ps)] >= 0).all()
        acc = rng.integers(0, n + 1, B).astype(np.int32)
        kp, _, table, lens, rel, nrel, st = oracle_mod.commit(kp, kp, table, lens, acc, k)
        assert st == 0
        returned = rel[:nrel]
        held = sorted([int(x) for x in table[table >= 0]] + [int(x) for x in free[:count]] +
                      [int(x) for x in returned])
        assert held == every
