"""Pins for the oracle's KV commit / evict (CPU only).

  * the hand-worked case in tests/golden/commit_ps4.txt;
  * invariants on random caches: rows below P+c untouched, rows P+c..P+n-1
    zero, every other byte untouched, seq_lens = P+c, page conservation (the
    released ids plus the ids left in the table are the ids before), released
    pages are exactly the step pages that hold no kept row, (b, i) order;
  * errors: an accept count out of range or an unmapped draft page leaves that
    sequence untouched.
"""
import numpy as np
import pytest

from conftest import read_golden


def _golden():
    hdr, seqs, zeroed, released, nrel = {}, [], [], None, None
    for ln in read_golden("commit_ps4.txt"):
        key, rest = ln.split(None, 1)
        if key == "seq":
            parts = [[int(v) for v in p.split()] for p in rest.split("|")]
            seqs.append(parts)
        elif key == "zeroed":
            zeroed.append(tuple(int(v) for v in rest.split()))
        elif key == "released":
            released = [int(v) for v in rest.split()]
        elif key == "num_released":
            nrel = int(rest)
        else:
            hdr[key] = int(rest)
    return hdr, seqs, zeroed, released, nrel


def test_golden_commit(oracle_mod):
    hdr, seqs, zeroed, released, nrel = _golden()
    ps, k, num_pages = hdr["ps"], hdr["k"], hdr["num_pages"]
    D = 2
    B = len(seqs)
    kp = (np.arange(num_pages * ps * D, dtype=np.float32).reshape(num_pages, 1, ps, D) + 1)
    vp = -kp
    table = np.array([s[1] for s in seqs], np.int32)
    seq_lens = np.array([s[0][0] for s in seqs], np.int32)
    acc = np.array([s[0][1] for s in seqs], np.int32)
    kp2, vp2, pt2, sl2, rel, nr, st = oracle_mod.commit(kp, vp, table, seq_lens, acc, k)
    assert st == 0
    np.testing.assert_array_equal(pt2, np.array([s[2] for s in seqs], np.int32))
    np.testing.assert_array_equal(sl2, np.array([s[3][0] for s in seqs], np.int32))
    np.testing.assert_array_equal(rel, np.array(released, np.int32))
    assert nr == nrel
    mask = np.zeros((num_pages, 1, ps), bool)
    for page, off in zeroed:
        mask[page, 0, off] = True
    assert (kp2[mask] == 0).all() and (vp2[mask] == 0).all()
    np.testing.assert_array_equal(kp2[~mask], kp[~mask])
    np.testing.assert_array_equal(vp2[~mask], vp[~mask])


def _random_state(rng, B, k, ps, Hkv=2, D=8):
    n = max(k, 1)
    P = rng.integers(0, 5 * ps, B)
    P[0] = ps - 1 if B > 1 else P[0]            # a tail that ends just before a boundary
    if B > 2:
        P[1] = 2 * ps                           # a prefix that ends on a boundary
    need = [-(-(int(p) + n) // ps) for p in P]
    num_pages = sum(need) + 3
    ids = rng.permutation(num_pages).astype(np.int32)
    max_pages = max(need) + 2
    table = np.full((B, max_pages), -1, np.int32)
    pos = 0
    for b, c in enumerate(need):
        table[b, :c] = ids[pos:pos + c]
        pos += c
    # a page reserved past the step's rows must survive the commit
    table[0, need[0]] = ids[pos]
    kp = rng.standard_normal((num_pages, Hkv, ps, D)).astype(np.float32)
    vp = rng.standard_normal((num_pages, Hkv, ps, D)).astype(np.float32)
    acc = rng.integers(0, n + 1, B).astype(np.int32)
    acc[0] = 0
    if B > 1:
        acc[-1] = n
    return kp, vp, table, P.astype(np.int32), acc


@pytest.mark.parametrize("k,ps,B", [(0, 4, 5), (1, 4, 6), (3, 4, 8), (8, 16, 12), (16, 64, 9),
                                    (5, 2, 7)])
def test_commit_invariants(oracle_mod, k, ps, B):
    rng = np.random.default_rng(k * 31 + ps)
    n = max(k, 1)
    kp, vp, table, P, acc = _random_state(rng, B, k, ps)
    kp2, vp2, pt2, sl2, rel, nr, st = oracle_mod.commit(kp, vp, table, P, acc, k)
    assert st == 0
    np.testing.assert_array_equal(sl2, P + acc)
    scrub = np.zeros(kp.shape[:1] + kp.shape[2:3], bool)       # [page][offset]
    expect_rel = []
    for b in range(B):
        for r in range(P[b] + acc[b], P[b] + n):
            scrub[table[b, r // ps], r % ps] = True
        for i in range(table.shape[1]):
            page = table[b, i]
            if page < 0:
                continue
            first_row = i * ps
            in_step = first_row < P[b] + n and (i + 1) * ps > P[b]
            holds_kept = first_row < P[b] + acc[b]
            if in_step and not holds_kept:
                expect_rel.append(page)
                assert pt2[b, i] == -1
            else:
                assert pt2[b, i] == page
    m = np.broadcast_to(scrub[:, None, :, None], kp.shape)
    assert (kp2[m] == 0).all() and (vp2[m] == 0).all()
    np.testing.assert_array_equal(kp2[~m], kp[~m])
    np.testing.assert_array_equal(vp2[~m], vp[~m])
    assert nr == len(expect_rel)
    np.testing.assert_array_equal(rel[:nr], expect_rel)        # (b, i) order
    assert (rel[nr:] == -1).all()
    # conservation of page ids
    before = sorted(table[table >= 0].tolist())
    after = sorted(pt2[pt2 >= 0].tolist() + rel[:nr].tolist())
    assert before == after


def test_commit_rejects_bad_count_and_unmapped_pages(oracle_mod):
    rng = np.random.default_rng(5)
    k, ps, B = 3, 4, 4
    kp, vp, table, P, acc = _random_state(rng, B, k, ps)
    acc[1] = k + 1                                  # out of range
    table2 = table.copy()
    r = P[2] + 1
    table2[2, r // ps] = -1                         # a draft row without a page
    kp2, vp2, pt2, sl2, rel, nr, st = oracle_mod.commit(kp, vp, table2, P, acc, k)
    assert st != 0
    assert sl2[1] == P[1] and sl2[2] == P[2]
    np.testing.assert_array_equal(pt2[1], table2[1])
    np.testing.assert_array_equal(pt2[2], table2[2])
    # the other sequences are still committed
    assert sl2[0] == P[0] + acc[0] and sl2[3] == P[3] + acc[3]
