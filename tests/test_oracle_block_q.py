"""Pins for the oracle's draft distributions taken from mask blocks (CPU only).

  * the hand-worked index table in tests/golden/block_q_k3.txt (which block and
    slot each q row comes from, and the fallback for a block outside 1..k);
  * through verification: when the selected block's slot rows are the AR rows
    (q_i = p_i) every draft is accepted whatever it is, and when they are a
    one-hot far from the drafts nothing is accepted -- the rule's two
    extremes, which fail if the wrong block or slot is read.
"""
import numpy as np
import pytest

from conftest import read_golden


def _cases():
    k, cases = None, []
    for ln in read_golden("block_q_k3.txt"):
        key, rest = ln.split(None, 1)
        if key == "k":
            k = int(rest)
        else:
            parts = [p.strip() for p in rest.split("|")]
            cases.append((int(parts[0]), [int(v) for v in parts[1].split()], len(parts) > 2))
    return k, cases


def test_golden_block_rows(oracle_mod):
    k, cases = _cases()
    V = 2
    bl = np.zeros((len(cases), k, k, V), np.float32)
    for j in range(1, k + 1):
        for s in range(1, k + 1):
            bl[:, j - 1, s - 1, :] = 10 * j + s
    db = np.array([c[0] for c in cases], np.int32)
    out, flags = oracle_mod.gather_block_q(bl, db, k)
    for b, (blk, want, flagged) in enumerate(cases):
        assert [int(x) for x in out[b, :, 0]] == want, (blk, out[b, :, 0])
    assert flags == (oracle_mod.GATHER_FLAG_BLOCK if any(c[2] for c in cases) else 0)
    ok, fl = oracle_mod.gather_block_q(bl[:3], db[:3], k)
    assert fl == 0


@pytest.mark.parametrize("k", [2, 4, 8])
def test_selected_block_drives_acceptance(oracle_mod, k):
    rng = np.random.default_rng(k)
    B, V = 6, 64
    logits = rng.normal(0, 3, (B, k, V)).astype(np.float32)
    drafts = rng.integers(0, V, (B, k)).astype(np.int32)
    uniforms = rng.random((B, k)).astype(np.float32) * 0.999
    db = rng.integers(1, k + 1, B).astype(np.int32)
    # other blocks: one-hot far away from every draft (q(d) ~ 0 would accept;
    # make them peaked ON the drafts so reading them would reject)
    bl = np.full((B, k, k, V), -30.0, np.float32)
    for b in range(B):
        for j in range(k):
            for s in range(1, k):
                bl[b, j, s, drafts[b, s]] = 30.0          # q(d) ~ 1: u*q < p fails
        for i in range(1, k):
            bl[b, db[b] - 1, i] = logits[b, i - 1]      # the selected block: q_i = p_i
    dl, flags = oracle_mod.gather_block_q(bl, db, k)
    assert flags == 0
    res = oracle_mod.verify(logits, drafts, k, oracle_mod.REJECTION, draft_logits=dl,
                            uniforms=uniforms)
    assert (res["accept_count"] == k).all()
    # reading any other block (or slot) would have rejected at the first draft
    wrong = np.where(db == k, 1, db + 1).astype(np.int32)
    dl2, _ = oracle_mod.gather_block_q(bl, wrong, k)
    res2 = oracle_mod.verify(logits, drafts, k, oracle_mod.REJECTION, draft_logits=dl2,
                             uniforms=uniforms)
    assert (res2["accept_count"] == 1).all()
