"""Pins for the oracle's sampling transform (temperature, nucleus top_p), the
verification that uses it and the draft sampling from the selected mask block
(CPU only).

  * the transform against a hand-worked five-token row
    (tests/golden/sampling_v5.txt), ties included;
  * properties checked with numpy, independently of the oracle's code: a tiny
    top_p keeps exactly the first maximal token; the kept set is the shortest
    run of the (logit desc, index asc) order -- built with numpy.lexsort --
    whose untruncated probability reaches top_p;
  * verification: greedy ignores the transform; with T = 1, top_p = 1 it is the
    pinned plain verification; chi-squared that the emitted tokens follow the
    transformed p_1, p_2 when the drafts are drawn from the transformed q; an
    exact enumeration for tiny vocabularies (every draft tuple weighted by the
    transformed q, every uniform region found by bisection) reproducing the
    transformed AR law;
  * draft sampling: argmax in greedy mode, the inverse CDF of the hand-worked
    row, a chi-squared test of the sampled drafts, and the fallback for a block
    index outside 1..k.
Targets are computed with numpy/scipy in fp64 (scipy.special.softmax, an
explicit sort for the truncation).
"""
import itertools

import numpy as np
import pytest
from scipy import special, stats

from conftest import read_golden

LN_ROW = np.log(np.array([4.0, 2.0, 2.0, 1.0, 1.0])).astype(np.float32)


def _golden_cases():
    out = []
    for ln in read_golden("sampling_v5.txt"):
        key, rest = ln.split(None, 1)
        assert key == "case"
        head, probs = rest.split("|")
        T, tp = (float(v) for v in head.split())
        out.append((T, tp, np.array([float(v) for v in probs.split()])))
    return out


def _np_transform(row, T, top_p):
    """Independent restatement for the properties below: softmax(l / T), then
    keep the tokens of the (logit desc, index asc) order while the mass before
    them is below top_p."""
    x = np.asarray(row, np.float64)
    p = special.softmax(x / T)
    if top_p >= 1.0:
        return p
    order = np.lexsort((np.arange(x.size), -x))        # last key primary: -x, then index
    before = np.concatenate([[0.0], np.cumsum(p[order])[:-1]])
    keep = np.zeros(x.size, bool)
    keep[order[before < top_p]] = True
    q = np.where(keep, p, 0.0)
    return q / q.sum()


@pytest.mark.parametrize("T,top_p,want", _golden_cases())
def test_golden_transform(oracle_mod, T, top_p, want):
    p, _ = oracle_mod.dist_row(LN_ROW, T, top_p)
    # the logits are fp32 roundings of ln(...): probabilities agree to ~1e-7
    np.testing.assert_allclose(p, want, rtol=0, atol=5e-7)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tiny_top_p_keeps_the_first_maximum(oracle_mod, dtype):
    rng = np.random.default_rng(5)
    for _ in range(50):
        x = (rng.standard_normal(300) * 2).astype(np.float32)
        if dtype == "bf16":
            bits = (x.view(np.uint32) >> 16).astype(np.uint16)
            x, row = (bits.astype(np.uint32) << 16).view(np.float32), bits
        else:
            row = x
        x[rng.integers(300)] = x.max()                   # a tie for the maximum
        if dtype == "bf16":
            row = (x.view(np.uint32) >> 16).astype(np.uint16)
        else:
            row = x
        p, _ = oracle_mod.dist_row(row, 0.7, 1e-9)
        want = np.zeros(300)
        want[int(np.argmax(x))] = 1.0                    # first maximal index
        np.testing.assert_array_equal(p, want)


@pytest.mark.parametrize("T,top_p", [(1.0, 0.9), (0.6, 0.5), (1.7, 0.95), (1.0, 1.0), (0.3, 0.99)])
def test_kept_set_is_the_shortest_reaching_run(oracle_mod, T, top_p):
    rng = np.random.default_rng(int(T * 100 + top_p * 1000))
    for _ in range(20):
        bits = (rng.standard_normal(2000).astype(np.float32) * 3).view(np.uint32) >> 16
        row = bits.astype(np.uint16)                    # bf16: many equal logits
        x = (bits.astype(np.uint32) << 16).view(np.float32)
        p, cm = oracle_mod.dist_row(row, T, top_p)
        if cm < 1e-9:
            continue                                     # a cut decided by rounding only
        np.testing.assert_allclose(p, _np_transform(x, T, top_p), rtol=1e-12, atol=1e-15)
        assert abs(p.sum() - 1.0) < 1e-12


def _rows(rng, n, V, std=1.5):
    return (rng.standard_normal((n, V)) * std).astype(np.float32)


def test_greedy_ignores_the_transform(oracle_mod):
    rng = np.random.default_rng(3)
    B, k, V = 40, 4, 50
    logits = (rng.standard_normal((B, k, V)) * 2).astype(np.float32)
    am = np.argmax(logits, axis=-1)
    drafts = rng.integers(0, V, (B, k)).astype(np.int32)
    drafts[:, 1:] = np.where(rng.random((B, k - 1)) < 0.6, am[:, :k - 1], drafts[:, 1:])
    g = rng.integers(0, V, (B, k, k)).astype(np.int32)
    a = oracle_mod.verify(logits, drafts, k, oracle_mod.GREEDY, block_guesses=g)
    b = oracle_mod.verify_sampled(logits, drafts, k, oracle_mod.GREEDY, temperature=0.3, top_p=0.5,
                                  block_guesses=g)
    for key in ("accept_count", "out_tokens", "next_drafts", "selected_block"):
        np.testing.assert_array_equal(a[key], b[key])


def test_untransformed_is_the_plain_verification(oracle_mod):
    rng = np.random.default_rng(4)
    B, k, V = 60, 4, 40
    logits = _rows(rng, B * k, V).reshape(B, k, V)
    dl = _rows(rng, B * (k - 1), V).reshape(B, k - 1, V)
    drafts = rng.integers(0, V, (B, k)).astype(np.int32)
    u = rng.random((B, k), dtype=np.float32)
    a = oracle_mod.verify(logits, drafts, k, oracle_mod.REJECTION, draft_logits=dl, uniforms=u)
    b = oracle_mod.verify_sampled(logits, drafts, k, oracle_mod.REJECTION, draft_logits=dl, uniforms=u)
    for key in ("accept_count", "out_tokens", "selected_block"):
        np.testing.assert_array_equal(a[key], b[key])


def test_chi2_emitted_tokens_follow_the_transformed_p(oracle_mod):
    rng = np.random.default_rng(2025)
    N, k, V, T, tp = 200_000, 4, 16, 0.7, 0.9
    n = k
    l1 = _rows(rng, n, V)
    # draft rows near the AR rows (as a good drafter's would be), so that the
    # truncated supports overlap and later tokens are emitted often enough
    q1 = (l1[:k - 1] + 0.6 * rng.standard_normal((k - 1, V))).astype(np.float32)
    p = np.stack([_np_transform(l1[i], T, tp) for i in range(n)])
    q = np.stack([_np_transform(q1[i], T, tp) for i in range(k - 1)])
    drafts = np.zeros((N, k), np.int32)
    for i in range(k - 1):
        drafts[:, i + 1] = rng.choice(V, size=N, p=q[i])
    u = rng.random((N, n), dtype=np.float32)
    r = oracle_mod.verify_sampled(np.broadcast_to(l1, (N, n, V)).copy(), drafts, k,
                                  oracle_mod.REJECTION, temperature=T, top_p=tp,
                                  draft_logits=np.broadcast_to(q1, (N, k - 1, V)).copy(), uniforms=u)
    assert (r["cut_margins"] > 1e-9).all()
    acc, toks = r["accept_count"], r["out_tokens"]
    rate = np.minimum(p[0], q[0]).sum()
    assert abs((acc >= 2).mean() - rate) < 4 * np.sqrt(rate * (1 - rate) / N)
    for m in range(3):
        sel = acc >= m + 1
        obs = np.bincount(toks[sel, m], minlength=V)
        keep = p[m] > 0
        assert obs[~keep].sum() == 0                      # truncated tokens never appear
        assert stats.chisquare(obs[keep], sel.sum() * p[m][keep]).pvalue > 1e-3


def _call(oracle_mod, l1, q1, drafts, u, k, T, tp):
    r = oracle_mod.verify_sampled(l1[None], np.array([drafts], np.int32), k, oracle_mod.REJECTION,
                                  temperature=T, top_p=tp,
                                  draft_logits=q1[None] if k > 1 else None,
                                  uniforms=np.array([u], np.float32))
    return int(r["accept_count"][0]), tuple(int(t) for t in r["out_tokens"][0])


def _bisect(f, lo, hi, iters=40):
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if f(mid):
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


@pytest.mark.parametrize("k,V,seed,T,tp", [(2, 4, 12, 0.8, 0.8), (3, 3, 13, 1.3, 0.9),
                                           (2, 3, 14, 0.5, 1.0)])
def test_exact_enumeration_equals_the_transformed_ar_law(oracle_mod, k, V, seed, T, tp):
    rng = np.random.default_rng(seed)
    n = k
    l1 = _rows(rng, n, V)
    q1 = _rows(rng, k - 1, V)
    p = np.stack([_np_transform(l1[i], T, tp) for i in range(n)])
    q = np.stack([_np_transform(q1[i], T, tp) for i in range(k - 1)])
    ONE = float(np.nextafter(np.float32(1), np.float32(0)))
    dist = {}
    for tail in itertools.product(range(V), repeat=n - 1):
        drafts = [0] + list(tail)
        w = float(np.prod([q[i, tail[i]] for i in range(n - 1)]))
        if w == 0.0:
            continue                                    # a draft the transformed q never proposes
        thr = []
        for i in range(1, n):
            def acc(x, i=i):
                u = [0.0] * n
                u[i - 1] = x
                return _call(oracle_mod, l1, q1, drafts, u, k, T, tp)[0] >= i + 1
            thr.append(1.0 if acc(ONE) else (0.0 if not acc(0.0) else _bisect(acc, 0.0, 1.0)))
        for j in range(1, n + 1):
            pj = w * float(np.prod(thr[:j - 1])) * ((1.0 - thr[j - 1]) if j < n else 1.0)
            if pj == 0.0:
                continue
            base = [0.0] * n
            if j < n:
                base[j - 1] = ONE
            def tok(x):
                u = list(base)
                u[n - 1] = x
                a, t = _call(oracle_mod, l1, q1, drafts, u, k, T, tp)
                assert a == j
                return t
            lo_u = 0.0
            while lo_u < 1.0:
                t0 = tok(lo_u)
                hi_u = 1.0 if tok(ONE) == t0 else _bisect(lambda x: tok(x) == t0, lo_u, 1.0)
                dist[t0] = dist.get(t0, 0.0) + pj * (hi_u - lo_u)
                if hi_u >= 1.0:
                    break
                lo_u = hi_u + 1e-12
    tol = 4 * 2.0 ** -24
    assert abs(sum(dist.values()) - 1.0) < tol
    first = np.zeros(V)
    for s, pr in dist.items():
        first[s[0]] += pr
    np.testing.assert_allclose(first, p[0], rtol=0, atol=tol)
    for m in range(1, n):
        for prefix in itertools.product(range(V), repeat=m):
            tot = sum(pr for s, pr in dist.items() if s[:m] == prefix and s[m] >= 0)
            if tot < 1e-9:
                continue
            cond = np.zeros(V)
            for s, pr in dist.items():
                if s[:m] == prefix and s[m] >= 0:
                    cond[s[m]] += pr / tot
            np.testing.assert_allclose(cond, p[m], rtol=0, atol=tol / tot)


# --- the next drafts from the selected mask block --------------------------------

def test_sample_drafts_greedy_is_the_slot_argmax(oracle_mod):
    rng = np.random.default_rng(8)
    B, k, V = 6, 4, 30
    bl = _rows(rng, B * k * k, V).reshape(B, k, k, V)
    sel = rng.integers(1, k + 1, B).astype(np.int32)
    prev = np.full((B, k), 77, np.int32)
    out, _, st = oracle_mod.sample_drafts(bl, sel, k, oracle_mod.GREEDY, temperature=0.2, top_p=0.3,
                                          next_drafts=prev)
    assert st == 0
    for b in range(B):
        assert out[b, 0] == 77                           # t* is the verification's
        for s in range(2, k + 1):
            assert out[b, s - 1] == int(np.argmax(bl[b, sel[b] - 1, s - 1]))


@pytest.mark.parametrize("T,top_p,want", _golden_cases())
def test_sample_drafts_inverse_cdf_of_the_golden_row(oracle_mod, T, top_p, want):
    # block 2, slot 2 holds the hand-worked row; a uniform inside each token's
    # interval of the cumulative sum picks that token
    k, V = 2, 5
    bl = np.zeros((1, k, k, V), np.float32)
    bl[0, 1, 1] = LN_ROW
    cdf = np.cumsum(want)
    lo = np.concatenate([[0.0], cdf[:-1]])
    for t in range(V):
        if want[t] < 1e-6:
            continue
        u = np.array([[0.0, 0.5 * (lo[t] + cdf[t])]], np.float32)
        out, _, st = oracle_mod.sample_drafts(bl, np.array([2], np.int32), k, oracle_mod.REJECTION,
                                              temperature=T, top_p=top_p, uniforms=u)
        assert st == 0 and out[0, 1] == t


def test_sample_drafts_chi2(oracle_mod):
    rng = np.random.default_rng(9)
    N, k, V, T, tp = 100_000, 3, 12, 0.9, 0.85
    row = _rows(rng, 1, V)[0]
    bl = np.zeros((N, k, k, V), np.float32)
    bl[:, 2, 1] = row                                   # block 3, slot 2
    u = rng.random((N, k), dtype=np.float32)
    out, marg, st = oracle_mod.sample_drafts(bl, np.full(N, 3, np.int32), k, oracle_mod.REJECTION,
                                             temperature=T, top_p=tp, uniforms=u)
    assert st == 0
    want = _np_transform(row, T, tp)
    obs = np.bincount(out[:, 1], minlength=V)
    keep = want > 0
    assert obs[~keep].sum() == 0
    assert stats.chisquare(obs[keep], N * want[keep]).pvalue > 1e-3


def test_sample_drafts_bad_block_reads_block_one(oracle_mod):
    rng = np.random.default_rng(10)
    k, V = 3, 20
    bl = _rows(rng, k * k, V).reshape(1, k, k, V)
    for bad in (0, 4, -1):
        out, _, st = oracle_mod.sample_drafts(bl, np.array([bad], np.int32), k, oracle_mod.GREEDY)
        assert st == 3                                   # ORACLE_ERR_COUNT
        for s in range(2, k + 1):
            assert out[0, s - 1] == int(np.argmax(bl[0, 0, s - 1]))
