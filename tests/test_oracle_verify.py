"""Pins for the oracle's verification / acceptance / selection (CPU only).

  * hand-worked golden cases (tests/golden/verify_*.txt);
  * greedy: the emitted tokens are exactly what plain AR argmax (numpy.argmax,
    first maximal index) produces on the same logits, up to and including the
    first disagreement;
  * rejection: the acceptance rate of d_2 equals the closed form
    sum_x min(p_1(x), q_1(x)); chi-squared tests that the first emitted token
    follows p_1 and the second (when emitted) follows p_2; and an exact
    enumeration for tiny vocabularies -- every draft tuple weighted by q, every
    uniform region found by bisection -- that reproduces the AR distribution to
    the resolution of the fp32 uniforms.
AR targets are computed with scipy.special.softmax in fp64.
"""
import itertools

import numpy as np
import pytest
from scipy import special, stats

from conftest import read_golden


def _parse_cases(name):
    lines = read_golden(name)
    hdr, rows, cases = {}, {}, []
    for ln in lines:
        key, rest = ln.split(None, 1)
        if key == "case":
            cases.append([[float(v) for v in part.split()] for part in rest.split("|")])
        elif key in ("V", "k"):
            hdr[key] = int(rest)
        else:
            rows.setdefault(key, []).append([float(v) for v in rest.split()])
    return hdr, rows, cases


def test_golden_greedy(oracle_mod):
    hdr, rows, cases = _parse_cases("verify_greedy_k4.txt")
    V, k = hdr["V"], hdr["k"]
    logits = np.array(rows["logits"], np.float32)[None]
    guesses = np.array(rows["guess"], np.int32)[None]
    for drafts, acc, toks, selb, nxt in cases:
        r = oracle_mod.verify(logits, np.array([drafts], np.int32), k, oracle_mod.GREEDY,
                              block_guesses=guesses)
        assert r["accept_count"][0] == int(acc[0])
        np.testing.assert_array_equal(r["out_tokens"][0], np.array(toks, np.int32))
        assert r["selected_block"][0] == int(selb[0])
        np.testing.assert_array_equal(r["next_drafts"][0], np.array(nxt, np.int32))


def test_golden_rejection(oracle_mod):
    hdr, rows, cases = _parse_cases("verify_rejection_v2.txt")
    k = hdr["k"]
    logits = np.array(rows["logits"], np.float32)[None]
    dl = np.array(rows["draft_logits"], np.float32)[None]
    for drafts, us, acc, toks in cases:
        r = oracle_mod.verify(logits, np.array([drafts], np.int32), k, oracle_mod.REJECTION,
                              draft_logits=dl, uniforms=np.array([us], np.float32))
        assert r["accept_count"][0] == int(acc[0])
        np.testing.assert_array_equal(r["out_tokens"][0], np.array(toks, np.int32))


@pytest.mark.parametrize("k,V,dtype", [(0, 512, "f32"), (1, 64, "f32"), (4, 512, "f32"),
                                       (8, 1000, "bf16"), (16, 300, "bf16")])
def test_greedy_equals_plain_ar_argmax(oracle_mod, k, V, dtype):
    rng = np.random.default_rng(k * 100 + V)
    B, n = 64, max(k, 1)
    lf = (rng.standard_normal((B, n, V)) * 3).astype(np.float32)
    if dtype == "bf16":
        bits = (lf.view(np.uint32) >> 16).astype(np.uint16)   # truncation: any bf16 values will do
        lf = (bits.astype(np.uint32) << 16).view(np.float32)
        logits = bits
    else:
        logits = lf
    am = np.argmax(lf, axis=-1)                                  # first maximal index
    drafts = rng.integers(0, V, (B, max(k, 1)), dtype=np.int32)[:, :k]
    # plant agreement so every accept count occurs
    for b in range(B):
        stop = rng.integers(0, n)
        for i in range(1, k):
            drafts[b, i] = am[b, i - 1] if i <= stop else (am[b, i - 1] + 1) % V
    guesses = rng.integers(0, V, (B, k, k), dtype=np.int32) if k else None
    r = oracle_mod.verify(logits, drafts if k else None, k, oracle_mod.GREEDY, block_guesses=guesses)
    for b in range(B):
        # plain AR: emit argmax of row 1, 2, ... while the drafts agree with it
        emitted, i = [], 1
        while True:
            t = int(am[b, i - 1])
            emitted.append(t)
            if i < n and drafts[b, i] == t:
                i += 1
                continue
            break
        j = len(emitted)
        assert r["accept_count"][b] == j
        np.testing.assert_array_equal(r["out_tokens"][b, :j], emitted)
        assert (r["out_tokens"][b, j:] == -1).all()
        if k:
            assert r["selected_block"][b] == j
            assert r["next_drafts"][b, 0] == emitted[-1]
            np.testing.assert_array_equal(r["next_drafts"][b, 1:], guesses[b, j - 1, 1:])


def _rejection_batch(rng, N, k, V, std=1.5):
    """N trials sharing one set of rows: logits [N][n][V], draft logits [N][k-1][V],
    drafts d_{i+1} ~ q_i, uniforms U[0,1)."""
    n = max(k, 1)
    l1 = (rng.standard_normal((n, V)) * std).astype(np.float32)
    q1 = (rng.standard_normal((max(k - 1, 1), V)) * std).astype(np.float32)[: k - 1]
    p = special.softmax(l1.astype(np.float64), axis=-1)
    q = special.softmax(q1.astype(np.float64), axis=-1)
    drafts = np.zeros((N, k), np.int32)
    for i in range(k - 1):
        drafts[:, i + 1] = rng.choice(V, size=N, p=q[i])
    u = rng.random((N, n), dtype=np.float32)
    return (np.broadcast_to(l1, (N, n, V)).copy(), np.broadcast_to(q1, (N, k - 1, V)).copy(),
            drafts, u, p, q)


def test_acceptance_rate_closed_form_and_chi2(oracle_mod):
    rng = np.random.default_rng(2024)
    N, k, V = 200_000, 4, 16
    logits, dl, drafts, u, p, q = _rejection_batch(rng, N, k, V)
    r = oracle_mod.verify(logits, drafts, k, oracle_mod.REJECTION, draft_logits=dl, uniforms=u)
    acc, toks = r["accept_count"], r["out_tokens"]
    # closed form: P(accept d_2) = sum_x min(p_1, q_1) = 1 - TV(p_1, q_1)
    rate = np.minimum(p[0], q[0]).sum()
    emp = (acc >= 2).mean()
    assert abs(emp - rate) < 4 * np.sqrt(rate * (1 - rate) / N)
    # first emitted token ~ p_1
    obs = np.bincount(toks[:, 0], minlength=V)
    assert stats.chisquare(obs, N * p[0]).pvalue > 1e-3
    # second emitted token (when emitted) ~ p_2
    sel = acc >= 2
    obs2 = np.bincount(toks[sel, 1], minlength=V)
    assert stats.chisquare(obs2, sel.sum() * p[1]).pvalue > 1e-3
    # third, given three emitted, ~ p_3
    sel3 = acc >= 3
    obs3 = np.bincount(toks[sel3, 2], minlength=V)
    assert stats.chisquare(obs3, sel3.sum() * p[2]).pvalue > 1e-3


def test_chi2_detects_a_planted_mistake(oracle_mod):
    # Power check of the chi-squared statistic used above: tokens drawn from q_1
    # instead of p_1 (what skipping the residual step would give) must fail.
    rng = np.random.default_rng(7)
    N, k, V = 200_000, 4, 16
    _, _, _, _, p, q = _rejection_batch(rng, N, k, V)
    wrong = rng.choice(V, size=N, p=q[0])
    assert stats.chisquare(np.bincount(wrong, minlength=V), N * p[0]).pvalue < 1e-6


def _call(oracle_mod, l1, q1, drafts, u, k):
    r = oracle_mod.verify(l1[None], np.array([drafts], np.int32), k, oracle_mod.REJECTION,
                          draft_logits=q1[None] if k > 1 else None,
                          uniforms=np.array([u], np.float32))
    return int(r["accept_count"][0]), tuple(int(t) for t in r["out_tokens"][0])


def _bisect(f, lo, hi, iters=40):
    """Largest-u boundary: f(lo) True, f(hi) False -> the switch point."""
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if f(mid):
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _exact_output_distribution(oracle_mod, l1, q1, k, V):
    """Exact law of the emitted token sequence: drafts enumerated with weight
    prod q_i(d_{i+1}); uniform regions found by bisection on the oracle itself
    (each accept test is a threshold in its own uniform; the final token is a
    nondecreasing step function of the last uniform)."""
    n = max(k, 1)
    q = special.softmax(q1.astype(np.float64), axis=-1) if k > 1 else None
    dist = {}
    ONE = float(np.nextafter(np.float32(1), np.float32(0)))
    for tail in itertools.product(range(V), repeat=n - 1):
        drafts = [0] + list(tail)
        w = 1.0
        for i in range(n - 1):
            w *= q[i, tail[i]]
        # thresholds of the accept tests: u below it accepts (earlier tests forced to accept)
        thr = []
        for i in range(1, n):
            def acc(x, i=i):
                u = [0.0] * n
                u[i - 1] = x
                return _call(oracle_mod, l1, q1, drafts, u, k)[0] >= i + 1
            if acc(ONE):
                thr.append(1.0)
            elif not acc(0.0):
                thr.append(0.0)
            else:
                thr.append(_bisect(acc, 0.0, 1.0))
        for j in range(1, n + 1):
            pj = w
            for i in range(1, j):
                pj *= thr[i - 1]
            if j < n:
                pj *= 1.0 - thr[j - 1]
            if pj == 0.0:
                continue
            base = [0.0] * n
            if j < n:
                base[j - 1] = ONE                       # force the rejection at test j
            def tok(x):
                u = list(base)
                u[n - 1] = x
                a, t = _call(oracle_mod, l1, q1, drafts, u, k)
                assert a == j
                return t
            lo_u = 0.0
            while lo_u < 1.0:
                t0 = tok(lo_u)
                if tok(ONE) == t0:
                    hi_u = 1.0
                else:
                    hi_u = _bisect(lambda x: tok(x) == t0, lo_u, 1.0)
                dist[t0] = dist.get(t0, 0.0) + pj * (hi_u - lo_u)
                if hi_u >= 1.0:
                    break
                lo_u = hi_u + 1e-12
    return dist


@pytest.mark.parametrize("k,V,seed", [(1, 4, 1), (2, 3, 2), (2, 4, 3), (3, 3, 4)])
def test_rejection_exact_enumeration_equals_ar(oracle_mod, k, V, seed):
    rng = np.random.default_rng(seed)
    n = max(k, 1)
    l1 = (rng.standard_normal((n, V)) * 1.5).astype(np.float32)
    q1 = (rng.standard_normal((max(k - 1, 1), V)) * 1.5).astype(np.float32)[: max(k - 1, 0)]
    if k <= 1:
        q1 = np.zeros((0, V), np.float32)
    p = special.softmax(l1.astype(np.float64), axis=-1)
    dist = _exact_output_distribution(oracle_mod, l1, q1, k, V)
    # The uniforms are fp32, so every region boundary is only defined to the fp32
    # grid near it (spacing <= 2**-24 ~ 6e-8); a few boundaries per probability.
    tol = 4 * 2.0 ** -24
    assert abs(sum(dist.values()) - 1.0) < tol
    # marginal law of the first token is p_1
    first = np.zeros(V)
    for seq, pr in dist.items():
        first[seq[0]] += pr
    np.testing.assert_allclose(first, p[0], rtol=0, atol=tol)
    # each later token, given the tokens before it and that it is emitted, follows p_m
    for m in range(1, n):
        for prefix in itertools.product(range(V), repeat=m):
            tot = sum(pr for s, pr in dist.items() if s[:m] == prefix and s[m] >= 0)
            if tot < 1e-12:
                continue
            cond = np.zeros(V)
            for s, pr in dist.items():
                if s[:m] == prefix and s[m] >= 0:
                    cond[s[m]] += pr / tot
            np.testing.assert_allclose(cond, p[m], rtol=0, atol=tol / tot)


def test_margins_reported(oracle_mod):
    rng = np.random.default_rng(11)
    logits, dl, drafts, u, p, q = _rejection_batch(rng, 100, 4, 16)
    r = oracle_mod.verify(logits, drafts, 4, oracle_mod.REJECTION, draft_logits=dl, uniforms=u,
                          with_margins=True)
    m = r["margins"]
    assert np.isfinite(m[:, -1]).all() and (m[:, -1] >= 0).all()
    for b in range(100):
        j = r["accept_count"][b]
        tested = min(j, 3)                     # accept tests that ran: j-1 accepted + 1 rejected
        assert np.isfinite(m[b, :tested]).all()
        assert np.isinf(m[b, tested:3]).all()


def test_k0_and_k1_sample_row_one(oracle_mod):
    logits = np.array([[[0.0, 3.0, 1.0]]], np.float32)
    for k in (0, 1):
        r = oracle_mod.verify(logits, np.array([[2]], np.int32)[:, :k], k, oracle_mod.GREEDY)
        assert r["accept_count"][0] == 1 and r["out_tokens"][0, 0] == 1
        assert r["selected_block"][0] == k
