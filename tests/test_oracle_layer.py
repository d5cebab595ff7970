"""Pins for the oracle's layer-level pieces (CPU only): zone positions, the
rotary embedding and the linear layer.

  * positions: the hand-worked table in tests/golden/positions_k3.txt; and the
    hand-off between steps -- with j drafts accepted the next step starts at
    P + j, and block j's slots must sit exactly where the next step's rows
    d_1 (= t*) .. d_k sit;
  * rotary embedding: against an independent formulation (each pair as a
    complex number times e^{i angle}, numpy complex128); norm preservation;
    position 0 is the identity; a score between a rotated query and key depends
    only on the difference of their positions;
  * linear: against numpy's matmul in fp64, bf16 inputs widened exactly.
"""
import numpy as np
import pytest

from conftest import read_golden


def _golden():
    lines = read_golden("positions_k3.txt")
    vals = {}
    for ln in lines:
        parts = ln.split()
        if parts[0] == "k0":
            vals["k0"] = (int(parts[2]), [int(v) for v in parts[4:]])
        elif parts[0] == "positions":
            vals["positions"] = [int(v) for v in parts[1:]]
        else:
            vals[parts[0]] = int(parts[1])
    return vals


def test_golden_positions(oracle_mod):
    g = _golden()
    assert list(oracle_mod.zone_positions(g["k"], g["P"])) == g["positions"]
    P0, want0 = g["k0"]
    assert list(oracle_mod.zone_positions(0, P0)) == want0


@pytest.mark.parametrize("k", [1, 2, 3, 8, 16])
def test_block_positions_hand_off_to_the_next_step(oracle_mod, k):
    P = 1000
    pos = oracle_mod.zone_positions(k, P)
    for j in range(1, k + 1):
        nxt = oracle_mod.zone_positions(k, P + j)      # j drafts accepted
        block = pos[k + (j - 1) * k: k + j * k]
        assert list(block) == list(nxt[:k]), j
    # drafts are consecutive after the prefix
    assert list(pos[:k]) == list(range(P, P + k))


def _rope_complex(x, pos, base):
    rows, H, D = x.shape
    half = D // 2
    f = np.arange(half)
    ang = np.asarray(pos, np.float64)[:, None] * base ** (-2.0 * f / D)[None, :]
    z = x[..., :half].astype(np.float64) + 1j * x[..., half:].astype(np.float64)
    z = z * np.exp(1j * ang)[:, None, :]
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("D,base", [(64, 10000.0), (128, 1e6), (8, 10.0)])
def test_rope_is_a_complex_rotation(oracle_mod, D, base):
    rng = np.random.default_rng(D)
    x = rng.normal(size=(7, 3, D)).astype(np.float32)
    pos = np.array([0, 1, 2, 17, 1000, 8191, 131071])
    got = oracle_mod.rope(x, pos, base)
    # angles reach ~1.3e5 rad, whose fp64 rounding (~1e-11) the two
    # formulations do differently; a wrong sign, pair or frequency is O(1)
    np.testing.assert_allclose(got, _rope_complex(x, pos, base), rtol=0, atol=1e-9)
    np.testing.assert_allclose(np.linalg.norm(got, axis=-1),
                               np.linalg.norm(x.astype(np.float64), axis=-1), rtol=1e-13)
    np.testing.assert_array_equal(got[0], x[0].astype(np.float64))     # position 0


def test_rope_scores_depend_on_relative_position(oracle_mod):
    rng = np.random.default_rng(3)
    D = 128
    q = rng.normal(size=(1, 1, D)).astype(np.float32)
    k = rng.normal(size=(1, 1, D)).astype(np.float32)
    def score(m, n):
        return float(np.dot(oracle_mod.rope(q, [m]).ravel(), oracle_mod.rope(k, [n]).ravel()))
    for m, n, t in [(5, 2, 100), (40, 40, 7), (3, 900, 2048)]:
        assert score(m, n) == pytest.approx(score(m + t, n + t), rel=1e-9, abs=1e-9)
    # and it does change with the difference
    assert abs(score(5, 2) - score(6, 2)) > 1e-6


def test_rope_bf16_input_widened_exactly(oracle_mod):
    import torch
    rng = np.random.default_rng(4)
    x32 = torch.tensor(rng.normal(size=(3, 2, 16)), dtype=torch.float32)
    xb = x32.to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle_mod.rope(bits, [0, 5, 9]),
                                  oracle_mod.rope(xb.float().numpy(), [0, 5, 9]))


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (5, 7, 3), (17, 33, 64)])
def test_linear_matches_numpy(oracle_mod, M, N, K):
    rng = np.random.default_rng(M * N + K)
    x = rng.normal(size=(M, K)).astype(np.float32)
    w = rng.normal(size=(N, K)).astype(np.float32)
    got = oracle_mod.linear(x, w)
    np.testing.assert_allclose(got, x.astype(np.float64) @ w.astype(np.float64).T, rtol=1e-12,
                               atol=1e-12)
