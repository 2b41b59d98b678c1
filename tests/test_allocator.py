"""Lifetime-aware width allocation: the oracle against what the pages and arithmetic fix, and the
library's host routine against the oracle (bit-exact; host code, no GPU)."""
import itertools
import math

import numpy as np
import pytest

from oracle import allocate as alo

D = 128
B4, B6, B8, B16 = (alo.head_block_bytes(b, D) for b in (4, 6, 8, 16))


def _convex_instance(rng, H):
    # distortion falling ~4x per 2 bits (convex in bytes), lifetimes log-uniform
    base = rng.lognormal(0.0, 0.5, size=H) * 1e-2
    dist = np.stack([base, base / 4.2 * rng.uniform(0.9, 1.1, H), base / 17.0 * rng.uniform(0.9, 1.1, H)], axis=1)
    half = np.exp(rng.uniform(0.0, math.log(4096.0), size=H))
    return dist, -1.0 / half


def _total_risk(widths, dist, lr):
    idx = {4: 0, 6: 1, 8: 2}
    return sum(0.0 if w == 16 else alo.risk(alo.lifetime_weight(lr[h]), dist[h][idx[w]]) for h, w in enumerate(widths))


def _bytes(widths):
    return sum({4: B4, 6: B6, 8: B8, 16: B16}[w] for w in widths)


def test_head_block_bytes_match_the_documented_layout():
    # codes b*d*d/8, padded to 16, + r and c in fp32, padded to 128; fp16 pivots 2*d*d
    assert (B4, B6, B8, B16) == (9216, 13312, 17408, 32768)
    assert alo.head_block_bytes(6, 16) == 384  # 192 code bytes + 128 scale bytes, padded to 128


def test_lifetime_weight_is_the_expected_memory_lifetime():
    # a memory kept with probability a per token lives 1/(1-a) tokens on average
    for a in (0.5, 0.9, 0.999):
        assert alo.lifetime_weight(math.log(a)) == pytest.approx(1.0 / (1.0 - a), rel=1e-12)
    assert alo.lifetime_weight(0.0) == pytest.approx(1e12)


@pytest.mark.parametrize("seed", range(6))
def test_greedy_matches_brute_force_on_convex_instances(seed):
    """With risk convex in bytes (each further step buys less), taking the best reduction per byte
    first is optimal: compare with every assignment of 6 heads that fits the budget."""
    rng = np.random.default_rng(seed)
    H = 6
    dist, lr = _convex_instance(rng, H)
    budget = int(B4 * H + rng.integers(1, 2 * H) * (B6 - B4))
    got = alo.allocate(dist, lr, D, 0, budget)
    best = min((c for c in itertools.product((4, 6, 8), repeat=H) if _bytes(c) <= budget),
               key=lambda c: _total_risk(c, dist, lr))
    assert _bytes(got) <= budget
    assert _total_risk(got, dist, lr) == pytest.approx(_total_risk(best, dist, lr), rel=1e-12)


def test_budget_pivots_and_degenerate_budgets():
    rng = np.random.default_rng(7)
    H = 40
    dist, lr = _convex_instance(rng, H)
    # the minimum budget gives pivots 16 bits and everyone else 4 bits
    w = alo.allocate(dist, lr, D, 3, 3 * B16 + 37 * B4)
    assert sorted(w).count(16) == 3 and w.count(4) == 37
    # pivots are the three largest 8-bit risks
    R8 = [alo.risk(alo.lifetime_weight(lr[h]), dist[h][2]) for h in range(H)]
    assert {h for h in range(H) if w[h] == 16} == set(np.argsort(R8)[-3:].tolist())
    # an unlimited budget gives every non-pivot head 8 bits
    w = alo.allocate(dist, lr, D, 3, 10 ** 12)
    assert w.count(8) == 37 and w.count(16) == 3
    with pytest.raises(ValueError):
        alo.allocate(dist, lr, D, 3, 3 * B16 + 37 * B4 - 128)


def test_longer_lifetime_never_gets_fewer_bits():
    # identical distortion curves: the allocation is monotone in lifetime
    H = 30
    dist = np.tile([1e-2, 2.5e-3, 6e-4], (H, 1))
    lr = -1.0 / np.exp(np.linspace(0.0, math.log(4096.0), H))
    w = alo.allocate(dist, lr, D, 2, H * B4 + 25 * (B6 - B4))
    order = {4: 0, 6: 1, 8: 2, 16: 3}
    assert all(order[w[h]] <= order[w[h + 1]] for h in range(H - 1))
    assert w[-2:] == [16, 16]


@pytest.mark.parametrize("seed", range(4))
def test_library_matches_oracle(seed):
    import quantized_linear_attention_stq_b200 as stq

    rng = np.random.default_rng(100 + seed)
    H = 300
    dist, lr = _convex_instance(rng, H)
    dist[::7] *= rng.uniform(0.5, 2.0, size=dist[::7].shape)  # some non-convex heads
    dist[5] = dist[6]
    lr[5] = lr[6]  # an exact tie
    npiv = 4
    budget = int(npiv * B16 + (H - npiv) * B4 + rng.integers(0, 2 * H) * (B6 - B4))
    ref = alo.allocate(dist, lr, D, npiv, budget)
    got = stq.allocate_widths(dist, lr, D, npiv, budget)
    assert got == ref


def test_library_rejects_bad_arguments():
    import quantized_linear_attention_stq_b200 as stq

    dist = np.full((4, 3), 1e-3)
    lr = np.full(4, -0.01)
    with pytest.raises(stq.StqError):
        stq.allocate_widths(dist, lr, D, 0, 4 * B4 - 128)
    with pytest.raises(stq.StqError):
        stq.allocate_widths(dist, np.full(4, 0.5), D, 0, 10 ** 9)
    with pytest.raises(stq.StqError):
        stq.allocate_widths(dist, lr, 100, 0, 10 ** 9)
    with pytest.raises(stq.StqError):
        stq.allocate_widths(dist, lr, D, 5, 10 ** 9)


@pytest.mark.parametrize("gate", [0, 1, 2])
def test_row_impact_is_the_readout_sensitivity_of_a_row_error(orc, gate):
    """The impact weight g_i of key row i is what a unit error in row i does to the next readout:
    perturb row i of the state by x, run the oracle's decode update and readout, compare."""
    rng = np.random.default_rng(11 + gate)
    d = 8
    S = rng.normal(size=(d, d))
    q, k, v = rng.normal(size=d), rng.normal(size=d), rng.normal(size=d)
    k /= np.linalg.norm(k)
    beta = 0.7
    alpha = 0.93 if gate == 0 else rng.uniform(0.5, 1.0, size=d)
    w = alo.row_impact([q], [k], [beta], [alpha] if gate == 0 else [alpha], gate)
    _, base = orc.update(gate, S, q, k, v, beta, alpha)
    for i in range(d):
        x = rng.normal(size=d)
        Sp = S.copy()
        Sp[i] += x
        _, o = orc.update(gate, Sp, q, k, v, beta, alpha)
        ratio = (o - base) / x
        # the readout moves by g_i * x: one common factor, whose square is w_i
        assert np.allclose(ratio, ratio[0], rtol=1e-9, atol=1e-12)
        assert ratio[0] ** 2 == pytest.approx(w[i], rel=1e-9, abs=1e-15)


def test_row_impact_special_cases():
    rng = np.random.default_rng(3)
    d, T = 6, 5
    q = rng.normal(size=(T, d))
    k = rng.normal(size=(T, d))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    # beta = 0: the weight is the decayed query
    w = alo.row_impact(q, k, np.zeros(T), np.full(T, 0.8))
    assert np.allclose(w, (0.64 * q ** 2).mean(axis=0), rtol=1e-12)
    # q = k (unit) and beta = 1: the delta rule erases what the query would read
    w = alo.row_impact(k, k, np.ones(T), np.ones(T))
    assert np.allclose(w, 0.0, atol=1e-24)
