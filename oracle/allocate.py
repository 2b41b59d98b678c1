"""Oracle of the lifetime-aware width allocation (plain Python, slow, obviously correct).

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` alone; the product library never imports it.

The pages' time dimension ("线性注意力状态量化难题" (aitest123.com/news/n1kj09), section 时间维度;
"K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), section 方法): errors of a state unit live as
long as its memory, so for every head two calibration quantities are estimated, the reconstruction
distortion at each candidate width and the mean log-retention of its gate; combined they give a
lifetime weight, and under a fixed bit budget the widths are chosen so that units with large error
and long lifetime get the higher precision. The few highest-risk heads, which no width tames, are
kept in FP16 as sparse pivots (about 1.4% of the heads).

Readings (the pages fix no formula):
  * lifetime weight  lam_h = 1 / max(1 - exp(l_h), 1e-12), the expected lifetime in tokens of a
    memory whose per-token retention is exp(l_h) (l_h = mean log-retention <= 0);
  * risk at a width  R_h(b) = lam_h * D_h(b);
  * pivots: the `num_pivots` heads of largest R_h(8) (ties: lower head index first);
  * the other heads start at 4 bits and are upgraded one step at a time (4 -> 6 -> 8), always the
    step of largest risk reduction per extra byte (ties: lower head index), skipping steps that
    would exceed the budget, until no step fits;
  * the budget is the state bytes of one request (head block bytes, layout of include/stq.h).
"""
from __future__ import annotations

import math

WIDTHS = (4, 6, 8)


def _round_up(x: int, a: int) -> int:
    return (x + a - 1) // a * a


def head_block_bytes(bits: int, d: int) -> int:
    """Bytes of one head block (codes, padding to 16 B, r and c in fp32, padding to 128 B)."""
    if bits == 16:
        return _round_up(2 * d * d, 128)
    codes = (bits * d * d + 7) // 8
    return _round_up(_round_up(codes, 16) + 8 * d, 128)


def lifetime_weight(mean_log_retention: float) -> float:
    return 1.0 / max(-math.expm1(mean_log_retention), 1e-12)


def risk(lam: float, dist: float) -> float:
    if dist == 0.0:
        return 0.0
    return lam * dist


def allocate(distortion, mean_log_retention, d: int, num_pivots: int, budget_bytes: int):
    """Widths per head (4, 6, 8 or 16). distortion[h][k] is D_h at width WIDTHS[k]."""
    H = len(mean_log_retention)
    if not (0 <= num_pivots <= H):
        raise ValueError("num_pivots out of range")
    lam = [lifetime_weight(float(x)) for x in mean_log_retention]
    R = [[risk(lam[h], float(distortion[h][k])) for k in range(3)] for h in range(H)]
    # pivots: largest 8-bit risk, lower head index first on ties
    order = sorted(range(H), key=lambda h: (-R[h][2], h))
    pivots = set(order[:num_pivots])
    level = [None if h in pivots else 0 for h in range(H)]
    total = 0
    for h in range(H):
        total += head_block_bytes(16, d) if h in pivots else head_block_bytes(WIDTHS[0], d)
    total = _round_up(total, 128)
    if total > budget_bytes:
        raise ValueError("budget below the smallest allocation")
    blocked = set()
    while True:
        best = None
        for h in range(H):
            if level[h] is None or level[h] == 2 or h in blocked:
                continue
            k = level[h]
            extra = head_block_bytes(WIDTHS[k + 1], d) - head_block_bytes(WIDTHS[k], d)
            gain = (R[h][k] - R[h][k + 1]) / extra
            if best is None or gain > best[0]:
                best = (gain, h, extra)
        if best is None:
            break
        _, h, extra = best
        if total + extra <= budget_bytes:
            level[h] += 1
            total += extra
        else:
            blocked.add(h)
    return [16 if level[h] is None else WIDTHS[level[h]] for h in range(H)]


def row_impact(q, k, beta, alpha, gate: int = 0):
    """Key-row impact scores of one head over calibration tokens ("线性注意力状态量化难题",
    section 空间维度: the output error is the sum over key rows of each row's accumulated error
    times a weight set by the current key, query and gate; the row impact score is that weight's
    mean square). One update S' = A(S) carries a state error E to E' and the next readout error
    is E'^T q = E^T g, so row i's weight is g_i:
      scalar gate            g = a (q - b (k.q) k)
      channel gate (literal) g = a*q - b (k.(a*q)) k          (S' = diag(a)(S - b k k^T S) + ...)
      channel, decay first   g = a * (q - b (k.q) k)          (S' = diag(a) S - b k k^T diag(a) S + ...)
    q, k: [T][d]; beta: [T]; alpha: [T] (scalar gate) or [T][d]. Returns w[d] = mean_t g_t^2."""
    T = len(q)
    d = len(q[0])
    acc = [0.0] * d
    for t in range(T):
        qt = [float(x) for x in q[t]]
        kt = [float(x) for x in k[t]]
        b = float(beta[t])
        a = [float(alpha[t])] * d if gate == 0 else [float(x) for x in alpha[t]]
        if gate == 1:
            aq = [a[i] * qt[i] for i in range(d)]
            kaq = sum(kt[i] * aq[i] for i in range(d))
            g = [aq[i] - b * kaq * kt[i] for i in range(d)]
        else:
            kq = sum(kt[i] * qt[i] for i in range(d))
            g = [a[i] * (qt[i] - b * kq * kt[i]) for i in range(d)]
        for i in range(d):
            acc[i] += g[i] * g[i]
    return [x / T for x in acc]
