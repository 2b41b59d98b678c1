"""Helpers shared by the GPU parity tests: oracle-side pool assembly and tile comparison.

The parity rule (codes, scales, readout):
  * every integer code equal to the oracle's, except a difference of exactly 1 where the oracle
    flags the real-valued code as a rounding near-tie (|frac(x) - 1/2| <= 1e-3); such differences
    stay below 1e-4 of the codes checked;
  * stored fp32 scales within 2e-3 relative (expected: a few fp32 ulps);
  * readout o within 2e-3 of max|o| of the oracle's fp64 readout rounded to fp32;
  * FP16 pivot values are floating-point state, compared as such. After one decode update: every
    value within one fp16 quantum of the oracle's plus the fp32 evaluation error of the update,
    2^-18 * M_ij, where M_ij = |alpha| |S_ij| + beta |k_i| (|v_j| + |alpha| sum_l |k_l| |S_lj|)
    is the magnitude of the terms that form S'_ij (an element born of cancellation has a tiny fp16
    quantum but an fp32 error set by those terms); and at most 1e-3 of the values not
    bit-identical (a wrong rounding mode or a dropped term would move far more). After a prefill
    chunk of T fp32 updates (compare_pivot_exact): each GPU value must be a correct fp16 rounding
    of some value within a per-element bound b_ij of the exact fp64 state, the bound carried
    through the chunk's updates by pivot_chunk_exact; the oracle's own value must satisfy the same
    rule with b = 0; and at most PIVOT_CHUNK_DIFF_BUDGET of the values may differ from the
    oracle's bit for bit, whatever T (the bound alone, sound but loose, would not catch a wrong
    rounding mode).
Inputs always flow from the generator (or the oracle) to the GPU, never back into the oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

CODE_TIE_BUDGET = 1e-4
SCALE_RTOL = 2e-3
O_TOL = 2e-3
PIVOT_DIFF_BUDGET = 1e-3
PIVOT_EVAL_ERR = 2.0 ** -18  # fp32 evaluation error of one update, relative to its term magnitude
# Pivot values after a prefill chunk that may differ from the oracle's, whatever the chunk length.
# An fp32 emulation of 64-token chunks (d = 32 and 128, all three gates) differs in 0.03% to 0.23%
# of the values; rounding toward zero instead of to nearest would differ in about half.
PIVOT_CHUNK_DIFF_BUDGET = 1e-2
FIT_OUTLIER_BUDGET = 1e-2


@dataclasses.dataclass
class Tally:
    codes: int = 0
    tie_flips: int = 0
    max_scale_rel: float = 0.0
    max_o_rel: float = 0.0
    pivot_values: int = 0        # pivot values checked after one update (budgeted rule)
    pivot_diffs: int = 0
    pivot_exact_values: int = 0  # pivot values checked by the per-value rule after a chunk
    pivot_exact_diffs: int = 0   # of which not bit-identical to the oracle's
    scales: int = 0              # bf16 scales checked
    scale_flips: int = 0         # of which one bf16 step off the oracle's, at a flagged near-tie
    fit_scale_outliers: int = 0  # jointly refined scales beyond SCALE_RTOL (within 10x)

    def check_budget(self):
        assert self.codes + self.pivot_values + self.pivot_exact_values > 0
        assert self.tie_flips <= CODE_TIE_BUDGET * self.codes, f"{self.tie_flips} tie flips in {self.codes} codes"
        assert self.pivot_diffs <= PIVOT_DIFF_BUDGET * self.pivot_values, \
            f"{self.pivot_diffs} of {self.pivot_values} fp16 pivot values differ"
        assert self.pivot_exact_diffs <= PIVOT_CHUNK_DIFF_BUDGET * self.pivot_exact_values, \
            f"{self.pivot_exact_diffs} of {self.pivot_exact_values} fp16 pivot values differ after a chunk"
        assert self.fit_scale_outliers <= FIT_OUTLIER_BUDGET * self.scales + 2, \
            f"{self.fit_scale_outliers} of {self.scales} refined scales beyond {SCALE_RTOL}"
        assert self.scale_flips <= SCALE_FLIP_BUDGET * self.scales + 2, \
            f"{self.scale_flips} of {self.scales} bf16 scales one step off"


def oracle_pool(orc, head_bits, d, blocks_per_request):
    """Assemble request blocks (list over requests of list over heads of block bytes)."""
    offs, total = orc.request_layout(head_bits, d, d)
    pool = np.zeros(len(blocks_per_request) * total, dtype=np.uint8)
    for r, blocks in enumerate(blocks_per_request):
        for h, blk in enumerate(blocks):
            pool[r * total + offs[h]: r * total + offs[h] + blk.size] = blk
    return pool


def tile_bytes(orc, pool, head_bits, d, slot, h):
    offs, total = orc.request_layout(head_bits, d, d)
    n = orc.block_bytes(int(head_bits[h]), d, d)
    start = slot * total + offs[h]
    return np.asarray(pool[start: start + n])


def update_magnitude(S, k, v, beta, alpha):
    """M_ij of the pivot tolerance: magnitude of the terms of one update of S (fp64)."""
    a = float(np.max(np.abs(alpha)))
    S, k, v = np.abs(S), np.abs(np.asarray(k, dtype=np.float64)), np.abs(np.asarray(v, dtype=np.float64))
    return a * S + beta * k[:, None] * (v[None, :] + a * (k @ S)[None, :])


def fp16_quantum(x):
    ax = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(ax)) - 10)


def pivot_chunk_exact(orc, gate, S0, q, k, v, beta, alpha):
    """The exact (fp64, oracle) state after a chunk's updates of S0, and a per-element bound on
    how far a kernel's fp32 state can be from it.

    Each update t adds a fresh error e_t with |e_t| <= PIVOT_EVAL_ERR * M(t) elementwise (M from
    update_magnitude on the state before the update) and carries the error E so far through the
    linear map A_t of the update: A X = a (X - beta k k^T X) for the scalar gate, diag(alpha)(X -
    beta k k^T X) or (I - beta k k^T) diag(alpha) X for the channel gates. Elementwise,
    |(A X)_ij| <= a (|X_ij| + beta |k_i| |k| |X_:j|) with a = max |alpha|, and column norms obey
    |(A X)_:j| <= a max(1, |1 - beta |k|^2|) |X_:j|. Carrying an elementwise bound b and a
    column-norm bound n through the chunk gives b, sound for every element (a bound by column
    norms alone would be loose on small elements; one by elementwise absolute values alone grows
    by (1 + beta |k_i| sum |k_l|) per update)."""
    S = np.asarray(S0, dtype=np.float64).copy()
    b = np.zeros_like(S)
    n = np.zeros(S.shape[1])
    for t in range(len(beta)):
        at = np.atleast_1d(np.asarray(alpha[t], dtype=np.float64))
        kt = np.asarray(k[t], dtype=np.float64)
        bt = float(beta[t])
        eps = PIVOT_EVAL_ERR * update_magnitude(S, kt, v[t], bt, at)
        a = float(np.max(np.abs(at)))
        kn = float(np.linalg.norm(kt))
        b = a * (b + bt * kn * np.abs(kt)[:, None] * n[None, :]) + eps
        n = a * max(1.0, abs(1.0 - bt * kn * kn)) * n + np.sqrt((eps ** 2).sum(axis=0))
        S, _ = orc.update(gate, S, q[t], kt, v[t], bt, at)
    return S, b


def compare_pivot_exact(orc, d, got, ref_block, S_exact, bound, tally: Tally, what=""):
    """A pivot block after a chunk: every GPU fp16 value must round some value within `bound` of
    the exact state S_exact (|g - S| <= bound + half an fp16 step at g); values equal to the
    oracle's bit for bit always pass (both overflowed to the same infinity included). The
    oracle's own values must pass with bound 0, which checks that S_exact is the state the oracle
    rounded."""
    gb = orc.pivot_values(d, d, np.asarray(got, dtype=np.uint8))
    rb = orc.pivot_values(d, d, np.asarray(ref_block, dtype=np.uint8))
    gv = gb.view(np.float16).astype(np.float64)
    rv = rb.view(np.float16).astype(np.float64)
    half = 0.5 * (1.0 + 2.0 ** -9)
    fin = np.isfinite(rv)
    assert (np.abs(rv - S_exact) <= half * fp16_quantum(rv))[fin].all(), f"{what}: oracle state sequence mismatch"
    ok = (gb == rb) | (np.abs(gv - S_exact) <= bound + half * fp16_quantum(gv))
    if not ok.all():
        i, j = np.argwhere(~ok)[0]
        raise AssertionError(f"{what}: {int((~ok).sum())} fp16 values outside the rounding rule, first at ({i},{j}): "
                             f"gpu {gv[i, j]!r} oracle {rv[i, j]!r} exact {S_exact[i, j]!r} bound {bound[i, j]!r}")
    tally.pivot_exact_values += gb.size
    tally.pivot_exact_diffs += int((gb != rb).sum())


def compare_block(orc, bits, d, got, ref_block, ref_tie, tally: Tally, what="", err_scale=None):
    got = np.asarray(got, dtype=np.uint8)
    ref_block = np.asarray(ref_block, dtype=np.uint8)
    if bits == 16:
        gb = orc.pivot_values(d, d, got)
        rb = orc.pivot_values(d, d, ref_block)
        gv = gb.view(np.float16).astype(np.float64)
        rv = rb.view(np.float16).astype(np.float64)
        tol = fp16_quantum(rv) + (0.0 if err_scale is None else PIVOT_EVAL_ERR * err_scale)
        bad = ~(np.abs(gv - rv) <= tol)
        if bad.any():
            i, j = np.argwhere(bad)[0]
            raise AssertionError(f"{what}: {int(bad.sum())} fp16 values outside tolerance, first at ({i},{j}): "
                                 f"gpu {gv[i, j]!r} oracle {rv[i, j]!r} tol {tol[i, j]!r}")
        tally.pivot_values += gb.size
        tally.pivot_diffs += int((gb != rb).sum())
        return
    Qg = orc.codes(bits, d, d, got)
    Qr = orc.codes(bits, d, d, ref_block)
    diff = np.abs(Qg - Qr)
    bad = (diff > 1) | ((diff == 1) & ~ref_tie)
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} codes differ off a tie, first at ({i},{j}): "
                             f"gpu {Qg[i, j]} oracle {Qr[i, j]}")
    tally.codes += Qg.size
    tally.tie_flips += int((diff == 1).sum())
    rg, cg = orc.scales(bits, d, d, got)
    rr, cr = orc.scales(bits, d, d, ref_block)
    rel = max(np.max(np.abs(rg.astype(np.float64) - rr) / np.abs(rr)),
              np.max(np.abs(cg.astype(np.float64) - cr) / np.abs(cr)))
    assert rel <= SCALE_RTOL, f"{what}: scale rel error {rel}"
    tally.max_scale_rel = max(tally.max_scale_rel, float(rel))
    # bytes outside codes and scales (padding) must stay zero
    n_used = orc.scale_offset(bits, d, d) + 8 * d
    pad_start = orc.codes_bytes(bits, d, d)
    assert not got[pad_start: orc.scale_offset(bits, d, d)].any()
    assert not got[n_used:].any()


def uniform_request_layout(orc, head_bits, d):
    """Offsets and request bytes of a uniformly scaled layout: 4/6/8-bit heads take the
    single-scale block, FP16 pivot heads their usual block, the request padded to 128 bytes."""
    offs, pos = [], 0
    for b in head_bits:
        offs.append(pos)
        pos += orc.block_bytes(16, d, d) if int(b) == 16 else orc.uniform_block_bytes(int(b), d, d)
    return offs, (pos + 127) // 128 * 128


def compare_uniform_block(orc, bits, d, got, ref_block, ref_tie, tally: Tally, what=""):
    """Codes and the one scale of a uniformly scaled head (the rule above, with the single scale
    in place of the row and column scales); padding stays zero."""
    got = np.asarray(got, dtype=np.uint8)
    ref_block = np.asarray(ref_block, dtype=np.uint8)
    Qg = orc.codes(bits, d, d, got)
    Qr = orc.codes(bits, d, d, ref_block)
    diff = np.abs(Qg - Qr)
    bad = (diff > 1) | ((diff == 1) & ~ref_tie)
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} codes differ off a tie, first at ({i},{j}): "
                             f"gpu {Qg[i, j]} oracle {Qr[i, j]}")
    tally.codes += Qg.size
    tally.tie_flips += int((diff == 1).sum())
    sg = orc.uniform_scale(bits, d, d, got)
    sr = orc.uniform_scale(bits, d, d, ref_block)
    rel = abs(sg - sr) / abs(sr)
    assert rel <= SCALE_RTOL, f"{what}: scale rel error {rel}"
    tally.max_scale_rel = max(tally.max_scale_rel, float(rel))
    so = orc.scale_offset(bits, d, d)
    assert not got[orc.codes_bytes(bits, d, d): so].any()
    assert not got[so + 4:].any()


SCALE_FLIP_BUDGET = 2e-3


def _bf16_neighbours(orc, a, b):
    """a and b are adjacent bf16 values (patterns one apart, same sign)."""
    ha, hb = orc.double_to_bf16(float(a)), orc.double_to_bf16(float(b))
    return (ha & 0x8000) == (hb & 0x8000) and abs(ha - hb) == 1


def compare_block_bf16s(orc, bits, d, got, S_new, w, tally: Tally, what=""):
    """A head block with bf16 row and column scales against the oracle's requantization of the
    same updated state S_new (fp64). A stored bf16 scale may differ from the oracle's by one bf16
    step only where the oracle flags the exact scale as a rounding near-tie; the oracle then
    continues with the GPU's stored scales (column scales first, then rows: codes follow the
    stored scales), and the codes are compared with the code rule above. Flipped scales stay
    below SCALE_FLIP_BUDGET of the scales checked (counted in tally.scale_flips)."""
    got = np.asarray(got, dtype=np.uint8)
    sf = orc.SCALE_BF16
    rg, cg = orc.scales_s(bits, sf, d, d, got)
    blk, x, tie, stie, st = orc.quantize_s(bits, sf, S_new, w)
    assert st == orc.OK
    ro, co = orc.scales_s(bits, sf, d, d, blk)
    for name, gv, ov, flags in (("column", cg, co, stie[d:]), ):
        diff = gv != ov
        bad = diff & ~(flags & np.array([_bf16_neighbours(orc, a, b) for a, b in zip(gv, ov)]))
        assert not bad.any(), f"{what}: {name} scale {int(np.argmax(bad))} gpu {gv[bad][0]!r} oracle {ov[bad][0]!r}"
        tally.scale_flips += int(diff.sum())
    if (cg != co).any():
        blk, x, tie, stie, st = orc.quantize_s(bits, sf, S_new, w, c_given=cg)
        ro = orc.scales_s(bits, sf, d, d, blk)[0]
    diff = rg != ro
    bad = diff & ~(stie[:d] & np.array([_bf16_neighbours(orc, a, b) for a, b in zip(rg, ro)]))
    assert not bad.any(), f"{what}: row scale {int(np.argmax(bad))} gpu {rg[bad][0]!r} oracle {ro[bad][0]!r}"
    tally.scale_flips += int(diff.sum())
    tally.scales += 2 * d
    if diff.any():
        blk, x, tie, _, st = orc.quantize_s(bits, sf, S_new, w, c_given=cg, r_given=rg)
    Qg = orc.codes(bits, d, d, got)
    Qr = orc.codes(bits, d, d, blk)
    cdiff = np.abs(Qg - Qr)
    badc = (cdiff > 1) | ((cdiff == 1) & ~tie)
    if badc.any():
        i, j = np.argwhere(badc)[0]
        raise AssertionError(f"{what}: {int(badc.sum())} codes differ off a tie, first at ({i},{j}): "
                             f"gpu {Qg[i, j]} oracle {Qr[i, j]} x {x[i, j]!r}")
    tally.codes += Qg.size
    tally.tie_flips += int((cdiff == 1).sum())
    so = orc.scale_offset(bits, d, d)
    assert not got[orc.codes_bytes(bits, d, d): so].any()
    assert not got[so + 4 * d:].any()


def compare_block_fit(orc, bits, d, got, S_new, w, rounds, tally: Tally, what="", sfmt=0):
    """A head block whose fp32 scales went through `rounds` rounds of the joint refinement,
    against the oracle's refinement of the same updated state S_new (fp64). The refinement
    recomputes codes between its least-squares steps, so a code that flips at a near-tie in an
    intermediate round moves the later scales: most in a column or row with few nonzero codes,
    where one code carries a large share of the least-squares sums (an fp32 emulation of the
    refinement moves about one scale in 10^4 by up to 4e-3 relative). So the stored scales are
    within the scale tolerance above except at most FIT_OUTLIER_BUDGET of them, which stay within
    10x that; the codes must be the oracle's requantization with the GPU's stored scales (code rule
    above); and the impact-weighted reconstruction error of the GPU's block, the quantity the
    refinement minimises, may exceed the oracle's by at most 1e-3 relative."""
    got = np.asarray(got, dtype=np.uint8)
    blk, _, _, st = orc.quantize_fit(bits, sfmt, rounds, S_new, w)
    assert st == orc.OK
    rg, cg = orc.scales_s(bits, sfmt, d, d, got)
    ro, co = orc.scales_s(bits, sfmt, d, d, blk)
    rels = np.concatenate([np.abs(rg - ro) / ro, np.abs(cg - co) / co])
    # with bf16 storage a refitted scale may also land one bf16 step (<= 2^-7 relative) away
    tol = SCALE_RTOL if sfmt == orc.SCALE_F32 else SCALE_RTOL + 2.0 ** -7
    assert rels.max() <= 10 * tol, f"{what}: scale rel error {rels.max()}"
    tally.scales += rels.size
    tally.fit_scale_outliers += int((rels > tol).sum())
    tally.max_scale_rel = max(tally.max_scale_rel, float(rels.max()))
    req, x, tie, _, st = orc.quantize_s(bits, sfmt, S_new, w, c_given=cg, r_given=rg)
    Qg = orc.codes(bits, d, d, got)
    Qr = orc.codes(bits, d, d, req)
    cdiff = np.abs(Qg - Qr)
    badc = (cdiff > 1) | ((cdiff == 1) & ~tie)
    if badc.any():
        i, j = np.argwhere(badc)[0]
        raise AssertionError(f"{what}: {int(badc.sum())} codes differ off a tie, first at ({i},{j}): "
                             f"gpu {Qg[i, j]} oracle {Qr[i, j]} x {x[i, j]!r}")
    tally.codes += Qg.size
    tally.tie_flips += int((cdiff == 1).sum())

    def werr(r, c, Q):
        return float((w[:, None] * (S_new - r[:, None] * c[None, :] * Q) ** 2).sum())

    e_gpu, e_orc = werr(rg, cg, Qg), werr(ro, co, orc.codes(bits, d, d, blk))
    assert e_gpu <= e_orc * (1 + 1e-3) + 1e-300, f"{what}: weighted error {e_gpu} against the oracle's {e_orc}"
    so = orc.scale_offset(bits, d, d)
    assert not got[orc.codes_bytes(bits, d, d): so].any()
    assert not got[so + (8 if sfmt == orc.SCALE_F32 else 4) * d:].any()


def compare_o(got, ref, tally: Tally, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = max(np.max(np.abs(ref)), 1e-30)
    rel = np.max(np.abs(got - ref)) / scale
    assert rel <= O_TOL, f"{what}: o rel error {rel}"
    tally.max_o_rel = max(tally.max_o_rel, float(rel))


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()
