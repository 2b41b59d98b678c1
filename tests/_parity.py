"""Helpers shared by the GPU parity tests: oracle-side pool assembly and tile comparison.

The parity rule (codes, scales, readout):
  * every integer code equal to the oracle's, except a difference of exactly 1 where the oracle
    flags the real-valued code as a rounding near-tie (|frac(x) - 1/2| <= 1e-3); such differences
    stay below 1e-4 of the codes checked;
  * stored fp32 scales within 2e-3 relative (expected: a few fp32 ulps);
  * readout o within 2e-3 of max|o| of the oracle's fp64 readout rounded to fp32;
  * FP16 pivot values equal, or one fp16 quantum apart where the oracle flags a near-tie.
Inputs always flow from the generator (or the oracle) to the GPU, never back into the oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

CODE_TIE_BUDGET = 1e-4
SCALE_RTOL = 2e-3
O_TOL = 2e-3


@dataclasses.dataclass
class Tally:
    codes: int = 0
    tie_flips: int = 0
    max_scale_rel: float = 0.0
    max_o_rel: float = 0.0
    pivot_values: int = 0
    pivot_flips: int = 0

    def check_budget(self):
        total = self.codes + self.pivot_values
        flips = self.tie_flips + self.pivot_flips
        assert total > 0
        assert flips <= CODE_TIE_BUDGET * total, f"{flips} tie flips in {total} codes"


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


def compare_block(orc, bits, d, got, ref_block, ref_tie, tally: Tally, what=""):
    got = np.asarray(got, dtype=np.uint8)
    ref_block = np.asarray(ref_block, dtype=np.uint8)
    if bits == 16:
        g = orc.pivot_values(d, d, got).astype(np.int32)
        r = orc.pivot_values(d, d, ref_block).astype(np.int32)
        diff = np.abs(g - r)
        bad = (diff > 1) | ((diff == 1) & ~ref_tie)
        assert not bad.any(), f"{what}: {int(bad.sum())} fp16 values differ off a tie"
        tally.pivot_values += g.size
        tally.pivot_flips += int((diff == 1).sum())
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


def compare_o(got, ref, tally: Tally, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = max(np.max(np.abs(ref)), 1e-30)
    rel = np.max(np.abs(got - ref)) / scale
    assert rel <= O_TOL, f"{what}: o rel error {rel}"
    tally.max_o_rel = max(tally.max_o_rel, float(rel))


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()
