"""Seeded synthetic workloads for the quantized-state decode and prefill path.

This module only draws inputs. It holds none of the method's arithmetic (no update, readout,
scale fit or quantization) and imports nothing else from this package, so the tests can hand the
same arrays to the CUDA path and to the CPU oracle.

The distributions stand in for the pages' calibration traces (C4 / WikiText-2 over the 2304
recurrent heads of Qwen3.8-27B; "线性注意力状态量化难题" (aitest123.com/news/n1kj09), sections
时间维度 and 空间维度; "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), section 方法), which
are not available here:
  q, k ~ N(0, I), then L2-normalised;  v ~ N(0, I);  beta = sigmoid(N(0, 1)) per token and head;
  w_i ~ lognormal(0, 1) per head and key row;  S0 = diag(a) G diag(b), G ~ N(0, 1),
  a, b ~ lognormal(0, 0.8);  gate half-life h ~ log-uniform[1, 4096] tokens, alpha = exp(-1/h).
The full 2304-head workload also plants the row / column outliers the pages measure on Qwen's
states (row max/median ~10.3x, column ~19.4x; section 空间维度) and the per-head widths 4/6/8 bits
with ~1.4% FP16 pivot heads on the longest half-lives (section 时间维度).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

GATE_SCALAR, GATE_CHANNEL, GATE_CHANNEL_DECAY_FIRST = 0, 1, 2

# stream ids of the seeded generators (one independent stream per tensor kind)
_S_HALF, _S_BITS, _S_W, _S_A, _S_B, _S_G, _S_Q, _S_K, _S_V, _S_BETA = range(10)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    d: int
    steps: int
    bits: Optional[int]          # uniform width, or None for the mixed 2304-head workload
    in_dtype: torch.dtype
    gate: int
    seed: int
    fixed_half_life: Optional[float] = None
    outliers: bool = False
    prompt: int = 0
    chunk: int = 64

    @property
    def tiles(self) -> int:
        return self.batch * self.heads


WORKLOADS = {
    # 1 request x 1 head, d=16, 64 steps, 6-bit, fp32 inputs, h = 256: the small parity case
    "pr1_d16_6bit": Workload("pr1_d16_6bit", 1, 1, 16, 64, 6, torch.float32, GATE_SCALAR, 0,
                             fixed_half_life=256.0),
    # one layer of 48 heads, d=128, 8 requests, 512 steps, 4-bit, bf16
    "layer48_b8_4bit": Workload("layer48_b8_4bit", 8, 48, 128, 512, 4, torch.bfloat16,
                                GATE_SCALAR, 1),
    # 48 layers x 48 heads, d=128, 70 requests, 256 tokens, mixed 4/6/8 + FP16 pivots, bf16
    "full2304_b70_mixed": Workload("full2304_b70_mixed", 70, 2304, 128, 256, None,
                                   torch.bfloat16, GATE_SCALAR, 2, outliers=True),
    # channel-wise gate, 32 heads, d=128, 128 requests, 2048 steps, 4-bit, bf16
    "channel32_b128_4bit": Workload("channel32_b128_4bit", 128, 32, 128, 2048, 4,
                                    torch.bfloat16, GATE_CHANNEL, 3),
    # chunked prefill of 8192 tokens (chunks of 64), then 1024 decode steps; 16 heads, 16 req.
    "prefill16_b16_6bit": Workload("prefill16_b16_6bit", 16, 16, 128, 1024, 6, torch.bfloat16,
                                   GATE_SCALAR, 4, prompt=8192),
}

# exact head counts of the mixed workload: largest-remainder rounding of 40 / 45 / 13.6 / 1.4 %
MIXED_COUNTS = {4: 922, 6: 1037, 8: 313, 16: 32}
ROW_OUTLIER, COL_OUTLIER = 10.3, 19.4


def _gen(wl: Workload, stream: int, index: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((wl.seed * 1_000_003 + stream * 10_007 + index * 7_919 + 12345) % (2 ** 62))
    return g


def half_lives(wl: Workload) -> torch.Tensor:
    """Gate half-life per head [H] (or per head and key row [H, d] for the channel gate)."""
    shape = (wl.heads, wl.d) if wl.gate != GATE_SCALAR else (wl.heads,)
    if wl.fixed_half_life is not None:
        return torch.full(shape, wl.fixed_half_life, dtype=torch.float64)
    u = torch.rand(shape, generator=_gen(wl, _S_HALF, 0, "cpu"), dtype=torch.float64)
    return torch.exp(u * math.log(4096.0))


def gate_values(wl: Workload) -> torch.Tensor:
    """alpha = exp(-1/h), constant over tokens: [H] or [H, d] (fp32)."""
    return torch.exp(-1.0 / half_lives(wl)).to(torch.float32)


def head_bits(wl: Workload) -> list:
    if wl.bits is not None:
        return [wl.bits] * wl.heads
    assert sum(MIXED_COUNTS.values()) == wl.heads
    h = half_lives(wl)
    order = torch.argsort(h, descending=True)
    bits = [0] * wl.heads
    pivots = order[: MIXED_COUNTS[16]].tolist()
    for p in pivots:
        bits[p] = 16
    rest = order[MIXED_COUNTS[16]:]
    pool = [4] * MIXED_COUNTS[4] + [6] * MIXED_COUNTS[6] + [8] * MIXED_COUNTS[8]
    perm = torch.randperm(len(pool), generator=_gen(wl, _S_BITS, 0, "cpu")).tolist()
    for slot, p in zip(rest.tolist(), perm):
        bits[slot] = pool[p]
    return bits


def impact_weights(wl: Workload, device="cpu") -> torch.Tensor:
    """w [H, d] fp32, lognormal(0, 1)."""
    z = torch.randn((wl.heads, wl.d), generator=_gen(wl, _S_W, 0, "cpu"), dtype=torch.float32)
    return torch.exp(z).to(device)


def initial_state(wl: Workload, request: int, device="cpu") -> torch.Tensor:
    """S0 of one request, [H, d, d] fp32: diag(a) G diag(b) per head."""
    H, d = wl.heads, wl.d
    a = torch.exp(0.8 * torch.randn((H, d), generator=_gen(wl, _S_A, request, device), device=device))
    b = torch.exp(0.8 * torch.randn((H, d), generator=_gen(wl, _S_B, request, device), device=device))
    if wl.outliers:
        a.scatter_(1, a.argmax(dim=1, keepdim=True), ROW_OUTLIER * a.median(dim=1, keepdim=True).values)
        b.scatter_(1, b.argmax(dim=1, keepdim=True), COL_OUTLIER * b.median(dim=1, keepdim=True).values)
    G = torch.randn((H, d, d), generator=_gen(wl, _S_G, request, device), device=device)
    return a[:, :, None] * G * b[:, None, :]


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def decode_inputs(wl: Workload, token: int, device="cpu", batch: Optional[int] = None,
                  heads: Optional[slice] = None) -> dict:
    """Inputs of one decode token: q, k, v [B, H, d] (wl.in_dtype), beta [B, H] fp32,
    alpha [B, H] or [B, H, d] fp32 (the per-head gate broadcast over requests)."""
    B = wl.batch if batch is None else batch
    H, d = wl.heads, wl.d
    idx = 1_000_000 + token
    q = _unit(torch.randn((B, H, d), generator=_gen(wl, _S_Q, idx, device), device=device))
    k = _unit(torch.randn((B, H, d), generator=_gen(wl, _S_K, idx, device), device=device))
    v = torch.randn((B, H, d), generator=_gen(wl, _S_V, idx, device), device=device)
    beta = torch.sigmoid(torch.randn((B, H), generator=_gen(wl, _S_BETA, idx, device), device=device))
    a = gate_values(wl).to(device)
    alpha = a.expand((B,) + tuple(a.shape)).contiguous()
    out = dict(q=q.to(wl.in_dtype), k=k.to(wl.in_dtype), v=v.to(wl.in_dtype),
               beta=beta.float(), alpha=alpha)
    if heads is not None:
        out = {n: t[:, heads].contiguous() for n, t in out.items()}
    return out


def prefill_inputs(wl: Workload, t0: int, T: int, device="cpu", batch: Optional[int] = None) -> dict:
    """Inputs of prompt tokens [t0, t0+T): q, k, v [B, H, T, d], beta [B, H, T] fp32, alpha
    [B, H, T] fp32 (scalar gate) or [B, H, T, d] (channel gates: the per-key-row gate of the head,
    constant over tokens)."""
    B = wl.batch if batch is None else batch
    H, d = wl.heads, wl.d
    idx = 2_000_000 + t0 * 7 + T
    q = _unit(torch.randn((B, H, T, d), generator=_gen(wl, _S_Q, idx, device), device=device))
    k = _unit(torch.randn((B, H, T, d), generator=_gen(wl, _S_K, idx, device), device=device))
    v = torch.randn((B, H, T, d), generator=_gen(wl, _S_V, idx, device), device=device)
    beta = torch.sigmoid(torch.randn((B, H, T), generator=_gen(wl, _S_BETA, idx, device), device=device))
    a = gate_values(wl).to(device)
    if a.dim() == 1:
        alpha = a[None, :, None].expand(B, H, T).contiguous()
    else:
        alpha = a[None, :, None, :].expand(B, H, T, d).contiguous()
    return dict(q=q.to(wl.in_dtype), k=k.to(wl.in_dtype), v=v.to(wl.in_dtype),
                beta=beta.float(), alpha=alpha)


def scaled(wl: Workload, **changes) -> Workload:
    """A smaller copy of a workload with the same distributions (for parity tests)."""
    return dataclasses.replace(wl, **changes)
