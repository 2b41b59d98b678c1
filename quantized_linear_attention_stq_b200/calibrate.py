"""Offline calibration for the lifetime-aware width allocation (the method's time dimension).

For every head: the reconstruction distortion of its calibration states at each candidate width
(quantized and dequantized by the library's own kernels, stq_init_state + stq_dequantize) and the
mean log-retention of its gate; stq_allocate_widths then spends a byte budget where distortion and
lifetime are both large and keeps the highest-risk heads FP16 ("线性注意力状态量化难题"
(aitest123.com/news/n1kj09), section 时间维度; "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09),
section 方法). The pages calibrate on 32 WikiText-2 segments; here the calibration states are the
caller's (synthetic ones in this repository). Host-side orchestration only: the relative error
reduction below is bookkeeping over two device tensors, not part of the decode path.
"""
from __future__ import annotations

import numpy as np
import torch

from . import api

WIDTHS = (4, 6, 8)


def distortion_by_width(S_calib: torch.Tensor, w: torch.Tensor, chunk: int = 8) -> np.ndarray:
    """D[h][k] = mean over calibration states of ||S - deq(quant_b(S))||_F^2 / ||S||_F^2 at width
    WIDTHS[k]. S_calib: device fp32 [R][H][d][d]; w: device fp32 [H][d]."""
    R, H, d, _ = S_calib.shape
    dev = S_calib.device
    out = np.zeros((H, len(WIDTHS)), dtype=np.float64)
    for k, b in enumerate(WIDTHS):
        lay = api.Layout([b] * H, d)
        acc = torch.zeros(H, dtype=torch.float64, device=dev)
        for r0 in range(0, R, chunk):
            n = min(chunk, R - r0)
            pool = lay.alloc_pool(n, dev)
            slots = torch.arange(n, dtype=torch.int32, device=dev)
            S = S_calib[r0:r0 + n].contiguous()
            api.init_state(lay, pool, slots, S, w)
            Sh = torch.empty_like(S)
            api.dequantize(lay, pool, slots, Sh)
            num = (S.double() - Sh.double()).pow(2).sum(dim=(2, 3))
            den = S.double().pow(2).sum(dim=(2, 3)).clamp_min(1e-300)
            acc += (num / den).sum(dim=0)
        out[:, k] = (acc / R).cpu().numpy()
    return out


def lifetime_widths(S_calib: torch.Tensor, w: torch.Tensor, mean_log_retention, budget_bytes: int,
                    num_pivots: int) -> list:
    """Widths per head from the calibration states and the gates' mean log-retention."""
    D = distortion_by_width(S_calib, w)
    return api.allocate_widths(D, np.asarray(mean_log_retention, dtype=np.float64), S_calib.shape[-1], num_pivots,
                               budget_bytes)
