"""Quantized linear-attention recurrent state on B200.

Per-token decode (and chunked prefill) of gated-delta-rule linear attention whose per-request
state lives in HBM as 4/6/8-bit codes with key-row x value-column scales, plus FP16 pivot heads.
All computation is in ``libstq.so`` (hand-written CUDA for sm_100a, C ABI in include/stq.h);
``api`` marshals torch tensors into it and ``workloads`` draws seeded synthetic inputs.
"""
from .api import (GATE_CHANNEL, GATE_CHANNEL_DECAY_FIRST, GATE_SCALAR, SCALES_ROW_COLUMN, SCALES_UNIFORM,  # noqa: F401
                  Layout, StqError,
                  allocate_widths, decode_step, dequantize, init_state, lib, prefill_chunk, prefill_chunk_noalloc,
                  prefill_workspace_bytes,
                  row_impact, selftest_wait_timeout, status_flags, status_string)
