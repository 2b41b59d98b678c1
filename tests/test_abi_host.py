"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function that
include/stq.h declares, lays the pool out exactly as the oracle's independent layout does, and
rejects bad arguments before anything is enqueued."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def stq():
    from quantized_linear_attention_stq_b200 import build

    build.build()
    import quantized_linear_attention_stq_b200 as m

    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "stq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(stq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ("stq_init_state", "stq_decode_step", "stq_prefill_chunk", "stq_dequantize"):
        assert n in names


def test_library_exports_every_declared_symbol(stq):
    L = stq.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value
    assert sorted(stq.api.EXPORTS) == declared_functions()
    assert L.stq_abi_version() == 4


def test_status_strings(stq):
    assert stq.status_string(0) == "ok"
    assert "non-finite" in stq.status_string(4)
    assert stq.status_string(99) == "unknown status"


@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_layout_matches_oracle_layout(stq, orc, d):
    rng = np.random.default_rng(d)
    bits = [int(b) for b in rng.choice([4, 6, 8, 16], size=37)]
    lay = stq.Layout(bits, d)
    offs, total = orc.request_layout(bits, d, d)
    assert lay.bytes_per_request == total
    for h, b in enumerate(bits):
        assert lay.head_offset(h) == offs[h]
        assert lay.head_bytes(h) == orc.block_bytes(b, d, d)
        assert lay.head_bits_of(h) == b
    assert lay.bytes_per_request % 128 == 0


@pytest.mark.parametrize("d", [16, 128])
def test_uniform_layout_matches_oracle_layout(stq, orc, d):
    """Uniformly scaled heads hold the codes, padding, one fp32 scale and padding to 128 bytes;
    FP16 pivot heads keep their block."""
    bits = [4, 6, 8, 16, 6]
    lay = stq.Layout(bits, d, scale_mode=stq.SCALES_UNIFORM)
    pos = 0
    for h, b in enumerate(bits):
        nb = orc.block_bytes(16, d, d) if b == 16 else orc.uniform_block_bytes(b, d, d)
        assert lay.head_offset(h) == pos and lay.head_bytes(h) == nb
        pos += nb
    assert lay.bytes_per_request == pos
    # 6-bit 128 x 128: 12,288 code bytes + 4 scale bytes -> 12,416 (vs 13,312 with row x column scales)
    if d == 128:
        assert lay.head_bytes(1) == 12416
    with pytest.raises(stq.StqError) as e:
        stq.Layout([4], d, scale_mode=2)
    assert e.value.status == stq.api.STQ_ERR_INVALID_ARG


def test_mixed_workload_bytes_per_token(stq):
    """The 2304-head mixed workload moves 57,597,952 state bytes (read + write) per request-token."""
    from quantized_linear_attention_stq_b200 import workloads as wl

    w = wl.WORKLOADS["full2304_b70_mixed"]
    bits = wl.head_bits(w)
    lay = stq.Layout(bits, 128)
    moved = 2 * sum(lay.head_bytes(h) for h in range(len(bits)))
    assert moved == 922 * 18432 + 1037 * 26624 + 313 * 34816 + 32 * 65536 == 57_597_952


def test_compression_against_pages(stq, orc):
    """The pages report ~5.03x (Qwen) / 5.08x (Kimi) state compression at 6 bits
    (tests/golden/page_facts.txt). This layout keeps fp32 scales: 4.92x per 128x128 head; 16-bit
    scales would give 5.12x."""
    fp32_state = 128 * 128 * 4
    ours = fp32_state / orc.block_bytes(6, 128, 128)
    assert abs(ours - 4.923) < 1e-3
    with_half_scales = fp32_state / (128 * 128 * 6 / 8 + 2 * 256)
    assert abs(with_half_scales - 5.12) < 1e-2


def test_layout_rejects_bad_descriptors(stq):
    with pytest.raises(stq.StqError) as e:
        stq.Layout([4, 5], 128)
    assert e.value.status == stq.api.STQ_ERR_UNSUPPORTED
    with pytest.raises(stq.StqError) as e:
        stq.Layout([4], 96)
    assert e.value.status == stq.api.STQ_ERR_UNSUPPORTED
    with pytest.raises(stq.StqError) as e:
        stq.Layout([], 128)
    assert e.value.status == stq.api.STQ_ERR_INVALID_ARG
    with pytest.raises(stq.StqError):
        stq.Layout([4], 128, gate=7)
    with pytest.raises(stq.StqError) as e:
        stq.Layout([4], 128, fit_rounds=9)
    assert e.value.status == stq.api.STQ_ERR_INVALID_ARG
    with pytest.raises(stq.StqError) as e:
        stq.Layout([4], 128, fit_rounds=-1)
    assert e.value.status == stq.api.STQ_ERR_INVALID_ARG
    with pytest.raises(stq.StqError) as e:
        stq.Layout([4], 128, scale_mode=stq.SCALES_UNIFORM, fit_rounds=1)
    assert e.value.status == stq.api.STQ_ERR_UNSUPPORTED
    with pytest.raises(TypeError):
        stq.Layout([4], 128, scale_dtype=torch.float16)
    # the scale format and the refinement leave the pool layout of row x column heads as specified
    assert stq.Layout([6], 128, fit_rounds=3).head_bytes(0) == 13312
    assert stq.Layout([6], 128, scale_dtype=torch.bfloat16).head_bytes(0) == 12800


def test_calls_reject_bad_arguments_before_enqueueing(stq):
    """Argument checks happen on the host before any CUDA call, so they run without a GPU."""
    L = stq.lib()
    lay = stq.Layout([4, 6], 128)
    h = lay.handle
    P = ctypes.c_void_p
    fake = P(0x10000)       # aligned, never dereferenced
    odd = P(0x10004)        # misaligned for the pool / bulk-copied rows
    # decode: bad head range, negative B, NULL pointers, misaligned pool / rows
    assert L.stq_decode_step(h, fake, 4, fake, 2, 1, 2, fake, fake, fake, fake, fake, fake, fake, None, None) == 1
    assert L.stq_decode_step(h, fake, 4, fake, -1, 0, 2, fake, fake, fake, fake, fake, fake, fake, None, None) == 1
    assert L.stq_decode_step(h, None, 4, fake, 2, 0, 2, fake, fake, fake, fake, fake, fake, fake, None, None) == 1
    assert L.stq_decode_step(h, odd, 4, fake, 2, 0, 2, fake, fake, fake, fake, fake, fake, fake, None, None) == 1
    assert L.stq_decode_step(h, fake, 4, fake, 2, 0, 2, odd, fake, fake, fake, fake, fake, fake, None, None) == 1
    assert L.stq_decode_step(None, fake, 4, fake, 2, 0, 2, fake, fake, fake, fake, fake, fake, fake, None, None) == 1
    # B == 0 and head_count == 0 are no-ops that succeed without touching CUDA
    assert L.stq_decode_step(h, None, 0, None, 0, 0, 2, None, None, None, None, None, None, None, None, None) == 0
    assert L.stq_decode_step(h, fake, 4, fake, 3, 2, 0, None, None, None, None, None, None, None, None, None) == 0
    # init / dequantize / prefill
    assert L.stq_init_state(h, fake, 4, fake, 2, None, fake, None, None) == 1
    assert L.stq_init_state(h, None, 0, None, 0, None, None, None, None) == 0
    assert L.stq_dequantize(h, odd, 4, fake, 2, fake, None, None) == 1
    assert L.stq_prefill_chunk(h, fake, 4, fake, 2, 8, 0, fake, fake, fake, fake, fake, fake, fake, None, 0, None,
                               None) == 1
    assert L.stq_prefill_chunk(h, fake, 4, fake, 2, 0, 64, None, None, None, None, None, None, None, None, 0, None,
                               None) == 0
    # the bounded-wait self-test needs a status word to report into
    assert L.stq_selftest_wait_timeout(None, None) == 1


def test_prefill_workspace_sizes(stq):
    """The three-kernel prefill asks for one record per (request, head, chunk of a segment of at
    most 32 chunks), FP16 pivot heads included; the shapes that run as one kernel ask for none. A
    workspace that is given must be large enough and 256-byte aligned (checked on the host, before
    any CUDA call)."""
    SEG = 32
    bf = torch.bfloat16
    REC = stq.prefill_workspace_bytes(stq.Layout([6], 128, in_dtype=bf), 1, 64, 64)
    assert REC > 0 and REC % 1024 == 0
    lay = stq.Layout([6, 16, 4, 8], 128, in_dtype=bf)
    assert stq.prefill_workspace_bytes(lay, 3, 64, 64) == 3 * 4 * 1 * REC
    assert stq.prefill_workspace_bytes(lay, 3, 65, 64) == 3 * 4 * 2 * REC
    assert stq.prefill_workspace_bytes(lay, 2, 8192, 64) == 2 * 4 * SEG * REC
    assert stq.prefill_workspace_bytes(stq.Layout([16, 16], 128, in_dtype=bf), 3, 640, 64) == 3 * 2 * 10 * REC
    assert stq.prefill_workspace_bytes(lay, 0, 64, 64) == 0
    assert stq.prefill_workspace_bytes(lay, 3, 0, 64) == 0
    assert stq.prefill_workspace_bytes(lay, 3, 64, 32) == 0
    for other in (stq.Layout([6, 4], 128, in_dtype=torch.float32), stq.Layout([6, 4], 64, in_dtype=bf),
                  stq.Layout([6, 4], 128, gate=1, in_dtype=bf), stq.Layout([6, 4], 128, in_dtype=bf, fit_rounds=1)):
        assert stq.prefill_workspace_bytes(other, 3, 640, 64) == 0
    L = stq.lib()
    P = ctypes.c_void_p
    fake = P(0x10000)
    need = stq.prefill_workspace_bytes(lay, 3, 64, 64)
    args = (lay.handle, fake, 4, fake, 3, 64, 64, fake, fake, fake, fake, fake, fake, fake)
    assert L.stq_prefill_chunk(*args, P(0x1000000), need - 1, None, None) == 1
    assert L.stq_prefill_chunk(*args, P(0x1000080), need, None, None) == 1


def test_python_binding_checks_shapes(stq):
    lay = stq.Layout([4, 4], 128)
    pool = torch.zeros(lay.bytes_per_request, dtype=torch.uint8)
    slots = torch.zeros(1, dtype=torch.int32)
    q = torch.zeros(1, 2, 128, dtype=torch.bfloat16)
    bad = torch.zeros(1, 2, 64, dtype=torch.bfloat16)
    f = torch.zeros(1, 2, dtype=torch.float32)
    with pytest.raises(ValueError):
        stq.decode_step(lay, pool, slots, q, bad, q, f, f, torch.zeros(2, 128), torch.zeros(1, 2, 128))
    with pytest.raises(TypeError):
        stq.decode_step(lay, pool, slots, q.float(), q, q, f, f, torch.zeros(2, 128), torch.zeros(1, 2, 128))


def test_product_path_does_not_reference_the_oracle():
    """The CUDA path and its binding never import or load the oracle."""
    pkg = os.path.join(ROOT, "quantized_linear_attention_stq_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "stq_oracle" not in text and "orc_" not in text, f
