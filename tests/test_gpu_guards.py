"""Out-of-block writes (needs a B200): every kernel writes only the bytes of the head blocks it owns.

A pool sits between two guard bands, and everything is filled with a poison byte first: the guard
bands, an unused pool slot, and every padding byte of the request and head blocks. Then init, three
decode steps, a two-chunk prefill and a dequantize run over three requests at permuted slots. Every
kernel family is covered: the tuned decode and streaming init at d = 128, the tcgen05 prefill, the
plain kernels at small d, bf16 scales, uniform layouts and FP16 pivots. Afterwards every poisoned
byte must still hold the poison. The bytes a head may write are its codes and its scales (or its
fp16 values); the rest of its 128-byte-padded block is padding.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"
POISON = 0xA5
GUARD = 4096


@pytest.fixture(scope="module")
def stq():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    import quantized_linear_attention_stq_b200 as m

    m.lib()
    return m


def _written_ranges(lay, bits, d, scale_bytes, uniform):
    """Byte ranges of one request block that the kernels may write."""
    out = []
    for h, b in enumerate(bits):
        off = lay.head_offset(h)
        if b == 16:
            out.append((off, off + 2 * d * d))
            continue
        codes = (b * d * d + 7) // 8
        so = (codes + 15) // 16 * 16
        out.append((off, off + codes))
        out.append((off + so, off + so + (4 if uniform else scale_bytes * 2 * d)))
    return out


CASES = [
    ("d128 mixed widths, pivots", [4, 6, 8, 16, 6, 4], 128, torch.bfloat16, {}),
    ("d128 mixed widths, prefill with a workspace", [4, 6, 8, 16, 6, 4], 128, torch.bfloat16, {"ws": True}),
    ("d128 bf16 scales", [4, 6, 8, 16], 128, torch.bfloat16, {"scale_dtype": torch.bfloat16}),
    ("d128 bf16 scales, prefill with a workspace", [4, 6, 8, 16], 128, torch.bfloat16,
     {"scale_dtype": torch.bfloat16, "ws": True}),
    ("d128 uniform", [4, 6, 8, 16], 128, torch.bfloat16, {"scale_mode": 1}),
    ("d64 mixed widths", [4, 6, 8, 16], 64, torch.bfloat16, {}),
    ("d16 fp32 inputs", [6, 4, 16], 16, torch.float32, {}),
]


@pytest.mark.parametrize("name,bits,d,in_dtype,kw", CASES, ids=[c[0] for c in CASES])
def test_kernels_write_only_their_head_bytes(stq, name, bits, d, in_dtype, kw):
    kw = dict(kw)
    use_ws = kw.pop("ws", False)
    lay = stq.Layout(bits, d, in_dtype=in_dtype, **kw)
    H, B, nslots = len(bits), 3, 4
    R = lay.bytes_per_request
    buf = torch.full((GUARD + nslots * R + GUARD,), POISON, dtype=torch.uint8, device=DEV)
    pool = buf[GUARD:GUARD + nslots * R]
    assert pool.data_ptr() % 128 == 0
    slots = torch.tensor([2, 0, 1], dtype=torch.int32, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(7)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    w = torch.rand(H, d, generator=g, device=DEV) + 0.5
    S0 = torch.randn(B, H, d, d, generator=g, device=DEV)
    stq.init_state(lay, pool, slots, S0, w, status=status)
    unit = lambda x: torch.nn.functional.normalize(x, dim=-1)
    for _ in range(3):
        q = unit(torch.randn(B, H, d, generator=g, device=DEV)).to(in_dtype)
        k = unit(torch.randn(B, H, d, generator=g, device=DEV)).to(in_dtype)
        v = torch.randn(B, H, d, generator=g, device=DEV).to(in_dtype)
        beta = torch.sigmoid(torch.randn(B, H, generator=g, device=DEV))
        alpha = torch.full((B, H), 0.95, device=DEV)
        o = torch.empty(B, H, d, device=DEV)
        stq.decode_step(lay, pool, slots, q, k, v, beta, alpha, w, o, status=status)
    T = 70  # one full and one short chunk
    q = unit(torch.randn(B, H, T, d, generator=g, device=DEV)).to(in_dtype)
    k = unit(torch.randn(B, H, T, d, generator=g, device=DEV)).to(in_dtype)
    v = torch.randn(B, H, T, d, generator=g, device=DEV).to(in_dtype)
    beta = torch.sigmoid(torch.randn(B, H, T, generator=g, device=DEV))
    alpha = torch.full((B, H, T), 0.95, device=DEV)
    o = torch.empty(B, H, T, d, device=DEV)
    ws = None
    if use_ws:  # the three-kernel form; its workspace lies outside the guarded buffer
        assert stq.prefill_workspace_bytes(lay, B, T, 64) > 0
        ws = torch.empty(stq.prefill_workspace_bytes(lay, B, T, 64), dtype=torch.uint8, device=DEV)
    stq.prefill_chunk(lay, pool, slots, q, k, v, beta, alpha, w, o, chunk=64, workspace=ws, status=status)
    out = torch.empty(B, H, d, d, device=DEV)
    stq.dequantize(lay, pool, slots, out, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.isfinite(out).all()

    host = buf.cpu().numpy()
    assert np.all(host[:GUARD] == POISON), "write before the pool"
    assert np.all(host[GUARD + nslots * R:] == POISON), "write after the pool"
    p = host[GUARD:GUARD + nslots * R].reshape(nslots, R)
    assert np.all(p[3] == POISON), "write into a slot no request uses"
    allowed = np.zeros(R, dtype=bool)
    sb = 2 if kw.get("scale_dtype") == torch.bfloat16 else 4
    for lo, hi in _written_ranges(lay, bits, d, sb, kw.get("scale_mode") == 1):
        allowed[lo:hi] = True
    for s in range(3):
        bad = np.nonzero((p[s] != POISON) & ~allowed)[0]
        assert bad.size == 0, f"slot {s}: {bad.size} padding bytes written, first at {bad[:8].tolist()}"
    # the written ranges did take the new state (not left poisoned)
    assert np.mean(p[:3][:, allowed] == POISON) < 0.05
