"""Lifetime-aware widths on the 2304-head workload (needs a B200): calibration by the library's own
quantize/dequantize kernels, allocation within the random mix's byte budget, and the effect the
pages claim for it: long-lived state keeps its error in check."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def stq():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    import quantized_linear_attention_stq_b200 as m

    m.lib()
    return m


def test_lifetime_widths_budget_order_and_error_growth(stq):
    from quantized_linear_attention_stq_b200 import calibrate
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl = wlm.WORKLOADS["full2304_b70_mixed"]
    H, d = wl.heads, wl.d
    rand_bits = wlm.head_bits(wl)
    w = wlm.impact_weights(wl, DEV)
    log_ret = np.log(wlm.gate_values(wl).double().numpy())
    lay_r = stq.Layout(rand_bits, d)
    S_cal = torch.stack([wlm.initial_state(wl, 100 + r, DEV) for r in range(4)])
    D = calibrate.distortion_by_width(S_cal, w)
    assert np.all(D[:, 0] > D[:, 1]) and np.all(D[:, 1] > D[:, 2])  # more bits, less distortion
    bits = calibrate.lifetime_widths(S_cal, w, log_ret, lay_r.bytes_per_request, 32)
    lay_l = stq.Layout(bits, d)
    assert lay_l.bytes_per_request <= lay_r.bytes_per_request
    assert bits.count(16) == 32
    half = -1.0 / log_ret
    med = [np.median([half[h] for h in range(H) if bits[h] == b]) for b in (4, 6, 8, 16)]
    assert med[0] < med[1] < med[2] < med[3]
    # same inputs, same bytes: after the workload's 256 tokens the lifetime-aware pool's readout has
    # grown far less than the random one's
    B = 2
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    toks = [wlm.decode_inputs(wl, t, DEV, batch=B) for t in range(8)]
    peak = {}
    for name, lay in (("random", lay_r), ("lifetime", lay_l)):
        pool = lay.alloc_pool(B)
        stq.init_state(lay, pool, slots, torch.stack([wlm.initial_state(wl, r, DEV) for r in range(B)]), w)
        o = torch.empty(B, H, d, device=DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        for t in range(256):
            x = toks[t % 8]
            stq.decode_step(lay, pool, slots, x["q"], x["k"], x["v"], x["beta"], x["alpha"], w, o, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0, stq.status_flags(st)
        peak[name] = o.abs().max().item()
    assert peak["lifetime"] * 100 < peak["random"], peak


@pytest.mark.parametrize("d,gate,dtype", [(128, 0, torch.bfloat16), (128, 1, torch.float32), (64, 2, torch.bfloat16),
                                          (16, 0, torch.float32)])
def test_row_impact_matches_oracle(stq, d, gate, dtype):
    from oracle import allocate as alo

    g = torch.Generator().manual_seed(d + gate)
    T, H = 37, 5
    q = torch.randn(T, H, d, generator=g).to(dtype)
    k = torch.nn.functional.normalize(torch.randn(T, H, d, generator=g), dim=-1).to(dtype)
    beta = torch.sigmoid(torch.randn(T, H, generator=g))
    alpha = torch.rand(T, H, generator=g) * 0.5 + 0.5 if gate == 0 else torch.rand(T, H, d, generator=g) * 0.5 + 0.5
    w = stq.row_impact(q.to(DEV), k.to(DEV), beta.to(DEV), alpha.to(DEV), gate=gate)
    torch.cuda.synchronize()
    got = w.cpu().double().numpy()
    for h in range(H):
        ref = alo.row_impact(q[:, h].double().numpy(), k[:, h].double().numpy(), beta[:, h].double().numpy(),
                             alpha[:, h].double().numpy(), gate)
        np.testing.assert_allclose(got[h], ref, rtol=2e-5, atol=1e-12)
