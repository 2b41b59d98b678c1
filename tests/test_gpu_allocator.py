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


def test_study_time_and_space_dimensions_over_2048_tokens(stq):
    """The method's two dimensions together, over 2048 decode tokens of all 2304 heads of one
    request (the pages follow their states for 2048 decode steps: "线性注意力状态量化难题", section
    空间维度): random widths (the workload as specified) or lifetime-aware widths within the same
    bytes (time dimension), each with the one-pass scales or one round of the impact-weighted joint
    refit (space dimension), beside the exact fp64 recurrence. Per configuration and checkpoint:
    the median and p90 over heads of the relative state error, and the heads no longer finite."""
    from quantized_linear_attention_stq_b200 import calibrate
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl = wlm.WORKLOADS["full2304_b70_mixed"]
    H, d = wl.heads, wl.d
    rand_bits = wlm.head_bits(wl)
    w = wlm.impact_weights(wl, DEV)
    log_ret = np.log(wlm.gate_values(wl).double().numpy())
    budget = stq.Layout(rand_bits, d).bytes_per_request
    S_cal = torch.stack([wlm.initial_state(wl, 100 + r, DEV) for r in range(4)])
    life_bits = calibrate.lifetime_widths(S_cal, w, log_ret, budget, 32)
    del S_cal
    S0 = wlm.initial_state(wl, 0, DEV)
    slots = torch.zeros(1, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    runs = {}
    for wname, bits in (("random", rand_bits), ("lifetime", life_bits)):
        for rounds in (0, 1):
            lay = stq.Layout(bits, d, fit_rounds=rounds)
            pool = lay.alloc_pool(1, DEV)
            stq.init_state(lay, pool, slots, S0[None].contiguous(), w, status=status)
            runs[wname, rounds] = (lay, pool)
    S = S0.double()
    checkpoints = (256, 1024, 2048)
    rows = []
    for t in range(checkpoints[-1]):
        inp = wlm.decode_inputs(wl, t, DEV, batch=1)
        k, v = inp["k"][0].double(), inp["v"][0].double()
        beta, alpha = inp["beta"][0].double()[:, None, None], inp["alpha"][0].double()[:, None, None]
        u = torch.einsum("hi,hij->hj", k, S)
        S = alpha * (S - beta * k[:, :, None] * u[:, None, :]) + beta * k[:, :, None] * v[:, None, :]
        o = torch.empty(1, H, d, device=DEV)
        for lay, pool in runs.values():
            stq.decode_step(lay, pool, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w, o,
                            status=status)
        if t + 1 in checkpoints:
            for (wname, rounds), (lay, pool) in runs.items():
                Sq = torch.zeros(1, H, d, d, device=DEV)
                stq.dequantize(lay, pool, slots, Sq)
                err = ((Sq[0].double() - S).norm(dim=(1, 2)) / S.norm(dim=(1, 2))).cpu().numpy()
                fin = np.isfinite(err)
                rows.append((t + 1, wname, rounds, float(np.median(err[fin])) if fin.any() else float("nan"),
                             float(np.quantile(err[fin], 0.9)) if fin.any() else float("nan"), int((~fin).sum())))
    torch.cuda.synchronize()
    print()
    print("| tokens | widths | refit rounds | median state err | p90 state err | heads not finite |")
    print("|---|---|---|---|---|---|")
    for r in rows:
        print(f"| {r[0]} | {r[1]} | {r[2]} | {r[3]:.3e} | {r[4]:.3e} | {r[5]} |")
    final = {(r[1], r[2]): r for r in rows if r[0] == checkpoints[-1]}
    # the specified widths with one-pass scales blow up; either dimension alone keeps the tail
    # bounded; both together do best
    assert all(r[5] == 0 for r in final.values())
    assert final["random", 0][4] > 100.0
    assert final["random", 1][4] < 1.0 and final["lifetime", 0][4] < 1.0
    assert final["lifetime", 1][4] < min(final["random", 1][4], final["lifetime", 0][4])
