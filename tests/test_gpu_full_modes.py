"""Full-size sampled parity of the bench's optional modes (needs a B200).

`bench.py --scale-dtype bf16` and `bench.py --fit-rounds 1` time the batch-70, 2304-head
mixed-width decode step with 16-bit scales or with one round of the joint scale refit. As for the
default mode (test_gpu_decode.py), that exact launch is checked on sampled tiles: 24 per width get
their pre-step bytes from the oracle, every other tile is initialised on the GPU and only has to
stay finite, and the sampled tiles are compared with the oracle's step under the mode's rule of
tests/_parity.py.
"""
import numpy as np
import pytest
import torch

from _parity import Tally, compare_block, compare_block_bf16s, compare_block_fit, compare_o, update_magnitude

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def stq():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    import quantized_linear_attention_stq_b200 as m

    m.lib()  # fails loudly if libstq.so is missing
    return m


@pytest.mark.parametrize("mode", ["bf16_scales", "fit_one_round"])
def test_full_batch70_launch_sampled(stq, orc, mode):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    sfmt = orc.SCALE_BF16 if mode == "bf16_scales" else orc.SCALE_F32
    rounds = 1 if mode == "fit_one_round" else 0
    wl_ = wlm.WORKLOADS["full2304_b70_mixed"]
    B, H, d = wl_.batch, wl_.heads, wl_.d
    bits = wlm.head_bits(wl_)
    lay = stq.Layout(bits, d, scale_dtype=torch.bfloat16 if sfmt == orc.SCALE_BF16 else torch.float32,
                     fit_rounds=rounds)
    offs, pos = [], 0
    for b in bits:
        offs.append(pos)
        pos += orc.block_bytes_s(b, sfmt, d, d)
    total = (pos + 127) // 128 * 128
    assert lay.bytes_per_request == total
    w = wlm.impact_weights(wl_, DEV)
    pool = lay.alloc_pool(B)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    rng = np.random.default_rng(43)
    sample = []
    for b in (4, 6, 8, 16):
        hs = [h for h in range(H) if bits[h] == b]
        for h in rng.choice(hs, size=24, replace=False):
            sample.append((int(rng.integers(B)), int(h)))
    S0_sample = {}
    for r0 in range(0, B, 10):
        S0 = torch.stack([wlm.initial_state(wl_, r, DEV) for r in range(r0, min(r0 + 10, B))])
        stq.init_state(lay, pool, slots[r0:r0 + S0.shape[0]].clone(), S0, w)
        for (r, h) in sample:
            if r0 <= r < r0 + S0.shape[0]:
                S0_sample[(r, h)] = S0[r - r0, h].double().cpu().numpy()
        del S0
    wc = w.double().cpu().numpy()
    pre = {}
    for (r, h) in sample:
        if bits[h] == 16:
            blk = orc.quantize(16, S0_sample[(r, h)], wc[h])[0]
        else:
            blk, _, _, st = orc.quantize_fit(bits[h], sfmt, rounds, S0_sample[(r, h)], wc[h])
            assert st == orc.OK
        pre[(r, h)] = blk
        start = r * total + offs[h]
        pool[start: start + blk.size] = torch.from_numpy(blk).to(DEV)
    inp = wlm.decode_inputs(wl_, 0, DEV)
    o = torch.zeros(B, H, d, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.decode_step(lay, pool, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w, o, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.isfinite(o).all()
    tally = Tally()
    for (r, h) in sample:
        start = r * total + offs[h]
        got = pool[start: start + pre[(r, h)].size].cpu().numpy()
        q, k, v = (inp[n][r, h].double().cpu().numpy() for n in ("q", "k", "v"))
        beta, alpha = float(inp["beta"][r, h]), float(inp["alpha"][r, h])
        what = f"{mode} req {r} head {h}"
        if bits[h] == 16:
            res = orc.decode_step(16, 0, pre[(r, h)], q, k, v, beta, alpha, wc[h], d, d)
            M = update_magnitude(orc.dequantize(16, d, d, pre[(r, h)]), k, v, beta, alpha)
            compare_block(orc, 16, d, got, res["block"], res["tie"], tally, what, err_scale=M)
        else:
            res = orc.decode_step_s(bits[h], sfmt, 0, pre[(r, h)], q, k, v, beta, alpha, wc[h], d, d, rounds=rounds)
            if mode == "bf16_scales":
                compare_block_bf16s(orc, bits[h], d, got, res["S_new"], wc[h], tally, what)
            else:
                compare_block_fit(orc, bits[h], d, got, res["S_new"], wc[h], rounds, tally, what)
        assert res["status"] == orc.OK
        compare_o(o[r, h].cpu().numpy(), res["o"], tally, "o " + what)
    tally.check_budget()
