"""GPU parity of the impact-aware joint refinement of the scales against the oracle (needs a B200).

A layout with fit_rounds = n refits, after the one-pass fit, every column scale by impact-weighted
least squares and every row scale by least squares, n times, recomputing the codes in between
(the pages fit the two scales jointly and weight high-impact rows more: "线性注意力状态量化难题"
(aitest123.com/news/n1kj09), section 空间维度; "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09),
section 方法). A layout with one round decodes 128 x 128 heads on the tuned kernel; other layouts
with refinement run on the plain kernels. Teacher-forced protocol as in test_gpu_decode.py; blocks
are compared with the joint-fit rule of tests/_parity.py.
"""
import numpy as np
import pytest
import torch

from _parity import (Tally, as_f64, compare_block, compare_block_fit, compare_o, tile_bytes,
                     update_magnitude)

pytestmark = pytest.mark.gpu

DEV = "cuda"
ROUNDS = 2
STUDY_ROUNDS = (0, 1, 2)


@pytest.fixture(scope="module")
def stq():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    import quantized_linear_attention_stq_b200 as m

    m.lib()  # fails loudly if libstq.so is missing
    return m


def _wl(name, **changes):
    from quantized_linear_attention_stq_b200 import workloads as wl

    return wl.scaled(wl.WORKLOADS[name], **changes)


def _layout_s(orc, bits, d, sfmt):
    offs, pos = [], 0
    for b in bits:
        offs.append(pos)
        pos += orc.block_bytes_s(int(b), sfmt, d, d)
    return offs, (pos + 127) // 128 * 128


def _oracle_pool(orc, bits, d, S0, w, rounds, sfmt=0):
    B, H = S0.shape[0], S0.shape[1]
    offs, total = _layout_s(orc, bits, d, sfmt)
    pool = np.zeros(B * total, dtype=np.uint8)
    for r in range(B):
        for h in range(H):
            blk, _, _, st = orc.quantize_fit(bits[h], sfmt, 0 if bits[h] == 16 else rounds,
                                             as_f64(S0[r, h]), as_f64(w[h]))
            assert st == orc.OK
            pool[r * total + offs[h]: r * total + offs[h] + blk.size] = blk
    return pool


@pytest.mark.parametrize("d", [16, 128])
def test_init(stq, orc, d):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=3, heads=6, d=d)
    bits = [4, 6, 8, 16, 8, 6]
    lay = stq.Layout(bits, d, fit_rounds=ROUNDS)
    assert lay.bytes_per_request == stq.Layout(bits, d).bytes_per_request
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(3)])
    pool = lay.alloc_pool(3)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.init_state(lay, pool, torch.arange(3, dtype=torch.int32, device=DEV), S0.to(DEV), w.to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    gp = pool.cpu().numpy()
    tally = Tally()
    for r in range(3):
        for h in range(6):
            got = tile_bytes(orc, gp, bits, d, r, h)
            if bits[h] == 16:
                blk, _, tie, _ = orc.quantize(16, as_f64(S0[r, h]), as_f64(w[h]))
                compare_block(orc, 16, d, got, blk, tie, tally, f"init req {r} head {h}")
            else:
                compare_block_fit(orc, bits[h], d, got, as_f64(S0[r, h]), as_f64(w[h]), ROUNDS, tally,
                                  f"init req {r} head {h}")
    tally.check_budget()


def _decode_teacher_forced(stq, orc, wl_, bits, steps, rounds=ROUNDS, sfmt=0):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    B, H, d = wl_.batch, wl_.heads, wl_.d
    lay = stq.Layout(bits, d, gate=wl_.gate, in_dtype=wl_.in_dtype, fit_rounds=rounds,
                     scale_dtype=torch.bfloat16 if sfmt == orc.SCALE_BF16 else torch.float32)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(B)])
    opool = _oracle_pool(orc, bits, d, S0, w, rounds, sfmt)
    offs, total = _layout_s(orc, bits, d, sfmt)
    assert lay.bytes_per_request == total
    gpool = torch.zeros(B * total, dtype=torch.uint8, device=DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    tally = Tally()
    for t in range(steps):
        inp = wlm.decode_inputs(wl_, t)
        gpool.copy_(torch.from_numpy(opool.copy()).to(DEV))
        o = torch.zeros(B, H, d, device=DEV)
        g = {n: x.to(DEV) for n, x in inp.items()}
        stq.decode_step(lay, gpool, slots, g["q"], g["k"], g["v"], g["beta"], g["alpha"], w.to(DEV), o,
                        status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, stq.status_flags(status)
        gp, og = gpool.cpu().numpy(), o.cpu().numpy()
        for r in range(B):
            for h in range(H):
                n_b = orc.block_bytes_s(bits[h], sfmt, d, d)
                ref_blk = opool[r * total + offs[h]: r * total + offs[h] + n_b]
                q, k, v = as_f64(inp["q"][r, h]), as_f64(inp["k"][r, h]), as_f64(inp["v"][r, h])
                beta, alpha = float(inp["beta"][r, h]), inp["alpha"][r, h].double().numpy()
                hr = 0 if bits[h] == 16 else rounds
                res = orc.decode_step_s(bits[h], sfmt, wl_.gate, ref_blk, q, k, v, beta, alpha,
                                        as_f64(w[h]), d, d, rounds=hr)
                assert res["status"] == orc.OK
                got = gp[r * total + offs[h]: r * total + offs[h] + n_b]
                what = f"step {t} req {r} head {h}"
                if bits[h] == 16:
                    M = update_magnitude(orc.dequantize(16, d, d, ref_blk), k, v, beta, alpha)
                    compare_block(orc, 16, d, got, res["block"], res["tie"], tally, what, err_scale=M)
                else:
                    compare_block_fit(orc, bits[h], d, got, res["S_new"], as_f64(w[h]), rounds, tally, what, sfmt)
                compare_o(og[r, h], res["o"], tally, "o " + what)
                opool[r * total + offs[h]: r * total + offs[h] + res["block"].size] = res["block"]
    tally.check_budget()


@pytest.mark.parametrize("rounds", [1, 2])
def test_decode_d128_mixed_with_pivots(stq, orc, rounds):
    """One round runs on the tuned 128 x 128 kernel, two on the plain kernel."""
    wl_ = _wl("full2304_b70_mixed", batch=3, heads=8)
    _decode_teacher_forced(stq, orc, wl_, [4, 16, 6, 8, 4, 6, 8, 6], 2, rounds)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_decode_d128_tuned_one_round(stq, orc, bits):
    """The tuned kernel's refit at each width: 5 requests x 6 heads, 3 steps."""
    wl_ = _wl("layer48_b8_4bit", batch=5, heads=6, bits=bits)
    _decode_teacher_forced(stq, orc, wl_, [bits] * 6, 3, 1)


@pytest.mark.parametrize("gate", [1, 2])
def test_decode_d128_tuned_channel_gates(stq, orc, gate):
    wl_ = _wl("channel32_b128_4bit", batch=2, heads=4, gate=gate)
    _decode_teacher_forced(stq, orc, wl_, [4, 6, 8, 6], 2, 1)


@pytest.mark.parametrize("rounds", [1, 2])
def test_decode_d128_bf16_scales(stq, orc, rounds):
    """The refit with 16-bit scales: every refitted value is rounded to bf16 before it is used
    (one round on the tuned kernel, two on the plain kernel)."""
    wl_ = _wl("full2304_b70_mixed", batch=3, heads=6)
    _decode_teacher_forced(stq, orc, wl_, [4, 6, 8, 16, 6, 4], 2, rounds, orc.SCALE_BF16)


def test_zero_heads_keep_unit_scales(stq, orc):
    """An all-zero state stays all-zero through a step with v = 0: every refit denominator is 0,
    so the scales stay 1 and the codes 0, without a non-finite flag."""
    bits, d = [4, 6, 8], 128
    lay = stq.Layout(bits, d, fit_rounds=1)
    pool = lay.alloc_pool(2)
    slots = torch.arange(2, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    w = torch.ones(3, d, device=DEV)
    stq.init_state(lay, pool, slots, torch.zeros(2, 3, d, d, device=DEV), w, status=status)
    q = torch.randn(2, 3, d, device=DEV).bfloat16()
    k = torch.nn.functional.normalize(torch.randn(2, 3, d, device=DEV), dim=-1).bfloat16()
    v = torch.zeros(2, 3, d, device=DEV).bfloat16()
    beta = torch.full((2, 3), 0.5, device=DEV)
    alpha = torch.full((2, 3), 0.9, device=DEV)
    o = torch.full((2, 3, d), 7.0, device=DEV)
    stq.decode_step(lay, pool, slots, q, k, v, beta, alpha, w, o, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.all(o == 0)
    gp = pool.cpu().numpy()
    for r in range(2):
        for h, b in enumerate(bits):
            blk = tile_bytes(orc, gp, bits, d, r, h)
            assert np.all(orc.codes(b, d, d, blk) == 0)
            rs, cs = orc.scales(b, d, d, blk)
            assert np.all(rs == 1.0) and np.all(cs == 1.0)


@pytest.mark.parametrize("gate", [1, 2])
def test_decode_channel_gates(stq, orc, gate):
    wl_ = _wl("channel32_b128_4bit", batch=2, heads=3, gate=gate, d=32, in_dtype=torch.float32)
    _decode_teacher_forced(stq, orc, wl_, [4, 6, 8], 3)


@pytest.mark.parametrize("rounds", [1, 2])
def test_prefill_chunk(stq, orc, rounds):
    """A 64-token chunk, then a 30-token chunk from the oracle's bytes, one request x three heads at
    d = 128, bf16 inputs: one round runs in the tensor-core prefill's chunk-end requantization, two
    on the sequential kernel."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits, d, T = [4, 6, 8], 128, 94
    wl_ = _wl("prefill16_b16_6bit", batch=1, heads=3)
    lay = stq.Layout(bits, d, in_dtype=torch.bfloat16, fit_rounds=rounds)
    w = wlm.impact_weights(wl_)
    S0 = wlm.initial_state(wl_, 0)[None]
    opool = _oracle_pool(orc, bits, d, S0, w, rounds)
    inp = wlm.prefill_inputs(wl_, 0, T)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    tally = Tally()
    # the 64-token chunk alone
    pool = torch.from_numpy(opool.copy()).to(DEV)
    o = torch.zeros(1, 3, 64, d, device=DEV)
    stq.prefill_chunk(lay, pool, torch.zeros(1, dtype=torch.int32, device=DEV),
                      *(inp[n][:, :, :64].contiguous().to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV),
                      o, chunk=64, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    gp, og = pool.cpu().numpy(), o.cpu().numpy()
    offs, total = orc.request_layout(bits, d, d)
    for h, b in enumerate(bits):
        blk = tile_bytes(orc, opool, bits, d, 0, h)
        args = [as_f64(inp[n][0, h, :64]) for n in ("q", "k", "v", "beta", "alpha")]
        S = orc.dequantize(b, d, d, blk)
        for t in range(64):
            S, _ = orc.update(0, S, args[0][t], args[1][t], args[2][t], args[3][t], args[4][t])
        res = orc.prefill_seq_s(b, orc.SCALE_F32, 0, blk, *args, as_f64(w[h]), 64, d, d, rounds=rounds)
        compare_block_fit(orc, b, d, tile_bytes(orc, gp, bits, d, 0, h), S, as_f64(w[h]), rounds, tally,
                          f"chunk 0 head {h}")
        for t in range(64):
            compare_o(og[0, h, t], res["o"][t], tally, f"o token {t} head {h}")
        opool[offs[h]: offs[h] + res["block"].size] = res["block"]
    # the 30-token rest from the oracle's bytes
    pool = torch.from_numpy(opool.copy()).to(DEV)
    o = torch.zeros(1, 3, T - 64, d, device=DEV)
    stq.prefill_chunk(lay, pool, torch.zeros(1, dtype=torch.int32, device=DEV),
                      *(inp[n][:, :, 64:].contiguous().to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV),
                      o, chunk=64, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    gp = pool.cpu().numpy()
    for h, b in enumerate(bits):
        blk = tile_bytes(orc, opool, bits, d, 0, h)
        args = [as_f64(inp[n][0, h, 64:]) for n in ("q", "k", "v", "beta", "alpha")]
        S = orc.dequantize(b, d, d, blk)
        for t in range(T - 64):
            S, _ = orc.update(0, S, args[0][t], args[1][t], args[2][t], args[3][t], args[4][t])
        compare_block_fit(orc, b, d, tile_bytes(orc, gp, bits, d, 0, h), S, as_f64(w[h]), rounds, tally,
                          f"chunk 1 head {h}")
    tally.check_budget()


def test_study_joint_fit_error_accumulation(stq):
    """The joint refinement against the one-pass scales over 256 decode tokens of all 2304 heads
    of one request of the mixed workload, beside the exact fp64 recurrence (as the uniform
    baseline study in test_gpu_uniform.py): per head the relative state error at the end and the
    impact-weighted one, sum_i w_i |E_i|^2 / sum_i w_i |S_i|^2, the quantity the refinement fits."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=1)
    H, d, steps = wl_.heads, wl_.d, 256
    w = wlm.impact_weights(wl_).to(DEV)
    S0 = wlm.initial_state(wl_, 0).to(DEV)
    slots = torch.zeros(1, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    runs = {}
    for rounds in STUDY_ROUNDS:
        for b in (4, 6, 8):
            lay = stq.Layout([b] * H, d, fit_rounds=rounds)
            pool = lay.alloc_pool(1, DEV)
            stq.init_state(lay, pool, slots, S0[None].contiguous(), w, status=status)
            runs[rounds, b] = dict(lay=lay, pool=pool)
    S = S0.double()
    for t in range(steps):
        inp = {n: x.to(DEV) for n, x in wlm.decode_inputs(wl_, t).items()}
        k, v = inp["k"][0].double(), inp["v"][0].double()
        beta, alpha = inp["beta"][0].double()[:, None, None], inp["alpha"][0].double()[:, None, None]
        u = torch.einsum("hi,hij->hj", k, S)
        S = alpha * (S - beta * k[:, :, None] * u[:, None, :]) + beta * k[:, :, None] * v[:, None, :]
        for run in runs.values():
            o = torch.zeros(1, H, d, device=DEV)
            stq.decode_step(run["lay"], run["pool"], slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                            w, o, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    wd = w.double()[:, :, None]
    print()
    print("| width | fit rounds | median state err | p90 state err | median weighted err | p90 weighted err |")
    print("|---|---|---|---|---|---|")
    med = {}
    for (rounds, b), run in sorted(runs.items(), key=lambda kv: (kv[0][1], kv[0][0])):
        Sq = torch.zeros(1, H, d, d, device=DEV)
        stq.dequantize(run["lay"], run["pool"], slots, Sq)
        E = Sq[0].double() - S
        err = (E.norm(dim=(1, 2)) / S.norm(dim=(1, 2))).cpu().numpy()
        werr = ((wd * E ** 2).sum(dim=(1, 2)) / (wd * S ** 2).sum(dim=(1, 2))).sqrt().cpu().numpy()
        med[rounds, b] = float(np.median(werr))
        print(f"| {b} | {rounds} | {np.median(err):.3e} | {np.quantile(err, 0.9):.3e} | {np.median(werr):.3e} | "
              f"{np.quantile(werr, 0.9):.3e} |")
        assert np.isfinite(err).all()
    for b in (6, 8):
        assert med[ROUNDS, b] < med[0, b]
