"""GPU parity of the uniform per-head INT baseline (one symmetric scale per head) against the oracle.

The baseline is the direct quantization the method is compared with ("线性注意力状态量化难题"
(aitest123.com/news/n1kj09), sections 直接量化为什么会翻车 and 数据说话): the same read -> update
-> readout -> requantize cycle, with s = max |S| / qmax for the whole head. Layouts with
scale_mode = SCALES_UNIFORM run it through the C ABI; FP16 pivot heads inside such a layout keep
their floating-point block. Teacher-forced protocol as in test_gpu_decode.py: the oracle's bytes go
up before each checked step, and the GPU's bytes and readout after it are compared with the
oracle's step from the same bytes (rules in tests/_parity.py).
"""
import numpy as np
import pytest
import torch

from _parity import (Tally, as_f64, compare_block, compare_o, compare_uniform_block, uniform_request_layout,
                     update_magnitude)

pytestmark = pytest.mark.gpu

DEV = "cuda"


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


def _quantize(orc, b, S, w):
    if b == 16:
        blk, x, tie, st = orc.quantize(16, S, w)
    else:
        blk, x, tie, st = orc.quantize_uniform(b, S)
    assert st == orc.OK
    return blk, tie


def _oracle_pool(orc, bits, d, S0, w):
    offs, total = uniform_request_layout(orc, bits, d)
    B, H = S0.shape[0], S0.shape[1]
    pool = np.zeros(B * total, dtype=np.uint8)
    ties = {}
    for r in range(B):
        for h in range(H):
            blk, tie = _quantize(orc, bits[h], as_f64(S0[r, h]), as_f64(w[h]))
            pool[r * total + offs[h]: r * total + offs[h] + blk.size] = blk
            ties[r, h] = tie
    return pool, ties


def _tile(orc, pool, bits, d, slot, h):
    offs, total = uniform_request_layout(orc, bits, d)
    n = orc.block_bytes(16, d, d) if bits[h] == 16 else orc.uniform_block_bytes(bits[h], d, d)
    return np.asarray(pool[slot * total + offs[h]: slot * total + offs[h] + n])


def _compare(orc, bits, d, h, got, ref, tie, tally, what, M=None):
    if bits[h] == 16:
        compare_block(orc, 16, d, got, ref, tie, tally, what, err_scale=M)
    else:
        compare_uniform_block(orc, bits[h], d, got, ref, tie, tally, what)


@pytest.mark.parametrize("d", [16, 128])
def test_uniform_init_and_dequantize(stq, orc, d):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=3, heads=6, d=d)
    bits = [4, 6, 8, 16, 6, 4]
    lay = stq.Layout(bits, d, scale_mode=stq.SCALES_UNIFORM)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(3)])
    ref, ties = _oracle_pool(orc, bits, d, S0, w)
    assert lay.bytes_per_request == uniform_request_layout(orc, bits, d)[1]
    pool = lay.alloc_pool(3)
    slots = torch.arange(3, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.init_state(lay, pool, slots, S0.to(DEV), w.to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    gp = pool.cpu().numpy()
    tally = Tally()
    for r in range(3):
        for h in range(6):
            _compare(orc, bits, d, h, _tile(orc, gp, bits, d, r, h), _tile(orc, ref, bits, d, r, h), ties[r, h],
                     tally, f"init req {r} head {h}")
    tally.check_budget()
    # dequantize the oracle's bytes (slots reversed): s * Q in fp32 against the fp64 product
    pool = torch.from_numpy(ref).to(DEV)
    out = torch.zeros(3, 6, d, d, device=DEV)
    stq.dequantize(lay, pool, torch.tensor([2, 1, 0], dtype=torch.int32, device=DEV), out, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = out.cpu().double().numpy()
    for r in range(3):
        for h in range(6):
            blk = _tile(orc, ref, bits, d, 2 - r, h)
            want = orc.dequantize(16, d, d, blk) if bits[h] == 16 else orc.dequantize_uniform(bits[h], d, d, blk)
            # one fp32 rounding of the product
            assert np.all(np.abs(got[r, h] - want) <= 2.0 ** -24 * np.abs(want)), f"req {r} head {h}"


def test_uniform_zero_state(stq, orc):
    """An all-zero head gets s = 1 and the zero code everywhere (the oracle's convention)."""
    bits = [4, 6, 8]
    d = 32
    lay = stq.Layout(bits, d, scale_mode=stq.SCALES_UNIFORM)
    pool = lay.alloc_pool(1)
    stq.init_state(lay, pool, torch.zeros(1, dtype=torch.int32, device=DEV), torch.zeros(1, 3, d, d, device=DEV),
                   torch.ones(3, d, device=DEV))
    torch.cuda.synchronize()
    gp = pool.cpu().numpy()
    for h, b in enumerate(bits):
        blk = _tile(orc, gp, bits, d, 0, h)
        ref = orc.quantize_uniform(b, np.zeros((d, d)))[0]
        assert np.array_equal(blk, ref)
        assert orc.uniform_scale(b, d, d, blk) == 1.0


def _decode_teacher_forced(stq, orc, wl_, bits, steps):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    B, H, d = wl_.batch, wl_.heads, wl_.d
    lay = stq.Layout(bits, d, gate=wl_.gate, in_dtype=wl_.in_dtype, scale_mode=stq.SCALES_UNIFORM)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(B)])
    opool, _ = _oracle_pool(orc, bits, d, S0, w)
    offs, total = uniform_request_layout(orc, bits, d)
    slot_of = np.random.default_rng(9).permutation(B + 2)[:B].astype(np.int32)
    gpool = torch.zeros((B + 2) * total, dtype=torch.uint8, device=DEV)
    slots = torch.from_numpy(slot_of).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    tally = Tally()
    for t in range(steps):
        inp = wlm.decode_inputs(wl_, t)
        host = np.zeros((B + 2) * total, dtype=np.uint8)
        for r in range(B):
            host[slot_of[r] * total:(slot_of[r] + 1) * total] = opool[r * total:(r + 1) * total]
        gpool.copy_(torch.from_numpy(host).to(DEV))
        o = torch.zeros(B, H, d, device=DEV)
        g = {n: x.to(DEV) for n, x in inp.items()}
        stq.decode_step(lay, gpool, slots, g["q"], g["k"], g["v"], g["beta"], g["alpha"], w.to(DEV), o,
                        status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, stq.status_flags(status)
        gp, og = gpool.cpu().numpy(), o.cpu().numpy()
        for r in range(B):
            for h in range(H):
                ref_blk = _tile(orc, opool, bits, d, r, h)
                args = (as_f64(inp["q"][r, h]), as_f64(inp["k"][r, h]), as_f64(inp["v"][r, h]),
                        float(inp["beta"][r, h]), inp["alpha"][r, h].double().numpy())
                if bits[h] == 16:
                    res = orc.decode_step(16, wl_.gate, ref_blk, *args, as_f64(w[h]), d, d)
                    M = update_magnitude(orc.dequantize(16, d, d, ref_blk), args[1], args[2], args[3], args[4])
                else:
                    res = orc.decode_step_uniform(bits[h], wl_.gate, ref_blk, *args, d, d)
                    M = None
                assert res["status"] == orc.OK
                _compare(orc, bits, d, h, _tile(orc, gp, bits, d, int(slot_of[r]), h), res["block"], res["tie"],
                         tally, f"step {t} req {r} head {h}", M)
                compare_o(og[r, h], res["o"], tally, f"o step {t} req {r} head {h}")
                opool[r * total + offs[h]: r * total + offs[h] + res["block"].size] = res["block"]
    tally.check_budget()
    return tally


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_uniform_decode_d128(stq, orc, bits):
    """d = 128 heads with bf16 inputs and the scalar gate: 4 requests x 6 heads, 3 steps."""
    wl_ = _wl("layer48_b8_4bit", batch=4, heads=6, bits=bits)
    _decode_teacher_forced(stq, orc, wl_, [bits] * 6, 3)


def test_uniform_decode_mixed_with_pivots(stq, orc):
    wl_ = _wl("layer48_b8_4bit", batch=3, heads=5, bits=None, in_dtype=torch.float32)
    _decode_teacher_forced(stq, orc, wl_, [4, 16, 6, 8, 6], 2)


@pytest.mark.parametrize("gate", [1, 2])
def test_uniform_decode_channel_gates(stq, orc, gate):
    wl_ = _wl("channel32_b128_4bit", batch=3, heads=4, gate=gate)
    _decode_teacher_forced(stq, orc, wl_, [4, 6, 8, 6], 2)


def test_uniform_decode_d16_sixty_four_steps(stq, orc):
    wl_ = _wl("pr1_d16_6bit")
    t = _decode_teacher_forced(stq, orc, wl_, [6], 64)
    assert t.codes == 64 * 256


@pytest.mark.parametrize("d,T,in_dtype", [(32, 100, torch.float32), (128, 70, torch.bfloat16)])
def test_uniform_prefill_matches_composed_oracle(stq, orc, d, T, in_dtype):
    """Chunked prefill (64-token chunks, ragged tail): the oracle composes its own pieces,
    dequantize -> per-token fp64 update and readout -> uniform requantization at every chunk end."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    chunk = 64
    bits = [4, 6, 8]
    wl_ = _wl("prefill16_b16_6bit", batch=2, heads=3, d=d, in_dtype=in_dtype)
    lay = stq.Layout(bits, d, in_dtype=in_dtype, scale_mode=stq.SCALES_UNIFORM)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(2)])
    opool, _ = _oracle_pool(orc, bits, d, S0, w)
    inp = wlm.prefill_inputs(wl_, 0, T)
    pool = torch.from_numpy(opool.copy()).to(DEV)
    o = torch.zeros(2, 3, T, d, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.prefill_chunk(lay, pool, torch.arange(2, dtype=torch.int32, device=DEV),
                      *(inp[n].to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV), o, chunk=chunk,
                      status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    gp, og = pool.cpu().numpy(), o.cpu().numpy()
    tally = Tally()
    for r in range(2):
        for h, b in enumerate(bits):
            blk = _tile(orc, opool, bits, d, r, h)
            S = orc.dequantize_uniform(b, d, d, blk)
            ref_o = np.zeros((T, d))
            for t in range(T):
                S, ref_o[t] = orc.update(0, S, as_f64(inp["q"][r, h, t]), as_f64(inp["k"][r, h, t]),
                                         as_f64(inp["v"][r, h, t]), float(inp["beta"][r, h, t]),
                                         float(inp["alpha"][r, h, t]))
                if (t + 1) % chunk == 0 or t == T - 1:
                    blk, _, tie, st = orc.quantize_uniform(b, S)
                    assert st == orc.OK
                    if t != T - 1:
                        S = orc.dequantize_uniform(b, d, d, blk)
            compare_uniform_block(orc, b, d, _tile(orc, gp, bits, d, r, h), blk, tie, tally, f"req {r} head {h}")
            compare_o(og[r, h], ref_o.astype(np.float32), tally, f"o req {r} head {h}")
    tally.check_budget()


def _spearman(x, y):
    rx = np.argsort(np.argsort(x)).astype(np.float64)
    ry = np.argsort(np.argsort(y)).astype(np.float64)
    rx -= rx.mean()
    ry -= ry.mean()
    return float((rx @ ry) / np.sqrt((rx @ rx) * (ry @ ry)))


def test_study_error_accumulation_uniform_vs_row_column(stq):
    """Error accumulation of the uniform baseline against the method's row x column scales.

    All 2304 heads of one request (d = 128, bf16 inputs, the outlier states and gate half-lives of
    the mixed workload) run 256 decode tokens at one width through the library, beside an exact
    fp64 recurrence from the same initial state. Per head: the relative state error at the end and
    the mean relative readout error over the last 64 tokens. The pages measure, under uniform INT6
    over Qwen's 2304 heads, a Spearman correlation of 0.80 between a head's gate half-life and its
    accumulated error ("线性注意力状态量化难题", section 时间维度), and show dual-axis scales
    keeping the state where uniform scales lose it (sections 空间维度, 数据说话)."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=1)
    H, d, steps, window = wl_.heads, wl_.d, 256, 64
    hl = wlm.half_lives(wl_).numpy()
    w = wlm.impact_weights(wl_).to(DEV)
    S0 = wlm.initial_state(wl_, 0).to(DEV)
    slots = torch.zeros(1, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    runs = {}
    for mode, name in ((stq.SCALES_ROW_COLUMN, "row x column"), (stq.SCALES_UNIFORM, "uniform")):
        for b in (4, 6, 8):
            lay = stq.Layout([b] * H, d, scale_mode=mode)
            pool = lay.alloc_pool(1, DEV)
            stq.init_state(lay, pool, slots, S0[None].contiguous(), w, status=status)
            runs[name, b] = dict(lay=lay, pool=pool, oerr=torch.zeros(H, dtype=torch.float64, device=DEV))
    S = S0.double()
    for t in range(steps):
        inp = {n: x.to(DEV) for n, x in wlm.decode_inputs(wl_, t).items()}
        q, k, v = (inp[n][0].double() for n in ("q", "k", "v"))
        beta, alpha = inp["beta"][0].double()[:, None, None], inp["alpha"][0].double()[:, None, None]
        u = torch.einsum("hi,hij->hj", k, S)
        S = alpha * (S - beta * k[:, :, None] * u[:, None, :]) + beta * k[:, :, None] * v[:, None, :]
        o_ref = torch.einsum("hi,hij->hj", q, S)
        for run in runs.values():
            o = torch.zeros(1, H, d, device=DEV)
            stq.decode_step(run["lay"], run["pool"], slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                            w, o, status=status)
            if t >= steps - window:
                run["oerr"] += (o[0].double() - o_ref).norm(dim=1) / o_ref.norm(dim=1) / window
    torch.cuda.synchronize()
    print()
    print("| scales | width | median state err | p90 state err | median readout err | "
          "Spearman(half-life, state err) | heads non-finite |")
    print("|---|---|---|---|---|---|---|")
    res = {}
    for (name, b), run in runs.items():
        Sq = torch.zeros(1, H, d, d, device=DEV)
        stq.dequantize(run["lay"], run["pool"], slots, Sq)
        err = ((Sq[0].double() - S).norm(dim=(1, 2)) / S.norm(dim=(1, 2))).cpu().numpy()
        oerr = run["oerr"].cpu().numpy()
        fin = np.isfinite(err) & np.isfinite(oerr)
        rho = _spearman(hl[fin], err[fin])
        res[name, b] = (np.median(err[fin]), rho, int((~fin).sum()))
        print(f"| {name} | {b} | {np.median(err[fin]):.3e} | {np.quantile(err[fin], 0.9):.3e} | "
              f"{np.median(oerr[fin]):.3e} | {rho:.3f} | {int((~fin).sum())} |")
    # the method keeps the state closer than the baseline at the same width, and under uniform
    # scales a longer half-life means a larger accumulated error
    for b in (6, 8):
        assert res["row x column", b][2] == 0 and res["uniform", b][2] == 0
        assert res["row x column", b][0] < res["uniform", b][0]
    assert res["uniform", 6][1] > 0.3
