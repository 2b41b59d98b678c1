"""GPU parity of the decode step, init and dequantize against the CPU oracle (needs a B200).

Teacher-forced protocol: the oracle's own trajectory is authoritative. Before each checked step
the oracle's pre-step pool bytes are uploaded into the GPU pool, one GPU step runs through the C
ABI, and the GPU's post-step bytes and readout are compared with the oracle's step from the same
bytes and the same inputs (rules in tests/_parity.py).
"""
import numpy as np
import pytest
import torch

from _parity import (Tally, as_f64, compare_block, compare_block_bf16s, compare_o, oracle_pool, tile_bytes,
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


def _oracle_init(orc, wl_, bits, S0, w):
    """Oracle init of every tile: S0 [B,H,d,d] and w [H,d] as torch CPU tensors."""
    B, H, d = S0.shape[0], S0.shape[1], S0.shape[2]
    blocks = []
    for r in range(B):
        row = []
        for h in range(H):
            blk, _, _, st = orc.quantize(bits[h], as_f64(S0[r, h]), as_f64(w[h]))
            assert st == orc.OK
            row.append(blk)
        blocks.append(row)
    return oracle_pool(orc, bits, d, blocks)


def _decode_teacher_forced(stq, orc, wl_, bits, steps, head_begin=0, head_count=None, slots_perm=True, seed_tok=0):
    """Run `steps` teacher-forced steps; returns the tally."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    B, H, d = wl_.batch, wl_.heads, wl_.d
    hc = H - head_begin if head_count is None else head_count
    lay = stq.Layout(bits, d, gate=wl_.gate, in_dtype=wl_.in_dtype)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(B)])
    opool = _oracle_init(orc, wl_, bits, S0, w)
    nslots = B + 3
    total = lay.bytes_per_request
    # requests live at permuted slots of a larger pool (slot != request index)
    slot_of = (np.random.default_rng(5).permutation(nslots)[:B] if slots_perm else np.arange(B)).astype(np.int32)
    gpool = torch.zeros(nslots * total, dtype=torch.uint8, device=DEV)
    slots = torch.from_numpy(slot_of).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    tally = Tally()
    hs = slice(head_begin, head_begin + hc)
    w_call = w[hs].contiguous()
    for t in range(steps):
        inp = wlm.decode_inputs(wl_, seed_tok + t)
        inp_h = {n: x[:, hs].contiguous() for n, x in inp.items()}
        # upload the oracle's pre-step state into the permuted slots
        host = np.zeros(nslots * total, dtype=np.uint8)
        for r in range(B):
            host[slot_of[r] * total:(slot_of[r] + 1) * total] = opool[r * total:(r + 1) * total]
        gpool.copy_(torch.from_numpy(host).to(DEV))
        o = torch.zeros(B, hc, d, dtype=torch.float32, device=DEV)
        g = {n: x.to(DEV) for n, x in inp_h.items()}
        stq.decode_step(lay, gpool, slots, g["q"], g["k"], g["v"], g["beta"], g["alpha"], w_call.to(DEV), o,
                        head_begin=head_begin, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, stq.status_flags(status)
        gp = gpool.cpu().numpy()
        og = o.cpu().numpy()
        new_opool = opool.copy()
        for r in range(B):
            for h in range(H):
                ref_blk = tile_bytes(orc, opool, bits, d, r, h)
                got_blk = tile_bytes(orc, gp, bits, d, int(slot_of[r]), h)
                if not (head_begin <= h < head_begin + hc):
                    assert np.array_equal(got_blk, ref_blk), f"head {h} outside the call changed"
                    continue
                hr = h - head_begin
                alpha = inp["alpha"][r, h].double().numpy()
                res = orc.decode_step(bits[h], wl_.gate, ref_blk, as_f64(inp["q"][r, h]), as_f64(inp["k"][r, h]),
                                      as_f64(inp["v"][r, h]), float(inp["beta"][r, h]), alpha, as_f64(w[h]), d, d)
                assert res["status"] == orc.OK
                M = None
                if bits[h] == 16:
                    M = update_magnitude(orc.dequantize(16, d, d, ref_blk), as_f64(inp["k"][r, h]),
                                         as_f64(inp["v"][r, h]), float(inp["beta"][r, h]), alpha)
                compare_block(orc, bits[h], d, got_blk, res["block"], res["tie"], tally, f"step {t} req {r} head {h}",
                              err_scale=M)
                compare_o(og[r, hr], res["o"], tally, f"o step {t} req {r} head {h}")
                offs, _ = orc.request_layout(bits, d, d)
                new_opool[r * total + offs[h]: r * total + offs[h] + res["block"].size] = res["block"]
        opool = new_opool
    tally.check_budget()
    return tally


def test_pr1_d16_sixty_four_steps(stq, orc):
    """1 request x 1 head, d = 16, 6-bit, fp32 inputs, every one of the 64 steps."""
    wl_ = _wl("pr1_d16_6bit")
    t = _decode_teacher_forced(stq, orc, wl_, [6], 64)
    assert t.codes == 64 * 256


@pytest.mark.parametrize("bits", [4, 6, 8, 16])
def test_layer_d128_uniform_width(stq, orc, bits):
    """The 48-head layer workload (d = 128, bf16 inputs, scalar gate) at 5 requests x 12 heads."""
    wl_ = _wl("layer48_b8_4bit", batch=5, heads=12, bits=bits)
    _decode_teacher_forced(stq, orc, wl_, [bits] * 12, 4)


def test_mixed_widths_with_pivots_ragged(stq, orc):
    """Mixed 4/6/8/16 heads in one launch, 7 requests (ragged), fp32 inputs."""
    wl_ = _wl("layer48_b8_4bit", batch=7, heads=9, bits=None, in_dtype=torch.float32)
    bits = [4, 16, 6, 8, 4, 6, 16, 8, 4]
    _decode_teacher_forced(stq, orc, wl_, bits, 3)


@pytest.mark.parametrize("gate", [1, 2])
def test_channel_gates(stq, orc, gate):
    wl_ = _wl("channel32_b128_4bit", batch=3, heads=6, gate=gate)
    _decode_teacher_forced(stq, orc, wl_, [4, 8, 6, 16, 4, 6], 3)


@pytest.mark.parametrize("d", [32, 64])
def test_small_heads(stq, orc, d):
    wl_ = _wl("layer48_b8_4bit", batch=3, heads=5, d=d, in_dtype=torch.float32)
    _decode_teacher_forced(stq, orc, wl_, [4, 6, 8, 16, 6], 3)


def test_head_subset_leaves_other_heads_alone(stq, orc):
    wl_ = _wl("layer48_b8_4bit", batch=3, heads=10, bits=None)
    bits = [4, 6, 8, 16, 4, 6, 8, 16, 4, 6]
    _decode_teacher_forced(stq, orc, wl_, bits, 2, head_begin=3, head_count=4)


def test_many_requests_split_launches(stq, orc):
    """More requests than one launch caches (1024): the host splits the call."""
    wl_ = _wl("layer48_b8_4bit", batch=1030, heads=1, bits=4)
    _decode_teacher_forced(stq, orc, wl_, [4], 1, slots_perm=False)


def test_per_width_launches_equal_one_launch_for_all_widths(stq):
    """A large call (every width has at least 8192 tiles: one launch per width) and the same
    requests issued in calls of 2048 requests (one launch for all widths) give the same bytes and
    readouts, for both scale formats."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [4, 6, 16, 8]
    for scale_dtype in (torch.float32, torch.bfloat16):
        wl_ = _wl("full2304_b70_mixed", batch=8192, heads=len(bits), outliers=False)
        B, H, d = wl_.batch, wl_.heads, wl_.d
        lay = stq.Layout(bits, d, gate=wl_.gate, in_dtype=wl_.in_dtype, scale_dtype=scale_dtype)
        w = wlm.impact_weights(wl_).to(DEV)
        slots = torch.arange(B, dtype=torch.int32, device=DEV)
        pool0 = lay.alloc_pool(B)
        for b0 in range(0, B, 1024):
            S0 = torch.stack([wlm.initial_state(wl_, r, DEV) for r in range(b0, b0 + 1024)])
            stq.init_state(lay, pool0, slots[b0:b0 + 1024].clone(), S0, w)
        g = {n: x.to(DEV) for n, x in wlm.decode_inputs(wl_, 0).items()}
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        pool_a, o_a = pool0.clone(), torch.zeros(B, H, d, device=DEV)
        stq.decode_step(lay, pool_a, slots, g["q"], g["k"], g["v"], g["beta"], g["alpha"], w, o_a, status=status)
        pool_b, o_b = pool0.clone(), torch.zeros(B, H, d, device=DEV)
        for b0 in range(0, B, 2048):
            sl = slice(b0, b0 + 2048)
            stq.decode_step(lay, pool_b, slots[sl].contiguous(), g["q"][sl].contiguous(), g["k"][sl].contiguous(),
                            g["v"][sl].contiguous(), g["beta"][sl].contiguous(), g["alpha"][sl].contiguous(), w,
                            o_b[sl], status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, stq.status_flags(status)
        assert torch.equal(pool_a, pool_b)
        assert torch.equal(o_a, o_b)
        del pool0, pool_a, pool_b


def test_back_to_back_calls_without_sync(stq, orc):
    """Two stq_decode_step calls issued back to back on one stream with no synchronization between
    them (mixed widths with pivots and more than 256 requests: several width and request-group
    launches per call) give the same pool bytes and readouts as the same calls with a
    synchronization between them, and the second step matches the oracle from the first step's
    pool on sampled tiles."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [4, 6, 8, 16, 8, 6, 4, 16]
    wl_ = _wl("full2304_b70_mixed", batch=300, heads=len(bits), outliers=False)
    B, H, d = wl_.batch, wl_.heads, wl_.d
    lay = stq.Layout(bits, d, gate=wl_.gate, in_dtype=wl_.in_dtype)
    w = wlm.impact_weights(wl_).to(DEV)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(B)]).to(DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV).flip(0).contiguous()
    pool0 = lay.alloc_pool(B)
    stq.init_state(lay, pool0, slots, S0, w)
    ins = [{n: x.to(DEV) for n, x in wlm.decode_inputs(wl_, t).items()} for t in range(2)]

    def run(sync_between):
        pool = pool0.clone()
        outs = [torch.zeros(B, H, d, device=DEV) for _ in range(2)]
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        mid = None
        for t in range(2):
            g = ins[t]
            stq.decode_step(lay, pool, slots, g["q"], g["k"], g["v"], g["beta"], g["alpha"], w, outs[t],
                            status=status)
            if sync_between and t == 0:
                torch.cuda.synchronize()
                mid = pool.clone()
        torch.cuda.synchronize()
        assert status.item() == 0, stq.status_flags(status)
        return pool, outs, mid

    p_ref, o_ref, mid = run(True)
    p_b2b, o_b2b, _ = run(False)
    assert torch.equal(p_ref, p_b2b)
    assert torch.equal(o_ref[0], o_b2b[0]) and torch.equal(o_ref[1], o_b2b[1])
    # second step teacher forced from the first step's GPU pool, sampled tiles
    midh, finh, o1 = mid.cpu().numpy(), p_ref.cpu().numpy(), o_ref[1].cpu().numpy()
    inp = {n: x.cpu() for n, x in ins[1].items()}
    wc = w.cpu()
    tally = Tally()
    rng = np.random.default_rng(11)
    slot_of = slots.cpu().numpy()
    for r, h in zip(rng.integers(0, B, 24), rng.integers(0, H, 24)):
        r, h = int(r), int(h)
        pre = tile_bytes(orc, midh, bits, d, int(slot_of[r]), h)
        alpha = inp["alpha"][r, h].double().numpy()
        res = orc.decode_step(bits[h], wl_.gate, pre, as_f64(inp["q"][r, h]), as_f64(inp["k"][r, h]),
                              as_f64(inp["v"][r, h]), float(inp["beta"][r, h]), alpha, as_f64(wc[h]), d, d)
        M = None
        if bits[h] == 16:
            M = update_magnitude(orc.dequantize(16, d, d, pre), as_f64(inp["k"][r, h]), as_f64(inp["v"][r, h]),
                                 float(inp["beta"][r, h]), alpha)
        compare_block(orc, bits[h], d, tile_bytes(orc, finh, bits, d, int(slot_of[r]), h), res["block"], res["tie"],
                      tally, f"req {r} head {h}", err_scale=M)
        compare_o(o1[r, h], res["o"], tally, f"o req {r} head {h}")
    tally.check_budget()


# ------------------------------------------------------------------------------------------------
# init and dequantize
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("d,aligned", [(16, True), (32, True), (64, True), (128, True), (128, False), (32, False)])
def test_init_matches_oracle(stq, orc, d, aligned):
    """Init at every head size. The states reach the kernel 16-byte aligned (staged by 16-byte
    loads for d >= 32), or one float past a 16-byte boundary (staged element by element)."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=3, heads=8, d=d)
    bits = [4, 6, 8, 16, 8, 6, 4, 16]
    lay = stq.Layout(bits, d, in_dtype=torch.bfloat16)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(3)])
    ref = _oracle_init(orc, wl_, bits, S0, w)
    pool = lay.alloc_pool(3)
    slots = torch.arange(3, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if aligned:
        S0_dev = S0.to(DEV)
        assert S0_dev.data_ptr() % 16 == 0
    else:
        flat = torch.zeros(S0.numel() + 1, device=DEV)
        S0_dev = flat[1:].view(S0.shape)
        S0_dev.copy_(S0.to(DEV))
        assert S0_dev.data_ptr() % 16 == 4
    stq.init_state(lay, pool, slots, S0_dev, w.to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    gp = pool.cpu().numpy()
    tally = Tally()
    for r in range(3):
        for h in range(8):
            _, _, tie, _ = orc.quantize(bits[h], as_f64(S0[r, h]), as_f64(w[h]))
            compare_block(orc, bits[h], d, tile_bytes(orc, gp, bits, d, r, h), tile_bytes(orc, ref, bits, d, r, h),
                          tie, tally, f"init req {r} head {h}")
    tally.check_budget()


def _init_two_ways(stq, lay, S0, w, nslots=None):
    """Init the same states twice: 16-byte aligned (the streaming kernel takes the 128 x 128 row x
    column heads) and one float off (every head takes the plain kernel)."""
    B = S0.shape[0]
    out = []
    for aligned in (True, False):
        pool = lay.alloc_pool(nslots or B)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        if aligned:
            S_dev = S0.to(DEV).contiguous()
        else:
            flat = torch.zeros(S0.numel() + 1, device=DEV)
            S_dev = flat[1:].view(S0.shape)
            S_dev.copy_(S0.to(DEV))
        stq.init_state(lay, pool, torch.arange(B, dtype=torch.int32, device=DEV), S_dev, w.to(DEV), status=status)
        torch.cuda.synchronize()
        out.append((pool.cpu(), status.item()))
    return out


@pytest.mark.parametrize("scale_dtype", [torch.float32, torch.bfloat16])
def test_init_degenerate_tiles_same_bytes_both_kernels(stq, scale_dtype):
    """All-zero tiles (unit scales, zero codes) and subnormal tiles: every column energy underflows
    to 0 (column scale 1) and the row scale is subnormal, so its reciprocal overflows and the codes
    take the element-by-element form. Both init kernels reach these bytes exactly."""
    bits = [4, 6, 8, 16]
    lay = stq.Layout(bits, 128, scale_dtype=scale_dtype)
    g = torch.Generator().manual_seed(11)
    S0 = torch.randn(2, 4, 128, 128, generator=g) * 1e-39
    S0[0, 0] = 0.0
    S0[1, 2] = 0.0
    w = torch.rand(4, 128, generator=g) + 0.5
    (pa, sa), (pb, sb) = _init_two_ways(stq, lay, S0, w)
    # fp32 scales stay finite and non-zero; a bf16 row scale may round to zero and be flagged
    assert sa == sb and (sa == 0 or scale_dtype == torch.bfloat16)
    assert torch.equal(pa, pb)


def test_init_out_of_range_slots_flagged_others_written(stq, orc):
    """Requests with an out-of-range pool slot are flagged and skipped by init; the others are
    written as the oracle quantizes them, by both init kernels."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=3, heads=4)
    bits = [4, 6, 8, 16]
    lay = stq.Layout(bits, 128)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(3)])
    total = lay.bytes_per_request
    for aligned in (True, False):
        pool = lay.alloc_pool(2)
        pool.fill_(7)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        slots = torch.tensor([1, 5, -1], dtype=torch.int32, device=DEV)
        if aligned:
            S_dev = S0.to(DEV)
        else:
            flat = torch.zeros(S0.numel() + 1, device=DEV)
            S_dev = flat[1:].view(S0.shape)
            S_dev.copy_(S0.to(DEV))
        stq.init_state(lay, pool, slots, S_dev, w.to(DEV), status=status)
        torch.cuda.synchronize()
        assert status.item() & (1 << stq.api.STQ_ERR_BOUNDS)
        gp = pool.cpu().numpy()
        assert np.all(gp[:total] == 7), "slot 0 belongs to no request and stays untouched"
        ref = _oracle_init(orc, wl_, bits, S0[:1], w)
        tally = Tally()
        for h in range(4):
            _, _, tie, _ = orc.quantize(bits[h], as_f64(S0[0, h]), as_f64(w[h]))
            compare_block(orc, bits[h], 128, tile_bytes(orc, gp, bits, 128, 1, h), tile_bytes(orc, ref, bits, 128, 0, h),
                          tie, tally, f"init slot 1 head {h} aligned={aligned}")
        tally.check_budget()


@pytest.mark.parametrize("scale_dtype", [torch.float32, torch.bfloat16])
def test_init_several_tiles_per_cta_with_skipped_requests(stq, orc, scale_dtype):
    """Init with several tiles per CTA of the streaming kernel (40 requests x 14 row x column heads
    = 560 tiles over at most 148 CTAs: both groups of a CTA take tiles, and the three ring slots
    are each reused), mixed widths, and every seventh request on an out-of-range slot. The skipped
    requests are flagged and leave the pool untouched; every written tile matches the oracle."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    B = 40
    bits = [4, 6, 8, 16, 8, 6, 4, 4, 6, 8, 6, 4, 8, 16, 6, 4]
    wl_ = _wl("full2304_b70_mixed", batch=B, heads=len(bits), outliers=False)
    H, d = len(bits), 128
    lay = stq.Layout(bits, d, scale_dtype=scale_dtype)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(B)])
    total = lay.bytes_per_request
    pool = lay.alloc_pool(B + 1)
    pool.fill_(7)
    slot_of = [-1 if r % 7 == 3 else r + 1 for r in range(B)]  # slot 0 belongs to no request
    slots = torch.tensor(slot_of, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    S_dev = S0.to(DEV)
    assert S_dev.data_ptr() % 16 == 0
    stq.init_state(lay, pool, slots, S_dev, w.to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() & (1 << stq.api.STQ_ERR_BOUNDS)
    assert status.item() & ~(1 << stq.api.STQ_ERR_BOUNDS) == 0, stq.status_flags(status)
    gp = pool.cpu().numpy()
    assert np.all(gp[:total] == 7), "slot 0 belongs to no request and stays untouched"
    written = [r for r in range(B) if slot_of[r] >= 0]
    assert sorted(slot_of[r] for r in written) == [r + 1 for r in written]
    for r in range(B):
        if slot_of[r] < 0:
            assert np.all(gp[(r + 1) * total:(r + 2) * total] == 7), f"skipped request {r}'s slot was written"
    sb16 = scale_dtype == torch.bfloat16
    tally = Tally()
    for r in written:
        for h in range(H):
            base = slot_of[r] * total + lay.head_offset(h)
            got = gp[base: base + lay.head_bytes(h)]
            if sb16 and bits[h] != 16:
                compare_block_bf16s(orc, bits[h], d, got, as_f64(S0[r, h]), as_f64(w[h]), tally,
                                    f"init req {r} head {h}")
            else:
                blk, _, tie, st = orc.quantize(bits[h], as_f64(S0[r, h]), as_f64(w[h]))
                assert st == orc.OK
                compare_block(orc, bits[h], d, got[:blk.size], blk, tie, tally, f"init req {r} head {h}")
    tally.check_budget()


def test_init_nonfinite_state_is_flagged(stq, orc):
    """A state with an infinite entry raises the non-finite flag in either init kernel; the other
    heads of the call still match the oracle."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=1, heads=3)
    bits = [6, 4, 8]
    lay = stq.Layout(bits, 128)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, 0)])
    S0[0, 1, 5, 9] = float("inf")
    ref = _oracle_init(orc, wl_, [bits[0]], S0[:, :1], w[:1])
    for (pool, status) in _init_two_ways(stq, lay, S0, w):
        assert status & (1 << stq.api.STQ_ERR_NONFINITE)
        gp = pool.numpy()
        tally = Tally()
        _, _, tie, _ = orc.quantize(bits[0], as_f64(S0[0, 0]), as_f64(w[0]))
        compare_block(orc, bits[0], 128, tile_bytes(orc, gp, bits, 128, 0, 0), tile_bytes(orc, ref, [bits[0]], 128, 0, 0),
                      tie, tally, "init head 0 beside a non-finite head")
        tally.check_budget()


def test_dequantize_matches_oracle(stq, orc):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=2, heads=6)
    bits = [4, 6, 8, 16, 4, 8]
    lay = stq.Layout(bits, 128)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(2)])
    ref = _oracle_init(orc, wl_, bits, S0, w)
    pool = torch.from_numpy(ref).to(DEV)
    slots = torch.tensor([1, 0], dtype=torch.int32, device=DEV)
    out = torch.zeros(2, 6, 128, 128, device=DEV)
    stq.dequantize(lay, pool, slots, out)
    got = out.cpu().double().numpy()
    for r, slot in enumerate([1, 0]):
        for h in range(6):
            S = orc.dequantize(bits[h], 128, 128, tile_bytes(orc, ref, bits, 128, slot, h))
            assert np.all(np.abs(got[r, h] - S) <= 2.0 ** -22 * np.abs(S))


# ------------------------------------------------------------------------------------------------
# edge cases and device status
# ------------------------------------------------------------------------------------------------

def test_zero_state_first_write(stq, orc):
    """A zero state (scales 1, codes 0) takes a rank-1 write on its first step."""
    lay = stq.Layout([6, 4], 128, in_dtype=torch.float32)
    w = torch.ones(2, 128)
    pool = lay.alloc_pool(1)
    slots = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.init_state(lay, pool, slots, torch.zeros(1, 2, 128, 128, device=DEV), w.to(DEV))
    ref0 = pool.cpu().numpy().copy()
    rng = np.random.default_rng(0)
    q, k, v = (torch.from_numpy(rng.standard_normal((1, 2, 128))).float() for _ in range(3))
    beta = torch.full((1, 2), 0.5)
    alpha = torch.full((1, 2), 0.9)
    o = torch.zeros(1, 2, 128, device=DEV)
    stq.decode_step(lay, pool, slots, q.to(DEV), k.to(DEV), v.to(DEV), beta.to(DEV), alpha.to(DEV), w.to(DEV), o)
    gp = pool.cpu().numpy()
    tally = Tally()
    for h, b in enumerate([6, 4]):
        blk = tile_bytes(orc, ref0, [6, 4], 128, 0, h)
        assert not orc.codes(b, 128, 128, blk).any()
        res = orc.decode_step(b, 0, blk, as_f64(q[0, h]), as_f64(k[0, h]), as_f64(v[0, h]), 0.5, 0.9,
                              np.ones(128), 128, 128)
        compare_block(orc, b, 128, tile_bytes(orc, gp, [6, 4], 128, 0, h), res["block"], res["tie"], tally)
        compare_o(o[0, h].cpu().numpy(), res["o"], tally)


def test_out_of_range_slot_is_flagged_and_skipped(stq):
    lay = stq.Layout([4, 8], 128, in_dtype=torch.float32)
    pool = lay.alloc_pool(2)
    pool.fill_(7)
    before = pool.clone()
    slots = torch.tensor([5, -1], dtype=torch.int32, device=DEV)
    B, H = 2, 2
    z = torch.zeros(B, H, 128, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.decode_step(lay, pool, slots, z, z, z, torch.zeros(B, H, device=DEV), torch.ones(B, H, device=DEV),
                    torch.ones(H, 128, device=DEV), torch.zeros(B, H, 128, device=DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() & (1 << stq.api.STQ_ERR_BOUNDS)
    assert torch.equal(pool, before)


def test_nonfinite_input_is_flagged(stq, orc):
    lay = stq.Layout([6, 16], 128, in_dtype=torch.float32)
    pool = lay.alloc_pool(1)
    slots = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.init_state(lay, pool, slots, torch.randn(1, 2, 128, 128, device=DEV), torch.ones(2, 128, device=DEV))
    v = torch.full((1, 2, 128), float("inf"), device=DEV)
    k = torch.nn.functional.normalize(torch.randn(1, 2, 128, device=DEV), dim=-1)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.decode_step(lay, pool, slots, k, k, v, torch.full((1, 2), 0.5, device=DEV), torch.full((1, 2), 0.9, device=DEV),
                    torch.ones(2, 128, device=DEV), torch.zeros(1, 2, 128, device=DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() & (1 << stq.api.STQ_ERR_NONFINITE)


def test_bounded_wait_gives_up_and_reports_timeout(stq):
    """A wait that nothing completes gives up after the library's cap (~2 s of clock) and reports
    STQ_ERR_TIMEOUT in the status word; the context stays usable for the next call."""
    import time

    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    stq.selftest_wait_timeout(status)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert status.item() == 1 << stq.api.STQ_ERR_TIMEOUT
    assert 0.5 < waited < 30.0
    # a normal call afterwards runs and reports nothing
    lay = stq.Layout([4, 16], 128)
    pool = lay.alloc_pool(1)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    S0 = torch.randn(1, 2, 128, 128, device=DEV)
    stq.init_state(lay, pool, torch.zeros(1, dtype=torch.int32, device=DEV), S0, torch.ones(2, 128, device=DEV),
                   status=st2)
    out = torch.zeros_like(S0)
    stq.dequantize(lay, pool, torch.zeros(1, dtype=torch.int32, device=DEV), out, status=st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    assert torch.equal(out[0, 1], S0[0, 1].half().float())  # the pivot head round-trips through fp16


def test_empty_calls_are_noops(stq):
    lay = stq.Layout([4], 128)
    pool = lay.alloc_pool(1)
    e = torch.zeros(0, 1, 128, dtype=torch.bfloat16, device=DEV)
    stq.decode_step(lay, pool, torch.zeros(0, dtype=torch.int32, device=DEV), e, e, e,
                    torch.zeros(0, 1, device=DEV), torch.zeros(0, 1, device=DEV), torch.ones(1, 128, device=DEV),
                    torch.zeros(0, 1, 128, device=DEV))
    torch.cuda.synchronize()
    assert not pool.any()


def test_step_is_deterministic(stq):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("full2304_b70_mixed", batch=9, heads=40)
    bits = wlm.head_bits(wlm.WORKLOADS["full2304_b70_mixed"])[:40]
    lay = stq.Layout(bits, 128)
    w = wlm.impact_weights(wl_).to(DEV)
    pool = lay.alloc_pool(9)
    slots = torch.arange(9, dtype=torch.int32, device=DEV)
    stq.init_state(lay, pool, slots, torch.stack([wlm.initial_state(wl_, r, DEV) for r in range(9)]), w)
    inp = wlm.decode_inputs(wl_, 0, DEV)
    outs = []
    for _ in range(2):
        p = pool.clone()
        o = torch.zeros(9, 40, 128, device=DEV)
        stq.decode_step(lay, p, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w, o)
        outs.append((p, o))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_free_running_error_statistics_match_oracle(stq, orc):
    """Over 48 free-running steps, the GPU and oracle trajectories each drift from the unquantized
    fp64 recurrence by the same amount (mean and p99 of the readout error within 10%)."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = _wl("layer48_b8_4bit", batch=2, heads=4, bits=6, in_dtype=torch.float32)
    bits = [6, 4, 8, 6]
    B, H, d = 2, 4, 128
    lay = stq.Layout(bits, d, in_dtype=torch.float32)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(B)])
    opool = _oracle_init(orc, wl_, bits, S0, w)
    gpool = torch.from_numpy(opool.copy()).to(DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    Sref = {(r, h): orc.dequantize(bits[h], d, d, tile_bytes(orc, opool, bits, d, r, h)) for r in range(B) for h in range(H)}
    err_g, err_o = [], []
    total = lay.bytes_per_request
    offs, _ = orc.request_layout(bits, d, d)
    for t in range(48):
        inp = wlm.decode_inputs(wl_, t)
        o = torch.zeros(B, H, d, device=DEV)
        stq.decode_step(lay, gpool, slots, *(inp[n].to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV), o)
        og = o.cpu().numpy()
        for r in range(B):
            for h in range(H):
                a = float(inp["alpha"][r, h])
                q, k, v = (as_f64(inp[n][r, h]) for n in ("q", "k", "v"))
                Sn, oref = orc.update(0, Sref[(r, h)], q, k, v, float(inp["beta"][r, h]), a)
                Sref[(r, h)] = Sn
                blk = tile_bytes(orc, opool, bits, d, r, h)
                res = orc.decode_step(bits[h], 0, blk, q, k, v, float(inp["beta"][r, h]), a, as_f64(w[h]), d, d)
                opool[r * total + offs[h]: r * total + offs[h] + blk.size] = res["block"]
                n = np.linalg.norm(oref)
                err_o.append(np.linalg.norm(res["o"] - oref) / n)
                err_g.append(np.linalg.norm(og[r, h] - oref) / n)
    err_g, err_o = np.array(err_g), np.array(err_o)
    assert abs(err_g.mean() / err_o.mean() - 1) < 0.10
    assert abs(np.percentile(err_g, 99) / np.percentile(err_o, 99) - 1) < 0.10


def test_partially_invalid_slots(stq, orc):
    """Tiles of an out-of-range slot are skipped and flagged; the others of the same launch are
    still computed correctly."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [4, 16, 8, 6]
    wl_ = _wl("layer48_b8_4bit", batch=3, heads=4, bits=None)
    lay = stq.Layout(bits, 128)
    w = wlm.impact_weights(wl_)
    S0 = torch.stack([wlm.initial_state(wl_, r) for r in range(3)])
    opool = _oracle_init(orc, wl_, bits, S0, w)
    gpool = torch.from_numpy(opool.copy()).to(DEV)
    slots = torch.tensor([2, 7, 0], dtype=torch.int32, device=DEV)  # request 1 has no valid slot
    inp = wlm.decode_inputs(wl_, 3)
    o = torch.zeros(3, 4, 128, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.decode_step(lay, gpool, slots, *(inp[n].to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV), o,
                    status=status)
    torch.cuda.synchronize()
    assert status.item() == (1 << stq.api.STQ_ERR_BOUNDS)
    gp = gpool.cpu().numpy()
    tally = Tally()
    for r, slot in ((0, 2), (2, 0)):
        for h in range(4):
            pre = tile_bytes(orc, opool, bits, 128, slot, h)
            res = orc.decode_step(bits[h], 0, pre, as_f64(inp["q"][r, h]), as_f64(inp["k"][r, h]),
                                  as_f64(inp["v"][r, h]), float(inp["beta"][r, h]), float(inp["alpha"][r, h]),
                                  as_f64(w[h]), 128, 128)
            M = update_magnitude(orc.dequantize(16, 128, 128, pre), as_f64(inp["k"][r, h]), as_f64(inp["v"][r, h]),
                                 float(inp["beta"][r, h]), float(inp["alpha"][r, h])) if bits[h] == 16 else None
            compare_block(orc, bits[h], 128, tile_bytes(orc, gp, bits, 128, slot, h), res["block"], res["tie"],
                          tally, err_scale=M)
            compare_o(o[r, h].cpu().numpy(), res["o"], tally)
    # slot 1 (not addressed by any request) is untouched
    assert np.array_equal(gp[lay.bytes_per_request: 2 * lay.bytes_per_request],
                          opool[lay.bytes_per_request: 2 * lay.bytes_per_request])


def test_full_batch70_launch_sampled(stq, orc):
    """The bench's launch (70 requests x 2304 mixed heads, ~545 tiles per CTA through the staging
    ring) checked on 96 sampled tiles: their pre-step bytes come from the oracle, every other tile
    is initialised on the GPU and only has to stay finite."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = wlm.WORKLOADS["full2304_b70_mixed"]
    B, H, d = wl_.batch, wl_.heads, wl_.d
    bits = wlm.head_bits(wl_)
    lay = stq.Layout(bits, d)
    w = wlm.impact_weights(wl_, DEV)
    pool = lay.alloc_pool(B)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    rng = np.random.default_rng(42)
    heads_by_width = {b: [h for h in range(H) if bits[h] == b] for b in (4, 6, 8, 16)}
    sample = []
    for b, hs in heads_by_width.items():
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
    offs, total = orc.request_layout(bits, d, d)
    pre = {}
    for (r, h) in sample:
        blk, _, _, _ = orc.quantize(bits[h], S0_sample[(r, h)], wc[h])
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
        args = [inp[n][r, h].double().cpu().numpy() for n in ("q", "k", "v")]
        beta, alpha = float(inp["beta"][r, h]), float(inp["alpha"][r, h])
        res = orc.decode_step(bits[h], 0, pre[(r, h)], *args, beta, alpha, wc[h], d, d)
        M = update_magnitude(orc.dequantize(16, d, d, pre[(r, h)]), args[1], args[2], beta, alpha) \
            if bits[h] == 16 else None
        compare_block(orc, bits[h], d, got, res["block"], res["tie"], tally, f"req {r} head {h}", err_scale=M)
        compare_o(o[r, h].cpu().numpy(), res["o"], tally, f"o req {r} head {h}")
    tally.check_budget()


def test_per_layer_calls_equal_one_call_and_graph_replay(stq):
    """A token issued as one stq_decode_step per layer of 48 heads (the serving shape) gives the
    same bytes and readout as one call over all heads, eagerly and replayed from a CUDA graph."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl_ = wlm.scaled(wlm.WORKLOADS["full2304_b70_mixed"], batch=3)
    B, H, d = wl_.batch, wl_.heads, wl_.d
    bits = wlm.head_bits(wl_)
    lay = stq.Layout(bits, d)
    w = wlm.impact_weights(wl_, DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    pool0 = lay.alloc_pool(B)
    stq.init_state(lay, pool0, slots, torch.stack([wlm.initial_state(wl_, r, DEV) for r in range(B)]), w)
    inp = wlm.decode_inputs(wl_, 0, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pool_a = pool0.clone()
    o_a = torch.zeros(B, H, d, device=DEV)
    stq.decode_step(lay, pool_a, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], w, o_a,
                    status=status)
    per = 48
    parts = [{n: x[:, l * per:(l + 1) * per].contiguous() for n, x in inp.items()} for l in range(H // per)]
    w_l = [w[l * per:(l + 1) * per].contiguous() for l in range(H // per)]
    o_l = [torch.zeros(B, per, d, device=DEV) for _ in range(H // per)]

    def token(pool):
        for l, x in enumerate(parts):
            stq.decode_step(lay, pool, slots, x["q"], x["k"], x["v"], x["beta"], x["alpha"], w_l[l], o_l[l],
                            head_begin=l * per, status=status)

    pool_b = pool0.clone()
    token(pool_b)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.equal(pool_a, pool_b)
    assert torch.equal(o_a, torch.cat(o_l, dim=1))
    pool_c = pool0.clone()
    for t in o_l:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        token(pool_c)
    pool_c.copy_(pool0)
    g.replay()
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.equal(pool_a, pool_c)
    assert torch.equal(o_a, torch.cat(o_l, dim=1))


def test_more_heads_than_one_launch_table(stq, orc):
    """3200 heads of one width in one call: the host splits the head table (3072 entries per
    launch) for init, decode and dequantize. Sampled heads on both sides of the split match the
    oracle, and every head stays finite."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    H, d, B = 3200, 128, 1
    wl_ = _wl("layer48_b8_4bit", batch=B, heads=H, bits=4)
    bits = [4] * H
    lay = stq.Layout(bits, d)
    w = wlm.impact_weights(wl_)
    S0 = wlm.initial_state(wl_, 0)[None]
    pool = lay.alloc_pool(B)
    slots = torch.zeros(1, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.init_state(lay, pool, slots, S0.to(DEV), w.to(DEV), status=status)
    sample = [0, 1, 3071, 3072, 3073, 3199]
    offs, total = orc.request_layout(bits, d, d)
    pre = {}
    for h in sample:
        blk = orc.quantize(4, as_f64(S0[0, h]), as_f64(w[h]))[0]
        pre[h] = blk
        pool[offs[h]: offs[h] + blk.size] = torch.from_numpy(blk).to(DEV)
    inp = wlm.decode_inputs(wl_, 0)
    o = torch.zeros(B, H, d, device=DEV)
    g = {n: x.to(DEV) for n, x in inp.items()}
    stq.decode_step(lay, pool, slots, g["q"], g["k"], g["v"], g["beta"], g["alpha"], w.to(DEV), o, status=status)
    out = torch.zeros(B, H, d, d, device=DEV)
    stq.dequantize(lay, pool, slots, out, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.isfinite(o).all() and torch.isfinite(out).all()
    gp = pool.cpu().numpy()
    tally = Tally()
    for h in sample:
        res = orc.decode_step(4, 0, pre[h], as_f64(inp["q"][0, h]), as_f64(inp["k"][0, h]), as_f64(inp["v"][0, h]),
                              float(inp["beta"][0, h]), float(inp["alpha"][0, h]), as_f64(w[h]), d, d)
        got = gp[offs[h]: offs[h] + pre[h].size]
        compare_block(orc, 4, d, got, res["block"], res["tie"], tally, f"head {h}")
        compare_o(o[0, h].cpu().numpy(), res["o"], tally, f"o head {h}")
        want = orc.dequantize(4, d, d, got)
        assert np.all(np.abs(out[0, h].cpu().double().numpy() - want) <= 2.0 ** -23 * np.abs(want)), f"head {h}"
    tally.check_budget()
