"""GPU parity of the chunked prefill against the oracle's sequential prefill (needs a B200).

Teacher-forced per chunk: the oracle's pre-chunk pool is uploaded, one single-chunk GPU call runs,
and the GPU's requantized state and every token's readout are compared with the oracle's chunk
from the same bytes. A multi-chunk call must be bit-identical to the same chunks issued one call
each.
"""
import numpy as np
import pytest
import torch

from _parity import (Tally, as_f64, compare_block, compare_o, compare_pivot_exact, oracle_pool, pivot_chunk_exact,
                     tile_bytes)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def stq():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    import quantized_linear_attention_stq_b200 as m

    m.lib()
    return m


def _setup(orc, B, bits, d=128, dtype=torch.bfloat16, base="prefill16_b16_6bit", gate=None):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    extra = {} if gate is None else {"gate": gate}
    wl_ = wlm.scaled(wlm.WORKLOADS[base], batch=B, heads=len(bits), d=d, in_dtype=dtype, **extra)
    w = wlm.impact_weights(wl_)
    blocks = []
    for r in range(B):
        S0 = wlm.initial_state(wl_, r)
        row = []
        for h, b in enumerate(bits):
            blk, _, _, st = orc.quantize(b, as_f64(S0[h]), as_f64(w[h]))
            assert st == orc.OK
            row.append(blk)
        blocks.append(row)
    return wl_, w, oracle_pool(orc, bits, d, blocks)


def _oracle_chunk(orc, pool, bits, d, r, h, inp, t0, T, w, chunk, gate=0):
    blk = tile_bytes(orc, pool, bits, d, r, h)
    sl = slice(t0, t0 + T)
    return orc.prefill_seq(bits[h], gate, blk, as_f64(inp["q"][r, h, sl]), as_f64(inp["k"][r, h, sl]),
                           as_f64(inp["v"][r, h, sl]), as_f64(inp["beta"][r, h, sl]), as_f64(inp["alpha"][r, h, sl]),
                           as_f64(w[h]), chunk, d, d)


def _check_chunk(orc, opool, gp, og, bits, d, B, inp, T, w, gate, tally):
    """Teacher-forced check of one single-chunk call: codes and scales (or, for a pivot, the
    per-value fp16 rule with the error bound carried through the chunk) and every readout."""
    for r in range(B):
        for h in range(len(bits)):
            what = f"req {r} head {h}"
            res = _oracle_chunk(orc, opool, bits, d, r, h, inp, 0, T, w, 64, gate)
            assert res["status"] == orc.OK
            got = tile_bytes(orc, gp, bits, d, r, h)
            if bits[h] == 16:
                S0 = orc.dequantize(16, d, d, tile_bytes(orc, opool, bits, d, r, h))
                args = [as_f64(inp[n][r, h, :T]) for n in ("q", "k", "v", "beta", "alpha")]
                S_ex, bound = pivot_chunk_exact(orc, gate, S0, *args)
                compare_pivot_exact(orc, d, got, res["block"], S_ex, bound, tally, what)
            else:
                compare_block(orc, bits[h], d, got, res["block"], res["tie"], tally, what)
            for t in range(T):
                compare_o(og[r, h, t], res["o"][t], tally, f"token {t} " + what)


def _workspace(stq, lay, B, T, C, form):
    """The three-kernel form gets a workspace of the size the library asks for; the one-kernel form
    gets none."""
    if form == "one_kernel":
        return None
    n = stq.prefill_workspace_bytes(lay, B, T, C)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("form", ["workspace", "one_kernel"])
@pytest.mark.parametrize("T", [64, 37, 1])
def test_single_chunk_teacher_forced(stq, orc, T, form):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [6, 4, 8, 16]
    B, d = 3, 128
    wl_, w, opool = _setup(orc, B, bits)
    lay = stq.Layout(bits, d, in_dtype=torch.bfloat16)
    inp = wlm.prefill_inputs(wl_, 0, T)
    gpool = torch.from_numpy(opool.copy()).to(DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    o = torch.zeros(B, len(bits), T, d, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = _workspace(stq, lay, B, T, 64, form)
    assert form == "one_kernel" or stq.prefill_workspace_bytes(lay, B, T, 64) > 0
    stq.prefill_chunk(lay, gpool, slots, *(inp[n].to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV), o,
                      chunk=64, workspace=ws, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    gp = gpool.cpu().numpy()
    og = o.cpu().numpy()
    tally = Tally()
    _check_chunk(orc, opool, gp, og, bits, d, B, inp, T, w, 0, tally)
    tally.check_budget()


@pytest.mark.parametrize("gate", [1, 2])
@pytest.mark.parametrize("d,T", [(128, 64), (128, 23), (32, 64), (32, 37)])
def test_channel_gate_single_chunk_teacher_forced(stq, orc, gate, d, T):
    """Both channel gates (alpha per key row: [B][H][T][d_k]) through stq_prefill_chunk, full and
    short chunks, mixed widths with an FP16 pivot, against the oracle's sequential prefill."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [6, 4, 8, 16]
    B = 2
    wl_, w, opool = _setup(orc, B, bits, d=d, base="channel32_b128_4bit", gate=gate)
    lay = stq.Layout(bits, d, gate=gate, in_dtype=torch.bfloat16)
    inp = wlm.prefill_inputs(wl_, 0, T)
    assert inp["alpha"].shape == (B, len(bits), T, d)
    # permuted slots: request 0 lives in slot 1 and request 1 in slot 0
    offs, total = orc.request_layout(bits, d, d)
    swap = lambda a: np.concatenate([a[total:2 * total], a[:total]])  # noqa: E731
    gpool = torch.from_numpy(swap(opool)).to(DEV)
    slots = torch.tensor([1, 0], dtype=torch.int32, device=DEV)
    o = torch.zeros(B, len(bits), T, d, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.prefill_chunk(lay, gpool, slots, *(inp[n].to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV), o,
                      chunk=64, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    gp, og = swap(gpool.cpu().numpy()), o.cpu().numpy()
    tally = Tally()
    _check_chunk(orc, opool, gp, og, bits, d, B, inp, T, w, gate, tally)
    tally.check_budget()


@pytest.mark.parametrize("gate", [1, 2])
def test_channel_gate_multi_chunk_equals_single_chunk_calls(stq, orc, gate):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [6, 16, 4]
    B, d, T, C = 2, 64, 80, 32
    wl_, w, opool = _setup(orc, B, bits, d=d, base="channel32_b128_4bit", gate=gate)
    lay = stq.Layout(bits, d, gate=gate, in_dtype=torch.bfloat16)
    inp = {n: x.to(DEV) for n, x in wlm.prefill_inputs(wl_, 0, T).items()}
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    wd = w.to(DEV)
    p_full = torch.from_numpy(opool.copy()).to(DEV)
    o_full = torch.zeros(B, 3, T, d, device=DEV)
    stq.prefill_chunk(lay, p_full, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], wd, o_full, chunk=C)
    p_seq = torch.from_numpy(opool.copy()).to(DEV)
    outs = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        part = {n: x[:, :, sl].contiguous() for n, x in inp.items()}
        o_part = torch.zeros(B, 3, sl.stop - sl.start, d, device=DEV)
        stq.prefill_chunk(lay, p_seq, slots, part["q"], part["k"], part["v"], part["beta"], part["alpha"], wd, o_part,
                          chunk=C)
        outs.append(o_part)
    torch.cuda.synchronize()
    assert torch.equal(p_full, p_seq)
    assert torch.equal(o_full, torch.cat(outs, dim=2))


@pytest.mark.parametrize("form", ["workspace", "one_kernel"])
def test_multi_chunk_equals_single_chunk_calls(stq, orc, form):
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [6, 8, 4]
    B, d, T, C = 2, 128, 150, 64
    wl_, w, opool = _setup(orc, B, bits)
    lay = stq.Layout(bits, d, in_dtype=torch.bfloat16)
    inp = {n: x.to(DEV) for n, x in wlm.prefill_inputs(wl_, 0, T).items()}
    slots = torch.tensor([1, 0], dtype=torch.int32, device=DEV)
    wd = w.to(DEV)
    ws = _workspace(stq, lay, B, T, C, form)
    p_full = torch.from_numpy(opool.copy()).to(DEV)
    o_full = torch.zeros(B, 3, T, d, device=DEV)
    stq.prefill_chunk(lay, p_full, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], wd, o_full,
                      chunk=C, workspace=ws)
    p_seq = torch.from_numpy(opool.copy()).to(DEV)
    outs = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        part = {n: x[:, :, sl].contiguous() for n, x in inp.items()}
        o_part = torch.zeros(B, 3, sl.stop - sl.start, d, device=DEV)
        stq.prefill_chunk(lay, p_seq, slots, part["q"], part["k"], part["v"], part["beta"], part["alpha"], wd, o_part,
                          chunk=C, workspace=ws)
        outs.append(o_part)
    torch.cuda.synchronize()
    assert torch.equal(p_full, p_seq)
    assert torch.equal(o_full, torch.cat(outs, dim=2))


def test_segments_equal_single_chunk_calls(stq, orc):
    """A three-kernel call over more than one segment of workspace records (34 chunks, the last one
    short; mixed widths with an FP16 pivot) equals the same chunks issued one call each, bit for
    bit, and its status stays clear."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [6, 16, 4, 8]
    B, d, C = 2, 128, 64
    T = 33 * C + 10
    wl_, w, opool = _setup(orc, B, bits)
    lay = stq.Layout(bits, d, in_dtype=torch.bfloat16)
    inp = {n: x.to(DEV) for n, x in wlm.prefill_inputs(wl_, 0, T).items()}
    slots = torch.tensor([1, 0], dtype=torch.int32, device=DEV)
    wd = w.to(DEV)
    rec = stq.prefill_workspace_bytes(stq.Layout([6], d, in_dtype=torch.bfloat16), 1, C, C)
    assert stq.prefill_workspace_bytes(lay, B, T, C) == B * 4 * 32 * rec  # two segments: 32 + 2 chunks
    ws = _workspace(stq, lay, B, T, C, "workspace")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    p_full = torch.from_numpy(opool.copy()).to(DEV)
    o_full = torch.zeros(B, len(bits), T, d, device=DEV)
    stq.prefill_chunk(lay, p_full, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], wd, o_full,
                      chunk=C, workspace=ws, status=status)
    p_seq = torch.from_numpy(opool.copy()).to(DEV)
    outs = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        part = {n: x[:, :, sl].contiguous() for n, x in inp.items()}
        o_part = torch.zeros(B, len(bits), sl.stop - sl.start, d, device=DEV)
        stq.prefill_chunk(lay, p_seq, slots, part["q"], part["k"], part["v"], part["beta"], part["alpha"], wd, o_part,
                          chunk=C, workspace=ws, status=status)
        outs.append(o_part)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.equal(p_full, p_seq)
    assert torch.equal(o_full, torch.cat(outs, dim=2))


@pytest.mark.parametrize("form", ["workspace", "one_kernel"])
def test_full_geometry_chunk_chain_and_sampled_first_chunk(stq, orc, form):
    """The 16-request x 16-head, 6-bit prefill workload in its bench launch shape (all tiles in
    one launch, more tiles than SMs), over 4 chunks: the multi-chunk call equals the chain of
    single-chunk calls bit for bit, and sampled tiles match the oracle on the first chunk."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl = wlm.WORKLOADS["prefill16_b16_6bit"]
    B, H, d, T, C = wl.batch, wl.heads, wl.d, 256, 64
    bits = wlm.head_bits(wl)
    lay = stq.Layout(bits, d, in_dtype=wl.in_dtype)
    w = wlm.impact_weights(wl)
    blocks = []
    for r in range(B):
        S0 = wlm.initial_state(wl, r)
        blocks.append([orc.quantize(bits[h], as_f64(S0[h]), as_f64(w[h]))[0] for h in range(H)])
    opool = oracle_pool(orc, bits, d, blocks)
    inp = {n: x.to(DEV) for n, x in wlm.prefill_inputs(wl, 0, T).items()}
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    wd = w.to(DEV)
    ws = _workspace(stq, lay, B, T, C, form)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    p_full = torch.from_numpy(opool.copy()).to(DEV)
    o_full = torch.zeros(B, H, T, d, device=DEV)
    stq.prefill_chunk(lay, p_full, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], wd, o_full,
                      chunk=C, workspace=ws, status=status)
    p_seq = torch.from_numpy(opool.copy()).to(DEV)
    outs = []
    first_pool = None
    for c0 in range(0, T, C):
        part = {n: x[:, :, c0:c0 + C].contiguous() for n, x in inp.items()}
        o_part = torch.zeros(B, H, C, d, device=DEV)
        stq.prefill_chunk(lay, p_seq, slots, part["q"], part["k"], part["v"], part["beta"], part["alpha"], wd,
                          o_part, chunk=C, workspace=ws, status=status)
        outs.append(o_part)
        if first_pool is None:
            torch.cuda.synchronize()
            first_pool = p_seq.cpu().numpy()
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(p_full, p_seq)
    assert torch.equal(o_full, torch.cat(outs, dim=2))
    # teacher-forced first chunk of sampled tiles
    cpu_inp = {n: x[:, :, :C].cpu() for n, x in inp.items()}
    o0 = outs[0].cpu().numpy()
    tally = Tally()
    rng = np.random.default_rng(5)
    for r, h in zip(rng.integers(0, B, 6), rng.integers(0, H, 6)):
        res = _oracle_chunk(orc, opool, bits, d, int(r), int(h), cpu_inp, 0, C, w, C)
        assert res["status"] == orc.OK
        compare_block(orc, bits[h], d, tile_bytes(orc, first_pool, bits, d, int(r), int(h)), res["block"],
                      res["tie"], tally, f"req {r} head {h}")
        for t in range(C):
            compare_o(o0[r, h, t], res["o"][t], tally, f"token {t} req {r} head {h}")
    tally.check_budget()


def test_bench_size_call_equals_segment_calls_and_first_chunk_parity(stq, orc):
    """The bench's prefill in its launch configuration: 16 requests x 16 heads, 6-bit, an
    8192-token prompt through the workspace (four segments of 32 chunks, 256 tiles in every
    launch). The whole call equals four 2048-token calls (one segment each) bit for bit, and
    sampled tiles match the oracle on the call's first chunk."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    wl = wlm.WORKLOADS["prefill16_b16_6bit"]
    B, H, d, C, T = wl.batch, wl.heads, wl.d, wl.chunk, wl.prompt
    bits = wlm.head_bits(wl)
    lay = stq.Layout(bits, d, in_dtype=wl.in_dtype)
    w = wlm.impact_weights(wl)
    blocks = []
    for r in range(B):
        S0 = wlm.initial_state(wl, r)
        blocks.append([orc.quantize(bits[h], as_f64(S0[h]), as_f64(w[h]))[0] for h in range(H)])
    opool = oracle_pool(orc, bits, d, blocks)
    inp = {n: x.to(DEV) for n, x in wlm.prefill_inputs(wl, 0, T).items()}
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    wd = w.to(DEV)
    ws = _workspace(stq, lay, B, T, C, "workspace")
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    p_full = torch.from_numpy(opool.copy()).to(DEV)
    o_full = torch.empty(B, H, T, d, device=DEV)
    stq.prefill_chunk(lay, p_full, slots, inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], wd, o_full,
                      chunk=C, workspace=ws, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    o_first = o_full[:, :, :C].cpu().numpy()
    p_seg = torch.from_numpy(opool.copy()).to(DEV)
    seg = 32 * C
    for t0 in range(0, T, seg):
        part = {n: x[:, :, t0:t0 + seg].contiguous() for n, x in inp.items()}
        o_part = torch.empty(B, H, seg, d, device=DEV)
        stq.prefill_chunk(lay, p_seg, slots, part["q"], part["k"], part["v"], part["beta"], part["alpha"], wd,
                          o_part, chunk=C, workspace=ws, status=status)
        assert torch.equal(o_part, o_full[:, :, t0:t0 + seg]), f"readouts of tokens {t0}.. differ"
        del o_part, part
    torch.cuda.synchronize()
    assert status.item() == 0, stq.status_flags(status)
    assert torch.equal(p_full, p_seg)
    # the first chunk of sampled tiles against the oracle, from a one-chunk call's pool
    p_one = torch.from_numpy(opool.copy()).to(DEV)
    part = {n: x[:, :, :C].contiguous() for n, x in inp.items()}
    o_one = torch.empty(B, H, C, d, device=DEV)
    stq.prefill_chunk(lay, p_one, slots, part["q"], part["k"], part["v"], part["beta"], part["alpha"], wd, o_one,
                      chunk=C, workspace=ws, status=status)
    torch.cuda.synchronize()
    assert torch.equal(o_one.cpu(), torch.from_numpy(o_first))
    first_pool = p_one.cpu().numpy()
    cpu_inp = {n: x[:, :, :C].cpu() for n, x in inp.items()}
    del inp, o_full, ws, p_seg
    tally = Tally()
    rng = np.random.default_rng(11)
    for r, h in zip(rng.integers(0, B, 6), rng.integers(0, H, 6)):
        res = _oracle_chunk(orc, opool, bits, d, int(r), int(h), cpu_inp, 0, C, w, C)
        assert res["status"] == orc.OK
        compare_block(orc, bits[h], d, tile_bytes(orc, first_pool, bits, d, int(r), int(h)), res["block"],
                      res["tie"], tally, f"req {r} head {h}")
        for t in range(C):
            compare_o(o_first[r, h, t], res["o"][t], tally, f"token {t} req {r} head {h}")
    tally.check_budget()


def test_fp32_inputs_sequential_form(stq, orc):
    """fp32 inputs (the sequential kernel) on a short single chunk, teacher forced."""
    from quantized_linear_attention_stq_b200 import workloads as wlm

    bits = [6, 4]
    B, d, T = 2, 128, 23
    wl_, w, opool = _setup(orc, B, bits, dtype=torch.float32)
    lay = stq.Layout(bits, d, in_dtype=torch.float32)
    inp = wlm.prefill_inputs(wl_, 0, T)
    gpool = torch.from_numpy(opool.copy()).to(DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    o = torch.zeros(B, len(bits), T, d, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    stq.prefill_chunk(lay, gpool, slots, *(inp[n].to(DEV) for n in ("q", "k", "v", "beta", "alpha")), w.to(DEV), o,
                      chunk=64, workspace=torch.empty(1, dtype=torch.uint8, device=DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    gp, og = gpool.cpu().numpy(), o.cpu().numpy()
    tally = Tally()
    _check_chunk(orc, opool, gp, og, bits, d, B, inp, T, w, 0, tally)
    tally.check_budget()
