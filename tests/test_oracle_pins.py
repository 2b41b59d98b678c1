"""Pins of the oracle against facts fixed outside the oracle itself (CPU only).

Each group checks the oracle against one of: a hand derivation from a layout or format
definition, a library routine that implements the same special case (numpy's LSB-first bit
packing, numpy's IEEE float16 conversion, numpy's round-half-to-even ``rint``, a numpy matrix
product), a closed form, an invariant, or brute force on tiny heads. The groups are chosen so
that a dropped term, a wrong sign, a wrong index or a transposed operand anywhere in the oracle
fails at least one of them.
"""
import itertools

import numpy as np
import pytest

BITS = (4, 6, 8)


# ----------------------------------------------------------------------------------------------
# Packing: code (i,j) at bit offset b*(i*dv+j) of a little-endian bitstream, offset-binary
# ----------------------------------------------------------------------------------------------

def test_pack_hand_derived_bytes(orc):
    # 4-bit: two codes per byte, the first in the low nibble.
    assert list(orc.pack(4, [1, 2, 3, 4, 15, 0, 10, 5])) == [0x21, 0x43, 0x0F, 0x5A]
    # 6-bit: four codes fill three bytes; 1 + 2*64 + 3*4096 + 4*262144 = 0x103081.
    assert list(orc.pack(6, [1, 2, 3, 4])) == [0x81, 0x30, 0x10]
    # 63 + 63*4096 = 0x03F03F.
    assert list(orc.pack(6, [63, 0, 63, 0])) == [0x3F, 0xF0, 0x03]
    # 8-bit: one code per byte.
    assert list(orc.pack(8, [1, 255, 128])) == [0x01, 0xFF, 0x80]
    # A 6-bit code straddling a byte boundary: code 1 occupies bits 6..11.
    assert list(orc.pack(6, [0, 63])) == [0xC0, 0x0F]


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("n", [16, 256, 300])
def test_pack_matches_numpy_lsb_first_bitstream(orc, bits, n):
    rng = np.random.default_rng(bits * 1000 + n)
    u = rng.integers(0, 1 << bits, size=n)
    # Expand every code into its bits, least significant first, and let numpy pack them.
    stream = ((u[:, None] >> np.arange(bits)[None, :]) & 1).astype(np.uint8).ravel()
    ref = np.packbits(stream, bitorder="little")
    assert np.array_equal(orc.pack(bits, u), ref)
    assert np.array_equal(orc.unpack(bits, n, ref), u)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("d", [4, 16])
def test_pack_every_value_every_position(orc, bits, d):
    n = d * d
    rng = np.random.default_rng(7 + bits + d)
    base = rng.integers(0, 1 << bits, size=n)
    packed_base = orc.pack(bits, base)
    positions = range(n) if d == 4 else rng.choice(n, size=24, replace=False)
    for p in positions:
        for val in range(1 << bits):
            u = base.copy()
            u[p] = val
            pk = orc.pack(bits, u)
            back = orc.unpack(bits, n, pk)
            assert np.array_equal(back, u)
            # Only the bits of position p may differ from the base stream.
            diff = np.unpackbits(pk ^ packed_base, bitorder="little")
            changed = np.nonzero(diff)[0]
            assert np.all((changed >= bits * p) & (changed < bits * (p + 1)))


def test_block_sizes_from_layout_definition(orc):
    # codes bytes, padded to 16, + 4*dk + 4*dv scale bytes, padded to 128.
    assert orc.block_bytes(4, 128, 128) == 8192 + 1024          # 9216
    assert orc.block_bytes(6, 128, 128) == 12288 + 1024         # 13312
    assert orc.block_bytes(8, 128, 128) == 16384 + 1024         # 17408
    assert orc.block_bytes(16, 128, 128) == 32768
    # 6-bit 16x16: 1536 bits = 192 bytes (16-aligned), + 128 scale bytes = 320 -> 384.
    assert orc.block_bytes(6, 16, 16) == 384
    # 4-bit 5x5: 100 bits -> 13 bytes -> 16, + 40 scale bytes = 56 -> 128.
    assert orc.block_bytes(4, 5, 5) == 128


# ----------------------------------------------------------------------------------------------
# IEEE binary16 (pivot heads)
# ----------------------------------------------------------------------------------------------

def test_half_decode_all_patterns_match_numpy(orc):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(h)) for h in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_half_encode_matches_numpy(orc):
    rng = np.random.default_rng(3)
    vals = [0.0, -0.0, 65504.0, 65519.99, 65520.0, 70000.0, 1e-8, 2.0 ** -24, 2.0 ** -25,
            3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, np.inf, -np.inf]
    # exact ties between neighbouring halves, in the normal and the subnormal range
    for e in range(-14, 15):
        for m in (0, 1, 2, 3, 1022, 1023):
            lo = (1024 + m) * 2.0 ** (e - 10)
            vals.append(lo + 2.0 ** (e - 11))
            vals.append(-(lo + 2.0 ** (e - 11)))
    for m in range(0, 1024, 37):
        vals.append((m + 0.5) * 2.0 ** -24)
    vals += list(rng.standard_normal(2000) * 10.0 ** rng.uniform(-8, 5, 2000))
    for x in vals:
        ref = int(np.array([x], dtype=np.float64).astype(np.float16).view(np.uint16)[0])
        assert orc.double_to_half(x) == ref, x


def test_round_half_even_matches_numpy_rint(orc):
    ys = [n + 0.5 for n in range(-300, 300)] + list(np.random.default_rng(1).uniform(-200, 200, 3000))
    ys += [0.49999999999999994, -0.49999999999999994, 2.5000000000000004]
    for y in ys:
        assert orc.round_half_even(y) == np.rint(y), y


# ----------------------------------------------------------------------------------------------
# Quantizer
# ----------------------------------------------------------------------------------------------

TIE_CASES = {
    # circulant base rows whose squares sum to 5 * 4^-e, each containing +-qmax once:
    # 49+20.25+6.25+2.25+2.25 = 80; 961+306.25+12.25+.25+.25 = 1280; 16129+4290.25+56.25+2.25+2.25 = 20480
    4: ([7, 4.5, 2.5, 1.5, 1.5], -2),
    6: ([31, 17.5, 3.5, 0.5, 0.5], -4),
    8: ([127, 65.5, 7.5, 1.5, 1.5], -6),
}


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_exact_planted_ties(orc, bits):
    """S = 2^e X diag(C) with X a signed circulant of half-integers: every fitted scale and
    every real code is exact, so each half-integer is an exact rounding tie."""
    g, e = TIE_CASES[bits]
    d = 5
    X = np.array([[g[(i - j) % d] for j in range(d)] for i in range(d)], dtype=np.float64)
    X *= np.where(np.random.default_rng(bits).random((d, d)) < 0.5, -1.0, 1.0)
    C = np.array([1.0, 0.75, 3.0, 0.125, 1.5])
    S = X * C[None, :] * 2.0 ** e
    for w in (np.full(d, 3.0), np.full(d, 0.25)):
        block, x, tie, st = orc.quantize(bits, S, w)
        assert st == orc.OK
        r, c = orc.scales(bits, d, d, block)
        assert np.array_equal(x, X)
        assert np.array_equal(r, np.full(d, 2.0 ** e, dtype=np.float32))
        assert np.array_equal(c, C.astype(np.float32))
        Q = orc.codes(bits, d, d, block)
        assert np.array_equal(Q, np.rint(X).astype(int))  # numpy rint rounds half to even
        assert np.array_equal(tie, X != np.round(X + 0.25))  # ties exactly at the half-integers
        assert tie.sum() == 20


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("d", [16, 128])
def test_quantizer_sign_pattern_gives_full_scale(orc, bits, d):
    """S = diag(a) Sigma diag(b), Sigma in {+-1}: every code is +-qmax with Sigma's sign."""
    rng = np.random.default_rng(d + bits)
    a = np.exp(rng.normal(0, 0.8, d))
    b = np.exp(rng.normal(0, 0.8, d))
    sig = np.where(rng.random((d, d)) < 0.5, -1.0, 1.0)
    w = np.exp(rng.normal(0, 1, d))
    block, x, tie, st = orc.quantize(bits, a[:, None] * sig * b[None, :], w)
    assert st == orc.OK
    Q = orc.codes(bits, d, d, block)
    assert np.array_equal(Q, orc.qmax(bits) * sig.astype(int))


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("d", [4, 16, 128])
def test_quantizer_integer_circulant_round_trip(orc, bits, d):
    """S = rho * circ(g) * diag(c) with integer g, max|g| = qmax and equal w: codes are g exactly
    and dequantization reproduces S to a few fp32 ulps."""
    rng = np.random.default_rng(100 + d + bits)
    qm = orc.qmax(bits)
    g = rng.integers(-qm, qm + 1, size=d)
    g[rng.integers(d)] = qm * (1 if rng.random() < 0.5 else -1)
    G = np.array([[g[(j - i) % d] for j in range(d)] for i in range(d)])
    cvec = np.exp(rng.normal(0, 1.0, d))
    rho = 0.37
    S = rho * G * cvec[None, :]
    block, x, tie, st = orc.quantize(bits, S, np.full(d, 2.5))
    assert st == orc.OK
    assert np.array_equal(orc.codes(bits, d, d, block), G)
    Sd = orc.dequantize(bits, d, d, block)
    nz = S != 0
    assert np.max(np.abs(Sd[nz] - S[nz]) / np.abs(S[nz])) < 4 * 2.0 ** -23


def _outlier_state(rng, d, row_ratio=10.3, col_ratio=19.4):
    a = np.exp(rng.normal(0, 0.8, d))
    b = np.exp(rng.normal(0, 0.8, d))
    a[np.argmax(a)] = row_ratio * np.median(a)
    b[np.argmax(b)] = col_ratio * np.median(b)
    return a[:, None] * rng.standard_normal((d, d)) * b[None, :]


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_closed_form_bounds(orc, bits):
    rng = np.random.default_rng(bits)
    dk, dv = 128, 96
    S = _outlier_state(rng, 128)[:, :dv]
    w = np.exp(rng.normal(0, 1, dk))
    block, x, tie, st = orc.quantize(bits, S, w)
    assert st == orc.OK
    Q = orc.codes(bits, dk, dv, block)
    r, c = orc.scales(bits, dk, dv, block)
    step = r.astype(np.float64)[:, None] * c.astype(np.float64)[None, :]
    # reconstruction error at most half a step (plus fp64 slack)
    assert np.all(np.abs(S - step * Q) <= 0.5 * step * (1 + 1e-9))
    # every row reaches full scale
    assert np.all(np.abs(Q).max(axis=1) == orc.qmax(bits))
    # the column scale is the impact-weighted RMS: c_j^2 * sum(w) == sum_i w_i S_ij^2
    lhs = c.astype(np.float64) ** 2 * w.sum()
    rhs = (w[:, None] * S ** 2).sum(axis=0)
    assert np.max(np.abs(lhs - rhs) / rhs) < 2.5e-7
    # the row scale is the largest column-normalised magnitude over qmax
    t = np.abs(S / c.astype(np.float64)[None, :]).max(axis=1) / orc.qmax(bits)
    assert np.max(np.abs(r - t) / t) < 1e-7


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_weight_roles(orc, bits):
    """Weight concentrated on one key row: the column scale becomes that row's magnitude (catches
    a row/column index swap or a missing square); scaling all weights by 4 changes nothing."""
    rng = np.random.default_rng(11)
    dk, dv = 12, 20
    S = rng.standard_normal((dk, dv))
    m = 5
    w = np.full(dk, 1e-12)
    w[m] = 1.0
    block, _, _, st = orc.quantize(bits, S, w)
    _, c = orc.scales(bits, dk, dv, block)
    assert np.allclose(c, np.abs(S[m]), rtol=1e-5)
    w2 = np.exp(rng.normal(0, 1, dk))
    b1, _, _, _ = orc.quantize(bits, S, w2)
    b2, _, _, _ = orc.quantize(bits, S, 4.0 * w2)
    assert np.array_equal(b1, b2)


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_zero_rows_and_columns(orc, bits):
    rng = np.random.default_rng(5)
    S = rng.standard_normal((8, 8))
    S[3, :] = 0.0
    S[:, 6] = 0.0
    block, _, _, st = orc.quantize(bits, S, np.ones(8))
    assert st == orc.OK
    r, c = orc.scales(bits, 8, 8, block)
    Q = orc.codes(bits, 8, 8, block)
    assert r[3] == 1.0 and c[6] == 1.0
    assert np.all(Q[3] == 0) and np.all(Q[:, 6] == 0)
    blk0, _, _, st0 = orc.quantize(bits, np.zeros((4, 4)), np.ones(4))
    assert st0 == orc.OK and np.all(orc.codes(bits, 4, 4, blk0) == 0)
    assert np.all(np.concatenate(orc.scales(bits, 4, 4, blk0)) == 1.0)


@pytest.mark.parametrize("bits", BITS)
def test_quantizer_brute_force_4x4(orc, bits):
    """On 4x4 heads every code is the argmin over all integers in [-qmax, qmax] of the distance
    to the real code, ties to the even integer."""
    qm = orc.qmax(bits)
    cands = np.arange(-qm, qm + 1)
    rng = np.random.default_rng(bits + 40)
    for trial in range(200):
        S = rng.standard_normal((4, 4)) * np.exp(rng.normal(0, 1, (4, 1)))
        block, x, tie, st = orc.quantize(bits, S, np.exp(rng.normal(0, 1, 4)))
        Q = orc.codes(bits, 4, 4, block)
        for i, j in itertools.product(range(4), range(4)):
            dist = np.abs(x[i, j] - cands)
            best = cands[dist == dist.min()]
            want = best[0] if best.size == 1 else best[best % 2 == 0][0]
            assert Q[i, j] == want


def test_quantizer_pivot_is_numpy_float16(orc):
    rng = np.random.default_rng(9)
    S = rng.standard_normal((16, 24)) * 300.0
    block, _, _, st = orc.quantize(16, S)
    assert st == orc.OK
    assert np.array_equal(orc.pivot_values(16, 24, block), S.astype(np.float16).view(np.uint16))
    S[2, 3] = 1e6  # overflows fp16
    _, _, _, st = orc.quantize(16, S)
    assert st == orc.ENONFINITE


def test_quantizer_rejects_bad_weights(orc):
    S = np.ones((4, 4))
    for w in ([1, 1, 0, 1], [1, -1, 1, 1], [1, np.nan, 1, 1], [np.inf, 1, 1, 1]):
        assert orc.quantize(6, S, np.array(w, dtype=float))[3] == orc.EINVAL


# ----------------------------------------------------------------------------------------------
# Decode step: gated delta rule update and readout
# ----------------------------------------------------------------------------------------------

def _random_block(orc, bits, dk, dv, seed):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((dk, dv)) * np.exp(rng.normal(0, 0.8, (dk, 1)))
    w = np.exp(rng.normal(0, 1, dk))
    block, _, _, st = orc.quantize(bits, S, w)
    assert st == orc.OK
    return block, w


@pytest.mark.parametrize("bits", BITS + (16,))
@pytest.mark.parametrize("shape", [(16, 16), (8, 12)])
@pytest.mark.parametrize("gate", [0, 1, 2])
def test_unit_key_write(orc, bits, shape, gate):
    """alpha=1, beta=1, k = e_m: row m of the updated state is v exactly, the other rows are the
    dequantized state exactly, and a query q = e_m reads back v."""
    dk, dv = shape
    block, w = _random_block(orc, bits, dk, dv, 1)
    S = orc.dequantize(bits, dk, dv, block)
    rng = np.random.default_rng(2)
    v = rng.standard_normal(dv)
    m = 3
    k = np.zeros(dk)
    k[m] = 1.0
    alpha = 1.0 if gate == 0 else np.ones(dk)
    res = orc.decode_step(bits, gate, block, k, k, v, 1.0, alpha, w, dk, dv)
    Sn = res["S_new"]
    assert np.array_equal(Sn[m], v)
    others = np.arange(dk) != m
    assert np.array_equal(Sn[others], S[others])
    assert np.array_equal(res["o"], v.astype(np.float32))


@pytest.mark.parametrize("bits", (4, 8))
def test_unit_key_write_general_direction(orc, bits):
    """For any unit k with alpha=1, beta=1: S'^T k = v."""
    dk = dv = 32
    block, w = _random_block(orc, bits, dk, dv, 3)
    rng = np.random.default_rng(4)
    k = rng.standard_normal(dk)
    k /= np.linalg.norm(k)
    v = rng.standard_normal(dv)
    res = orc.decode_step(bits, 0, block, k, k, v, 1.0, 1.0, w, dk, dv)
    assert np.allclose(res["S_new"].T @ k, v, atol=1e-12, rtol=0)
    assert np.allclose(res["o"], v, atol=1e-6, rtol=1e-6)


@pytest.mark.parametrize("gate", [0, 1, 2])
def test_beta_zero_is_pure_decay(orc, gate):
    dk, dv = 16, 24
    block, w = _random_block(orc, 6, dk, dv, 5)
    S = orc.dequantize(6, dk, dv, block)
    rng = np.random.default_rng(6)
    q, k, v = rng.standard_normal(dk), rng.standard_normal(dk), rng.standard_normal(dv)
    alpha = 0.9 if gate == 0 else np.exp(-1.0 / rng.uniform(1, 100, dk))
    res = orc.decode_step(6, gate, block, q, k, v, 0.0, alpha, w, dk, dv)
    a = np.atleast_1d(alpha)[:, None] if gate else alpha
    assert np.array_equal(res["S_new"], a * S)


def test_readout_is_transposed_state_times_query(orc):
    """alpha=1, beta=0: o = deq(S)^T q, checked against numpy's matrix product, d_k != d_v."""
    dk, dv = 24, 40
    block, w = _random_block(orc, 8, dk, dv, 7)
    S = orc.dequantize(8, dk, dv, block)
    rng = np.random.default_rng(8)
    q, k, v = rng.standard_normal(dk), rng.standard_normal(dk), rng.standard_normal(dv)
    res = orc.decode_step(8, 0, block, q, k, v, 0.0, 1.0, w, dk, dv)
    ref = (S.T @ q).astype(np.float32)
    assert np.allclose(res["o"], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_update_is_non_expansive_plus_write(orc):
    rng = np.random.default_rng(10)
    dk = dv = 32
    for t in range(50):
        S = rng.standard_normal((dk, dv))
        k = rng.standard_normal(dk)
        k /= np.linalg.norm(k)
        v = rng.standard_normal(dv)
        beta, alpha = rng.uniform(0, 1), rng.uniform(0.2, 1)
        Sn, _ = orc.update(0, S, k, k, v, beta, alpha)
        assert np.linalg.norm(Sn) <= np.linalg.norm(S) + beta * np.linalg.norm(v) + 1e-12


@pytest.mark.parametrize("bits", (4, 16))
def test_channel_gate_with_equal_entries_is_scalar_gate(orc, bits):
    dk, dv = 16, 16
    block, w = _random_block(orc, bits, dk, dv, 12)
    rng = np.random.default_rng(13)
    q, k, v = rng.standard_normal(dk), rng.standard_normal(dk), rng.standard_normal(dv)
    a = 0.875
    r0 = orc.decode_step(bits, 0, block, q, k, v, 0.6, a, w, dk, dv)
    r1 = orc.decode_step(bits, 1, block, q, k, v, 0.6, np.full(dk, a), w, dk, dv)
    assert np.array_equal(r0["S_new"], r1["S_new"])
    assert np.array_equal(r0["block"], r1["block"])
    # decay-first with equal entries: alpha*(S - beta k u) == alpha S - beta k (alpha u)
    r2 = orc.decode_step(bits, 2, block, q, k, v, 0.6, np.full(dk, a), w, dk, dv)
    assert np.allclose(r2["S_new"], r0["S_new"], rtol=1e-13, atol=1e-13)


def test_channel_gate_orders_differ_in_general(orc):
    dk = dv = 16
    block, w = _random_block(orc, 6, dk, dv, 14)
    rng = np.random.default_rng(15)
    q, k, v = rng.standard_normal(dk), rng.standard_normal(dk), rng.standard_normal(dv)
    alpha = np.exp(-1.0 / rng.uniform(1, 50, dk))
    r1 = orc.decode_step(6, 1, block, q, k, v, 0.7, alpha, w, dk, dv)
    r2 = orc.decode_step(6, 2, block, q, k, v, 0.7, alpha, w, dk, dv)
    assert not np.allclose(r1["S_new"], r2["S_new"])


def test_fp16_pivot_tracks_unquantized_recurrence(orc):
    """A pivot head (fp16 storage) follows the unquantized fp64 recurrence over 64 steps of the
    d=16 test workload (h = 256): every single step stores each element within half an fp16
    quantum of the exact update of the stored state, and over the trajectory the relative error
    is at most 1e-3 (RMS over the 64 readouts, and mean of the per-step state errors; the
    per-step drift is a random walk of fp16 roundings and reaches ~1.2e-3 at single steps)."""
    rng = np.random.default_rng(0)
    d = 16
    a = np.exp(rng.normal(0, 0.8, d))
    b = np.exp(rng.normal(0, 0.8, d))
    S0 = a[:, None] * rng.standard_normal((d, d)) * b[None, :]
    w = np.exp(rng.normal(0, 1, d))
    alpha = np.exp(-1.0 / 256)
    block, _, _, _ = orc.quantize(16, S0)
    Sref = orc.dequantize(16, d, d, block)
    O, Oref, s_err = [], [], []
    for t in range(64):
        q = rng.standard_normal(d)
        q /= np.linalg.norm(q)
        k = rng.standard_normal(d)
        k /= np.linalg.norm(k)
        v = rng.standard_normal(d)
        beta = 1.0 / (1.0 + np.exp(-rng.standard_normal()))
        Sprev = orc.dequantize(16, d, d, block)
        res = orc.decode_step(16, 0, block, q, k, v, beta, alpha, w, d, d)
        block = res["block"]
        Sd = orc.dequantize(16, d, d, block)
        # single step: exact update of the stored state, then one fp16 rounding
        exact = alpha * (Sprev - beta * np.outer(k, k @ Sprev)) + beta * np.outer(k, v)
        quantum = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0 ** -14))) - 10)
        assert np.all(np.abs(Sd - exact) <= 0.5 * quantum * (1 + 1e-9))
        Sref = alpha * (Sref - beta * np.outer(k, k @ Sref)) + beta * np.outer(k, v)
        O.append(res["o"])
        Oref.append(Sref.T @ q)
        s_err.append(np.linalg.norm(Sd - Sref) / np.linalg.norm(Sref))
    O, Oref = np.array(O, dtype=np.float64), np.array(Oref)
    assert np.linalg.norm(O - Oref) <= 1e-3 * np.linalg.norm(Oref)
    assert np.mean(s_err) <= 1e-3
    assert np.max(s_err) <= 2e-3


def test_decode_flags(orc):
    block, w = _random_block(orc, 6, 8, 8, 16)
    z = np.zeros(8)
    bad = w.copy()
    bad[0] = 0.0
    assert orc.decode_step(6, 0, block, z, z, z, 0.5, 0.9, bad, 8, 8)["status"] == orc.EINVAL
    v = np.full(8, np.inf)
    assert orc.decode_step(6, 0, block, z, np.ones(8), v, 0.5, 0.9, w, 8, 8)["status"] == orc.ENONFINITE


# ----------------------------------------------------------------------------------------------
# Chunked prefill
# ----------------------------------------------------------------------------------------------

def _chunk_inputs(rng, C, dk, dv):
    q = rng.standard_normal((C, dk))
    k = rng.standard_normal((C, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((C, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(C)))
    alpha = np.exp(-1.0 / rng.uniform(1, 400, C))
    return q, k, v, beta, alpha


@pytest.mark.parametrize("C,dk,dv", [(1, 16, 16), (7, 16, 16), (64, 16, 24), (64, 64, 64)])
def test_wy_form_matches_token_recurrence(orc, C, dk, dv):
    rng = np.random.default_rng(C + dk)
    S0 = rng.standard_normal((dk, dv))
    q, k, v, beta, alpha = _chunk_inputs(rng, C, dk, dv)
    S_end, O = orc.chunk_wy(S0, q, k, v, beta, alpha)
    S = S0.copy()
    Oseq = np.zeros((C, dv))
    for t in range(C):
        S, Oseq[t] = orc.update(0, S, q[t], k[t], v[t], beta[t], alpha[t])
    assert np.max(np.abs(S_end - S)) <= 1e-10 * np.max(np.abs(S))
    assert np.max(np.abs(O - Oseq)) <= 1e-10 * np.max(np.abs(Oseq))


def test_wy_pure_decay(orc):
    rng = np.random.default_rng(21)
    C, d = 64, 16
    S0 = rng.standard_normal((d, d))
    q, k, v, _, _ = _chunk_inputs(rng, C, d, d)
    a = 0.97
    S_end, _ = orc.chunk_wy(S0, q, k, v, np.zeros(C), np.full(C, a))
    assert np.allclose(S_end, a ** C * S0, rtol=1e-12, atol=0)


@pytest.mark.parametrize("bits", BITS + (16,))
def test_prefill_chunk_of_one_is_decode(orc, bits):
    dk, dv, T = 16, 16, 9
    block, w = _random_block(orc, bits, dk, dv, 22)
    rng = np.random.default_rng(23)
    q, k, v, beta, alpha = _chunk_inputs(rng, T, dk, dv)
    res = orc.prefill_seq(bits, 0, block, q, k, v, beta, alpha, w, 1, dk, dv)
    blk = block.copy()
    for t in range(T):
        r = orc.decode_step(bits, 0, blk, q[t], k[t], v[t], beta[t], alpha[t], w, dk, dv)
        blk = r["block"]
        assert np.array_equal(res["o"][t], r["o"])
    assert np.array_equal(res["block"], blk)


def test_prefill_multi_chunk_equals_single_chunk_calls(orc):
    dk, dv, T, C = 16, 16, 150, 64
    block, w = _random_block(orc, 6, dk, dv, 24)
    rng = np.random.default_rng(25)
    q, k, v, beta, alpha = _chunk_inputs(rng, T, dk, dv)
    full = orc.prefill_seq(6, 0, block, q, k, v, beta, alpha, w, C, dk, dv)
    blk = block.copy()
    outs = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        r = orc.prefill_seq(6, 0, blk, q[sl], k[sl], v[sl], beta[sl], alpha[sl], w, C, dk, dv)
        blk = r["block"]
        outs.append(r["o"])
    assert np.array_equal(full["block"], blk)
    assert np.array_equal(full["o"], np.concatenate(outs))


def test_prefill_empty_call_is_identity(orc):
    block, w = _random_block(orc, 4, 16, 16, 26)
    e = np.zeros((0, 16))
    res = orc.prefill_seq(4, 0, block, e, e, e, np.zeros(0), np.zeros(0), w, 64, 16, 16)
    assert np.array_equal(res["block"], block)


# ---------------------------------------------------------------------------------------------
# Uniform baseline quantizer (one scale per head)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 6, 8])
def test_uniform_integer_multiples_round_trip_exactly(orc, bits):
    # S = s * G with integer G, max |G| = qmax: the scale is s and the codes are G exactly
    rng = np.random.default_rng(bits)
    qm = orc.qmax(bits)
    G = rng.integers(-qm, qm + 1, size=(9, 7)).astype(float)
    G[3, 2] = -qm
    s = 2.0 ** -5 * 3
    blk, x, tie, st = orc.quantize_uniform(bits, s * G)
    assert st == orc.OK
    assert orc.uniform_scale(bits, 9, 7, blk) == s
    assert np.array_equal(orc.unpack(bits, 63, blk).reshape(9, 7) - (1 << (bits - 1)), G.astype(int))
    assert np.array_equal(orc.dequantize_uniform(bits, 9, 7, blk), s * G)


@pytest.mark.parametrize("bits", [4, 6])
def test_uniform_rounds_half_to_even_and_bounds_the_error(orc, bits):
    qm = orc.qmax(bits)
    # a planted tie: max entry qmax*s, another entry at exactly 2.5*s
    S = np.zeros((3, 4))
    S[0, 0] = qm * 0.25
    S[1, 1] = 2.5 * 0.25
    S[2, 3] = -1.5 * 0.25
    blk, x, tie, st = orc.quantize_uniform(bits, S)
    codes = orc.unpack(bits, 12, blk).reshape(3, 4) - (1 << (bits - 1))
    assert codes[1, 1] == 2 and codes[2, 3] == -2 and tie[1, 1] and tie[2, 3]
    # random states: |S - s Q| <= s/2 everywhere, and the largest entry maps to +-qmax
    rng = np.random.default_rng(5)
    S = rng.normal(size=(16, 16)) * np.exp(rng.normal(size=(16, 1)))
    blk, x, tie, st = orc.quantize_uniform(bits, S)
    s = orc.uniform_scale(bits, 16, 16, blk)
    Sh = orc.dequantize_uniform(bits, 16, 16, blk)
    assert np.max(np.abs(S - Sh)) <= s / 2 * (1 + 1e-12)
    assert np.max(np.abs(orc.unpack(bits, 256, blk) - (1 << (bits - 1)))) == qm


def test_uniform_block_layout_and_zero_state(orc):
    # codes padded to 16 bytes, one fp32 scale, padding to 128 bytes
    assert orc.uniform_block_bytes(4, 128, 128) == 8320
    assert orc.uniform_block_bytes(6, 128, 128) == 12416
    assert orc.uniform_block_bytes(8, 16, 16) == 384
    blk, _, _, st = orc.quantize_uniform(6, np.zeros((4, 4)))
    assert st == orc.OK and orc.uniform_scale(6, 4, 4, blk) == 1.0
    assert np.all(orc.dequantize_uniform(6, 4, 4, blk) == 0.0)


def test_uniform_decode_step_is_update_then_uniform_requantization(orc):
    rng = np.random.default_rng(9)
    d = 8
    S = rng.normal(size=(d, d))
    blk, _, _, _ = orc.quantize_uniform(8, S)
    q, k, v = rng.normal(size=d), rng.normal(size=d), rng.normal(size=d)
    k /= np.linalg.norm(k)
    res = orc.decode_step_uniform(8, 0, blk, q, k, v, 0.6, 0.97, d, d)
    S_deq = orc.dequantize_uniform(8, d, d, blk)
    S_new, o = orc.update(0, S_deq, q, k, v, 0.6, 0.97)
    assert np.array_equal(res["o"], o.astype(np.float32))
    ref_blk, _, _, _ = orc.quantize_uniform(8, S_new)
    assert np.array_equal(res["block"], ref_blk)


# ----------------------------------------------------------------------------------------------
# 16-bit (bf16) scale storage
# ----------------------------------------------------------------------------------------------

def _fp32_rne_to_bf16(x32):
    """Textbook round-to-nearest-even of binary32 patterns to their upper 16 bits (add 0x7fff
    plus the lowest kept bit, then truncate): correct for every finite input."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_bf16_decode_all_patterns_are_fp32_upper_halves(orc):
    pats = np.arange(65536, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        ref = (pats << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    got = np.array([orc.bf16_to_double(int(h)) for h in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_encode_matches_fp32_rne_on_fp32_values(orc):
    """For values exactly representable in fp32, rounding to bf16 is the textbook bit rounding;
    exact ties go to the even pattern, and 255.5 * 2^120 (half an ulp above the largest finite
    value) overflows to infinity."""
    rng = np.random.default_rng(21)
    vals = [0.0, 1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -133, 2.0 ** -134,
            3 * 2.0 ** -134, 2.0 ** -126, 255.0 * 2.0 ** 120, 255.5 * 2.0 ** 120 - 2.0 ** 104, 255.5 * 2.0 ** 120]
    for e in (-130, -126, -20, -1, 0, 7, 100, 126):
        for m in (0, 1, 2, 126, 127):
            vals.append((128 + m + 0.5) * 2.0 ** (e - 7))  # exact ties
    vals += list((rng.standard_normal(3000) * 10.0 ** rng.uniform(-30, 30, 3000)).astype(np.float32))
    x32 = np.array(vals, dtype=np.float32)
    assert np.array_equal(x32.astype(np.float64), np.array(vals, dtype=np.float64))  # all fp32-exact
    ref = _fp32_rne_to_bf16(x32)
    for x, h in zip(vals, ref):
        assert orc.double_to_bf16(float(x)) == int(h), x
    assert orc.double_to_bf16(255.5 * 2.0 ** 120) == 0x7F80
    assert orc.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80 and orc.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82


def test_bf16_encode_rounds_the_exact_value_once(orc):
    """READING: a scale is rounded to bf16 from its exact value in one step, not through fp32: just
    above a bf16 tie by less than an fp32 half-ulp rounds up."""
    assert orc.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert orc.double_to_bf16(1.0 + 2.0 ** -8 - 2.0 ** -40) == 0x3F80


def test_bf16_scale_block_layout(orc):
    """Codes, padding to 16 bytes, r[dk] and c[dv] in bf16, padding to 128 bytes: at 128 x 128 a
    6-bit head is 12,800 bytes, 5.12x smaller than fp32, and with 1.4% FP16 pivot heads the state
    is 5.01x smaller (the pages report 5.03x / 5.08x at 6 bits)."""
    for bits, want in ((4, 8704), (6, 12800), (8, 16896)):
        assert orc.block_bytes_s(bits, orc.SCALE_BF16, 128, 128) == want
        assert orc.block_bytes_s(bits, orc.SCALE_F32, 128, 128) == orc.block_bytes(bits, 128, 128)
    assert orc.block_bytes_s(16, orc.SCALE_BF16, 128, 128) == 32768
    assert abs(65536 / 12800 - 5.12) < 1e-12
    mixed = 0.986 * 12800 + 0.014 * 32768
    assert abs(65536 / mixed - 5.01) < 0.01
    assert orc.block_bytes_s(6, 2, 128, 128) == 0  # unknown format


# rows g with max |g| = qmax and sum g^2 = 8 * 4^k: a circulant of g has column RMS exactly 2^k
EXACT_ROWS = {4: ([7, 5, 5, 3, 3, 3, 1, 1], 2), 6: ([31, 23, 17, 13, 9, 3, 3, 1], 4),
              8: ([127, 121, 44, 7, 3, 2, 0, 0], 6)}


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("sfmt", [0, 1])
def test_scales_exact_round_trip(orc, bits, sfmt):
    """S = circ(+-g) diag(c) with bf16-exact c and equal weights: the fitted column scale is
    2^k c_j, the row scale 2^-k, both exact in either format, the codes are the integers and
    dequantization gives S back exactly."""
    g, k = EXACT_ROWS[bits]
    assert sum(x * x for x in g) == 8 * 4 ** k and max(g) == orc.qmax(bits)
    d = 8
    rng = np.random.default_rng(bits * 10 + sfmt)
    G = np.array([[g[(j - i) % d] for j in range(d)] for i in range(d)], dtype=np.float64)
    G *= np.where(rng.random((d, d)) < 0.5, -1.0, 1.0)
    c = (128 + rng.integers(0, 128, d)) / 128.0 * 2.0 ** rng.integers(-6, 6, d)
    S = G * c[None, :]
    block, x, tie, stie, st = orc.quantize_s(bits, sfmt, S, np.full(d, 0.7))
    assert st == orc.OK
    r_s, c_s = orc.scales_s(bits, sfmt, d, d, block)
    assert np.array_equal(c_s, c * 2.0 ** k) and np.array_equal(r_s, np.full(d, 2.0 ** -k))
    assert np.array_equal(orc.codes(bits, d, d, block), G.astype(int))
    assert np.array_equal(orc.dequantize_s(bits, sfmt, d, d, block), S)
    assert not stie.any()


@pytest.mark.parametrize("bits", BITS)
def test_bf16_scales_bounds(orc, bits):
    """On an outlier state: every stored scale is a bf16 value within half a bf16 ulp of its
    defining quantity (the column's impact-weighted RMS; the row's largest magnitude over the
    stored column scales, over qmax), and every code is within half a step of the stored step."""
    rng = np.random.default_rng(60 + bits)
    dk, dv = 128, 96
    S = _outlier_state(rng, 128)[:, :dv]
    w = np.exp(rng.normal(0, 1, dk))
    block, x, tie, stie, st = orc.quantize_s(bits, orc.SCALE_BF16, S, w)
    assert st == orc.OK
    r, c = orc.scales_s(bits, orc.SCALE_BF16, dk, dv, block)
    rc = np.concatenate([r, c])
    assert np.array_equal(rc.astype(np.float32).astype(np.float64), rc)
    assert not (rc.astype(np.float32).view(np.uint32) & 0xFFFF).any()  # bf16 values: low half zero
    def half_ulp(v):  # half the bf16 quantum of the binade [2^e, 2^(e+1)) holding v
        return 2.0 ** (np.floor(np.log2(v)) - 8)

    rms = np.sqrt((w[:, None] * S ** 2).sum(axis=0) / w.sum())
    assert np.all(np.abs(c - rms) <= half_ulp(rms) * (1 + 1e-9))
    t = np.abs(S / c[None, :]).max(axis=1) / orc.qmax(bits)
    assert np.all(np.abs(r - t) <= half_ulp(t) * (1 + 1e-9))
    Q = orc.codes(bits, dk, dv, block)
    step = r[:, None] * c[None, :]
    assert np.all(np.abs(S - step * Q) <= 0.5 * step * (1 + 1e-9))
    assert np.all(np.abs(Q).max(axis=1) >= orc.qmax(bits) - 1)


@pytest.mark.parametrize("bits", BITS)
def test_bf16_sign_pattern_gives_full_scale(orc, bits):
    """S = diag(a) Sigma diag(b): with bf16 scales every code has Sigma's sign and magnitude within
    qmax (1 - 2^-7) of qmax (the stored column scales carry up to 2^-8 relative rounding each way),
    so qmax at 4 and 6 bits and 126 or 127 at 8 bits; every row reaches qmax."""
    d = 64
    rng = np.random.default_rng(70 + bits)
    a = np.exp(rng.normal(0, 0.8, d))
    b = np.exp(rng.normal(0, 0.8, d))
    sig = np.where(rng.random((d, d)) < 0.5, -1.0, 1.0)
    block, _, _, _, st = orc.quantize_s(bits, orc.SCALE_BF16, a[:, None] * sig * b[None, :], np.exp(rng.normal(0, 1, d)))
    assert st == orc.OK
    Q = orc.codes(bits, d, d, block)
    qm = orc.qmax(bits)
    assert np.array_equal(np.sign(Q), sig.astype(int))
    assert np.all(np.abs(Q) >= np.ceil(qm * (1 - 2.0 ** -7) - 0.5)) and np.all(np.abs(Q).max(axis=1) == qm)
    if bits < 8:
        assert np.all(np.abs(Q) == qm)


def test_bf16_given_scales_are_used_as_stored(orc):
    """Scales passed in replace the fitted ones: with the fitted scales given back the block is
    identical, and with another column scale the codes follow it."""
    rng = np.random.default_rng(77)
    S = _outlier_state(rng, 32)
    w = np.exp(rng.normal(0, 1, 32))
    blk, _, _, _, _ = orc.quantize_s(6, orc.SCALE_BF16, S, w)
    r, c = orc.scales_s(6, orc.SCALE_BF16, 32, 32, blk)
    again, _, _, _, _ = orc.quantize_s(6, orc.SCALE_BF16, S, w, c_given=c, r_given=r)
    assert np.array_equal(again, blk)
    c2 = c.copy()
    c2[5] = orc.bf16_to_double(orc.double_to_bf16(c[5]) + 1)  # one bf16 ulp up
    other, _, _, _, _ = orc.quantize_s(6, orc.SCALE_BF16, S, w, c_given=c2)
    r3, c3 = orc.scales_s(6, orc.SCALE_BF16, 32, 32, other)
    assert np.array_equal(c3, c2)
    Q = orc.codes(6, 32, 32, other)
    step = r3[:, None] * c3[None, :]
    assert np.all(np.abs(S - step * Q) <= 0.5 * step * (1 + 1e-9))


def test_bf16_decode_step_is_update_then_requantization(orc):
    rng = np.random.default_rng(78)
    d = 16
    S0 = _outlier_state(rng, d)
    w = np.exp(rng.normal(0, 1, d))
    blk = orc.quantize_s(4, orc.SCALE_BF16, S0, w)[0]
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    q, k = q / np.linalg.norm(q), k / np.linalg.norm(k)
    v = rng.standard_normal(d)
    res = orc.decode_step_s(4, orc.SCALE_BF16, 0, blk, q, k, v, 0.6, 0.97, w, d, d)
    assert res["status"] == orc.OK
    S1, o = orc.update(0, orc.dequantize_s(4, orc.SCALE_BF16, d, d, blk), q, k, v, 0.6, 0.97)
    assert np.array_equal(res["o"], o.astype(np.float32))
    assert np.array_equal(res["block"], orc.quantize_s(4, orc.SCALE_BF16, S1, w)[0])
    assert res["block"].size == orc.block_bytes_s(4, orc.SCALE_BF16, d, d)



# ----------------------------------------------------------------------------------------------
# Impact-aware joint refinement of the scales (alternating weighted least squares)
# ----------------------------------------------------------------------------------------------

def _weighted_error(orc, bits, sfmt, S, w, block):
    d_k, d_v = S.shape
    r, c = orc.scales_s(bits, sfmt, d_k, d_v, block)
    Q = orc.codes(bits, d_k, d_v, block)
    return float((w[:, None] * (S - r[:, None] * c[None, :] * Q) ** 2).sum())


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("sfmt", [0, 1])
def test_fit_rounds_never_raise_the_weighted_error(orc, bits, sfmt):
    """Each least-squares step minimises the impact-weighted error for fixed codes and each code
    step picks the nearest codes for fixed scales, so the error cannot rise from round to round
    (up to the rounding of the stored scales); on an outlier state it falls."""
    rng = np.random.default_rng(90 + bits + 10 * sfmt)
    S = _outlier_state(rng, 64)
    w = np.exp(rng.normal(0, 1, 64))
    E = [_weighted_error(orc, bits, sfmt, S, w, orc.quantize_fit(bits, sfmt, k, S, w)[0]) for k in range(4)]
    slack = 1e-6 if sfmt == 0 else 3e-2
    for a, b in zip(E, E[1:]):
        assert b <= a * (1 + slack), E
    assert E[3] < E[0], E
    assert np.array_equal(orc.quantize_fit(bits, sfmt, 0, S, w)[0], orc.quantize_s(bits, sfmt, S, w)[0])


@pytest.mark.parametrize("bits", BITS)
def test_fit_rounds_keep_an_exact_fit(orc, bits):
    """An exactly representable state (the exact round-trip fixture) is a fixed point."""
    g, k = EXACT_ROWS[bits]
    d = 8
    rng = np.random.default_rng(bits)
    G = np.array([[g[(j - i) % d] for j in range(d)] for i in range(d)], dtype=np.float64)
    G *= np.where(rng.random((d, d)) < 0.5, -1.0, 1.0)
    c = (128 + rng.integers(0, 128, d)) / 128.0 * 2.0 ** rng.integers(-6, 6, d)
    S = G * c[None, :]
    w = np.full(d, 0.7)
    for sfmt in (0, 1):
        blk = orc.quantize_fit(bits, sfmt, 3, S, w)[0]
        assert np.array_equal(blk, orc.quantize_fit(bits, sfmt, 0, S, w)[0])
        assert np.array_equal(orc.dequantize_s(bits, sfmt, d, d, blk), S)


@pytest.mark.parametrize("bits", BITS)
def test_fit_follows_the_impact_weights(orc, bits):
    """The weight on two key rows: two rounds of the joint fit cut those rows' error to a small
    fraction of the one-pass error, and of the error left by the same fit run with equal weights
    (a dropped weight, or a transposed index in the column step, would not)."""
    rng = np.random.default_rng(95 + bits)
    d = 24
    S = _outlier_state(rng, d)
    w = np.full(d, 1e-9)
    w[[3, 11]] = 1.0
    e_one = _weighted_error(orc, bits, 0, S, w, orc.quantize_fit(bits, 0, 0, S, w)[0])
    e_fit = _weighted_error(orc, bits, 0, S, w, orc.quantize_fit(bits, 0, 2, S, w)[0])
    e_eq = _weighted_error(orc, bits, 0, S, w, orc.quantize_fit(bits, 0, 2, S, np.ones(d))[0])
    assert e_fit < 0.2 * e_one and e_fit < 0.2 * e_eq, (e_one, e_fit, e_eq)
