"""Host check of a bound the tensor-core prefill's state kernel relies on: with an fp32 row scale
that is a normal number, the value a code is rounded from never exceeds qmax + 1/2, so the clamp
to +-qmax can be left out there. The kernel's fp32 steps are replayed in numpy float32 (each
operation rounded to nearest, as on the GPU): t = S * rcp(c), m = max |t|, r = m / qmax,
x = t * rcp(r). A bf16 row scale may undershoot m / qmax by up to 2^-8 (relative), which puts x
outside this fp32 argument (it comes within 0.01 of qmax + 1/2 for qmax = 127), so the kernel keeps
the clamp there; the last check shows that bf16 case leaves the fp32 bound."""
import numpy as np
import pytest


def _f32_rows(rng, n, d, scale_exp):
    mag = np.float32(2.0) ** rng.integers(-scale_exp, scale_exp, size=(n, 1)).astype(np.float32)
    return (rng.standard_normal((n, d)).astype(np.float32) * mag).astype(np.float32)


def _x(S, c, qmax, bf16_r=False):
    rc = (np.float32(1.0) / c).astype(np.float32)          # __frcp_rn
    t = (S * rc).astype(np.float32)
    m = np.max(np.abs(t), axis=1, keepdims=True)
    r = (m / np.float32(qmax)).astype(np.float32)            # IEEE division
    if bf16_r:  # round half to even to bf16
        u = r.view(np.uint32)
        u = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
        r = u.view(np.float32)
    r = np.where(r == 0, np.float32(1.0), r)
    rri = (np.float32(1.0) / r).astype(np.float32)
    return (t * rri).astype(np.float32), r


@pytest.mark.parametrize("qmax", [7, 31, 127])
def test_scaled_value_stays_below_qmax_plus_half_with_fp32_scales(qmax):
    rng = np.random.default_rng(qmax)
    d = 128
    worst = 0.0
    for scale_exp in (2, 30, 100):
        S = _f32_rows(rng, 4096, d, scale_exp)
        c = np.abs(_f32_rows(rng, 1, d, 4)) + np.float32(1e-3)
        x, r = _x(S, c.astype(np.float32), qmax)
        normal = (r >= np.float32(1.17549435e-38)).ravel()
        worst = max(worst, float(np.max(np.abs(x[normal]))))
    # three roundings of 2^-24 each at most
    assert worst <= qmax * (1 + 3 * 2.0 ** -24)
    assert worst < qmax + 0.5


def test_bf16_row_scale_leaves_the_fp32_bound():
    """With the row scale rounded to bf16, |x| goes well past the fp32 bound qmax (1 + 3 * 2^-24)
    (up to qmax / (1 - 2^-8)), so the fp32 argument does not cover it."""
    rng = np.random.default_rng(1)
    S = _f32_rows(rng, 20000, 128, 8)
    c = np.ones((1, 128), dtype=np.float32)
    x, _ = _x(S, c, 127, bf16_r=True)
    worst = float(np.max(np.abs(x)))
    assert worst > 127 * (1 + 2.0 ** -10)
    assert worst <= 127 / (1 - 2.0 ** -8) * (1 + 3 * 2.0 ** -24)
