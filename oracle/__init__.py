"""The oracle: a plain fp64 CPU implementation of the quantized-state decode path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package. The product library
(``quantized_linear_attention_stq_b200``) never imports, loads or calls it, and the two share
no code: the arithmetic lives in ``stq_oracle.c`` (plain C99, fp64, no FMA contraction); this
module only builds that file with gcc and marshals numpy arrays through ctypes.

Every function follows the pages it cites in ``stq_oracle.c``:
  "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), sections 方法 / 實驗結果, and
  "线性注意力状态量化难题" (aitest123.com/news/n1kj09), sections 直接量化为什么会翻车 / 时间维度 /
  空间维度 / 工程落地.
Parity of the accuracy claims (perplexity, benchmark scores, generation lengths) is unpinned:
those need the models and evaluation suites, which this library does not have.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "stq_oracle.c")
_HDR = os.path.join(_HERE, "stq_oracle.h")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libstq_oracle.so")

OK, EINVAL, ENONFINITE = 0, 1, 4
GATE_SCALAR, GATE_CHANNEL, GATE_CHANNEL_DECAY_FIRST = 0, 1, 2
SCALE_F32, SCALE_BF16 = 0, 1  # storage format of the row and column scales
TIE_DELTA = 1e-3

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``stq_oracle.c`` into ``_build/libstq_oracle.so`` (gcc, -O2, no FMA contraction)."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            L = ctypes.CDLL(path)
            P = ctypes.c_void_p
            i32, f64, sz = ctypes.c_int, ctypes.c_double, ctypes.c_size_t
            L.orc_qmax.argtypes, L.orc_qmax.restype = [i32], i32
            L.orc_round_half_even.argtypes, L.orc_round_half_even.restype = [f64], f64
            for name in ("orc_codes_bytes", "orc_scale_offset", "orc_block_bytes"):
                getattr(L, name).argtypes = [i32, i32, i32]
                getattr(L, name).restype = sz
            L.orc_pack.argtypes, L.orc_pack.restype = [i32, sz, P, P], None
            L.orc_unpack.argtypes, L.orc_unpack.restype = [i32, sz, P, P], None
            L.orc_half_to_double.argtypes, L.orc_half_to_double.restype = [ctypes.c_uint16], f64
            L.orc_double_to_half.argtypes, L.orc_double_to_half.restype = [f64], ctypes.c_uint16
            L.orc_quantize.argtypes = [i32, i32, i32, P, P, P, P, P, f64]
            L.orc_quantize.restype = i32
            L.orc_dequantize.argtypes, L.orc_dequantize.restype = [i32, i32, i32, P, P], i32
            L.orc_update.argtypes = [i32, i32, i32, P, P, P, P, f64, P, P]
            L.orc_update.restype = None
            L.orc_decode_step.argtypes = [i32, i32, i32, i32, P, P, P, P, f64, P, P, P, P, P, P, f64]
            L.orc_decode_step.restype = i32
            L.orc_prefill_seq.argtypes = [i32, i32, i32, i32, P, i32, i32, P, P, P, P, P, P, P, P, P, f64]
            L.orc_prefill_seq.restype = i32
            L.orc_chunk_wy.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P]
            L.orc_chunk_wy.restype = i32
            L.orc_uniform_block_bytes.argtypes, L.orc_uniform_block_bytes.restype = [i32, i32, i32], sz
            L.orc_quantize_uniform.argtypes = [i32, i32, i32, P, P, P, P, f64]
            L.orc_quantize_uniform.restype = i32
            L.orc_dequantize_uniform.argtypes, L.orc_dequantize_uniform.restype = [i32, i32, i32, P, P], i32
            L.orc_decode_step_uniform.argtypes = [i32, i32, i32, i32, P, P, P, P, f64, P, P, P, P, f64]
            L.orc_decode_step_uniform.restype = i32
            L.orc_block_bytes_s.argtypes, L.orc_block_bytes_s.restype = [i32, i32, i32, i32], sz
            L.orc_bf16_to_double.argtypes, L.orc_bf16_to_double.restype = [ctypes.c_uint16], f64
            L.orc_double_to_bf16.argtypes, L.orc_double_to_bf16.restype = [f64], ctypes.c_uint16
            L.orc_quantize_s.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P, P, P, f64]
            L.orc_quantize_s.restype = i32
            L.orc_dequantize_s.argtypes, L.orc_dequantize_s.restype = [i32, i32, i32, i32, P, P], i32
            L.orc_decode_step_s.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P, f64, P, P, P, P, P, P, P, f64]
            L.orc_decode_step_s.restype = i32
            L.orc_prefill_seq_s.argtypes = [i32, i32, i32, i32, i32, i32, P, i32, i32, P, P, P, P, P, P, P, P, P, P,
                                            f64]
            L.orc_quantize_fit.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, f64]
            L.orc_quantize_fit.restype = i32
            L.orc_prefill_seq_s.restype = i32
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


# ----------------------------------------------------------------------------------------------
# Elementary pieces
# ----------------------------------------------------------------------------------------------

def qmax(bits: int) -> int:
    return lib().orc_qmax(bits)


def round_half_even(y: float) -> float:
    return lib().orc_round_half_even(float(y))


def codes_bytes(bits: int, dk: int, dv: int) -> int:
    return lib().orc_codes_bytes(bits, dk, dv)


def scale_offset(bits: int, dk: int, dv: int) -> int:
    return lib().orc_scale_offset(bits, dk, dv)


def block_bytes(bits: int, dk: int, dv: int) -> int:
    return lib().orc_block_bytes(bits, dk, dv)


def pack(bits: int, u) -> np.ndarray:
    u = np.ascontiguousarray(np.asarray(u, dtype=np.int32).ravel())
    out = np.zeros((bits * u.size + 7) // 8, dtype=np.uint8)
    lib().orc_pack(bits, u.size, _p(u), _p(out))
    return out


def unpack(bits: int, n: int, data) -> np.ndarray:
    data = np.ascontiguousarray(np.asarray(data, dtype=np.uint8))
    assert data.size * 8 >= bits * n
    u = np.zeros(n, dtype=np.int32)
    lib().orc_unpack(bits, n, _p(data), _p(u))
    return u


def bf16_to_double(h: int) -> float:
    return lib().orc_bf16_to_double(int(h))


def double_to_bf16(x: float) -> int:
    return lib().orc_double_to_bf16(float(x))


def half_to_double(h: int) -> float:
    return lib().orc_half_to_double(int(h))


def double_to_half(x: float) -> int:
    return lib().orc_double_to_half(float(x))


# ----------------------------------------------------------------------------------------------
# One head block
# ----------------------------------------------------------------------------------------------

def quantize(bits: int, S, w=None, delta: float = TIE_DELTA):
    """Quantize an fp64 state into a fresh head block. Returns (block, x, tie, status)."""
    S = _f64(S)
    dk, dv = S.shape
    w = _f64(np.ones(dk) if w is None else w)
    block = np.zeros(block_bytes(bits, dk, dv), dtype=np.uint8)
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    st = lib().orc_quantize(bits, dk, dv, _p(S), _p(w), _p(block), _p(x), _p(tie), float(delta))
    return block, x, tie.astype(bool), st


def dequantize(bits: int, dk: int, dv: int, block) -> np.ndarray:
    block = np.ascontiguousarray(np.asarray(block, dtype=np.uint8))
    assert block.size >= block_bytes(bits, dk, dv)
    S = np.zeros((dk, dv))
    st = lib().orc_dequantize(bits, dk, dv, _p(block), _p(S))
    assert st == OK
    return S


def codes(bits: int, dk: int, dv: int, block) -> np.ndarray:
    """Signed integer codes Q (dk x dv) of a quantized head block."""
    u = unpack(bits, dk * dv, np.asarray(block, dtype=np.uint8)[: codes_bytes(bits, dk, dv)])
    return (u - (1 << (bits - 1))).reshape(dk, dv)


def scales(bits: int, dk: int, dv: int, block):
    """(r, c) fp32 scales of a quantized head block."""
    off = scale_offset(bits, dk, dv)
    raw = np.asarray(block, dtype=np.uint8)
    r = raw[off: off + 4 * dk].view(np.float32).copy()
    c = raw[off + 4 * dk: off + 4 * dk + 4 * dv].view(np.float32).copy()
    return r, c


def pivot_values(dk: int, dv: int, block) -> np.ndarray:
    return np.asarray(block, dtype=np.uint8)[: 2 * dk * dv].view(np.uint16).reshape(dk, dv).copy()


def update(gate: int, S, q, k, v, beta: float, alpha):
    """Unquantized fp64 gated-delta-rule update (returns S', o); no rounding of any kind."""
    S = _f64(S).copy()
    dk, dv = S.shape
    o = np.zeros(dv)
    a = _f64(np.atleast_1d(alpha))
    lib().orc_update(dk, dv, gate, _p(S), _p(_f64(q)), _p(_f64(k)), _p(_f64(v)), float(beta), _p(a), _p(o))
    return S, o


def decode_step(bits: int, gate: int, block, q, k, v, beta: float, alpha, w,
                dk: int, dv: int, delta: float = TIE_DELTA):
    """One decode step on a copy of ``block``.

    Returns dict(block, o (fp32), S_new (fp64, before requantization), x, tie, status)."""
    blk = np.ascontiguousarray(np.asarray(block, dtype=np.uint8)).copy()
    o = np.zeros(dv, dtype=np.float32)
    S_new = np.zeros((dk, dv))
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    a = _f64(np.atleast_1d(alpha))
    wv = _f64(np.ones(dk) if w is None else w)
    st = lib().orc_decode_step(bits, dk, dv, gate, _p(blk), _p(_f64(q)), _p(_f64(k)), _p(_f64(v)),
                               float(beta), _p(a), _p(wv), _p(o), _p(S_new), _p(x), _p(tie),
                               float(delta))
    return dict(block=blk, o=o, S_new=S_new, x=x, tie=tie.astype(bool), status=st)


def prefill_seq(bits: int, gate: int, block, q, k, v, beta, alpha, w, chunk: int,
                dk: int, dv: int, delta: float = TIE_DELTA):
    """Sequential chunked prefill on a copy of ``block`` (q,k: [T][dk], v: [T][dv])."""
    blk = np.ascontiguousarray(np.asarray(block, dtype=np.uint8)).copy()
    q, k, v = _f64(q), _f64(k), _f64(v)
    T = q.shape[0]
    o = np.zeros((T, dv), dtype=np.float32)
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    st = lib().orc_prefill_seq(bits, dk, dv, gate, _p(blk), T, chunk, _p(q), _p(k), _p(v),
                               _p(_f64(beta)), _p(_f64(alpha)), _p(_f64(w)), _p(o), _p(x), _p(tie),
                               float(delta))
    return dict(block=blk, o=o, x=x, tie=tie.astype(bool), status=st)


def chunk_wy(S0, q, k, v, beta, alpha):
    """fp64 WY/UT evaluation of one chunk (scalar gate, no quantization) -> (S_end, O)."""
    S0 = _f64(S0)
    dk, dv = S0.shape
    q, k, v = _f64(q), _f64(k), _f64(v)
    C = q.shape[0]
    S_end = np.zeros((dk, dv))
    O = np.zeros((C, dv))
    st = lib().orc_chunk_wy(dk, dv, C, _p(S0), _p(q), _p(k), _p(v), _p(_f64(beta)), _p(_f64(alpha)),
                            _p(S_end), _p(O))
    assert st == OK
    return S_end, O


# ----------------------------------------------------------------------------------------------
# Request blocks (a request's head blocks back to back, padded to 128 bytes)
# ----------------------------------------------------------------------------------------------

def request_layout(head_bits, dk: int, dv: int):
    """Per-head byte offsets inside one request block, and the request block size."""
    offs, pos = [], 0
    for b in head_bits:
        offs.append(pos)
        pos += block_bytes(int(b), dk, dv)
    total = (pos + 127) // 128 * 128
    return np.array(offs, dtype=np.int64), total


# ---------------------------------------------------------------------------------------------
# Uniform baseline quantizer (one scale per head; see stq_oracle.c)
# ---------------------------------------------------------------------------------------------

def uniform_block_bytes(bits: int, dk: int, dv: int) -> int:
    return int(lib().orc_uniform_block_bytes(bits, dk, dv))


def quantize_uniform(bits: int, S, delta: float = TIE_DELTA):
    """Uniform per-head quantization into a fresh block. Returns (block, x, tie, status)."""
    S = _f64(S)
    dk, dv = S.shape
    block = np.zeros(uniform_block_bytes(bits, dk, dv), dtype=np.uint8)
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    st = lib().orc_quantize_uniform(bits, dk, dv, _p(S), _p(block), _p(x), _p(tie), float(delta))
    return block, x, tie.astype(bool), st


def dequantize_uniform(bits: int, dk: int, dv: int, block) -> np.ndarray:
    block = np.ascontiguousarray(np.asarray(block, dtype=np.uint8))
    S = np.zeros((dk, dv))
    lib().orc_dequantize_uniform(bits, dk, dv, _p(block), _p(S))
    return S


def uniform_scale(bits: int, dk: int, dv: int, block) -> float:
    off = scale_offset(bits, dk, dv)
    return float(np.asarray(block, dtype=np.uint8)[off:off + 4].view(np.float32)[0])


def decode_step_uniform(bits: int, gate: int, block, q, k, v, beta: float, alpha, dk: int, dv: int,
                        delta: float = TIE_DELTA):
    """One decode step of a uniformly quantized head on a copy of ``block``."""
    blk = np.ascontiguousarray(np.asarray(block, dtype=np.uint8)).copy()
    o = np.zeros(dv, dtype=np.float32)
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    a = _f64(np.atleast_1d(alpha))
    st = lib().orc_decode_step_uniform(bits, dk, dv, gate, _p(blk), _p(_f64(q)), _p(_f64(k)), _p(_f64(v)),
                                       float(beta), _p(a), _p(o), _p(x), _p(tie), float(delta))
    return dict(block=blk, o=o, x=x, tie=tie.astype(bool), status=st)


# ---------------------------------------------------------------------------------------------
# Scale storage formats (fp32, or bf16 for 16-bit scales; see stq_oracle.c)
# ---------------------------------------------------------------------------------------------

def block_bytes_s(bits: int, sfmt: int, dk: int, dv: int) -> int:
    return int(lib().orc_block_bytes_s(bits, sfmt, dk, dv))


def quantize_s(bits: int, sfmt: int, S, w=None, c_given=None, r_given=None, delta: float = TIE_DELTA):
    """Quantize with scales stored in format sfmt; c_given / r_given replace the fitted stored
    scales. Returns (block, x, tie, scale_tie, status); scale_tie holds dk row flags, then dv
    column flags."""
    S = _f64(S)
    dk, dv = S.shape
    w = _f64(np.ones(dk) if w is None else w)
    block = np.zeros(block_bytes_s(bits, sfmt, dk, dv), dtype=np.uint8)
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    stie = np.zeros(dk + dv, dtype=np.uint8)
    cg = None if c_given is None else _f64(c_given)
    rg = None if r_given is None else _f64(r_given)
    st = lib().orc_quantize_s(bits, sfmt, dk, dv, _p(S), _p(w), _p(cg), _p(rg), _p(block), _p(x), _p(tie),
                              _p(stie), float(delta))
    return block, x, tie.astype(bool), stie.astype(bool), st


def dequantize_s(bits: int, sfmt: int, dk: int, dv: int, block) -> np.ndarray:
    block = np.ascontiguousarray(np.asarray(block, dtype=np.uint8))
    assert block.size >= block_bytes_s(bits, sfmt, dk, dv)
    S = np.zeros((dk, dv))
    st = lib().orc_dequantize_s(bits, sfmt, dk, dv, _p(block), _p(S))
    assert st == OK
    return S


def scales_s(bits: int, sfmt: int, dk: int, dv: int, block):
    """(r, c) stored scales of a head block as fp64 values."""
    if sfmt == SCALE_F32:
        r, c = scales(bits, dk, dv, block)
        return r.astype(np.float64), c.astype(np.float64)
    off = scale_offset(bits, dk, dv)
    raw = np.asarray(block, dtype=np.uint8)[off: off + 2 * (dk + dv)].view(np.uint16)
    vals = np.array([bf16_to_double(int(h)) for h in raw])
    return vals[:dk], vals[dk:]


def decode_step_s(bits: int, sfmt: int, gate: int, block, q, k, v, beta: float, alpha, w, dk: int, dv: int,
                  delta: float = TIE_DELTA, rounds: int = 0):
    """One decode step on a copy of ``block`` with scales in format sfmt. Returns dict(block, o,
    S_new (fp64 before requantization), x, tie, scale_tie, status)."""
    blk = np.ascontiguousarray(np.asarray(block, dtype=np.uint8)).copy()
    o = np.zeros(dv, dtype=np.float32)
    S_new = np.zeros((dk, dv))
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    stie = np.zeros(dk + dv, dtype=np.uint8)
    a = _f64(np.atleast_1d(alpha))
    wv = _f64(np.ones(dk) if w is None else w)
    st = lib().orc_decode_step_s(bits, sfmt, rounds, dk, dv, gate, _p(blk), _p(_f64(q)), _p(_f64(k)), _p(_f64(v)),
                                 float(beta), _p(a), _p(wv), _p(o), _p(S_new), _p(x), _p(tie), _p(stie),
                                 float(delta))
    return dict(block=blk, o=o, S_new=S_new, x=x, tie=tie.astype(bool), scale_tie=stie.astype(bool), status=st)


def prefill_seq_s(bits: int, sfmt: int, gate: int, block, q, k, v, beta, alpha, w, chunk: int, dk: int, dv: int,
                  delta: float = TIE_DELTA, rounds: int = 0):
    """Sequential chunked prefill on a copy of ``block`` with scales in format sfmt."""
    blk = np.ascontiguousarray(np.asarray(block, dtype=np.uint8)).copy()
    q, k, v = _f64(q), _f64(k), _f64(v)
    T = q.shape[0]
    o = np.zeros((T, dv), dtype=np.float32)
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    stie = np.zeros(dk + dv, dtype=np.uint8)
    st = lib().orc_prefill_seq_s(bits, sfmt, rounds, dk, dv, gate, _p(blk), T, chunk, _p(q), _p(k), _p(v),
                                 _p(_f64(beta)), _p(_f64(alpha)), _p(_f64(w)), _p(o), _p(x), _p(tie), _p(stie),
                                 float(delta))
    return dict(block=blk, o=o, x=x, tie=tie.astype(bool), scale_tie=stie.astype(bool), status=st)


def quantize_fit(bits: int, sfmt: int, rounds: int, S, w=None, delta: float = TIE_DELTA):
    """One-pass fit plus `rounds` rounds of the impact-weighted joint refinement (stq_oracle.c).
    Returns (block, x, tie, status)."""
    S = _f64(S)
    dk, dv = S.shape
    w = _f64(np.ones(dk) if w is None else w)
    block = np.zeros(block_bytes_s(bits, sfmt, dk, dv), dtype=np.uint8)
    x = np.zeros((dk, dv))
    tie = np.zeros((dk, dv), dtype=np.uint8)
    st = lib().orc_quantize_fit(bits, sfmt, rounds, dk, dv, _p(S), _p(w), _p(block), _p(x), _p(tie), None,
                                float(delta))
    return block, x, tie.astype(bool), st
