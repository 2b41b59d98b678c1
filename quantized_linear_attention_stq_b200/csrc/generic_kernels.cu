// generic_kernels.cu -- one CTA per (request, head) tile, the state staged in shared memory as
// fp32 and every step written out directly: dequantization, the decode step for the small head
// sizes (d < 128), the sequential prefill, and the initial quantization of the heads the streaming
// init kernel does not take (FP16 pivots, uniform and multi-round layouts, d < 128, states that
// are not 16-byte aligned). The tuned d = 128 decode lives in decode_d128.cu, the streaming init
// of 128 x 128 row x column heads in init_d128.cu.
//
// Method (formulas in include/stq.h): per-step read -> gated delta rule update -> readout ->
// requantize -> store ("线性注意力状态量化难题" (aitest123.com/news/n1kj09), section
// 直接量化为什么会翻车); key-row x value-column scales with the impact-weighted column fit
// (same page, section 空间维度; "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), section 方法);
// FP16 pivot heads (k1 page, section 方法).
#include "stq_internal.cuh"

namespace stq {
namespace {

constexpr int kThreads = 256;

struct TileRef {
    bool ok;
    bool uniform;  // one scale for the whole head (the baseline quantizer)
    int sb16;      // row and column scales stored as bf16
    int rounds;    // rounds of the impact-weighted joint refinement of the scales
    int b, head, bits;
    uint8_t *block;
};

__device__ __forceinline__ TileRef tile_ref(const TileParams &p, int b, int pos)
{
    TileRef t;
    const TileEntry e = p.table[pos];
    t.b = b;
    t.head = entry_head(e);
    t.bits = entry_bits(e);
    t.uniform = entry_uniform(e);
    t.sb16 = p.scale_bf16;
    t.rounds = p.fit_rounds;
    const int slot = p.slots[b];
    t.ok = slot >= 0 && slot < p.pool_slots;
    t.block = t.ok ? p.pool + (uint64_t)slot * p.req_bytes + e.off : nullptr;
    return t;
}

// (row, column) of flat element e of a dk x dv tile; dv is a power of two (16 .. 128)
__device__ __forceinline__ int row_of(int e, int dv) { return e >> (__ffs(dv) - 1); }
__device__ __forceinline__ int col_of(int e, int dv) { return e & (dv - 1); }

// Code n (offset-binary) of a b-bit little-endian bitstream. Reads at most two bytes; the byte
// after the last code is inside the block (scales follow the codes).
__device__ __forceinline__ int read_code(const uint8_t *codes, int bits, int n)
{
    const uint32_t bit = (uint32_t)bits * (uint32_t)n;
    const uint32_t lo = codes[bit >> 3];
    const uint32_t hi = codes[(bit >> 3) + 1];
    return (int)(((lo | (hi << 8)) >> (bit & 7)) & ((1u << bits) - 1u));
}

// Pack the offset-binary codes of a dk x dv tile into `block` with whole 32-bit stores: a thread
// takes a group of codes that fills whole words (8 x 4-bit, 16 x 6-bit = 3 words, 4 x 8-bit), so
// every group starts 4-byte aligned. code(e) returns the signed code of flat element e.
template <int BITS, typename CodeOf>
__device__ __forceinline__ void pack_codes_words(uint8_t *block, int n, CodeOf code)
{
    constexpr int CW = BITS == 6 ? 16 : 32 / BITS;  // codes per group
    constexpr int WW = BITS == 6 ? 3 : 1;           // words per group
    constexpr int OFF = 1 << (BITS - 1);
    uint32_t *out = reinterpret_cast<uint32_t *>(block);
    for (int g = threadIdx.x; g < n / CW; g += blockDim.x) {
        uint32_t w[WW];
#pragma unroll
        for (int k = 0; k < WW; ++k) w[k] = 0u;
#pragma unroll
        for (int t = 0; t < CW; ++t) {
            const uint32_t u = (uint32_t)(code(g * CW + t) + OFF);
            const int bit = BITS * t;
            w[bit >> 5] |= u << (bit & 31);
            if ((bit & 31) + BITS > 32) w[(bit >> 5) + 1] |= u >> (32 - (bit & 31));
        }
#pragma unroll
        for (int k = 0; k < WW; ++k) out[g * WW + k] = w[k];
    }
}

template <typename CodeOf>
__device__ __forceinline__ void pack_codes(uint8_t *block, int bits, int n, CodeOf code)
{
    if (bits == 4)
        pack_codes_words<4>(block, n, code);
    else if (bits == 6)
        pack_codes_words<6>(block, n, code);
    else
        pack_codes_words<8>(block, n, code);
}

// Dequantize a tile from global memory into S (row stride ld): S_ij = fp32(r_i c_j) * Q_ij, or
// S_ij = s * Q_ij for a uniformly scaled head.
__device__ void dequant_to_smem(const uint8_t *block, int bits, bool uniform, int sb16, int dk, int dv, float *S,
                                int ld)
{
    const int n = dk * dv;
    if (bits == 16) {
        const __half *h = reinterpret_cast<const __half *>(block);
        for (int e = threadIdx.x; e < n; e += blockDim.x) S[row_of(e, dv) * ld + col_of(e, dv)] = __half2float(h[e]);
        return;
    }
    if (uniform) {
        const float su = *reinterpret_cast<const float *>(block + scale_offset(bits, dk, dv));
        const int off = 1 << (bits - 1);
        for (int e = threadIdx.x; e < n; e += blockDim.x)
            S[row_of(e, dv) * ld + col_of(e, dv)] = su * (float)(read_code(block, bits, e) - off);
        return;
    }
    const uint8_t *sc = block + scale_offset(bits, dk, dv);
    const int off = 1 << (bits - 1);
    const int shv = __ffs(dv) - 1;  // dv is a power of two
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
        const int i = e >> shv, j = e & (dv - 1);
        const float rc = load_scale(sc, i, sb16) * load_scale(sc, dk + j, sb16);
        S[i * ld + j] = rc * (float)(read_code(block, bits, e) - off);
    }
}

// Fit scales to the fp32 state in S and write codes + scales into `block` (or fp16 values for a
// pivot head). `wv` holds the impact weights of the head in shared memory. Needs a CTA-wide
// barrier before (S complete) and provides one after.
// Signed code of x = (s / c) / r, rounded half to even and clamped (0 for a non-finite x).
__device__ __forceinline__ float code_of(float s, float c, float r, float qmax)
{
    const float x = (s / c) / r;
    return isfinite(x) ? fminf(fmaxf(rintf(x), -qmax), qmax) : 0.f;
}

// Rounds of alternating impact-weighted least squares on the stored scales cs[dv], rs[dk] (the
// one-pass fit on entry): each round refits every column scale c_j = sum_i w_i a_i S_ij /
// sum_i w_i a_i^2 with a_i = r_i Q_ij, then every row scale r_i = sum_j b_j S_ij / sum_j b_j^2
// with b_j = c~_j Q_ij, both with the codes Q of the round's starting scales; each new value is
// rounded to the storage format and kept only if finite and positive (else the old one stays).
// Needs a CTA-wide barrier before and provides one after.
__device__ void refine_scales(const float *S, int ld, const float *wv, float qmax, int sb16, int rounds, int dk,
                              int dv, float *cs, float *rs)
{
    __shared__ float cn[128], rn[128];
    for (int round = 0; round < rounds; ++round) {
        for (int j = threadIdx.x; j < dv; j += blockDim.x) {
            float num = 0.f, den = 0.f;
            for (int i = 0; i < dk; ++i) {
                const float s = S[i * ld + j];
                const float a = rs[i] * code_of(s, cs[j], rs[i], qmax);
                num += wv[i] * a * s;
                den += wv[i] * a * a;
            }
            const float c = den > 0.f ? round_scale(num / den, sb16) : 0.f;
            cn[j] = (isfinite(c) && c > 0.f) ? c : cs[j];
        }
        __syncthreads();
        for (int i = threadIdx.x; i < dk; i += blockDim.x) {
            float num = 0.f, den = 0.f;
            for (int j = 0; j < dv; ++j) {
                const float s = S[i * ld + j];
                const float b = cn[j] * code_of(s, cs[j], rs[i], qmax);
                num += b * s;
                den += b * b;
            }
            const float r = den > 0.f ? round_scale(num / den, sb16) : 0.f;
            rn[i] = (isfinite(r) && r > 0.f) ? r : rs[i];
        }
        __syncthreads();
        for (int j = threadIdx.x; j < dv; j += blockDim.x) cs[j] = cn[j];
        for (int i = threadIdx.x; i < dk; i += blockDim.x) rs[i] = rn[i];
        __syncthreads();
    }
}

__device__ void quantize_from_smem(float *S, int ld, const float *wv, int bits, bool uniform, int sb16, int rounds,
                                   int dk, int dv, uint8_t *block, float *cs, float *rs, int32_t *status)
{
    const int n = dk * dv;
    __shared__ uint32_t smax;
    if (bits == 16) {
        __half *h = reinterpret_cast<__half *>(block);
        bool bad = false;
        for (int e = threadIdx.x; e < n; e += blockDim.x) {
            const float x = S[row_of(e, dv) * ld + col_of(e, dv)];
            bad |= !(fabsf(x) < 65520.0f);  // overflows fp16 (or is NaN)
            h[e] = __float2half_rn(x);
        }
        if (__syncthreads_or(bad) && threadIdx.x == 0) flag(status, kFlagNonfinite);
        return;
    }
    const float qmax = (float)((1 << (bits - 1)) - 1);
    if (uniform) {
        // one symmetric scale per head: s = max |S_ij| / qmax (1 when the head is all zero). The
        // magnitudes are non-negative, so their fp32 bit patterns order like their values and an
        // integer max reduces them; a NaN is skipped by fmaxf and caught by the finiteness flag.
        if (threadIdx.x == 0) smax = 0u;
        __syncthreads();
        float m = 0.f;
        bool bad = false;
        for (int e = threadIdx.x; e < n; e += blockDim.x) {
            const float x = S[row_of(e, dv) * ld + col_of(e, dv)];
            m = fmaxf(m, fabsf(x));
            bad |= !isfinite(x);
        }
        for (int sh = 16; sh > 0; sh >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, sh));
        if ((threadIdx.x & 31) == 0) atomicMax(&smax, __float_as_uint(m));
        __syncthreads();
        float su = __uint_as_float(smax) / qmax;
        if (su == 0.f) su = 1.f;
        bad |= !isfinite(su);
        if (threadIdx.x == 0) *reinterpret_cast<float *>(block + scale_offset(bits, dk, dv)) = su;
        const float isu = __frcp_rn(su);
        const int shv = __ffs(dv) - 1;
        pack_codes(block, bits, n, [&](int e) {
            const float xr = S[(e >> shv) * ld + (e & (dv - 1))] * isu;
            return (int)(isfinite(xr) ? fminf(fmaxf(rintf(xr), -qmax), qmax) : 0.f);  // rintf: half to even
        });
        if (__syncthreads_or(bad) && threadIdx.x == 0) flag(status, kFlagNonfinite);
        return;
    }
    // column scales: impact-weighted RMS over the key rows. Every thread takes one column and
    // every P-th row of it (P = threads / dv row classes, two running sums each); the partials are
    // added per column after a barrier. W = sum_i w_i is the same for every column.
    __shared__ float part[kThreads], wsum;
    {
        const int P = (int)blockDim.x / dv, j = (int)threadIdx.x % dv, cls = (int)threadIdx.x / dv;
        float E0 = 0.f, E1 = 0.f;
        int i = cls;
        for (; i + P < dk; i += 2 * P) {
            const float x0 = S[i * ld + j], x1 = S[(i + P) * ld + j];
            E0 += wv[i] * x0 * x0;
            E1 += wv[i + P] * x1 * x1;
        }
        if (i < dk) {
            const float x0 = S[i * ld + j];
            E0 += wv[i] * x0 * x0;
        }
        part[threadIdx.x] = E0 + E1;
        if (threadIdx.x < 32) {
            float W = 0.f;
            for (int r = (int)threadIdx.x; r < dk; r += 32) W += wv[r];
            for (int sh = 16; sh > 0; sh >>= 1) W += __shfl_xor_sync(0xffffffffu, W, sh);
            if (threadIdx.x == 0) wsum = W;
        }
    }
    __syncthreads();
    __shared__ float ic1[128];
    for (int j = threadIdx.x; j < dv; j += blockDim.x) {
        const int P = (int)blockDim.x / dv;
        float E = 0.f;
        for (int c = 0; c < P; ++c) E += part[c * dv + j];
        float c = sqrtf(E / wsum);
        if (c == 0.f) c = 1.f;
        cs[j] = round_scale(c, sb16);  // the codes use the stored value
        ic1[j] = __frcp_rn(cs[j]);
    }
    __syncthreads();
    // row scales: largest column-normalised magnitude over qmax. Every thread takes one row and
    // every P-th column of it; the partial maxima meet after a barrier (max is exact in any order).
    {
        const int P = (int)blockDim.x / dk, i = (int)threadIdx.x % dk, cls = (int)threadIdx.x / dk;
        float m0 = 0.f, m1 = 0.f;
        int j = cls;
        for (; j + P < dv; j += 2 * P) {
            m0 = fmaxf(m0, fabsf(S[i * ld + j] * ic1[j]));
            m1 = fmaxf(m1, fabsf(S[i * ld + j + P] * ic1[j + P]));
        }
        if (j < dv) m0 = fmaxf(m0, fabsf(S[i * ld + j] * ic1[j]));
        part[threadIdx.x] = fmaxf(m0, m1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        const int P = (int)blockDim.x / dk;
        float m = 0.f;
        for (int c = 0; c < P; ++c) m = fmaxf(m, part[c * dk + i]);
        float r = m / qmax;
        if (r == 0.f) r = 1.f;
        rs[i] = round_scale(r, sb16);
    }
    __syncthreads();
    if (rounds > 0) refine_scales(S, ld, wv, qmax, sb16, rounds, dk, dv, cs, rs);
    bool bad = false;
    uint8_t *sg = block + scale_offset(bits, dk, dv);
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        store_scale(sg, i, rs[i], sb16);
        bad |= !isfinite(rs[i]) || rs[i] == 0.f;
    }
    for (int j = threadIdx.x; j < dv; j += blockDim.x) {
        store_scale(sg, dk + j, cs[j], sb16);
        bad |= !isfinite(cs[j]);
    }
    // reciprocals of the stored scales (correctly rounded): x = S * (1/c) * (1/r) is within a few
    // fp32 ulps of (S / c) / r, ~10^-4 of a code step at most, far inside the rounding-tie window
    __shared__ float ics[128], irs[128];
    for (int j = threadIdx.x; j < dv; j += blockDim.x) ics[j] = __frcp_rn(cs[j]);
    for (int i = threadIdx.x; i < dk; i += blockDim.x) irs[i] = __frcp_rn(rs[i]);
    __syncthreads();
    // codes: whole 32-bit words per thread (pack_codes)
    const int shv = __ffs(dv) - 1;
    pack_codes(block, bits, n, [&](int e) {
        const int i = e >> shv, j = e & (dv - 1);
        const float xr = (S[i * ld + j] * ics[j]) * irs[i];
        return (int)(isfinite(xr) ? fminf(fmaxf(rintf(xr), -qmax), qmax) : 0.f);  // rintf: half to even
    });
    if (__syncthreads_or(bad) && threadIdx.x == 0) flag(status, kFlagNonfinite);
}

// ------------------------------------------------------------------------------------------
// Initial quantization: S0 fp32 [B][H][dk][dv] -> pool
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) init_kernel(const __grid_constant__ TileParams p)
{
    extern __shared__ __align__(16) float sm[];
    const int b = blockIdx.x, pos = blockIdx.y;
    const TileRef t = tile_ref(p, b, pos);
    if (!t.ok) {
        if (threadIdx.x == 0) flag(p.status, kFlagBounds);
        return;
    }
    const int dk = p.dk, dv = p.dv, ld = dv + 1;
    float *S = sm;
    float *wv = S + dk * ld;
    float *cs = wv + dk;
    float *rs = cs + dv;
    const float *src = p.S0 + ((uint64_t)b * p.head_count + t.head) * dk * dv;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) wv[i] = p.w[(uint64_t)t.head * dk + i];
    if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0 && dv >= 32) {
        // 16-byte loads, 8 in flight per thread. Lane l of a warp takes chunk (l % 8) of row (l / 8)
        // of a 4-row x 8-chunk block: rows are read 128 contiguous bytes at a time, and the scalar
        // stores into the (dv + 1)-float rows fall on 32 different banks.
        constexpr int U = 8;
        const int cpr = dv / 4, gpr = cpr / 8, n4 = dk * cpr;
        const float4 *s4 = reinterpret_cast<const float4 *>(src);
        for (int base = threadIdx.x; base < n4; base += U * blockDim.x) {
            float4 v[U];
            int at[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int g = base + u * (int)blockDim.x;
                at[u] = -1;
                if (g < n4) {
                    const int wg = g >> 5, l = g & 31;
                    const int i = 4 * (wg / gpr) + (l >> 3), q = 8 * (wg % gpr) + (l & 7);
                    v[u] = s4[i * cpr + q];
                    at[u] = i * ld + 4 * q;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (at[u] >= 0) {
                    float *d = S + at[u];
                    d[0] = v[u].x;
                    d[1] = v[u].y;
                    d[2] = v[u].z;
                    d[3] = v[u].w;
                }
            }
        }
    } else {
        const int shv = __ffs(dv) - 1;  // dv is a power of two
        for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) S[(e >> shv) * ld + (e & (dv - 1))] = src[e];
    }
    __syncthreads();
    quantize_from_smem(S, ld, wv, t.bits, t.uniform, t.sb16, t.rounds, dk, dv, t.block, cs, rs, p.status);
}

// ------------------------------------------------------------------------------------------
// Dequantization: pool -> S_out fp32 [B][H][dk][dv]
// ------------------------------------------------------------------------------------------
// Row x column codes of width BITS (scales bf16 if SB16), 8 consecutive elements of a row per
// thread: the group's BITS * 8 code bits are BITS bytes at byte offset BITS * g, unpacked at once,
// and the 8 column scales are one or two 16-byte loads (8 | d_v, and the scales start on a 16-byte
// boundary); S_ij = fp32(r_i c_j) Q_ij.
template <int BITS, int SB16>
__device__ __forceinline__ void dequant_rc(const uint8_t *block, const uint8_t *sc, int dk, int dv, float *dst)
{
    constexpr int off = 1 << (BITS - 1);
    constexpr uint32_t mask = (1u << BITS) - 1u;
    const int shv = __ffs(dv) - 1;
    for (int g = threadIdx.x; g < dk * dv / 8; g += blockDim.x) {
        const int e0 = 8 * g, i = e0 >> shv, j0 = e0 & (dv - 1);
        uint32_t lo, hi;
        if constexpr (BITS == 8) {
            const uint2 wd = *reinterpret_cast<const uint2 *>(block + 8 * g);
            lo = wd.x;
            hi = wd.y;
        } else if constexpr (BITS == 4) {
            lo = *reinterpret_cast<const uint32_t *>(block + 4 * g);
            hi = 0u;
        } else {  // 6 bytes at 6g, 2-byte aligned
            const uint16_t *h = reinterpret_cast<const uint16_t *>(block + 6 * g);
            lo = (uint32_t)h[0] | ((uint32_t)h[1] << 16);
            hi = h[2];
        }
        const float r = load_scale(sc, i, SB16);
        float c[8];
        if constexpr (SB16) {
            const uint4 cw = *reinterpret_cast<const uint4 *>(sc + 2 * (dk + j0));
            const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                c[2 * k] = __uint_as_float(w4[k] << 16);              // bf16 -> fp32: the high half of the word
                c[2 * k + 1] = __uint_as_float(w4[k] & 0xffff0000u);
            }
        } else {
            const float4 a = *reinterpret_cast<const float4 *>(sc + 4 * (dk + j0));
            const float4 b = *reinterpret_cast<const float4 *>(sc + 4 * (dk + j0) + 16);
            c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w;
            c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
        }
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int bit = BITS * k;  // position in the 64-bit (hi:lo) group
            const uint32_t u = (bit < 32 ? (bit + BITS <= 32 ? lo >> bit : __funnelshift_r(lo, hi, bit))
                                         : hi >> (bit - 32)) & mask;
            v[k] = (r * c[k]) * (float)((int)u - off);
        }
        float4 *o4 = reinterpret_cast<float4 *>(dst + e0);
        o4[0] = make_float4(v[0], v[1], v[2], v[3]);
        o4[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
}

__global__ void __launch_bounds__(kThreads) dequant_kernel(const __grid_constant__ TileParams p)
{
    const int b = blockIdx.x, pos = blockIdx.y;
    const TileRef t = tile_ref(p, b, pos);
    if (!t.ok) {
        if (threadIdx.x == 0) flag(p.status, kFlagBounds);
        return;
    }
    const int dk = p.dk, dv = p.dv;
    float *dst = p.S_out + ((uint64_t)b * p.head_count + t.head) * dk * dv;
    if (t.bits == 16 || t.uniform || (reinterpret_cast<uintptr_t>(dst) & 15u) != 0) {
        dequant_to_smem(t.block, t.bits, t.uniform, t.sb16, dk, dv, dst, dv);  // straight to global, row stride dv
        return;
    }
    const uint8_t *sc = t.block + scale_offset(t.bits, dk, dv);
    switch (2 * t.bits + t.sb16) {
    case 8: dequant_rc<4, 0>(t.block, sc, dk, dv, dst); break;
    case 9: dequant_rc<4, 1>(t.block, sc, dk, dv, dst); break;
    case 12: dequant_rc<6, 0>(t.block, sc, dk, dv, dst); break;
    case 13: dequant_rc<6, 1>(t.block, sc, dk, dv, dst); break;
    case 16: dequant_rc<8, 0>(t.block, sc, dk, dv, dst); break;
    default: dequant_rc<8, 1>(t.block, sc, dk, dv, dst); break;
    }
}

// ------------------------------------------------------------------------------------------
// Decode step, plain form
// ------------------------------------------------------------------------------------------
template <int IN_BF16>
__global__ void __launch_bounds__(kThreads) decode_generic_kernel(const __grid_constant__ TileParams p)
{
    extern __shared__ __align__(16) float sm[];
    const int b = blockIdx.x, pos = blockIdx.y;
    const TileRef t = tile_ref(p, b, pos);
    if (!t.ok) {
        if (threadIdx.x == 0) flag(p.status, kFlagBounds);
        return;
    }
    const int dk = p.dk, dv = p.dv, ld = dv + 1;
    float *S = sm;
    float *kv = S + dk * ld;
    float *qv = kv + dk;
    float *av = qv + dk;
    float *wv = av + dk;
    float *vv = wv + dk;
    float *uv = vv + dv;
    float *cs = uv + dv;
    float *rs = cs + dv;
    const uint64_t tile = (uint64_t)b * p.head_count + t.head;
    const bool channel = p.gate != 0;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        kv[i] = load_in<IN_BF16>(p.k, tile * dk + i);
        qv[i] = load_in<IN_BF16>(p.q, tile * dk + i);
        av[i] = channel ? p.alpha[tile * dk + i] : p.alpha[tile];
        wv[i] = p.w[(uint64_t)t.head * dk + i];
    }
    for (int j = threadIdx.x; j < dv; j += blockDim.x) vv[j] = load_in<IN_BF16>(p.v, tile * dv + j);
    dequant_to_smem(t.block, t.bits, t.uniform, t.sb16, dk, dv, S, ld);
    __syncthreads();
    const float beta = p.beta[tile];
    const bool decay_first = p.gate == 2;
    // u = k^T S   (decay-first: k^T diag(alpha) S)
    for (int j = threadIdx.x; j < dv; j += blockDim.x) {
        float acc = 0.f;
        for (int i = 0; i < dk; ++i) acc += kv[i] * (decay_first ? av[i] : 1.f) * S[i * ld + j];
        uv[j] = acc;
    }
    __syncthreads();
    // S' = alpha (S - beta k u^T) + beta k v^T   (decay-first: alpha S - beta k u^T + beta k v^T)
    for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
        const int i = row_of(e, dv), j = col_of(e, dv);
        const float s = S[i * ld + j];
        S[i * ld + j] = decay_first ? av[i] * s - beta * kv[i] * uv[j] + beta * kv[i] * vv[j]
                                    : av[i] * (s - beta * kv[i] * uv[j]) + beta * kv[i] * vv[j];
    }
    __syncthreads();
    // o = S'^T q
    bool bad = false;
    for (int j = threadIdx.x; j < dv; j += blockDim.x) {
        float acc = 0.f;
        for (int i = 0; i < dk; ++i) acc += qv[i] * S[i * ld + j];
        p.o[tile * dv + j] = acc;
        bad |= !isfinite(acc);
    }
    if (bad) flag(p.status, kFlagNonfinite);
    quantize_from_smem(S, ld, wv, t.bits, t.uniform, t.sb16, t.rounds, dk, dv, t.block, cs, rs, p.status);
}

// ------------------------------------------------------------------------------------------
// Chunked prefill, sequential form: the state is carried unquantized in shared memory through a
// chunk (token-by-token gated delta rule, o_t = S_t^T q_t per token) and requantized into the
// pool at the end of every chunk; the next chunk starts from the dequantized state.
// ------------------------------------------------------------------------------------------
template <int IN_BF16>
__global__ void __launch_bounds__(kThreads) prefill_seq_kernel(const __grid_constant__ TileParams p, int T, int chunk)
{
    extern __shared__ __align__(16) float sm[];
    const int b = blockIdx.x, pos = blockIdx.y;
    const TileRef t = tile_ref(p, b, pos);
    if (!t.ok) {
        if (threadIdx.x == 0) flag(p.status, kFlagBounds);
        return;
    }
    const int dk = p.dk, dv = p.dv, ld = dv + 1;
    float *S = sm;
    float *kv = S + dk * ld;
    float *qv = kv + dk;
    float *av = qv + dk;
    float *wv = av + dk;
    float *vv = wv + dk;
    float *uv = vv + dv;
    float *cs = uv + dv;
    float *rs = cs + dv;
    const uint64_t tile = (uint64_t)b * p.head_count + t.head;
    const bool channel = p.gate != 0, decay_first = p.gate == 2;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) wv[i] = p.w[(uint64_t)t.head * dk + i];
    dequant_to_smem(t.block, t.bits, t.uniform, t.sb16, dk, dv, S, ld);
    bool bad = false;
    for (int tok = 0; tok < T; ++tok) {
        const uint64_t row = tile * T + tok;
        for (int i = threadIdx.x; i < dk; i += blockDim.x) {
            kv[i] = load_in<IN_BF16>(p.k, row * dk + i);
            qv[i] = load_in<IN_BF16>(p.q, row * dk + i);
            av[i] = channel ? p.alpha[row * dk + i] : p.alpha[row];
        }
        for (int j = threadIdx.x; j < dv; j += blockDim.x) vv[j] = load_in<IN_BF16>(p.v, row * dv + j);
        __syncthreads();
        const float beta = p.beta[row];
        for (int j = threadIdx.x; j < dv; j += blockDim.x) {
            float acc = 0.f;
            for (int i = 0; i < dk; ++i) acc += kv[i] * (decay_first ? av[i] : 1.f) * S[i * ld + j];
            uv[j] = acc;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
            const int i = row_of(e, dv), j = col_of(e, dv);
            const float s = S[i * ld + j];
            S[i * ld + j] = decay_first ? av[i] * s - beta * kv[i] * uv[j] + beta * kv[i] * vv[j]
                                        : av[i] * (s - beta * kv[i] * uv[j]) + beta * kv[i] * vv[j];
        }
        __syncthreads();
        for (int j = threadIdx.x; j < dv; j += blockDim.x) {
            float acc = 0.f;
            for (int i = 0; i < dk; ++i) acc += qv[i] * S[i * ld + j];
            p.o[row * dv + j] = acc;
            bad |= !isfinite(acc);
        }
        if ((tok + 1) % chunk == 0 || tok == T - 1) {
            __syncthreads();
            quantize_from_smem(S, ld, wv, t.bits, t.uniform, t.sb16, t.rounds, dk, dv, t.block, cs, rs, p.status);
            if (tok != T - 1) {
                __syncthreads();
                dequant_to_smem(t.block, t.bits, t.uniform, t.sb16, dk, dv, S, ld);
            }
        }
        __syncthreads();
    }
    if (bad) flag(p.status, kFlagNonfinite);
}

size_t generic_smem_bytes(const TileParams &p)
{
    return sizeof(float) * ((size_t)p.dk * (p.dv + 1) + 5 * (size_t)p.dk + 4 * (size_t)p.dv + 64);
}

template <typename K>
cudaError_t launch_tiles(K kernel, const TileParams &p, cudaStream_t s)
{
    const size_t smem = generic_smem_bytes(p);
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid((unsigned)p.B, (unsigned)p.npos);
    kernel<<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_init_generic(const TileParams &p, cudaStream_t s) { return launch_tiles(init_kernel, p, s); }

cudaError_t launch_dequant_generic(const TileParams &p, cudaStream_t s)
{
    dim3 grid((unsigned)p.B, (unsigned)p.npos);
    dequant_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_decode_generic(const TileParams &p, int in_bf16, cudaStream_t s)
{
    return in_bf16 ? launch_tiles(decode_generic_kernel<1>, p, s) : launch_tiles(decode_generic_kernel<0>, p, s);
}

cudaError_t launch_prefill_seq(const TileParams &p, int in_bf16, int T, int chunk, cudaStream_t s)
{
    const size_t smem = generic_smem_bytes(p);
    auto kernel = in_bf16 ? prefill_seq_kernel<1> : prefill_seq_kernel<0>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid((unsigned)p.B, (unsigned)p.npos);
    kernel<<<grid, kThreads, smem, s>>>(p, T, chunk);
    return cudaGetLastError();
}

}  // namespace stq
