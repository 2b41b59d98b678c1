// prefill_common.cuh -- device helpers shared by the chunked-prefill kernels of 128 x 128
// states: packed-code row load / store, bf16 term splitting of fp32 operands, the 64 x 64 unit
// lower-triangular inverse of the UT transform, bounded barrier waits and Tensor Memory loads.
#pragma once

#include "stq_internal.cuh"
#include "umma.cuh"

namespace stq {
namespace pf {

using umma::sw128_chunk;

constexpr int D = 128;
constexpr int C = 64;   // chunk length
constexpr int LDL = 68; // row stride (floats) of the fp32 L and T work matrices

template <int BITS>
struct PCfg {
    static constexpr int QMAX = (1 << (BITS - 1)) - 1;
    static constexpr int OFFS = 1 << (BITS - 1);
    static constexpr uint32_t ROWB = 16u * BITS;               // packed bytes of one 128-code row
    static constexpr uint32_t SOFF = scale_offset(BITS, D, D); // r[] then c[]
};

__device__ __forceinline__ float *smf(uint8_t *base, uint32_t off) { return reinterpret_cast<float *>(base + off); }
__device__ __forceinline__ double *smd(uint8_t *base, uint32_t off) { return reinterpret_cast<double *>(base + off); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------------------------------------
// State load / store (packed little-endian offset-binary bitstream, row-major). Thread (row i,
// quarter part) owns codes i, 32 part .. 32 part + 31: BITS 32-bit words at an 8-byte boundary.
// ---------------------------------------------------------------------------------------------
template <int BITS>
__device__ __forceinline__ void load_codes_row(const uint8_t *gblock, uint8_t *qc, int i, int part)
{
    using P = PCfg<BITS>;
    uint32_t wv[BITS + 1];
    const uint2 *src = reinterpret_cast<const uint2 *>(gblock + (size_t)i * P::ROWB + part * (4 * BITS));
#pragma unroll
    for (int k = 0; k < BITS / 2; ++k) {
        const uint2 x = src[k];
        wv[2 * k] = x.x;
        wv[2 * k + 1] = x.y;
    }
    wv[BITS] = 0u;
    uint8_t *atom = qc + (part >> 1) * 16384;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t packed[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float f[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                const int col = 8 * k + e + z, bit = BITS * col, wi = bit >> 5, sh = bit & 31;
                uint32_t u = wv[wi] >> sh;
                if (sh + BITS > 32) u |= wv[wi + 1] << (32 - sh);
                u &= (1u << BITS) - 1u;
                f[z] = (float)((int)u - P::OFFS);
            }
            packed[e >> 1] = umma::pack_bf16(__float2bfloat16_rn(f[0]), __float2bfloat16_rn(f[1]));
        }
        *reinterpret_cast<uint4 *>(atom + sw128_chunk(i, 4 * (part & 1) + k)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

template <int BITS>
__device__ __forceinline__ void store_codes_row(uint8_t *gblock, int i, int part, const float (&q)[32])
{
    using P = PCfg<BITS>;
    uint32_t wv[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) wv[k] = 0u;
#pragma unroll
    for (int col = 0; col < 32; ++col) {
        const uint32_t u = (uint32_t)((int)q[col] + P::OFFS);
        const int bit = BITS * col, wi = bit >> 5, sh = bit & 31;
        wv[wi] |= u << sh;
        if (sh + BITS > 32) wv[wi + 1] |= u >> (32 - sh);
    }
    uint2 *dst = reinterpret_cast<uint2 *>(gblock + (size_t)i * P::ROWB + part * (4 * BITS));
#pragma unroll
    for (int k = 0; k < BITS / 2; ++k) dst[k] = make_uint2(wv[2 * k], wv[2 * k + 1]);
}

// ---------------------------------------------------------------------------------------------
// bf16 term splitting, two values at a time (packed conversions, f32x2 residuals).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t *>(&h); }

// x = h + m + l exactly (three bf16 terms carry the 24 significand bits of each value).
__device__ __forceinline__ void split3_pair(float2 x, uint32_t &h, uint32_t &m, uint32_t &l)
{
    const float2 neg = make_float2(-1.f, -1.f);
    const __nv_bfloat162 hb = __floats2bfloat162_rn(x.x, x.y);
    const float2 r1 = __ffma2_rn(__bfloat1622float2(hb), neg, x);
    const __nv_bfloat162 mb = __floats2bfloat162_rn(r1.x, r1.y);
    const float2 r2 = __ffma2_rn(__bfloat1622float2(mb), neg, r1);
    h = bf2_bits(hb);
    m = bf2_bits(mb);
    l = bf2_bits(__floats2bfloat162_rn(r2.x, r2.y));
}

__device__ __forceinline__ void split2_pair(float2 x, uint32_t &h, uint32_t &l)
{
    const __nv_bfloat162 hb = __floats2bfloat162_rn(x.x, x.y);
    const float2 r1 = __ffma2_rn(__bfloat1622float2(hb), make_float2(-1.f, -1.f), x);
    h = bf2_bits(hb);
    l = bf2_bits(__floats2bfloat162_rn(r1.x, r1.y));
}

// Eight values -> one 16-byte chunk per term.
__device__ __forceinline__ void store_split3(uint8_t *t0, uint8_t *t1, uint8_t *t2, uint32_t off, const float (&x)[8])
{
    uint32_t a[4], b[4], c[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) split3_pair(make_float2(x[2 * e], x[2 * e + 1]), a[e], b[e], c[e]);
    *reinterpret_cast<uint4 *>(t0 + off) = make_uint4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<uint4 *>(t1 + off) = make_uint4(b[0], b[1], b[2], b[3]);
    *reinterpret_cast<uint4 *>(t2 + off) = make_uint4(c[0], c[1], c[2], c[3]);
}

__device__ __forceinline__ void store_split2(uint8_t *t0, uint8_t *t1, uint32_t off, const float (&x)[8])
{
    uint32_t a[4], b[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) split2_pair(make_float2(x[2 * e], x[2 * e + 1]), a[e], b[e]);
    *reinterpret_cast<uint4 *>(t0 + off) = make_uint4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<uint4 *>(t1 + off) = make_uint4(b[0], b[1], b[2], b[3]);
}

// x = h + m + l with three fp16 terms (33 significand bits: exact for an fp32 value whose terms
// stay normal; the caller keeps |x| below 2^15 so that none overflows).
__device__ __forceinline__ void store_split3_h(uint8_t *t0, uint8_t *t1, uint8_t *t2, uint32_t off,
                                               const float (&x)[8])
{
    uint32_t a[4], b[4], c[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 v = make_float2(x[2 * e], x[2 * e + 1]);
        const __half2 h = __floats2half2_rn(v.x, v.y);
        const float2 hf = __half22float2(h);
        const float2 r1 = make_float2(v.x - hf.x, v.y - hf.y);
        const __half2 m = __floats2half2_rn(r1.x, r1.y);
        const float2 mf = __half22float2(m);
        const __half2 l = __floats2half2_rn(r1.x - mf.x, r1.y - mf.y);
        a[e] = *reinterpret_cast<const uint32_t *>(&h);
        b[e] = *reinterpret_cast<const uint32_t *>(&m);
        c[e] = *reinterpret_cast<const uint32_t *>(&l);
    }
    *reinterpret_cast<uint4 *>(t0 + off) = make_uint4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<uint4 *>(t1 + off) = make_uint4(b[0], b[1], b[2], b[3]);
    *reinterpret_cast<uint4 *>(t2 + off) = make_uint4(c[0], c[1], c[2], c[3]);
}

__device__ __forceinline__ void f16x8_to_f32(uint4 raw, float (&x)[8])
{
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[e]));
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
    }
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 raw, float (&x)[8])
{
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(w[e] << 16);
        x[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}


__device__ __forceinline__ void named_bar(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}


// ---------------------------------------------------------------------------------------------
// T = (I + L)^-1 for a strictly lower triangular 64 x 64 L given transposed (Lt[s][t] = L_ts, row
// stride LDL; its entries on and above the diagonal are zero), by 16 x 16 blocks, run by the 128
// threads of warps W0..W0+3 (named barrier 2) with the work split evenly:
//   1. warp w inverts the diagonal block D_w = (I + L_ww)^-1 by forward substitution;
//   2-4. the blocks at distance 1, 2, 3 below the diagonal, T_ij = -D_i sum_{k=j}^{i-1} L_ik T_kj:
//        three blocks of 16 columns (one per warp), then two blocks as four jobs of 8 columns, then
//        one block as four jobs of 4 columns; a job forms M = sum_k L_ik T_kj, parks it in a
//        scratch block above the diagonal and multiplies by -D_i;
//   5. the six blocks above the diagonal are zeroed.
// In a job, lane (r = lane % 16, h = lane / 16) computes row r of the block, columns h nc/2 ..
// (h + 1) nc/2 - 1 of the job's nc. The result goes to T (row-major, stride LDL).
// ---------------------------------------------------------------------------------------------
// NH consecutive floats from shared memory, 8-byte aligned (16-byte aligned for NH >= 4)
template <int NH>
__device__ __forceinline__ void load_row(const float *src, float (&v)[NH])
{
    if constexpr (NH >= 4) {
#pragma unroll
        for (int e = 0; e < NH; e += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(src + e);
            v[e] = a.x;
            v[e + 1] = a.y;
            v[e + 2] = a.z;
            v[e + 3] = a.w;
        }
    } else {
        const float2 a = *reinterpret_cast<const float2 *>(src);
        v[0] = a.x;
        v[1] = a.y;
    }
}

template <int NC>
__device__ __forceinline__ void inverse_block_job(const float *Lt, float *T, float *scr, int i, int j, int c_lo)
{
    constexpr int NH = NC / 2;
    const int lane = threadIdx.x & 31, r = lane & 15, h = lane >> 4;
    const int col = 16 * j + c_lo + h * NH;  // first absolute column of this lane
    float m[NH];
#pragma unroll
    for (int e = 0; e < NH; ++e) m[e] = 0.f;
    for (int kb = j; kb < i; ++kb) {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float l = Lt[(16 * kb + k) * LDL + 16 * i + r];  // L(16i + r, 16kb + k)
            float tr[NH];
            load_row<NH>(T + (16 * kb + k) * LDL + col, tr);
#pragma unroll
            for (int e = 0; e < NH; ++e) m[e] = fmaf(l, tr[e], m[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < NH; ++e) scr[r * LDL + h * NH + e] = m[e];
    __syncwarp();
    float dr[16];  // row r of D_i
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
        const float4 v = *reinterpret_cast<const float4 *>(T + (16 * i + r) * LDL + 16 * i + 4 * k4);
        dr[4 * k4] = v.x;
        dr[4 * k4 + 1] = v.y;
        dr[4 * k4 + 2] = v.z;
        dr[4 * k4 + 3] = v.w;
    }
    float out[NH];
#pragma unroll
    for (int e = 0; e < NH; ++e) out[e] = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        float mk[NH];
        load_row<NH>(scr + k * LDL + h * NH, mk);
#pragma unroll
        for (int e = 0; e < NH; ++e) out[e] = fmaf(dr[k], mk[e], out[e]);
    }
#pragma unroll
    for (int e = 0; e < NH; ++e) T[(16 * i + r) * LDL + col + e] = -out[e];
    __syncwarp();  // the scratch block is read by every lane before the next job writes it
}

template <int W0>
__device__ __forceinline__ void invert_unit_lower(const float *Lt, float *T)
{
    const int wi = (threadIdx.x >> 5) - W0, lane = threadIdx.x & 31;
    // scratch: a 16 x 16 block above the diagonal, (0, 1 + wi) for warps 0..2 and (1, 3) for warp 3
    float *scr = wi < 3 ? T + 16 * (1 + wi) : T + 16 * LDL + 48;
    if (lane < 16) {
        // 1. D_wi by forward substitution, lane c < 16 keeping all of column c in registers (the
        //    chain of steps needs no data from other lanes; the L rows are the same for every lane)
        const int b = 16 * wi, c = lane;
        float x[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = (e == c) ? 1.f : 0.f;
#pragma unroll
        for (int sidx = 0; sidx < 15; ++sidx) {
            float l[16];  // L(b + e, b + sidx), zero for e <= sidx
            load_row<16>(Lt + (b + sidx) * LDL + b, l);
#pragma unroll
            for (int e = sidx + 1; e < 16; ++e) x[e] = fmaf(l[e], -x[sidx], x[e]);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) T[(b + e) * LDL + b + c] = x[e];
    }
    named_bar(2, 128);
    // 2. distance 1: blocks (1,0), (2,1), (3,2)
    if (wi < 3) inverse_block_job<16>(Lt, T, scr, wi + 1, wi, 0);
    named_bar(2, 128);
    // 3. distance 2: blocks (2,0) and (3,1), 8 columns per warp
    inverse_block_job<8>(Lt, T, scr, 2 + (wi >> 1), wi >> 1, 8 * (wi & 1));
    named_bar(2, 128);
    // 4. distance 3: block (3,0), 4 columns per warp
    inverse_block_job<4>(Lt, T, scr, 3, 0, 4 * wi);
    named_bar(2, 128);
    // 5. zeros above the diagonal: blocks (0,1..3), (1,2..3), (2,3)
    for (int e = threadIdx.x - 32 * W0; e < 6 * 256; e += 128) {
        const int blk = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
        const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
        const int bj = blk < 3 ? 1 + blk : (blk < 5 ? blk - 1 : 3);
        T[(16 * bi + rr) * LDL + 16 * bj + cc] = 0.f;
    }
    named_bar(2, 128);
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, int32_t *status)
{
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity));
    if (!ok && (threadIdx.x & 31) == 0) flag(status, kFlagTimeout);
    return ok;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}


}  // namespace pf
}  // namespace stq
