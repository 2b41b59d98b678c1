// init_d128.cu -- initial quantization (stq_init_state) of 128 x 128 heads with row x column
// scales. A persistent kernel, one 512-thread CTA per SM, streams whole fp32 tiles through a
// two-slot shared-memory ring, one bulk copy per tile. The first pass over a tile (its column
// energies) also moves it into a work tile whose rows are padded to 132 floats, where every later
// pass reads it without bank conflicts; that frees its ring slot for the tile after next, so two
// tiles are in flight while the current one is fitted, coded and stored.
//
// Method: the column scale is the impact-weighted RMS of the column over the key rows, the row
// scale the largest column-normalised magnitude of the row over qmax, the codes S / (r c) rounded
// half to even and clamped to +-qmax ("线性注意力状态量化难题" (aitest123.com/news/n1kj09),
// section 空间维度; "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), section 方法). The
// arithmetic is the plain init kernel's (generic_kernels.cu), in the same fp32 operations per
// element; only the order of the column-energy sums differs.
#include <cstddef>

#include "stq_internal.cuh"

namespace stq {
namespace {

constexpr int NTI = 512;                               // threads per CTA
constexpr int DI = 128;                                // d_k = d_v
constexpr int LDI = DI + 4;                            // padded row: 16-byte aligned, one bank quad apart
constexpr int NSI = 2;                                 // ring slots
constexpr uint32_t TILE_BYTES = DI * DI * 4;           // one fp32 tile of S0
constexpr uint32_t SLOT_BYTES = TILE_BYTES + DI * 4;   // + the head's impact weights
constexpr uint32_t TX_BYTES = SLOT_BYTES;              // bytes a slot's copies complete
constexpr uint32_t WORK_BYTES = DI * LDI * 4;          // the padded work tile

// The float arrays are read as float4: each starts 16-byte aligned.
struct InitFixed {
    alignas(16) float part[16 * DI];  // partial column energies (16 row classes)
    alignas(16) float cs[DI];
    alignas(16) float ics[DI];
    alignas(16) float rs[DI];
    alignas(16) float irs[DI];
    unsigned long long bars[NSI];
    unsigned long long gblock[NSI];  // head block the slot's tile is written to (0: skipped tile)
    int bits[NSI];
    float wsum;
    int slow;  // a reciprocal scale of the tile is not finite: code it element by element
};
static_assert(offsetof(InitFixed, ics) % 16 == 0 && offsetof(InitFixed, cs) % 16 == 0 &&
                  offsetof(InitFixed, part) % 16 == 0 && offsetof(InitFixed, bars) % 8 == 0,
              "float4 reads of ics and 8-byte mbarriers need these alignments");
constexpr uint32_t RING_OFF = (uint32_t)(sizeof(InitFixed) + 127) / 128 * 128;
constexpr uint32_t WORK_OFF = RING_OFF + NSI * SLOT_BYTES;
constexpr uint32_t SMEM_INIT = WORK_OFF + WORK_BYTES;
static_assert(SMEM_INIT <= 227 * 1024, "ring and work tile fit one CTA's shared memory");
static_assert(SLOT_BYTES % 16 == 0 && TILE_BYTES % 16 == 0 && (LDI * 4) % 16 == 0 && WORK_OFF % 16 == 0,
              "bulk-copy destinations and float4 rows stay 16-byte aligned");

// The CTA's k-th tile is global tile blockIdx.x + k * gridDim.x, requests fastest.
struct TileSrc {
    TileEntry e;
    int b, slot;
};
__device__ __forceinline__ TileSrc tile_src(const TileParams &p, int k)
{
    TileSrc t;
    const int tile = (int)blockIdx.x + k * (int)gridDim.x;
    const int pos = tile / p.B;
    t.b = tile - pos * p.B;
    t.e = p.table[pos];
    t.slot = p.slots[t.b];
    return t;
}

// Thread 0: stream the CTA's k-th tile (read by tile_src) into ring slot k % NSI: the tile and
// the head's weights, two bulk copies. A request whose pool slot is out of range is flagged and
// its slot completed without copies.
__device__ __forceinline__ void issue_tile(const TileParams &p, InitFixed &sm, uint8_t *smem, int k, int my_count,
                                           const TileSrc &t)
{
    if (k >= my_count) return;
    const TileEntry e = t.e;
    const int b = t.b, slot = t.slot;
    const int si = k % NSI, h = entry_head(e);
    const uint32_t bar = smem_u32(&sm.bars[si]);
    sm.bits[si] = entry_bits(e);
    if (slot < 0 || slot >= p.pool_slots) {
        flag(p.status, kFlagBounds);
        sm.gblock[si] = 0ull;
        mbar_arrive(bar);
        return;
    }
    sm.gblock[si] = reinterpret_cast<unsigned long long>(p.pool + (uint64_t)slot * p.req_bytes + e.off);
    mbar_arrive_expect_tx(bar, TX_BYTES);
    const float *src = p.S0 + ((uint64_t)b * (uint64_t)p.head_count + (uint64_t)h) * (DI * DI);
    const uint32_t dst = smem_u32(smem + RING_OFF + (uint32_t)si * SLOT_BYTES);
    bulk_g2s(dst, src, TILE_BYTES, bar);
    bulk_g2s(dst + TILE_BYTES, p.w + (uint64_t)h * DI, DI * 4, bar);
}

// Pack 16 offset-binary codes (u < 2^bits) into 2 * bits bytes at dst: code k at bits
// bits * k .. of a little-endian bitstream.
template <int BITS>
__device__ __forceinline__ void store_group(uint8_t *dst, const uint32_t (&u)[16])
{
    if constexpr (BITS == 4) {
        uint2 w;
        w.x = u[0] | (u[1] << 4) | (u[2] << 8) | (u[3] << 12) | (u[4] << 16) | (u[5] << 20) | (u[6] << 24) |
              (u[7] << 28);
        w.y = u[8] | (u[9] << 4) | (u[10] << 8) | (u[11] << 12) | (u[12] << 16) | (u[13] << 20) | (u[14] << 24) |
              (u[15] << 28);
        *reinterpret_cast<uint2 *>(dst) = w;
    } else if constexpr (BITS == 6) {
        uint32_t *d32 = reinterpret_cast<uint32_t *>(dst);
        d32[0] = u[0] | (u[1] << 6) | (u[2] << 12) | (u[3] << 18) | (u[4] << 24) | (u[5] << 30);
        d32[1] = (u[5] >> 2) | (u[6] << 4) | (u[7] << 10) | (u[8] << 16) | (u[9] << 22) | (u[10] << 28);
        d32[2] = (u[10] >> 4) | (u[11] << 2) | (u[12] << 8) | (u[13] << 14) | (u[14] << 20) | (u[15] << 26);
    } else {
        uint4 w;
        w.x = u[0] | (u[1] << 8) | (u[2] << 16) | (u[3] << 24);
        w.y = u[4] | (u[5] << 8) | (u[6] << 16) | (u[7] << 24);
        w.z = u[8] | (u[9] << 8) | (u[10] << 16) | (u[11] << 24);
        w.w = u[12] | (u[13] << 8) | (u[14] << 16) | (u[15] << 24);
        *reinterpret_cast<uint4 *>(dst) = w;
    }
}

// Phase 1 of a tile: move it from its ring slot (raw: 128 x 128 floats, then the head's
// weights) into the padded work tile S, and form the partial column energies and the weight sum.
// The caller's barrier after it frees the ring slot.
__device__ __forceinline__ void energies(InitFixed &sm, const float *raw, float *S)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *wv = raw + DI * DI;
    if (tid == 0) sm.slow = 0;
    // columns 4 (tid % 32) .. +3 over rows 8 (tid / 32) .. +7, as w_i x x in packed pairs; the 16
    // partials of a column are added after the barrier
    {
        const int jq = tid & 31, rb = tid >> 5;
        const float4 wa = *reinterpret_cast<const float4 *>(wv + 8 * rb);
        const float4 wb = *reinterpret_cast<const float4 *>(wv + 8 * rb + 4);
        const float wr[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
        float2 e01 = make_float2(0.f, 0.f), e23 = make_float2(0.f, 0.f);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int i = 8 * rb + r;
            const float4 x = *reinterpret_cast<const float4 *>(raw + i * DI + 4 * jq);
            *reinterpret_cast<float4 *>(S + i * LDI + 4 * jq) = x;
            const float2 ww = make_float2(wr[r], wr[r]);
            const float2 x01 = make_float2(x.x, x.y), x23 = make_float2(x.z, x.w);
            e01 = __ffma2_rn(__fmul2_rn(ww, x01), x01, e01);
            e23 = __ffma2_rn(__fmul2_rn(ww, x23), x23, e23);
        }
        *reinterpret_cast<float4 *>(sm.part + rb * DI + 4 * jq) = make_float4(e01.x, e01.y, e23.x, e23.y);
        if (warp == 0) {
            float W = (wv[lane] + wv[lane + 32]) + (wv[lane + 64] + wv[lane + 96]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
            if (lane == 0) sm.wsum = W;
        }
    }
}

// The rest of a tile (in the padded work tile S, after the energies and a barrier): scales,
// codes and stores. Returns whether a stored scale is non-finite (or a row scale zero).
template <int BITS, int SB16>
__device__ __forceinline__ bool quantize_tile(InitFixed &sm, const float *S, uint8_t *gblock)
{
    constexpr int bits = BITS, sb16 = SB16;
    const int tid = threadIdx.x;
    constexpr float qmax = (float)((1 << (BITS - 1)) - 1);
    bool nf = false;  // a non-finite stored scale (or a zero row scale) met by this thread
    if (tid < DI) {
        float a[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) a[r] = sm.part[r * DI + tid] + sm.part[(r + 8) * DI + tid];
        const float E = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
        float c = sqrtf(E / sm.wsum);
        if (c == 0.f) c = 1.f;
        c = round_scale(c, sb16);  // the codes follow the stored value
        const float ic = __frcp_rn(c);
        sm.cs[tid] = c;
        sm.ics[tid] = ic;
        nf = !isfinite(c);
        if (!isfinite(ic)) atomicOr(&sm.slow, 1);
    }
    __syncthreads();
    // ---- row maxima of |S_ij / c_j|: row i = tid / 4, columns 32 (tid % 4) .. +31 as float4,
    // taken in a rotated order so that the eight lanes of a load phase hit eight bank quads
    {
        const int i = tid >> 2, q = tid & 3;
        const float4 *row = reinterpret_cast<const float4 *>(S + i * LDI + 32 * q);
        const float4 *ic = reinterpret_cast<const float4 *>(sm.ics + 32 * q);
        float m0 = 0.f, m1 = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int kk = (k + 2 * q) & 7;
            const float4 x = row[kk], c = ic[kk];
            const float2 t01 = __fmul2_rn(make_float2(x.x, x.y), make_float2(c.x, c.y));
            const float2 t23 = __fmul2_rn(make_float2(x.z, x.w), make_float2(c.z, c.w));
            m0 = fmaxf(m0, fmaxf(fabsf(t01.x), fabsf(t01.y)));
            m1 = fmaxf(m1, fmaxf(fabsf(t23.x), fabsf(t23.y)));
        }
        float m = fmaxf(m0, m1);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        if (q == 0) {
            float r = m / qmax;
            if (r == 0.f) r = 1.f;
            r = round_scale(r, sb16);
            const float ir = __frcp_rn(r);
            sm.rs[i] = r;
            sm.irs[i] = ir;
            nf |= !isfinite(r) || r == 0.f;
            if (!isfinite(ir)) atomicOr(&sm.slow, 1);
        }
    }
    const bool bad = __syncthreads_or(nf);
    const bool fast = !bad && sm.slow == 0;
    // ---- codes: 16 consecutive elements of row i = g % 128 (columns 16 (g / 128) ..) per group g;
    // x = (S * (1/c)) * (1/r) with the correctly rounded reciprocals, rounded half to even
    constexpr int off = 1 << (BITS - 1);
    constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll 1
    for (int g = tid; g < DI * DI / 16; g += NTI) {
        const int i = g & (DI - 1), cg = g >> 7;
        const float4 *row = reinterpret_cast<const float4 *>(S + i * LDI + 16 * cg);
        const float4 *ic = reinterpret_cast<const float4 *>(sm.ics + 16 * cg);
        const float ir = sm.irs[i];
        uint32_t u[16];
        if (fast) {
            // finite scales and reciprocals: x is finite and, with fp32 scales, |x| <= qmax (1 + 3 * 2^-24), so
            // adding 2^23 + 2^(b-1) rounds x half to even and leaves the offset-binary code in the
            // low bits; bf16 scales (a row scale up to 2^-8 below m / qmax) clamp first
            const float2 ir2 = make_float2(ir, ir);
            const float2 rnd = make_float2(8388608.f + (float)off, 8388608.f + (float)off);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 x = row[k], c = ic[k];
                float2 y01 = __fmul2_rn(__fmul2_rn(make_float2(x.x, x.y), make_float2(c.x, c.y)), ir2);
                float2 y23 = __fmul2_rn(__fmul2_rn(make_float2(x.z, x.w), make_float2(c.z, c.w)), ir2);
                if constexpr (SB16 != 0) {
                    y01 = make_float2(fminf(fmaxf(y01.x, -qmax), qmax), fminf(fmaxf(y01.y, -qmax), qmax));
                    y23 = make_float2(fminf(fmaxf(y23.x, -qmax), qmax), fminf(fmaxf(y23.y, -qmax), qmax));
                }
                const float2 f01 = __fadd2_rn(y01, rnd), f23 = __fadd2_rn(y23, rnd);
                u[4 * k] = __float_as_uint(f01.x) & mask;
                u[4 * k + 1] = __float_as_uint(f01.y) & mask;
                u[4 * k + 2] = __float_as_uint(f23.x) & mask;
                u[4 * k + 3] = __float_as_uint(f23.y) & mask;
            }
        } else {
            // a non-finite scale or reciprocal: the plain kernel's per-element form (code 0 where
            // x is not finite)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 x = row[k], c = ic[k];
                const float xs[4] = {x.x * c.x, x.y * c.y, x.z * c.z, x.w * c.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float xr = xs[e] * ir;
                    const float qv = isfinite(xr) ? fminf(fmaxf(rintf(xr), -qmax), qmax) : 0.f;
                    u[4 * k + e] = (uint32_t)((int)qv + off);
                }
            }
        }
        // the group's 16 codes are 2 * bits bytes at byte 2 * bits * (8 i + cg) of the bitstream
        store_group<BITS>(gblock + 2 * BITS * (8 * i + cg), u);
    }
    if (tid < DI) {
        uint8_t *sg = gblock + scale_offset(bits, DI, DI);
        store_scale(sg, tid, sm.rs[tid], sb16);
        store_scale(sg, DI + tid, sm.cs[tid], sb16);
    }
    return bad;
}

__global__ void __launch_bounds__(NTI, 1) init_d128_kernel(const __grid_constant__ TileParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    InitFixed &sm = *reinterpret_cast<InitFixed *>(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int G = (int)gridDim.x;
    const int my_count = (p.ntiles - (int)blockIdx.x + G - 1) / G;
    if (tid == 0) {
        for (int s = 0; s < NSI; ++s) mbar_init(smem_u32(&sm.bars[s]), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0)
        for (int k = 0; k < NSI && k < my_count; ++k) issue_tile(p, sm, smem, k, my_count, tile_src(p, k));
    float *work = reinterpret_cast<float *>(smem + WORK_OFF);
    int k = 0;
    bool failed = false;
    for (; k < my_count; ++k) {
        const int si = k % NSI;
        // thread 0 reads where the tile after next comes from now; it is issued after the repack
        TileSrc next = {};
        if (tid == 0 && k + NSI < my_count) next = tile_src(p, k + NSI);
        const bool got = mbar_wait_bounded(smem_u32(&sm.bars[si]), (uint32_t)(k / NSI) & 1u);
        if (__syncthreads_or(!got)) {
            failed = true;
            break;
        }
        const unsigned long long gb = sm.gblock[si];
        const int bits = sm.bits[si];
        if (gb != 0ull) energies(sm, reinterpret_cast<const float *>(smem + RING_OFF + (uint32_t)si * SLOT_BYTES), work);
        __syncthreads();  // the ring slot is free: it takes the tile after next
        if (tid == 0) issue_tile(p, sm, smem, k + NSI, my_count, next);
        bool bad = false;
        if (gb != 0ull) {
            uint8_t *g = reinterpret_cast<uint8_t *>(gb);
            switch (2 * bits + (p.scale_bf16 ? 1 : 0)) {
            case 8: bad = quantize_tile<4, 0>(sm, work, g); break;
            case 9: bad = quantize_tile<4, 1>(sm, work, g); break;
            case 12: bad = quantize_tile<6, 0>(sm, work, g); break;
            case 13: bad = quantize_tile<6, 1>(sm, work, g); break;
            case 16: bad = quantize_tile<8, 0>(sm, work, g); break;
            default: bad = quantize_tile<8, 1>(sm, work, g); break;
            }
        }
        if (bad && tid == 0) flag(p.status, kFlagNonfinite);
        __syncthreads();  // every thread is done with the work tile and the per-tile scratch
    }
    if (failed && tid == 0) {
        flag(p.status, kFlagTimeout);
        // let the copies still in flight (tiles k .. k + NSI - 1) land before shared memory is released
        for (int m = k; m < k + NSI && m < my_count; ++m)
            mbar_wait_bounded(smem_u32(&sm.bars[m % NSI]), (uint32_t)(m / NSI) & 1u);
    }
}

}  // namespace

// Tiles of p.table (128 x 128 row x column heads, no refinement rounds), S0 and w 16-byte
// aligned. One persistent CTA per SM.
cudaError_t launch_init_d128(const TileParams &p, cudaStream_t s)
{
    int dev = 0, sms = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(init_d128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_INIT);
    if (err != cudaSuccess) return err;
    const int grid = p.ntiles < sms ? p.ntiles : sms;
    if (grid <= 0) return cudaSuccess;
    init_d128_kernel<<<grid, NTI, SMEM_INIT, s>>>(p);
    return cudaGetLastError();
}

}  // namespace stq
