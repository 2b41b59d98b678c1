// init_d128.cu -- initial quantization (stq_init_state) of 128 x 128 heads with row x column
// scales. A persistent kernel, one CTA per SM of two independent groups of 256 threads. Each group
// fits, codes and stores one tile at a time (every other tile of the CTA), synchronised by its own
// named barrier, so that one group's barrier waits overlap the other group's work. Whole fp32
// tiles stream through a three-slot shared-memory ring: the two groups' tiles and the next one in
// flight. A tile arrives by four TMA tensor copies (32-column quarters, 128-byte swizzle: the
// 16-byte chunk c of row i of a quarter sits at chunk c ^ (i % 8)) and is read in place: each pass
// maps its lanes so that the 8 lanes of a 16-byte load phase of the tile hit 8 bank quads, with
// no padded copy.
//
// Method: the column scale is the impact-weighted RMS of the column over the key rows, the row
// scale the largest column-normalised magnitude of the row over qmax, the codes S / (r c) rounded
// half to even and clamped to +-qmax ("线性注意力状态量化难题" (aitest123.com/news/n1kj09),
// section 空间维度; "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), section 方法). The
// arithmetic is the plain init kernel's (generic_kernels.cu), in the same fp32 operations per
// element; only the order of the column-energy sums differs.
#include <cstddef>

#include <cuda.h>

#include "stq_internal.cuh"

namespace stq {
namespace {

constexpr int NTI = 512;                               // threads per CTA
constexpr int NTG = 256;                               // threads per group
constexpr int DI = 128;                                // d_k = d_v
constexpr int NSI = 3;                                 // ring slots
constexpr uint32_t QUARTER_BYTES = DI * 32 * 4;        // 32 columns of the 128 rows
constexpr uint32_t TILE_BYTES = DI * DI * 4;           // one fp32 tile of S0 (four quarters)
constexpr uint32_t TX_BYTES = TILE_BYTES + DI * 4;     // + the head's impact weights
constexpr uint32_t SLOT_BYTES = (TX_BYTES + 1023) / 1024 * 1024;  // quarters stay 1024-byte aligned

// One group's per-tile scratch. The float arrays are read as float4: each starts 16-byte aligned.
struct GroupScratch {
    alignas(16) float part[8 * DI];  // partial column energies (8 row classes)
    alignas(16) float cs[DI];
    alignas(16) float ics[DI];
    alignas(16) float rs[DI];
    alignas(16) float irs[DI];
    float wsum;
    int slow;  // a reciprocal scale of the tile is not finite: code it element by element
};

struct InitFixed {
    GroupScratch g[2];
    unsigned long long bars[NSI];
    unsigned long long gblock[NSI];  // head block the slot's tile is written to (0: skipped tile)
    int bits[NSI];
    int last[NSI];                   // the last tile issued into the slot (-1: none)
    int fail;                        // a wait timed out: both groups stop taking tiles
};
static_assert(offsetof(InitFixed, g) % 16 == 0 && sizeof(GroupScratch) % 16 == 0 &&
                  offsetof(GroupScratch, cs) % 16 == 0 && offsetof(GroupScratch, ics) % 16 == 0 &&
                  offsetof(InitFixed, bars) % 8 == 0,
              "float4 reads of the scratch arrays and 8-byte mbarriers need these alignments");
constexpr uint32_t RING_OFF = (uint32_t)(sizeof(InitFixed) + 1023) / 1024 * 1024;
constexpr uint32_t SMEM_INIT = RING_OFF + NSI * SLOT_BYTES;
static_assert(SMEM_INIT <= 227 * 1024, "ring and scratch fit one CTA's shared memory");
static_assert(RING_OFF % 1024 == 0 && SLOT_BYTES % 1024 == 0 && QUARTER_BYTES % 1024 == 0,
              "128-byte-swizzled TMA destinations start on 1024-byte boundaries");

// Byte offset of the float4 holding columns 4c .. 4c + 3 of quarter qt, row i, in a ring slot.
__device__ __forceinline__ uint32_t chunk_off(int qt, int i, int c)
{
    return (uint32_t)qt * QUARTER_BYTES + (uint32_t)i * 128u + ((uint32_t)(c ^ (i & 7)) << 4);
}

__device__ __forceinline__ void group_sync(int g)
{
    asm volatile("bar.sync %0, %1;" ::"r"(g + 1), "n"(NTG) : "memory");
}

// Named-barrier OR over the group's threads.
__device__ __forceinline__ bool group_or(int g, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(g + 1), "n"(NTG)
        : "memory");
    return r != 0;
}

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

// Stream the CTA's k-th tile (read by tile_src) into ring slot k % NSI: four 32-column quarters by
// TMA tensor copy and the head's weights by bulk copy. A request whose pool slot is out of range
// is flagged and its slot completed without copies.
__device__ __forceinline__ void issue_tile(const TileParams &p, const CUtensorMap *map, InitFixed &sm, uint8_t *smem,
                                           int k, int my_count, const TileSrc &t)
{
    if (k >= my_count) return;
    const TileEntry e = t.e;
    const int b = t.b, slot = t.slot;
    const int si = k % NSI, h = entry_head(e);
    const uint32_t bar = smem_u32(&sm.bars[si]);
    sm.bits[si] = entry_bits(e);
    sm.last[si] = k;
    if (slot < 0 || slot >= p.pool_slots) {
        flag(p.status, kFlagBounds);
        sm.gblock[si] = 0ull;
        mbar_arrive(bar);
        return;
    }
    sm.gblock[si] = reinterpret_cast<unsigned long long>(p.pool + (uint64_t)slot * p.req_bytes + e.off);
    mbar_arrive_expect_tx(bar, TX_BYTES);
    const uint32_t dst = smem_u32(smem + RING_OFF + (uint32_t)si * SLOT_BYTES);
    const int y = (b * p.head_count + h) * DI;  // the tile's first row in S0 seen as rows of 128 floats
#pragma unroll
    for (int qt = 0; qt < 4; ++qt)
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
            "[%4];" ::"r"(dst + (uint32_t)qt * QUARTER_BYTES),
            "l"(reinterpret_cast<uint64_t>(map)), "r"(32 * qt), "r"(y), "r"(bar)
            : "memory");
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

// Phase 1 of a tile (in its ring slot `T`, the head's weights after the four quarters): the partial
// column energies and the weight sum. Thread tg: columns 4 (tg % 32) .. +3 over rows 16 (tg / 32)
// .. +15; a warp reads whole rows. The 8 partials of a column are added after the group barrier.
__device__ __forceinline__ void energies(GroupScratch &gs, const uint8_t *T, int tg)
{
    const float *wv = reinterpret_cast<const float *>(T + TILE_BYTES);
    if (tg == 0) gs.slow = 0;
    const int jq = tg & 31, rb = tg >> 5, qt = jq >> 3, c = jq & 7;
    float2 e01 = make_float2(0.f, 0.f), e23 = make_float2(0.f, 0.f);
#pragma unroll
    for (int r4 = 0; r4 < 4; ++r4) {
        const float4 wq = *reinterpret_cast<const float4 *>(wv + 16 * rb + 4 * r4);
        const float wr[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int i = 16 * rb + 4 * r4 + r;
            const float4 x = *reinterpret_cast<const float4 *>(T + chunk_off(qt, i, c));
            const float2 ww = make_float2(wr[r], wr[r]);
            const float2 x01 = make_float2(x.x, x.y), x23 = make_float2(x.z, x.w);
            e01 = __ffma2_rn(__fmul2_rn(ww, x01), x01, e01);
            e23 = __ffma2_rn(__fmul2_rn(ww, x23), x23, e23);
        }
    }
    *reinterpret_cast<float4 *>(gs.part + rb * DI + 4 * jq) = make_float4(e01.x, e01.y, e23.x, e23.y);
    if (tg < 32) {
        float W = (wv[tg] + wv[tg + 32]) + (wv[tg + 64] + wv[tg + 96]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
        if (tg == 0) gs.wsum = W;
    }
}

// The rest of a tile (in its ring slot T, after the energies and a group barrier): scales, codes
// and stores. Returns whether a stored scale is non-finite (or a row scale zero).
template <int BITS, int SB16>
__device__ __forceinline__ bool quantize_tile(GroupScratch &gs, const uint8_t *T, uint8_t *gblock, int g, int tg)
{
    constexpr int bits = BITS, sb16 = SB16;
    constexpr float qmax = (float)((1 << (BITS - 1)) - 1);
    bool nf = false;  // a non-finite stored scale (or a zero row scale) met by this thread
    if (tg < DI) {
        float a[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) a[r] = gs.part[r * DI + tg];
        const float E = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
        float c = sqrtf(E / gs.wsum);
        if (c == 0.f) c = 1.f;
        c = round_scale(c, sb16);  // the codes follow the stored value
        const float ic = __frcp_rn(c);
        gs.cs[tg] = c;
        gs.ics[tg] = ic;
        nf = !isfinite(c);
        if (!isfinite(ic)) atomicOr(&gs.slow, 1);
    }
    group_sync(g);
    // ---- row maxima of |S_ij / c_j|: row i = tg / 2, quarters 2q and 2q + 1 (q = tg % 2); lanes
    // with q = 1 take the chunks in an order shifted by 4, so that the 8 lanes of a load phase (4
    // rows x 2 halves) hit 8 bank quads
    {
        const int i = tg >> 1, q = tg & 1;
        float m0 = 0.f, m1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int qt = 2 * q + (k >> 3), c = (k + 4 * q) & 7;
            const float4 x = *reinterpret_cast<const float4 *>(T + chunk_off(qt, i, c));
            const float4 cc = *reinterpret_cast<const float4 *>(gs.ics + 32 * qt + 4 * c);
            const float2 t01 = __fmul2_rn(make_float2(x.x, x.y), make_float2(cc.x, cc.y));
            const float2 t23 = __fmul2_rn(make_float2(x.z, x.w), make_float2(cc.z, cc.w));
            m0 = fmaxf(m0, fmaxf(fabsf(t01.x), fabsf(t01.y)));
            m1 = fmaxf(m1, fmaxf(fabsf(t23.x), fabsf(t23.y)));
        }
        float m = fmaxf(m0, m1);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        if (q == 0) {
            float r = m / qmax;
            if (r == 0.f) r = 1.f;
            r = round_scale(r, sb16);
            const float ir = __frcp_rn(r);
            gs.rs[i] = r;
            gs.irs[i] = ir;
            nf |= !isfinite(r) || r == 0.f;
            if (!isfinite(ir)) atomicOr(&gs.slow, 1);
        }
    }
    const bool bad = group_or(g, nf);
    const bool fast = !bad && gs.slow == 0;
    // ---- codes: per pass, 16 consecutive elements of row i = tg / 2, columns 16 cg .. with
    // cg = 2 pass + tg % 2 (quarter `pass`); x = (S * (1/c)) * (1/r) with the correctly rounded
    // reciprocals, rounded half to even. The 8 lanes of a load phase (4 rows x 2 column groups)
    // hit 8 bank quads in the swizzled quarter.
    constexpr int off = 1 << (BITS - 1);
    constexpr uint32_t mask = (1u << BITS) - 1u;
    const int i = tg >> 1;
    const float ir = gs.irs[i];
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int cg = 2 * pass + (tg & 1);
        const float4 *ic = reinterpret_cast<const float4 *>(gs.ics + 16 * cg);
        uint32_t u[16];
        if (fast) {
            // finite scales and reciprocals: x is finite and, with fp32 scales, |x| <= qmax (1 + 3 * 2^-24), so
            // adding 2^23 + 2^(b-1) rounds x half to even and leaves the offset-binary code in the
            // low bits; bf16 scales (a row scale up to 2^-8 below m / qmax) clamp first
            const float2 ir2 = make_float2(ir, ir);
            const float2 rnd = make_float2(8388608.f + (float)off, 8388608.f + (float)off);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 x = *reinterpret_cast<const float4 *>(T + chunk_off(pass, i, 4 * (tg & 1) + k));
                const float4 c = ic[k];
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
                const float4 x = *reinterpret_cast<const float4 *>(T + chunk_off(pass, i, 4 * (tg & 1) + k));
                const float4 c = ic[k];
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
    if (tg < DI) {
        uint8_t *sg = gblock + scale_offset(bits, DI, DI);
        store_scale(sg, tg, gs.rs[tg], sb16);
        store_scale(sg, DI + tg, gs.cs[tg], sb16);
    }
    return bad;
}

__global__ void __launch_bounds__(NTI, 1)
    init_d128_kernel(const __grid_constant__ TileParams p, const __grid_constant__ CUtensorMap map)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    InitFixed &sm = *reinterpret_cast<InitFixed *>(smem);
    const int tid = threadIdx.x, g = tid / NTG, tg = tid % NTG;
    const int G = (int)gridDim.x;
    const int my_count = (p.ntiles - (int)blockIdx.x + G - 1) / G;
    GroupScratch &gs = sm.g[g];
    if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled copies need 1024-byte aligned slots
        if (tid == 0) flag(p.status, kFlagBounds);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < NSI; ++s) {
            mbar_init(smem_u32(&sm.bars[s]), 1);
            sm.last[s] = -1;
        }
        sm.fail = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map)) : "memory");
        for (int k = 0; k < NSI && k < my_count; ++k) issue_tile(p, &map, sm, smem, k, my_count, tile_src(p, k));
    }
    __syncthreads();
    // group g takes the CTA's tiles k = g, g + 2, ...; the group that finishes tile k issues tile
    // k + NSI into the slot it frees (the other group will take it)
    for (int k = g; k < my_count; k += 2) {
        const int si = k % NSI;
        // the group's thread 0 reads where tile k + NSI comes from now; it is issued at the end
        TileSrc next = {};
        if (tg == 0 && k + NSI < my_count) next = tile_src(p, k + NSI);
        // Tile k is in flight once the group that took tile k - NSI has issued it (tiles below NSI:
        // before the loop). Only then is the slot's barrier in tile k's phase: a wait on its parity
        // before that would see the phase of tile k - 2 NSI as complete.
        bool got = true;
        if (tg == 0 && k >= NSI) {
            const long long start = clock64();
            while (*reinterpret_cast<volatile int *>(&sm.last[si]) != k)
                if (clock64() - start > kWaitTimeoutCycles) {
                    got = false;
                    break;
                }
        }
        if (!got) atomicOr(&sm.fail, 1);
        if (group_or(g, !got || *reinterpret_cast<volatile int *>(&sm.fail) != 0)) break;
        got = mbar_wait_bounded(smem_u32(&sm.bars[si]), (uint32_t)(k / NSI) & 1u);
        if (!got) atomicOr(&sm.fail, 1);
        if (group_or(g, !got)) break;
        const unsigned long long gb = sm.gblock[si];
        const int bits = sm.bits[si];
        const uint8_t *T = smem + RING_OFF + (uint32_t)si * SLOT_BYTES;
        bool bad = false;
        if (gb != 0ull) {
            energies(gs, T, tg);
            group_sync(g);
            uint8_t *gbp = reinterpret_cast<uint8_t *>(gb);
            switch (2 * bits + (p.scale_bf16 ? 1 : 0)) {
            case 8: bad = quantize_tile<4, 0>(gs, T, gbp, g, tg); break;
            case 9: bad = quantize_tile<4, 1>(gs, T, gbp, g, tg); break;
            case 12: bad = quantize_tile<6, 0>(gs, T, gbp, g, tg); break;
            case 13: bad = quantize_tile<6, 1>(gs, T, gbp, g, tg); break;
            case 16: bad = quantize_tile<8, 0>(gs, T, gbp, g, tg); break;
            default: bad = quantize_tile<8, 1>(gs, T, gbp, g, tg); break;
            }
        }
        if (bad && tg == 0) flag(p.status, kFlagNonfinite);
        group_sync(g);  // every thread of the group is done with the slot and the group's scratch
        if (tg == 0) issue_tile(p, &map, sm, smem, k + NSI, my_count, next);
    }
    __syncthreads();
    if (tid == 0) {
        if (sm.fail) flag(p.status, kFlagTimeout);
        // let every copy issued into a slot land before shared memory is released (an immediate
        // return for copies already consumed)
        for (int s = 0; s < NSI; ++s)
            if (sm.last[s] >= 0) mbar_wait_bounded(smem_u32(&sm.bars[s]), (uint32_t)(sm.last[s] / NSI) & 1u);
    }
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_tiled()
{
    // a function-local static: initialised once, safely across host threads
    static const EncodeTiled fn = []() -> EncodeTiled {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiled>(f);
        return nullptr;
    }();
    return fn;
}

}  // namespace

// Tiles of p.table (128 x 128 row x column heads, no refinement rounds), S0 [B][head_count][128][128]
// and w 16-byte aligned. One persistent CTA per SM.
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
    // S0 as rows of 128 floats, copied as boxes of 32 columns x 128 rows, 128-byte swizzle. Where
    // no tensor map can be made (no driver entry point, or more rows than 32-bit TMA coordinates
    // reach) the plain kernel takes the tiles.
    const EncodeTiled enc = encode_tiled();
    const uint64_t rows = (uint64_t)p.B * (uint64_t)p.head_count * DI;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)DI, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)DI * 4};
    const cuuint32_t box[2] = {32, (cuuint32_t)DI};
    const cuuint32_t estr[2] = {1, 1};
    if (!enc || rows > 0x7fffffffull ||
        enc(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(p.S0), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return launch_init_generic(p, s);
    init_d128_kernel<<<grid, NTI, SMEM_INIT, s>>>(p, map);
    return cudaGetLastError();
}

}  // namespace stq
