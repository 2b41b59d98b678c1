// decode_d128.cu -- the fused decode step for 128 x 128 head states: read the packed state once,
// dequantize, apply the gated delta rule, read out, refit the column and row scales, requantize
// and write the state back in place, one CTA per (request, head) tile at a time.
//
// Method (formulas in include/stq.h): every decode step reads the previous state, updates it,
// requantizes and stores it ("线性注意力状态量化难题" (aitest123.com/news/n1kj09), section
// 直接量化为什么会翻车); the scales are one per key row and one per value column, the column scale
// an impact-weighted fit (same page, section 空间维度; "K1 論文詳解"
// (k1-news.pages.dev/paper/2026-10-09), section 方法); widths per head from {4, 6, 8} and FP16
// pivot heads (k1 page, section 方法); quantization and state update fused to cut memory traffic
// (k1 page, section 方法; aitest123 page, section 工程落地).
//
// Design (B200):
//  * Persistent CTAs of 256 threads, two per SM, walking tiles round-robin over a list sorted by
//    block size (FP16 pivots first, then 8-, 6-, 4-bit), so all CTAs see the same width mix.
//  * A thread-0 producer streams each upcoming tile (packed codes + scales, and the q, k, v, w
//    rows) into a byte-addressed shared-memory ring with cp.async.bulk, one mbarrier per tile in
//    flight; every wait is bounded and reports STQ_ERR_TIMEOUT instead of hanging.
//  * Each thread owns an 8 x 8 sub-block (rows 16m + 2*warp + half, columns 8*lane16 .. +7) in
//    64 fp32 registers, so the state is read from HBM once and written once per step.
//  * The algebra runs in column-normalised coordinates: with y_ij = sqrt(w_i) S'_ij / c_j,
//      y_ij = rho_i Q_ij + kappa_i g_j   (rho = alpha sqrt(w) r, kappa = sqrt(w) k, g = h / c,
//                                         h = beta (v - alpha u))
//    so the update, the column energy, the row maximum and the rounding are 1-2 packed f32x2
//    operations per element each. Codes are unpacked with a LOP3/PRMT into the mantissa of
//    2^23 (exact; a per-column power-of-two factor sigma is folded back per column) and rounded
//    back with one FFMA against 2^23 + 2^(b-1), which rounds half to even for free.
//  * Column sums cross warps through shared memory; row maxima stay inside a warp.
#include "stq_internal.cuh"

namespace stq {
namespace {

constexpr int D = 128;
constexpr int NT = 256;
constexpr int NBAR = 8;                // tiles in flight per CTA (mbarriers)
constexpr uint32_t RING = 72 * 1024;   // bytes of the staging ring per CTA
constexpr int MAXB = 1024;             // requests per launch whose slots are cached in smem
constexpr uint32_t MAGIC = 0x4B000000u;  // bit pattern of 2^23

struct __align__(16) SmemD128 {
    uint8_t ring[RING];
    float red[16 * 2 * D];   // column partials per (warp, half); later the row-max partials
    float4 rowA[2][D];       // per tile parity: (k~, q~, rho, kappa)
    float2 rowB[2][D];       // per tile parity: (sqrt w, mu)
    float colG1[D];
    float colG2[D];
    float colH[D];           // rank-1 part of the readout
    float colB[D];           // c_j / (sigma_j c'_j)
    float2 rowS[D];          // (s_i, s_i), s_i = 1 / (sqrt(w_i) r'_i)
    float rsum[2][4][4];     // per parity, per precompute warp: sum w, q.k, q.(alpha*k)
    float scal[2][4];        // per parity: beta, alpha, skip
    int32_t slots[MAXB];
    uint32_t tpos[NBAR];     // ring position / wrap count of each tile in flight (producer only)
    uint32_t twrap[NBAR];
    unsigned long long bars[NBAR];
};

// ---------------------------------------------------------------------------------------------
// Static per-width facts
// ---------------------------------------------------------------------------------------------
template <int BITS>
struct Width {
    static constexpr int RB = 16 * BITS;                       // code bytes of one 128-wide row
    static constexpr uint32_t SOFF = scale_offset(BITS, D, D);  // byte offset of r[]
    static constexpr uint32_t BLK = head_block_bytes(BITS, D, D);
    static constexpr float QMAX = (float)((1 << (BITS - 1)) - 1);
    static constexpr float ROUND = 8388608.0f + (float)(1 << (BITS - 1));  // 2^23 + offset
    // power-of-two factor of column c (= j mod 8) left by the unpacking
    __device__ static constexpr float sigma(int c)
    {
        return BITS == 4 ? (float)(1 << (4 * (c & 3)))
             : BITS == 6 ? (float)(1 << (6 * (c % 3)))
                         : 1.0f;
    }
};

__device__ __forceinline__ float f_of(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t u_of(float x) { return __float_as_uint(x); }

// Unpack the 8 codes of one thread's row segment (in shared memory) into sigma_c * Q.
template <int BITS>
__device__ __forceinline__ void unpack_row(const uint8_t *src, int cg, float2 (&Q)[4])
{
    if constexpr (BITS == 4) {
        const uint32_t wd = *reinterpret_cast<const uint32_t *>(src);
        const uint32_t hi = wd >> 16;
        Q[0] = __fadd2_rn(make_float2(f_of((wd & 0x000Fu) | MAGIC), f_of((wd & 0x00F0u) | MAGIC)),
                          make_float2(-(8388608.0f + 8.0f), -(8388608.0f + 128.0f)));
        Q[1] = __fadd2_rn(make_float2(f_of((wd & 0x0F00u) | MAGIC), f_of((wd & 0xF000u) | MAGIC)),
                          make_float2(-(8388608.0f + 2048.0f), -(8388608.0f + 32768.0f)));
        Q[2] = __fadd2_rn(make_float2(f_of((hi & 0x000Fu) | MAGIC), f_of((hi & 0x00F0u) | MAGIC)),
                          make_float2(-(8388608.0f + 8.0f), -(8388608.0f + 128.0f)));
        Q[3] = __fadd2_rn(make_float2(f_of((hi & 0x0F00u) | MAGIC), f_of((hi & 0xF000u) | MAGIC)),
                          make_float2(-(8388608.0f + 2048.0f), -(8388608.0f + 32768.0f)));
    } else if constexpr (BITS == 6) {
        uint32_t lo, hi;
        if ((cg & 1) == 0) {
            lo = *reinterpret_cast<const uint32_t *>(src);
            hi = *reinterpret_cast<const uint16_t *>(src + 4);
        } else {
            const uint32_t w1 = *reinterpret_cast<const uint32_t *>(src + 2);
            lo = (uint32_t)(*reinterpret_cast<const uint16_t *>(src)) | (w1 << 16);
            hi = w1 >> 16;
        }
        const uint32_t t = __funnelshift_r(lo, hi, 18);
        const uint32_t t2 = hi >> 4;
        Q[0] = __fadd2_rn(make_float2(f_of((lo & 0x3Fu) | MAGIC), f_of((lo & 0xFC0u) | MAGIC)),
                          make_float2(-(8388608.0f + 32.0f), -(8388608.0f + 2048.0f)));
        Q[1] = __fadd2_rn(make_float2(f_of((lo & 0x3F000u) | MAGIC), f_of((t & 0x3Fu) | MAGIC)),
                          make_float2(-(8388608.0f + 131072.0f), -(8388608.0f + 32.0f)));
        Q[2] = __fadd2_rn(make_float2(f_of((t & 0xFC0u) | MAGIC), f_of((t & 0x3F000u) | MAGIC)),
                          make_float2(-(8388608.0f + 2048.0f), -(8388608.0f + 131072.0f)));
        Q[3] = __fadd2_rn(make_float2(f_of((t2 & 0x3Fu) | MAGIC), f_of((t2 & 0xFC0u) | MAGIC)),
                          make_float2(-(8388608.0f + 32.0f), -(8388608.0f + 2048.0f)));
    } else {
        const uint2 wd = *reinterpret_cast<const uint2 *>(src);
        const float2 off = make_float2(-(8388608.0f + 128.0f), -(8388608.0f + 128.0f));
        Q[0] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.x, MAGIC, 0x7650)), f_of(__byte_perm(wd.x, MAGIC, 0x7651))), off);
        Q[1] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.x, MAGIC, 0x7652)), f_of(__byte_perm(wd.x, MAGIC, 0x7653))), off);
        Q[2] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.y, MAGIC, 0x7650)), f_of(__byte_perm(wd.y, MAGIC, 0x7651))), off);
        Q[3] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.y, MAGIC, 0x7652)), f_of(__byte_perm(wd.y, MAGIC, 0x7653))), off);
    }
}

// Pack 8 rounded codes (bit patterns 2^23 + u, u < 2^b) and store them to the tile in HBM.
template <int BITS>
__device__ __forceinline__ void pack_store_row(uint8_t *dst, int cg, const float2 (&F)[4])
{
    const uint32_t f0 = u_of(F[0].x), f1 = u_of(F[0].y), f2 = u_of(F[1].x), f3 = u_of(F[1].y);
    const uint32_t f4 = u_of(F[2].x), f5 = u_of(F[2].y), f6 = u_of(F[3].x), f7 = u_of(F[3].y);
    if constexpr (BITS == 4) {
        // sum_c F_c << 4c minus the same sum of the 2^23 patterns (mod 2^32) leaves the nibbles
        constexpr uint32_t C = (uint32_t)(((uint64_t)MAGIC << 0) + ((uint64_t)MAGIC << 4) + ((uint64_t)MAGIC << 8) +
                                          ((uint64_t)MAGIC << 12) + ((uint64_t)MAGIC << 16) + ((uint64_t)MAGIC << 20) +
                                          ((uint64_t)MAGIC << 24) + ((uint64_t)MAGIC << 28));
        uint32_t acc = f7;
        acc = (acc << 4) + f6;
        acc = (acc << 4) + f5;
        acc = (acc << 4) + f4;
        acc = (acc << 4) + f3;
        acc = (acc << 4) + f2;
        acc = (acc << 4) + f1;
        acc = (acc << 4) + f0;
        *reinterpret_cast<uint32_t *>(dst) = acc - C;
    } else if constexpr (BITS == 6) {
        constexpr uint32_t C = (uint32_t)(((uint64_t)MAGIC << 0) + ((uint64_t)MAGIC << 6) + ((uint64_t)MAGIC << 12) +
                                          ((uint64_t)MAGIC << 18) + ((uint64_t)MAGIC << 24) + ((uint64_t)MAGIC << 30));
        const uint32_t lo = f0 + (f1 << 6) + (f2 << 12) + (f3 << 18) + (f4 << 24) + (f5 << 30) - C;
        // bits 32..47: the top 4 bits of code 5, codes 6 and 7 (garbage above bit 15 is dropped)
        const uint32_t hi = ((f5 >> 2) + (f6 << 4) + (f7 << 10)) & 0xFFFFu;
        if ((cg & 1) == 0) {
            *reinterpret_cast<uint32_t *>(dst) = lo;
            *reinterpret_cast<uint16_t *>(dst + 4) = (uint16_t)hi;
        } else {
            *reinterpret_cast<uint16_t *>(dst) = (uint16_t)(lo & 0xFFFFu);
            *reinterpret_cast<uint32_t *>(dst + 2) = (lo >> 16) | (hi << 16);
        }
    } else {
        uint2 wd;
        wd.x = __byte_perm(__byte_perm(f0, f1, 0x0040), __byte_perm(f2, f3, 0x0040), 0x5410);
        wd.y = __byte_perm(__byte_perm(f4, f5, 0x0040), __byte_perm(f6, f7, 0x0040), 0x5410);
        *reinterpret_cast<uint2 *>(dst) = wd;
    }
}

__device__ __forceinline__ float4 f4_of(float2 a, float2 b) { return make_float4(a.x, a.y, b.x, b.y); }

__host__ __device__ constexpr uint32_t tile_bytes(int bits, int in_bf16, int gate)
{
    return head_block_bytes(bits, D, D) + 3u * D * (in_bf16 ? 2u : 4u) + 4u * D + (gate != 0 ? 4u * D : 0u);
}

// Deterministic placement of the next tile in the ring: continue, or wrap to 0 if it does not fit.
__device__ __forceinline__ void ring_place(uint32_t &head, uint32_t &wrap, uint32_t len, uint32_t &pos)
{
    if (head + len > RING) {
        head = 0;
        ++wrap;
    }
    pos = head;
    head += len;
}

struct TileId {
    int b, hr, bits;
    uint32_t off;
};

__device__ __forceinline__ TileId tile_id(const TileParams &p, int t)
{
    TileId id;
    const int pos = t / p.B;
    id.b = t - pos * p.B;
    const TileEntry e = p.table[pos];
    id.hr = entry_head(e);
    id.bits = entry_bits(e);
    id.off = e.off;
    return id;
}

// Thread 0's producer state.
template <int GATE, int IN_BF16>
struct Producer {
    int issued = 0;
    uint32_t head = 0, wrap = 0;
    float nbeta = 0.f, nalpha = 0.f, nskip = 0.f;

    // Issue bulk copies for as many upcoming tiles as fit next to the live ones. Tiles before
    // `oldest` are dead (their ring bytes are no longer read). A tile always fits an empty ring,
    // so every tile is eventually issued.
    __device__ void issue_more(const TileParams &p, SmemD128 &sm, int my_count, int oldest)
    {
        constexpr uint32_t ROW_IN = D * (IN_BF16 ? 2 : 4);
        while (issued < my_count && issued - oldest < NBAR) {
            const TileId id = tile_id(p, (int)blockIdx.x + issued * (int)gridDim.x);
            const uint32_t len = tile_bytes(id.bits, IN_BF16, GATE);
            uint32_t h = head, wr = wrap, pos;
            ring_place(h, wr, len, pos);
            if (issued > oldest) {
                const uint32_t opos = sm.tpos[oldest % NBAR], owrap = sm.twrap[oldest % NBAR];
                const bool fits = (wr == owrap) || (wr == owrap + 1 && pos + len <= opos);
                if (!fits) break;
            }
            head = h;
            wrap = wr;
            sm.tpos[issued % NBAR] = pos;
            sm.twrap[issued % NBAR] = wr;
            const uint32_t bar = smem_u32(&sm.bars[issued % NBAR]);
            const int slot = sm.slots[id.b];
            if (slot < 0 || slot >= p.pool_slots) {
                flag(p.status, kFlagBounds);
                mbar_arrive(bar);
            } else {
                const uint32_t blk = head_block_bytes(id.bits, D, D);
                const uint32_t dst = smem_u32(sm.ring + pos);
                const size_t row = (size_t)id.b * p.head_count + id.hr;
                mbar_arrive_expect_tx(bar, len);
                bulk_g2s(dst, p.pool + (uint64_t)slot * p.req_bytes + id.off, blk, bar);
                bulk_g2s(dst + blk, (const uint8_t *)p.k + row * ROW_IN, ROW_IN, bar);
                bulk_g2s(dst + blk + ROW_IN, (const uint8_t *)p.q + row * ROW_IN, ROW_IN, bar);
                bulk_g2s(dst + blk + 2 * ROW_IN, (const uint8_t *)p.v + row * ROW_IN, ROW_IN, bar);
                bulk_g2s(dst + blk + 3 * ROW_IN, p.w + (size_t)id.hr * D, 4 * D, bar);
                if (GATE != 0) bulk_g2s(dst + blk + 3 * ROW_IN + 4 * D, p.alpha + row * D, 4 * D, bar);
            }
            ++issued;
        }
    }

    // Start loading the per-tile scalars of tile n (plain loads; consumed one sweep later).
    __device__ void load_scalars(const TileParams &p, const SmemD128 &sm, int n, int my_count)
    {
        if (n >= my_count) return;
        const TileId id = tile_id(p, (int)blockIdx.x + n * (int)gridDim.x);
        const size_t row = (size_t)id.b * p.head_count + id.hr;
        const int slot = sm.slots[id.b];
        nskip = (slot < 0 || slot >= p.pool_slots) ? 1.f : 0.f;
        nbeta = p.beta[row];
        nalpha = GATE == 0 ? p.alpha[row] : 1.f;
    }
    __device__ void store_scalars(SmemD128 &sm, int parity)
    {
        sm.scal[parity][0] = nbeta;
        sm.scal[parity][1] = nalpha;
        sm.scal[parity][2] = nskip;
    }
};

// Row factors of one tile (threads 0..127, row i = tid), and per-warp sums of w, q.k, q.(alpha k).
template <int GATE, int IN_BF16>
__device__ __forceinline__ void precompute_rows(SmemD128 &sm, const uint8_t *tile, int bits, int pb)
{
    constexpr uint32_t ROW_IN = D * (IN_BF16 ? 2 : 4);
    const int i = threadIdx.x;
    const uint32_t blk = head_block_bytes(bits, D, D);
    const uint8_t *rows = tile + blk;
    const bool pivot = bits == 16;
    const float r = pivot ? 1.f : reinterpret_cast<const float *>(tile + scale_offset(bits, D, D))[i];
    const float k = load_in<IN_BF16>(rows, i);
    const float q = load_in<IN_BF16>(rows + ROW_IN, i);
    const float w = reinterpret_cast<const float *>(rows + 3 * ROW_IN)[i];
    const float a = GATE == 0 ? sm.scal[pb][1] : reinterpret_cast<const float *>(rows + 3 * ROW_IN + 4 * D)[i];
    const float sw = pivot ? 1.f : sqrtf(w);
    const float kt = (GATE == 2 ? k * a : k) * r;
    sm.rowA[pb][i] = make_float4(kt, q * a * r, a * sw * r, sw * k);
    sm.rowB[pb][i] = make_float2(sw, -sw * a * k);
    float s0 = w, s1 = q * k, s2 = q * a * k;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    if ((i & 31) == 0) {
        sm.rsum[pb][i >> 5][0] = s0;
        sm.rsum[pb][i >> 5][1] = s1;
        sm.rsum[pb][i >> 5][2] = s2;
    }
}

// Column finals after the first sweep: threads 0..127 turn the column sums of k~ Q into g (and
// the readout's rank-1 part); threads 128..255 return the column sums of q~ Q (un-scaled).
template <int GATE, int IN_BF16>
__device__ __forceinline__ float finals_a(SmemD128 &sm, const uint8_t *tile, int bits, int pb, float cj,
                                          float inv_sig, float sig)
{
    constexpr uint32_t ROW_IN = D * (IN_BF16 ? 2 : 4);
    const int tid = threadIdx.x;
    const int j = tid & (D - 1);
    if (tid < D) {
        float U = 0.f;
#pragma unroll
        for (int s = 0; s < 16; ++s) U += sm.red[s * 2 * D + j];
        U *= inv_sig;
        const float beta = sm.scal[pb][0], alpha = sm.scal[pb][1];
        const float vj = load_in<IN_BF16>(tile + head_block_bytes(bits, D, D) + 2 * ROW_IN, j);
        const float qk = sm.rsum[pb][0][1] + sm.rsum[pb][1][1] + sm.rsum[pb][2][1] + sm.rsum[pb][3][1];
        const float u = cj * U;
        if (GATE == 1) {
            const float qak = sm.rsum[pb][0][2] + sm.rsum[pb][1][2] + sm.rsum[pb][2][2] + sm.rsum[pb][3][2];
            sm.colG1[j] = sig * (beta * vj / cj);
            sm.colG2[j] = sig * (beta * u / cj);
            sm.colH[j] = qk * beta * vj - qak * beta * u;
        } else {
            const float h = GATE == 0 ? beta * (vj - alpha * u) : beta * (vj - u);
            sm.colG1[j] = sig * (h / cj);
            sm.colH[j] = qk * h;
        }
        return 0.f;
    }
    float P = 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s) P += sm.red[s * 2 * D + D + j];
    return P * inv_sig;
}

// Sweep A (shared by quantized and pivot tiles): column sums of k~ Q and q~ Q from registers.
__device__ __forceinline__ void sweep_a_sums(SmemD128 &sm, const float2 (&Q)[8][4], int pb, int warp, int sub, int cg)
{
    float2 accU[4], accP[4];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) accU[pp] = accP[pp] = make_float2(0.f, 0.f);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int i = 16 * m + 2 * warp + sub;
        const float4 ra = sm.rowA[pb][i];
        const float2 kk = make_float2(ra.x, ra.x), qq = make_float2(ra.y, ra.y);
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            accU[pp] = __ffma2_rn(kk, Q[m][pp], accU[pp]);
            accP[pp] = __ffma2_rn(qq, Q[m][pp], accP[pp]);
        }
    }
    float *red = sm.red + (2 * warp + sub) * 2 * D + 8 * cg;
    *reinterpret_cast<float4 *>(red) = f4_of(accU[0], accU[1]);
    *reinterpret_cast<float4 *>(red + 4) = f4_of(accU[2], accU[3]);
    *reinterpret_cast<float4 *>(red + D) = f4_of(accP[0], accP[1]);
    *reinterpret_cast<float4 *>(red + D + 4) = f4_of(accP[2], accP[3]);
}

// y = rho Q + kappa g1 (+ mu g2), in place in Q; optionally accumulating the column energy.
template <int GATE, bool ENERGY>
__device__ __forceinline__ void sweep_b_update(SmemD128 &sm, float2 (&Q)[8][4], int pb, int warp, int sub, int cg,
                                               float2 (&accE)[4], bool &bad)
{
    float2 g1[4], g2[4];
    {
        const float4 a = *reinterpret_cast<const float4 *>(sm.colG1 + 8 * cg);
        const float4 b = *reinterpret_cast<const float4 *>(sm.colG1 + 8 * cg + 4);
        g1[0] = make_float2(a.x, a.y); g1[1] = make_float2(a.z, a.w);
        g1[2] = make_float2(b.x, b.y); g1[3] = make_float2(b.z, b.w);
    }
    if (GATE == 1) {
        const float4 a = *reinterpret_cast<const float4 *>(sm.colG2 + 8 * cg);
        const float4 b = *reinterpret_cast<const float4 *>(sm.colG2 + 8 * cg + 4);
        g2[0] = make_float2(a.x, a.y); g2[1] = make_float2(a.z, a.w);
        g2[2] = make_float2(b.x, b.y); g2[3] = make_float2(b.z, b.w);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int i = 16 * m + 2 * warp + sub;
        const float4 ra = sm.rowA[pb][i];
        const float2 rho = make_float2(ra.z, ra.z), kap = make_float2(ra.w, ra.w);
        float2 mu = make_float2(0.f, 0.f);
        if (GATE == 1) {
            const float mv = sm.rowB[pb][i].y;
            mu = make_float2(mv, mv);
        }
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            float2 t = __fmul2_rn(kap, g1[pp]);
            if (GATE == 1) t = __ffma2_rn(mu, g2[pp], t);
            const float2 y = __ffma2_rn(rho, Q[m][pp], t);
            Q[m][pp] = y;
            if (ENERGY) accE[pp] = __ffma2_rn(y, y, accE[pp]);
            else bad |= !(fabsf(y.x) < 65520.0f) || !(fabsf(y.y) < 65520.0f);
        }
    }
}

template <int BITS, int GATE, int IN_BF16>
__device__ __forceinline__ void tile_quant(const TileParams &p, SmemD128 &sm, const uint8_t *tile,
                                           uint8_t *gblock, float *orow, int pb, int n, int my_count,
                                           Producer<GATE, IN_BF16> &prod)
{
    using Wd = Width<BITS>;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, cg = lane & 15, sub = lane >> 4;
    float2 Q[8][4];
#pragma unroll
    for (int m = 0; m < 8; ++m) unpack_row<BITS>(tile + (16 * m + 2 * warp + sub) * Wd::RB + cg * BITS, cg, Q[m]);
    sweep_a_sums(sm, Q, pb, warp, sub, cg);
    if (tid == 0) prod.store_scalars(sm, pb ^ 1);
    __syncthreads();  // B1: column partials complete

    const int j = tid & (D - 1);
    const float cj = reinterpret_cast<const float *>(tile + Wd::SOFF)[D + j];
    const float sig = Wd::sigma(j & 7);
    const float inv_sig = 1.0f / sig;  // power of two: exact
    const float Pj = finals_a<GATE, IN_BF16>(sm, tile, BITS, pb, cj, inv_sig, sig);
    __syncthreads();  // B2: g, readout parts ready; this tile's ring bytes are no longer read
    if (tid == 0) prod.issue_more(p, sm, my_count, n + 1);

    if (tid >= D) {
        const float o = cj * Pj + sm.colH[j];
        orow[j] = o;
        if (!isfinite(o)) flag(p.status, kFlagNonfinite);
    }
    float2 accE[4];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) accE[pp] = make_float2(0.f, 0.f);
    bool bad_unused = false;
    sweep_b_update<GATE, true>(sm, Q, pb, warp, sub, cg, accE, bad_unused);
    {
        float *red = sm.red + (2 * warp + sub) * D + 8 * cg;
        *reinterpret_cast<float4 *>(red) = f4_of(accE[0], accE[1]);
        *reinterpret_cast<float4 *>(red + 4) = f4_of(accE[2], accE[3]);
    }
    __syncthreads();  // B3: column energies complete

    if (tid < D) {
        float E = 0.f;
#pragma unroll
        for (int s = 0; s < 16; ++s) E += sm.red[s * D + j];
        const float W = sm.rsum[pb][0][0] + sm.rsum[pb][1][0] + sm.rsum[pb][2][0] + sm.rsum[pb][3][0];
        float c = (cj * inv_sig) * sqrtf(E / W);
        if (c == 0.f) c = 1.f;
        reinterpret_cast<float *>(gblock + Wd::SOFF)[D + j] = c;
        if (!isfinite(c)) flag(p.status, kFlagNonfinite);
        sm.colB[j] = (cj * inv_sig) / c;
    }
    __syncthreads();  // B4: new column scales ready

    // Sweep C: column-normalised values z and the per-row maxima of |z|.
    float mx[8];
    {
        float2 bb[4];
        const float4 a = *reinterpret_cast<const float4 *>(sm.colB + 8 * cg);
        const float4 b = *reinterpret_cast<const float4 *>(sm.colB + 8 * cg + 4);
        bb[0] = make_float2(a.x, a.y); bb[1] = make_float2(a.z, a.w);
        bb[2] = make_float2(b.x, b.y); bb[3] = make_float2(b.z, b.w);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            float v = 0.f;
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                Q[m][pp] = __fmul2_rn(Q[m][pp], bb[pp]);
                v = fmaxf(v, fmaxf(fabsf(Q[m][pp].x), fabsf(Q[m][pp].y)));
            }
            mx[m] = v;
        }
    }
    float *rm = sm.red + (2 * warp + sub) * 128;
    *reinterpret_cast<float4 *>(rm + 8 * cg) = make_float4(mx[0], mx[1], mx[2], mx[3]);
    *reinterpret_cast<float4 *>(rm + 8 * cg + 4) = make_float4(mx[4], mx[5], mx[6], mx[7]);
    __syncwarp();
    {
        const int m = cg >> 1, half = cg & 1;
        float v = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) v = fmaxf(v, rm[(half * 8 + c8) * 8 + m]);
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
        const int i = 16 * m + 2 * warp + sub;
        const float sw = sm.rowB[pb][i].x;
        float r = v / (sw * Wd::QMAX);
        if (v == 0.f) r = 1.f;
        const float s = 1.0f / (sw * r);
        if (half == 0) {
            sm.rowS[i] = make_float2(s, s);
            reinterpret_cast<float *>(gblock + Wd::SOFF)[i] = r;
            if (!isfinite(r) || r == 0.f) flag(p.status, kFlagNonfinite);
        }
    }
    __syncwarp();

    // Sweep D: x = z s rounded half to even by the 2^23 + offset FFMA, packed and stored in place.
    const float2 rnd = make_float2(Wd::ROUND, Wd::ROUND);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int i = 16 * m + 2 * warp + sub;
        const float2 s2 = sm.rowS[i];
        float2 F[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) F[pp] = __ffma2_rn(Q[m][pp], s2, rnd);
        pack_store_row<BITS>(gblock + i * Wd::RB + cg * BITS, cg, F);
    }
}

template <int GATE, int IN_BF16>
__device__ __forceinline__ void tile_pivot(const TileParams &p, SmemD128 &sm, const uint8_t *tile,
                                           uint8_t *gblock, float *orow, int pb, int n, int my_count,
                                           Producer<GATE, IN_BF16> &prod)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, cg = lane & 15, sub = lane >> 4;
    float2 Q[8][4];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const uint4 raw = *reinterpret_cast<const uint4 *>(tile + (16 * m + 2 * warp + sub) * 256 + cg * 16);
        Q[m][0] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
        Q[m][1] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
        Q[m][2] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.z));
        Q[m][3] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.w));
    }
    sweep_a_sums(sm, Q, pb, warp, sub, cg);
    if (tid == 0) prod.store_scalars(sm, pb ^ 1);
    __syncthreads();  // B1

    const int j = tid & (D - 1);
    const float Pj = finals_a<GATE, IN_BF16>(sm, tile, 16, pb, 1.f, 1.f, 1.f);
    __syncthreads();  // B2: this tile's ring bytes are no longer read
    if (tid == 0) prod.issue_more(p, sm, my_count, n + 1);
    if (tid >= D) {
        const float o = Pj + sm.colH[j];
        orow[j] = o;
        if (!isfinite(o)) flag(p.status, kFlagNonfinite);
    }
    float2 accE[4];
    bool bad = false;
    sweep_b_update<GATE, false>(sm, Q, pb, warp, sub, cg, accE, bad);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        uint4 raw;
        __half2 h0 = __float22half2_rn(Q[m][0]), h1 = __float22half2_rn(Q[m][1]);
        __half2 h2 = __float22half2_rn(Q[m][2]), h3 = __float22half2_rn(Q[m][3]);
        raw.x = *reinterpret_cast<uint32_t *>(&h0);
        raw.y = *reinterpret_cast<uint32_t *>(&h1);
        raw.z = *reinterpret_cast<uint32_t *>(&h2);
        raw.w = *reinterpret_cast<uint32_t *>(&h3);
        *reinterpret_cast<uint4 *>(gblock + (16 * m + 2 * warp + sub) * 256 + cg * 16) = raw;
    }
    if (bad) flag(p.status, kFlagNonfinite);
}

template <int GATE, int IN_BF16>
__global__ void __launch_bounds__(NT, 2) decode_d128_kernel(const __grid_constant__ TileParams p)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SmemD128 &sm = *reinterpret_cast<SmemD128 *>(smem_raw);
    const int tid = threadIdx.x;
    const int G = (int)gridDim.x;
    const int my_count = (p.ntiles - (int)blockIdx.x + G - 1) / G;

    for (int b = tid; b < p.B; b += NT) sm.slots[b] = p.slots[b];
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(smem_u32(&sm.bars[i]), 1);
        fence_mbar_init();
    }
    __syncthreads();

    Producer<GATE, IN_BF16> prod;
    if (tid == 0) {
        prod.issue_more(p, sm, my_count, 0);
        prod.load_scalars(p, sm, 0, my_count);
        prod.store_scalars(sm, 0);
    }
    __syncthreads();

    uint32_t c_head = 0, c_wrap = 0;
    for (int n = 0; n < my_count; ++n) {
        const TileId id = tile_id(p, (int)blockIdx.x + n * G);
        uint32_t tpos;  // replays the producer's deterministic placement
        ring_place(c_head, c_wrap, tile_bytes(id.bits, IN_BF16, GATE), tpos);
        const uint8_t *tile = sm.ring + tpos;
        const int pb = n & 1;
        const bool skip = sm.scal[pb][2] != 0.f;
        const bool ok = mbar_wait_bounded(smem_u32(&sm.bars[n % NBAR]), (uint32_t)((n / NBAR) & 1));
        if (tid < D && !skip) precompute_rows<GATE, IN_BF16>(sm, tile, id.bits, pb);
        if (__syncthreads_or(!ok)) {  // B0
            if (tid == 0) {
                flag(p.status, kFlagTimeout);
                for (int m = n; m < prod.issued; ++m)  // let copies in flight land before exiting
                    mbar_wait_bounded(smem_u32(&sm.bars[m % NBAR]), (uint32_t)((m / NBAR) & 1));
            }
            return;
        }
        if (tid == 0) prod.load_scalars(p, sm, n + 1, my_count);
        if (skip) {
            if (tid == 0) {
                prod.store_scalars(sm, pb ^ 1);
                prod.issue_more(p, sm, my_count, n + 1);
            }
            __syncthreads();
            continue;
        }
        const int slot = sm.slots[id.b];
        uint8_t *gblock = p.pool + (uint64_t)slot * p.req_bytes + id.off;
        float *orow = p.o + ((size_t)id.b * p.head_count + id.hr) * D;
        switch (id.bits) {
        case 4: tile_quant<4, GATE, IN_BF16>(p, sm, tile, gblock, orow, pb, n, my_count, prod); break;
        case 6: tile_quant<6, GATE, IN_BF16>(p, sm, tile, gblock, orow, pb, n, my_count, prod); break;
        case 8: tile_quant<8, GATE, IN_BF16>(p, sm, tile, gblock, orow, pb, n, my_count, prod); break;
        default: tile_pivot<GATE, IN_BF16>(p, sm, tile, gblock, orow, pb, n, my_count, prod); break;
        }
    }
}

template <int GATE, int IN_BF16>
cudaError_t launch_t(const TileParams &p, cudaStream_t s)
{
    auto kernel = decode_d128_kernel<GATE, IN_BF16>;
    const int smem = (int)sizeof(SmemD128);
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    int sms = 0, per_sm = 0;
    err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, NT, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int grid = p.ntiles < sms * per_sm ? p.ntiles : sms * per_sm;
    kernel<<<grid, NT, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int decode_d128_max_requests() { return MAXB; }

cudaError_t launch_decode_d128(const TileParams &p, int in_bf16, cudaStream_t s)
{
    switch (p.gate * 2 + (in_bf16 ? 1 : 0)) {
    case 0: return launch_t<0, 0>(p, s);
    case 1: return launch_t<0, 1>(p, s);
    case 2: return launch_t<1, 0>(p, s);
    case 3: return launch_t<1, 1>(p, s);
    case 4: return launch_t<2, 0>(p, s);
    default: return launch_t<2, 1>(p, s);
    }
}

}  // namespace stq
