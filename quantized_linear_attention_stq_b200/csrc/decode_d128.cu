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
//  * One persistent kernel per width (FP16 pivots, 8-, 6-, 4-bit), launched largest first; CTAs of
//    128 threads (four per SM) walk the width's tiles round-robin.
//  * Thread 0 streams each upcoming tile into a shared-memory slot ring: the packed codes + scales
//    and the k, q, v, w (and alpha) rows by cp.async.bulk, the per-tile scalars by 4-byte cp.async,
//    all completing on the slot's mbarrier. Every wait is bounded and reports STQ_ERR_TIMEOUT.
//  * Thread (warp w, lane l) owns a 16 x 8 sub-block of the tile: rows 8m + 2w + l/16 (m < 16),
//    columns 8 (l%16) .. +7. Its 128 values live in its own lane of Tensor Memory (lane 32w + l,
//    128 columns) between the sweeps and pass through registers 8 or 16 at a time (tcgen05.st /
//    tcgen05.ld); the state is read from HBM once and written once per step.
//  * The algebra runs in column-normalised coordinates: with y_ij = sqrt(w_i) S'_ij / c_j,
//      y_ij = rho_i Q_ij + kappa_i g_j   (rho = alpha sqrt(w) r, kappa = sqrt(w) k, g = h / c,
//                                         h = beta (v - alpha u))
//    so the update, the column energy, the row maximum and the rounding are 1-2 packed f32x2
//    operations per element each. Codes are unpacked with a LOP3/PRMT into the mantissa of 2^23
//    (exact; odd columns carry a power-of-two factor sigma, folded back per column) and rounded
//    back with one FFMA against 2^23 + 2^(b-1), which rounds half to even for free.
//  * Four CTA barriers per tile: column sums of k~Q and q~Q (B1), the update coefficients (B2),
//    the column energies (B3) and the new column scales with the next tile's row factors (B4).
//    Every thread takes one column (and one row) in each of these steps. Column partials are
//    summed between the two half-warps by shuffles, then across the four warps through shared
//    memory; row maxima stay inside a half-warp.
//  * Scale arithmetic (reciprocals, square roots) uses the SFU approximations (a few ulp): the
//    codes are always computed from the scales this kernel stores.
#include "stq_internal.cuh"

namespace stq {
namespace {

constexpr int D = 128;
constexpr int NT = 128;                // threads per CTA: one tile at a time
constexpr int NSMAX = 4;               // slots (tiles in flight) per CTA
constexpr uint32_t MAGIC = 0x4B000000u;  // bit pattern of 2^23
constexpr uint32_t TMEM_COLS = 128;    // per CTA: 128 lanes x 128 columns of fp32 = one tile
// red[]: one region of RS floats per (warp, half) k = 2w + h. [0, 128): the half's column
// partials, column j at cpos(j) (k~Q for h = 0, q~Q for h = 1); [128, 256) of the h = 0 region:
// the warp's column energies; later the half's 16 row-max partial rows of RM floats. Only warp w writes its two
// regions while other warps may be reading, so a warp never overwrites data still in use.
constexpr int RM = 20;                 // row stride of the row-max partials (bank-conflict free)
constexpr int RS = 336;                // region stride (= 16 mod 32 banks: the halves do not collide)

// Thread 0's cursor over this CTA's tiles t = blockIdx.x + n * gridDim.x, kept as (table
// position, request) = (t / B, t % B) and advanced without a division.
struct Issuer {
    int n, pos, b, qG, rG;
    int next_slot;  // pool slot of the next tile's request, loaded one issue ahead
};

// Per tile, written by the issuing thread: where the tile lives and which input row it uses.
struct SlotMeta {
    unsigned long long gblock;  // address of the tile's head block in the pool
    uint32_t orow;              // request * head_count + head: the row of q, k, v, beta, alpha, o
    uint16_t skip;              // 1: out-of-range slot, nothing was loaded
    uint16_t bits;              // code width of the tile
};

struct __align__(16) SmemFixed {
    float red[8 * RS];
    float4 rowKQ[D];         // (k~, k~, q~, q~)
    float4 rowRK[D];         // (rho, rho, kappa, kappa)
    float rowRq[2][D];       // per tile parity: 1 / (sqrt(w_i) qmax)
    float2 rowS[D];          // (s_i, s_i), s_i = 1 / (sqrt(w_i) r'_i) = qmax / max_j |z_ij|, at rpos<FIT>(i)
    float colG1[D];          // per column j at cpos(j), as colB and colG2
    float colB[D];           // c_j / (sigma_j c'_j) = 1 / sqrt(x_j)
    float rsum[2][4][4];     // per parity, per warp: sum w, q.k, q.(alpha*k)
    float scal[NSMAX][2];    // per slot: beta, alpha
    SlotMeta meta[4];        // per tile n, at n % 4 (NS + 1 <= 4 tiles are live at a time)
    Issuer iss;              // thread 0's tile cursor
    unsigned long long bars[NSMAX];
    uint32_t magic;          // 0x4B000000, read at run time so the unpack keeps it in a register
                             // and forms each value with one LOP3 ((s & mask) | magic)
    uint32_t tmem_base;
};

// Only the literal channel gate (gate 1) needs these; they follow SmemFixed when present.
struct __align__(16) SmemChannel {
    float2 rowMu[D];         // (mu, mu)
    float colG2[D];
};

// Only the joint scale refinement (FIT) needs these; they follow SmemFixed (and SmemChannel).
// In the coordinates z_ij = sqrt(w_i) S'_ij / c'_j of the one-pass fit (c' its stored column
// scale), the impact-weighted error is sum_ij c'_j^2 (z_ij - rho_i K_j Q_ij)^2 with rho_i =
// sqrt(w_i) r_i and c_j = K_j c'_j.
// The refit's column factors reuse SmemFixed arrays that are dead by then: colB holds K~_j (the
// refitted stored column scale over c'_j) and colG1 holds c'_j^2 K~_j.
struct __align__(16) SmemFit {
    float rowRho[D];         // rho_i of the one-pass stored row scale
};

// ---------------------------------------------------------------------------------------------
// Per-width facts. A launch either has one compile-time width (BITS = 4, 6, 8 or 16: FP16 pivots)
// or takes each tile's width from the head table (BITS = 0: any mix of 4, 6 and 8 bits; the ring
// slots are then sized for 8-bit tiles and only the unpack and pack steps branch on the width).
// ---------------------------------------------------------------------------------------------
struct Width {
    int bits;
    uint32_t rb;    // bytes of one 128-wide row of codes
    uint32_t soff;  // byte offset of r[] in the head block
    float qmax;
    float round;    // 2^23 + 2^(b-1): the FFMA against it rounds half to even into the code bits
    float sig1;     // odd columns are unpacked scaled by sig1 (even columns by 1)
};

__device__ __forceinline__ Width width_of(int bits)
{
    Width w;
    w.bits = bits;
    w.rb = bits == 16 ? 256u : 16u * (uint32_t)bits;
    w.soff = bits == 16 ? 0u : 2048u * (uint32_t)bits;  // the codes of 128 x 128, a multiple of 16
    w.qmax = bits == 16 ? 0.f : (float)((1 << (bits - 1)) - 1);
    w.round = 8388608.0f + (bits == 16 ? 0.f : (float)(1 << (bits - 1)));
    w.sig1 = bits == 4 ? 16.f : bits == 6 ? 64.f : 1.f;
    return w;
}

template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
struct Cfg {
    static constexpr int RBITS = BITS == 0 ? 8 : BITS;                // the ring's slots fit this width
    static constexpr uint32_t BLK = head_block_bytes(RBITS, D, D);    // ring room (fp32 scales)
    static constexpr uint32_t ROW_IN = D * (IN_BF16 ? 2u : 4u);
    static constexpr uint32_t K_OFF = BLK, Q_OFF = BLK + ROW_IN, V_OFF = BLK + 2 * ROW_IN;
    static constexpr uint32_t W_OFF = BLK + 3 * ROW_IN, A_OFF = W_OFF + 4 * D;
    static constexpr uint32_t LEN = A_OFF + (GATE != 0 ? 4u * D : 0u);  // a multiple of 256
    static constexpr uint32_t FIT_OFF = (uint32_t)sizeof(SmemFixed) + (GATE == 1 ? (uint32_t)sizeof(SmemChannel) : 0u);
    static constexpr uint32_t RING = FIT_OFF + (FIT ? (uint32_t)sizeof(SmemFit) : 0u);
    // slots so that four CTAs fit an SM's 228 KB where they can
    static constexpr int NS = BITS == 4 ? 3 : 2;
    static constexpr size_t SMEM = RING + (size_t)NS * LEN;
};

__device__ __forceinline__ float f_of(uint32_t x) { return __uint_as_float(x); }
__device__ __forceinline__ uint32_t u_of(float x) { return __float_as_uint(x); }

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float fast_rcp(float x) { return __fdividef(1.0f, x); }

// ---------------------------------------------------------------------------------------------
// Tensor Memory: each thread keeps its values in consecutive columns of its own lane. The loads
// and stores carry no memory clobber (they touch only Tensor Memory), so shared-memory loads can
// be scheduled across them; their ordering with each other is kept by the waits.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float2 (&v)[8])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16};" ::"r"(taddr),
        "f"(v[0].x), "f"(v[0].y), "f"(v[1].x), "f"(v[1].y), "f"(v[2].x), "f"(v[2].y), "f"(v[3].x), "f"(v[3].y),
        "f"(v[4].x), "f"(v[4].y), "f"(v[5].x), "f"(v[5].y), "f"(v[6].x), "f"(v[6].y), "f"(v[7].x), "f"(v[7].y));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float2 (&v)[4])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "f"(v[0].x), "f"(v[0].y), "f"(v[1].x), "f"(v[1].y), "f"(v[2].x), "f"(v[2].y), "f"(v[3].x), "f"(v[3].y));
}
// Start loading 16 values; they may be read only after tmem_wait_ld on the same array.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, float2 (&v)[8])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=f"(v[0].x), "=f"(v[0].y), "=f"(v[1].x), "=f"(v[1].y), "=f"(v[2].x), "=f"(v[2].y), "=f"(v[3].x),
          "=f"(v[3].y), "=f"(v[4].x), "=f"(v[4].y), "=f"(v[5].x), "=f"(v[5].y), "=f"(v[6].x), "=f"(v[6].y),
          "=f"(v[7].x), "=f"(v[7].y)
        : "r"(taddr));
}
// Wait for this thread's outstanding Tensor Memory loads. The array is passed through as
// read-write operands so that no use of it can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(float2 (&v)[8])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(v[0].x), "+f"(v[0].y), "+f"(v[1].x), "+f"(v[1].y), "+f"(v[2].x), "+f"(v[2].y), "+f"(v[3].x),
                   "+f"(v[3].y), "+f"(v[4].x), "+f"(v[4].y), "+f"(v[5].x), "+f"(v[5].y), "+f"(v[6].x), "+f"(v[6].y),
                   "+f"(v[7].x), "+f"(v[7].y)
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Two adjacent codes at bits [0, BITS) and [BITS, 2*BITS) of s, as (2^23 + u0, 2^23 + u1 * 2^BITS).
template <int BITS>
__device__ __forceinline__ float2 code_pair(uint32_t s, uint32_t magic)
{
    constexpr uint32_t M = (1u << BITS) - 1u;
    return make_float2(f_of((s & M) | magic), f_of((s & (M << BITS)) | magic));
}

// Unpack the 8 codes of one thread's row segment (in shared memory) into (Q, SIG1 * Q) pairs;
// `off` = (-(2^23 + o), -(2^23 + o * SIG1)) with o = 2^(b-1). A pivot row holds 8 halves.
template <int BITS>
__device__ __forceinline__ void unpack_row(const uint8_t *src, int cg, float2 off, uint32_t magic, float2 *Q)
{
    if constexpr (BITS == 4) {
        const uint32_t wd = *reinterpret_cast<const uint32_t *>(src);
        Q[0] = __fadd2_rn(code_pair<4>(wd, magic), off);
        Q[1] = __fadd2_rn(code_pair<4>(wd >> 8, magic), off);
        Q[2] = __fadd2_rn(code_pair<4>(wd >> 16, magic), off);
        Q[3] = __fadd2_rn(code_pair<4>(wd >> 24, magic), off);
    } else if constexpr (BITS == 6) {
        // the 6-byte segment starts 4-byte aligned for even cg and 2 bytes past it for odd cg: load
        // the two aligned words around it and shift (no branch on the lane's parity; the bits of
        // hi above 15 belong to the next lane and are never used)
        const int odd = cg & 1;
        const uint32_t *a = reinterpret_cast<const uint32_t *>(src - 2 * odd);
        const uint32_t w0 = a[0], w1 = a[1];
        const uint32_t lo = __funnelshift_r(w0, w1, 16 * odd);
        const uint32_t hi = w1 >> (16 * odd);
        Q[0] = __fadd2_rn(code_pair<6>(lo, magic), off);
        Q[1] = __fadd2_rn(code_pair<6>(lo >> 12, magic), off);
        Q[2] = __fadd2_rn(code_pair<6>(__funnelshift_r(lo, hi, 24), magic), off);
        Q[3] = __fadd2_rn(code_pair<6>(hi >> 4, magic), off);
    } else if constexpr (BITS == 8) {
        const uint2 wd = *reinterpret_cast<const uint2 *>(src);
        Q[0] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.x, magic, 0x7650)), f_of(__byte_perm(wd.x, magic, 0x7651))), off);
        Q[1] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.x, magic, 0x7652)), f_of(__byte_perm(wd.x, magic, 0x7653))), off);
        Q[2] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.y, magic, 0x7650)), f_of(__byte_perm(wd.y, magic, 0x7651))), off);
        Q[3] = __fadd2_rn(make_float2(f_of(__byte_perm(wd.y, magic, 0x7652)), f_of(__byte_perm(wd.y, magic, 0x7653))), off);
    } else {
        const uint4 raw = *reinterpret_cast<const uint4 *>(src);
        Q[0] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
        Q[1] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
        Q[2] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.z));
        Q[3] = __half22float2(*reinterpret_cast<const __half2 *>(&raw.w));
    }
}

// Pack 8 rounded codes (bit patterns 2^23 + u, u < 2^b) and store them to the tile in HBM.
template <int BITS>
__device__ __forceinline__ void pack_store_row(uint8_t *dst, int cg, const float2 *F)
{
    const uint32_t f0 = u_of(F[0].x), f1 = u_of(F[0].y), f2 = u_of(F[1].x), f3 = u_of(F[1].y);
    const uint32_t f4 = u_of(F[2].x), f5 = u_of(F[2].y), f6 = u_of(F[3].x), f7 = u_of(F[3].y);
    if constexpr (BITS == 4) {
        // pair nibbles by shift-add (garbage above bit 8 is dropped), then gather the low bytes
        const uint32_t p0 = (f1 << 4) + f0, p1 = (f3 << 4) + f2, p2 = (f5 << 4) + f4, p3 = (f7 << 4) + f6;
        *reinterpret_cast<uint32_t *>(dst) = __byte_perm(__byte_perm(p0, p1, 0x0040), __byte_perm(p2, p3, 0x0040), 0x5410);
    } else if constexpr (BITS == 6) {
        // sum_c F_c << 6c minus the same sum of the 2^23 patterns (mod 2^32) leaves the codes
        constexpr uint32_t C = (uint32_t)(((uint64_t)MAGIC << 0) + ((uint64_t)MAGIC << 6) + ((uint64_t)MAGIC << 12) +
                                          ((uint64_t)MAGIC << 18) + ((uint64_t)MAGIC << 24) + ((uint64_t)MAGIC << 30));
        const uint32_t lo = f0 + (f1 << 6) + (f2 << 12) + (f3 << 18) + (f4 << 24) + (f5 << 30) - C;
        // bits 32..47: the top 4 bits of code 5, codes 6 and 7 (garbage above bit 15 is dropped)
        const uint32_t hi = (f5 >> 2) + (f6 << 4) + (f7 << 10);
        // three 2-byte stores fit every lane's alignment (no branch on the lane's parity)
        uint16_t *d16 = reinterpret_cast<uint16_t *>(dst);
        d16[0] = (uint16_t)lo;
        d16[1] = (uint16_t)(lo >> 16);
        d16[2] = (uint16_t)hi;
    } else {
        uint2 wd;
        wd.x = __byte_perm(__byte_perm(f0, f1, 0x0040), __byte_perm(f2, f3, 0x0040), 0x5410);
        wd.y = __byte_perm(__byte_perm(f4, f5, 0x0040), __byte_perm(f6, f7, 0x0040), 0x5410);
        *reinterpret_cast<uint2 *>(dst) = wd;
    }
}

// Column j's place in the per-column arrays (colG1, colB, colG2) and in the column-partial regions
// of red[]: lane cg keeps its columns 8 cg + 4 h + t (h < 2, t < 4) as two float4 at 4 cslot(cg, h),
// cslot(cg, h) = 8 (2 (cg / 8) + h) + (cg + 4 h) % 8. Then the float4 of 8 lanes with the same h
// and the floats of 32 threads j (column j each) both fall on 32 distinct banks. LIN: column j at
// j instead (two-way conflicts on the float4, two fewer live addresses; the refit kernels, which
// are short of registers, keep it).
template <int LIN>
__device__ __forceinline__ int cslot(int cg, int h)
{
    return LIN ? 2 * cg + h : 8 * (2 * (cg >> 3) + h) + ((cg + 4 * h) & 7);
}
template <int LIN>
__device__ __forceinline__ int cpos(int j)
{
    return LIN ? j : 4 * cslot<0>(j >> 3, (j >> 2) & 1) + (j & 3);
}

// Row i's place in rowS: [i % 8][i / 8], so that the 16 rows 8 m + rb of a half-warp are
// consecutive (lane m writes row 8 m + rb); LIN: row i at i.
template <int LIN>
__device__ __forceinline__ int rpos(int i) { return LIN ? i : (i & 7) * 16 + (i >> 3); }

// Lane cg's 8 columns of a per-column array (layout of cpos) as four pairs.
template <int LIN>
__device__ __forceinline__ void load_cols(const float *base, int cg, float2 (&out)[4])
{
    const float4 a = *reinterpret_cast<const float4 *>(base + 4 * cslot<LIN>(cg, 0));
    const float4 b = *reinterpret_cast<const float4 *>(base + 4 * cslot<LIN>(cg, 1));
    out[0] = make_float2(a.x, a.y);
    out[1] = make_float2(a.z, a.w);
    out[2] = make_float2(b.x, b.y);
    out[3] = make_float2(b.z, b.w);
}

template <int LIN>
__device__ __forceinline__ void store_cols(float *base, int cg, const float2 (&v)[4])
{
    *reinterpret_cast<float4 *>(base + 4 * cslot<LIN>(cg, 0)) = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
    *reinterpret_cast<float4 *>(base + 4 * cslot<LIN>(cg, 1)) = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
}

// Sum of the 4 per-warp partials at `stride` floats apart.
__device__ __forceinline__ float sum4(const float *src, int stride)
{
    return (src[0] + src[stride]) + (src[2 * stride] + src[3 * stride]);
}

template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
__device__ __forceinline__ uint8_t *ring_slot(uint8_t *smem, int slot_i)
{
    return smem + Cfg<BITS, GATE, IN_BF16, FIT, SB16>::RING + (size_t)slot_i * Cfg<BITS, GATE, IN_BF16, FIT, SB16>::LEN;
}

__device__ __forceinline__ SmemChannel &channel(uint8_t *smem)
{
    return *reinterpret_cast<SmemChannel *>(smem + sizeof(SmemFixed));
}

template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
__device__ __forceinline__ SmemFit &fitmem(uint8_t *smem)
{
    return *reinterpret_cast<SmemFit *>(smem + Cfg<BITS, GATE, IN_BF16, FIT, SB16>::FIT_OFF);
}

// Thread 0: stream this CTA's next tile into ring slot n % NS (codes + scales and the input rows
// by bulk copy, the per-tile scalars by 4-byte cp.async), completing on the slot's mbarrier (two
// arrivals: expect_tx + cp.async), and record where the tile lives and which row it reads.
template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
__device__ __forceinline__ void issue_next(const TileParams &p, SmemFixed &sm, uint8_t *smem, Issuer &it, int my_count)
{
    using C = Cfg<BITS, GATE, IN_BF16, FIT, SB16>;
    if (it.n >= my_count) return;
    const int n = it.n, slot_i = n % C::NS;
    const TileEntry e = p.table[it.pos];
    const int hr = entry_head(e), b = it.b;
    const int slot = it.next_slot;
    ++it.n;
    it.b += it.rG;
    it.pos += it.qG;
    if (it.b >= p.B) {
        it.b -= p.B;
        ++it.pos;
    }
    if (it.n < my_count) it.next_slot = p.slots[it.b];  // used at the next issue
    const uint32_t bar = smem_u32(&sm.bars[slot_i]);
    const uint32_t row = (uint32_t)b * (uint32_t)p.head_count + (uint32_t)hr;
    const int bits = BITS == 0 ? entry_bits(e) : BITS;
    SlotMeta &m = sm.meta[n & 3];
    m.orow = row;
    m.bits = (uint16_t)bits;
    if (slot < 0 || slot >= p.pool_slots) {
        flag(p.status, kFlagBounds);
        m.skip = 1u;
        m.gblock = 0ull;
        mbar_arrive(bar);
        mbar_arrive(bar);
        return;
    }
    const uint8_t *src = p.pool + (uint64_t)slot * p.req_bytes + e.off;
    m.skip = 0u;
    m.gblock = reinterpret_cast<unsigned long long>(src);
    cp_async4(smem_u32(&sm.scal[slot_i][0]), p.beta + row);
    if (GATE == 0) cp_async4(smem_u32(&sm.scal[slot_i][1]), p.alpha + row);
    cp_async_arrive(bar);
    const uint32_t dst = smem_u32(ring_slot<BITS, GATE, IN_BF16, FIT, SB16>(smem, slot_i));
    const uint32_t blk = SB16 ? head_block_bytes_bf16s(bits, D, D) : head_block_bytes(bits, D, D);
    mbar_arrive_expect_tx(bar, C::LEN - (C::BLK - blk));
    bulk_g2s(dst, src, blk, bar);
    bulk_g2s(dst + C::K_OFF, (const uint8_t *)p.k + (size_t)row * C::ROW_IN, C::ROW_IN, bar);
    bulk_g2s(dst + C::Q_OFF, (const uint8_t *)p.q + (size_t)row * C::ROW_IN, C::ROW_IN, bar);
    bulk_g2s(dst + C::V_OFF, (const uint8_t *)p.v + (size_t)row * C::ROW_IN, C::ROW_IN, bar);
    bulk_g2s(dst + C::W_OFF, p.w + (size_t)hr * D, 4 * D, bar);
    if (GATE != 0) bulk_g2s(dst + C::A_OFF, p.alpha + (size_t)row * D, 4 * D, bar);
}

// Wait for tile n (ring slot n % NS) and compute its row factors, row i = threadIdx.x, with
// per-warp sums of w, q.k and q.(alpha k). Returns false on a timeout.
template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
__device__ __forceinline__ bool precompute_rows(SmemFixed &sm, uint8_t *smem, int n, int my_count)
{
    using C = Cfg<BITS, GATE, IN_BF16, FIT, SB16>;
    if (n >= my_count) return true;
    const int slot_i = n % C::NS;
    const uint32_t phase = (uint32_t)(n / C::NS) & 1u;
    // the verdict is made warp-uniform before any warp-wide shuffle below
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&sm.bars[slot_i]), phase))) return false;
    if (sm.meta[n & 3].skip) return true;  // skipped tile: nothing was loaded
    const int pb = n & 1;
    const Width W = width_of(BITS == 0 ? (int)sm.meta[n & 3].bits : BITS);
    const uint8_t *tile = ring_slot<BITS, GATE, IN_BF16, FIT, SB16>(smem, slot_i);
    const int i = threadIdx.x;
    constexpr bool pivot = BITS == 16;
    const float r = pivot ? 1.f : load_scale(tile + W.soff, i, SB16);
    const float k = load_in<IN_BF16>(tile + C::K_OFF, i);
    const float q = load_in<IN_BF16>(tile + C::Q_OFF, i);
    const float w = reinterpret_cast<const float *>(tile + C::W_OFF)[i];
    const float a = GATE == 0 ? sm.scal[slot_i][1] : reinterpret_cast<const float *>(tile + C::A_OFF)[i];
    // sqrt(w) for w > 0 (the weights are positive) from the SFU reciprocal square root
    const float sw = pivot ? 1.f : w * rsqrtf(w);
    const float kt = (GATE == 2 ? k * a : k) * r;
    const float qt = q * a * r;
    const float rho = a * sw * r, kap = sw * k;
    sm.rowKQ[i] = make_float4(kt, kt, qt, qt);
    sm.rowRK[i] = make_float4(rho, rho, kap, kap);
    if (GATE == 1) {
        const float mu = -sw * a * k;
        channel(smem).rowMu[i] = make_float2(mu, mu);
    }
    if (!pivot) sm.rowRq[pb][i] = fast_rcp(sw * W.qmax);
    float s0 = w, s1 = q * k, s2 = q * a * k;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        if (GATE == 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    if ((i & 31) == 0) {
        sm.rsum[pb][i >> 5][0] = s0;
        sm.rsum[pb][i >> 5][1] = s1;
        sm.rsum[pb][i >> 5][2] = s2;
    }
    return true;
}

// One round of the impact-weighted joint refinement of the scales (the refit), on the tile's
// z_ij = sqrt(w_i) S'_ij / c'_j in Tensor Memory. With the one-pass codes Q_ij = round(z_ij s_i):
//   column step  K_j = sum_i rho_i Q_ij z_ij / sum_i (rho_i Q_ij)^2, c_j = K_j c'_j, stored as c~_j;
//   row step     rho_i = sum_j c'_j^2 K~_j Q_ij z_ij / sum_j c'_j^2 K~_j^2 Q_ij^2, r_i = rho_i /
//                sqrt(w_i), stored as r~_i,
// each kept only if finite and positive. Writes the stored scales, K~_j into colB, c'_j^2 K~_j into
// colG1 and the new s_i = 1 / (sqrt(w_i) r~_i) into rowS. Two CTA barriers; the row sums stay in
// each half-warp. c_one is this thread's column c'_j (j = threadIdx.x); r_one / s_one are the
// one-pass r and s of this lane's row i = 8 cg + rb.
template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
__device__ __forceinline__ bool refit_scales(const TileParams &p, SmemFixed &sm, uint8_t *smem, int n, uint32_t tcol,
                                             const Width &W, float c_one, float r_one, float s_one)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, cg = lane & 15, sub = lane >> 4;
    const int rb = 2 * warp + sub, pb = n & 1;
    constexpr int sb16 = SB16;
    const float *rho = fitmem<BITS, GATE, IN_BF16, FIT, SB16>(smem).rowRho;
    const float2 rnd = make_float2(W.round, W.round), nrnd = make_float2(-W.round, -W.round);
    uint8_t *gsc = reinterpret_cast<uint8_t *>(sm.meta[n & 3].gblock + W.soff);
    tmem_wait_st();
    // ---- column sums over this thread's 16 rows --------------------------------------------
    {
        float2 aN[4], aD[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) aN[pp] = aD[pp] = make_float2(0.f, 0.f);
        float2 cha[8], chb[8];
        tmem_ld16_async(tcol, cha);
        tmem_wait_ld(cha);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float2 (&ch)[8] = (k & 1) ? chb : cha;
            float2 (&nx)[8] = (k & 1) ? cha : chb;
            if (k + 1 < 8) tmem_ld16_async(tcol + 16 * (k + 1), nx);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int i = 8 * (2 * k + r) + rb;
                const float2 s2 = sm.rowS[rpos<FIT>(i)];
                const float2 rr = make_float2(rho[i], rho[i]);
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    const float2 z = ch[4 * r + pp];
                    const float2 q = __fadd2_rn(__ffma2_rn(z, s2, rnd), nrnd);  // the one-pass code
                    const float2 t = __fmul2_rn(q, rr);
                    aN[pp] = __ffma2_rn(t, z, aN[pp]);
                    aD[pp] = __ffma2_rn(t, t, aD[pp]);
                }
            }
            if (k + 1 < 8) tmem_wait_ld(nx);
        }
        // halves 0/1 hold the same columns: half 0 keeps the numerators, half 1 the denominators
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            const float2 send = sub ? aN[pp] : aD[pp];
            const float2 keep = sub ? aD[pp] : aN[pp];
            const float2 got = make_float2(__shfl_xor_sync(0xffffffffu, send.x, 16),
                                           __shfl_xor_sync(0xffffffffu, send.y, 16));
            aN[pp] = __fadd2_rn(keep, got);
        }
        store_cols<FIT>(sm.red + rb * RS, cg, aN);
    }
    __syncthreads();
    // ---- column j = tid: refitted stored scale --------------------------------------------
    {
        const int j = tid;
        const float N = sum4(sm.red + cpos<FIT>(j), 2 * RS), Dn = sum4(sm.red + RS + cpos<FIT>(j), 2 * RS);
        float cf = c_one;
        if (Dn > 0.f) {
            const float cn = round_scale(c_one * (N / Dn), sb16);
            if (isfinite(cn) && cn > 0.f) cf = cn;
        }
        store_scale(gsc, D + j, cf, sb16);
        const float K = cf / c_one;
        sm.colB[cpos<FIT>(j)] = K;
        sm.colG1[cpos<FIT>(j)] = c_one * c_one * K;
    }
    __syncthreads();
    // ---- row sums over this thread's 8 columns, then across the half-warp ---------------------
    float pn[16], pd[16];
    {
        float2 g[4], h[4];
        load_cols<FIT>(sm.colG1, cg, g);
        load_cols<FIT>(sm.colB, cg, h);
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) h[pp] = __fmul2_rn(g[pp], h[pp]);  // c'^2 K~^2
        float2 cha[8], chb[8];
        tmem_ld16_async(tcol, cha);
        tmem_wait_ld(cha);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float2 (&ch)[8] = (k & 1) ? chb : cha;
            float2 (&nx)[8] = (k & 1) ? cha : chb;
            if (k + 1 < 8) tmem_ld16_async(tcol + 16 * (k + 1), nx);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int m = 2 * k + r;
                const float2 s2 = sm.rowS[rpos<FIT>(8 * m + rb)];
                float2 n2 = make_float2(0.f, 0.f), d2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    const float2 z = ch[4 * r + pp];
                    const float2 q = __fadd2_rn(__ffma2_rn(z, s2, rnd), nrnd);
                    n2 = __ffma2_rn(__fmul2_rn(q, g[pp]), z, n2);
                    d2 = __ffma2_rn(__fmul2_rn(q, h[pp]), q, d2);
                }
                pn[m] = n2.x + n2.y;
                pd[m] = d2.x + d2.y;
            }
            if (k + 1 < 8) tmem_wait_ld(nx);
        }
    }
    float *rm = sm.red + rb * RS + cg;
    const float4 *src = reinterpret_cast<const float4 *>(sm.red + rb * RS + cg * RM);
#pragma unroll
    for (int m = 0; m < 16; ++m) rm[m * RM] = pn[m];
    __syncwarp();
    float num;
    {
        const float4 a = src[0], b = src[1], c = src[2], d = src[3];
        num = ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w)) + ((c.x + c.y) + (c.z + c.w)) +
              ((d.x + d.y) + (d.z + d.w));
    }
    __syncwarp();
#pragma unroll
    for (int m = 0; m < 16; ++m) rm[m * RM] = pd[m];
    __syncwarp();
    {
        const float4 a = src[0], b = src[1], c = src[2], d = src[3];
        const float den = ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w)) + ((c.x + c.y) + (c.z + c.w)) +
                          ((d.x + d.y) + (d.z + d.w));
        const int i = 8 * cg + rb;
        float rf = r_one, sf = s_one;
        if (den > 0.f) {
            const float rq = sm.rowRq[pb][i] * W.qmax;  // 1 / sqrt(w_i)
            const float rn = round_scale((num / den) * rq, sb16);
            if (isfinite(rn) && rn > 0.f) {
                rf = rn;
                sf = rq * fast_rcp(rn);
            }
        }
        store_scale(gsc, i, rf, sb16);
        sm.rowS[rpos<FIT>(i)] = make_float2(sf, sf);
    }
    __syncwarp();
    return true;
}

// Sweep A of a tile of width WB: unpack this thread's 16 row segments into Tensor Memory, with
// the column sums of k~Q and q~Q (accumulated into accU / accP).
template <int WB>
__device__ __forceinline__ void sweep_unpack(const uint8_t *tile, const SmemFixed &sm, uint32_t tcol, int rb, int cg,
                                             uint32_t magic, float2 (&accU)[4], float2 (&accP)[4])
{
    constexpr uint32_t RB = WB == 16 ? 256u : 16u * WB;
    constexpr float o = WB == 16 ? 0.f : (float)(1 << (WB - 1));
    constexpr float SIG1 = WB == 4 ? 16.f : WB == 6 ? 64.f : 1.f;
    const float2 off = make_float2(-(8388608.0f + o), -(8388608.0f + o * SIG1));
    const uint8_t *rowsrc = tile + rb * RB + cg * (WB == 16 ? 16 : WB);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
        float2 ch[4];
        unpack_row<WB>(rowsrc + 8 * m * RB, cg, off, magic, ch);
        const float4 kq = sm.rowKQ[8 * m + rb];
        const float2 kk = make_float2(kq.x, kq.y), qq = make_float2(kq.z, kq.w);
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            accU[pp] = __ffma2_rn(kk, ch[pp], accU[pp]);
            accP[pp] = __ffma2_rn(qq, ch[pp], accP[pp]);
        }
        tmem_st8(tcol + 8 * m, ch);
    }
}

// Sweep D of a tile of width WB: x = z s (z / K~_j first with the refit) rounded half to even by
// the FFMA against 2^23 + 2^(b-1), packed, stored to the head block in HBM.
template <int WB, int FIT>
__device__ __forceinline__ void sweep_pack(uint8_t *gblock, const SmemFixed &sm, uint32_t tcol, int rb, int cg)
{
    constexpr uint32_t RB = 16u * WB;
    constexpr float QMAX = (float)((1 << (WB - 1)) - 1);
    const float2 rnd = make_float2(8388608.0f + (float)(1 << (WB - 1)), 8388608.0f + (float)(1 << (WB - 1)));
    uint8_t *dstrow = gblock + rb * RB + cg * WB;
    float2 ik[4];  // 1 / K~_j of this thread's columns (refit only)
    if constexpr (FIT) {
        load_cols<FIT>(sm.colB, cg, ik);
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) ik[pp] = make_float2(fast_rcp(ik[pp].x), fast_rcp(ik[pp].y));
    }
    float2 cha[8], chb[8];
    tmem_ld16_async(tcol, cha);
    tmem_wait_ld(cha);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        float2 (&ch)[8] = (k & 1) ? chb : cha;
        float2 (&nx)[8] = (k & 1) ? cha : chb;
        if (k + 1 < 8) tmem_ld16_async(tcol + 16 * (k + 1), nx);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int m = 2 * k + r;
            const float2 s2 = sm.rowS[rpos<FIT>(8 * m + rb)];
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                if constexpr (FIT) {
                    // x = z / (K~_j rho~_i), clamped (refitted scales may clip), rounded by the add
                    float2 v = __fmul2_rn(__fmul2_rn(ch[4 * r + pp], ik[pp]), s2);
                    v.x = fminf(fmaxf(v.x, -QMAX), QMAX);
                    v.y = fminf(fmaxf(v.y, -QMAX), QMAX);
                    ch[4 * r + pp] = __fadd2_rn(v, rnd);
                } else {
                    ch[4 * r + pp] = __ffma2_rn(ch[4 * r + pp], s2, rnd);
                }
            }
            pack_store_row<WB>(dstrow + 8 * m * RB, cg, ch + 4 * r);
        }
        if (k + 1 < 8) tmem_wait_ld(nx);
    }
}

// Tile n (ring slot n % NS). Returns false if the wait for the next tile timed out.
template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
__device__ __forceinline__ bool process_tile(const TileParams &p, SmemFixed &sm, uint8_t *smem, int n, int my_count,
                                             uint32_t tcol)
{
    using C = Cfg<BITS, GATE, IN_BF16, FIT, SB16>;
    constexpr bool pivot = BITS == 16;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, cg = lane & 15, sub = lane >> 4;
    const int pb = n & 1, slot_i = n % C::NS;
    const int rb = 2 * warp + sub;  // this thread's rows: rb + 8m, m < 16
    const uint8_t *tile = ring_slot<BITS, GATE, IN_BF16, FIT, SB16>(smem, slot_i);
    // the tile's record (sm.meta[n & 3]) stays valid until the issue after the next tile's B2
    const int bits = BITS == 0 ? (int)sm.meta[n & 3].bits : BITS;
    const Width W = width_of(bits);

    // ---- Sweep A: unpack to TMEM, column sums of k~Q and q~Q -------------------------------
    {
        const uint32_t magic = sm.magic;
        float2 accU[4], accP[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) accU[pp] = accP[pp] = make_float2(0.f, 0.f);
        if constexpr (BITS != 0) {
            sweep_unpack<BITS>(tile, sm, tcol, rb, cg, magic, accU, accP);
        } else if (bits == 4) {
            sweep_unpack<4>(tile, sm, tcol, rb, cg, magic, accU, accP);
        } else if (bits == 6) {
            sweep_unpack<6>(tile, sm, tcol, rb, cg, magic, accU, accP);
        } else {
            sweep_unpack<8>(tile, sm, tcol, rb, cg, magic, accU, accP);
        }
        // halves 0/1 of a warp hold the same columns: half 0 keeps U, half 1 keeps P
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            const float2 send = sub ? accU[pp] : accP[pp];
            const float2 keep = sub ? accP[pp] : accU[pp];
            const float2 got = make_float2(__shfl_xor_sync(0xffffffffu, send.x, 16),
                                           __shfl_xor_sync(0xffffffffu, send.y, 16));
            accU[pp] = __fadd2_rn(keep, got);
        }
        store_cols<FIT>(sm.red + rb * RS, cg, accU);
    }
    __syncthreads();  // B1: column partials complete

    // ---- Column finals (column j = tid): update coefficients and the readout ---------------
    const int j = tid;
    constexpr int sb16 = SB16;
    const float cj = pivot ? 1.f : load_scale(tile + W.soff, D + j, sb16);
    const float inv_sig = (j & 1) ? 1.f / W.sig1 : 1.f;  // powers of two: exact
    {
        // k~Q partials in the half-0 regions (0, 2, 4, 6), q~Q partials in the half-1 regions
        const float U = sum4(sm.red + cpos<FIT>(j), 2 * RS) * inv_sig;
        const float P = sum4(sm.red + RS + cpos<FIT>(j), 2 * RS) * inv_sig;
        const float sig = (j & 1) ? W.sig1 : 1.f;
        const float beta = sm.scal[slot_i][0], alpha = sm.scal[slot_i][1];
        const float vj = load_in<IN_BF16>(tile + C::V_OFF, j);
        const float qk = sm.rsum[pb][0][1] + sm.rsum[pb][1][1] + sm.rsum[pb][2][1] + sm.rsum[pb][3][1];
        const float u = cj * U;
        const float rc = pivot ? 1.f : fast_rcp(cj);
        float o;
        if (GATE == 1) {
            const float qak = sm.rsum[pb][0][2] + sm.rsum[pb][1][2] + sm.rsum[pb][2][2] + sm.rsum[pb][3][2];
            sm.colG1[cpos<FIT>(j)] = sig * (beta * vj) * rc;
            channel(smem).colG2[cpos<FIT>(j)] = sig * (beta * u) * rc;
            o = cj * P + (qk * beta * vj - qak * beta * u);
        } else {
            const float h = GATE == 0 ? beta * (vj - alpha * u) : beta * (vj - u);
            sm.colG1[cpos<FIT>(j)] = sig * h * rc;
            o = cj * P + qk * h;
        }
        p.o[(size_t)sm.meta[n & 3].orow * D + j] = o;
        if (!isfinite(o)) flag(p.status, kFlagNonfinite);
    }
    __syncthreads();  // B2: coefficients ready; this tile's ring bytes are no longer read
    if (tid == 0) issue_next<BITS, GATE, IN_BF16, FIT, SB16>(p, sm, smem, sm.iss, my_count);

    // ---- Sweep B: y = rho Q + kappa g1 (+ mu g2), column energy ---------------------------
    tmem_wait_st();
    {
        float2 g1[4], g2[4], accE[4];
        load_cols<FIT>(sm.colG1, cg, g1);
        if (GATE == 1) load_cols<FIT>(channel(smem).colG2, cg, g2);
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) accE[pp] = make_float2(0.f, 0.f);
        bool bad = false;
        float2 cha[8], chb[8];
        tmem_ld16_async(tcol, cha);
        tmem_wait_ld(cha);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float2 (&ch)[8] = (k & 1) ? chb : cha;
            float2 (&nx)[8] = (k & 1) ? cha : chb;
            if (k + 1 < 8) tmem_ld16_async(tcol + 16 * (k + 1), nx);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int i = 8 * (2 * k + r) + rb;
                const float4 rk = sm.rowRK[i];
                const float2 rho = make_float2(rk.x, rk.y), kap = make_float2(rk.z, rk.w);
                float2 mu = make_float2(0.f, 0.f);
                if (GATE == 1) mu = channel(smem).rowMu[i];
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    float2 t = __fmul2_rn(kap, g1[pp]);
                    if (GATE == 1) t = __ffma2_rn(mu, g2[pp], t);
                    const float2 y = __ffma2_rn(rho, ch[4 * r + pp], t);
                    ch[4 * r + pp] = y;
                    if (!pivot) accE[pp] = __ffma2_rn(y, y, accE[pp]);
                    else bad |= !(fabsf(y.x) < 65520.0f) || !(fabsf(y.y) < 65520.0f);
                }
            }
            if constexpr (pivot) {
                // an FP16 pivot head stores S' directly
                uint8_t *gblock = reinterpret_cast<uint8_t *>(sm.meta[n & 3].gblock);
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    uint4 raw;
                    __half2 h0 = __float22half2_rn(ch[4 * r]), h1 = __float22half2_rn(ch[4 * r + 1]);
                    __half2 h2 = __float22half2_rn(ch[4 * r + 2]), h3 = __float22half2_rn(ch[4 * r + 3]);
                    raw.x = *reinterpret_cast<uint32_t *>(&h0);
                    raw.y = *reinterpret_cast<uint32_t *>(&h1);
                    raw.z = *reinterpret_cast<uint32_t *>(&h2);
                    raw.w = *reinterpret_cast<uint32_t *>(&h3);
                    const int i = 8 * (2 * k + r) + rb;
                    *reinterpret_cast<uint4 *>(gblock + i * 256 + cg * 16) = raw;
                }
            } else {
                tmem_st16(tcol + 16 * k, ch);
            }
            if (k + 1 < 8) tmem_wait_ld(nx);
        }
        if (pivot) {
            if (bad) flag(p.status, kFlagNonfinite);
        } else {
            // both halves of a warp add their partner's energies; half 0 publishes
#pragma unroll
            for (int pp = 0; pp < 4; ++pp)
                accE[pp] = __fadd2_rn(accE[pp], make_float2(__shfl_xor_sync(0xffffffffu, accE[pp].x, 16),
                                                            __shfl_xor_sync(0xffffffffu, accE[pp].y, 16)));
            if (sub == 0) store_cols<FIT>(sm.red + 2 * warp * RS + D, cg, accE);
        }
    }
    __syncthreads();  // B3: column energies complete

    // ---- New column scale of column j, then the next tile's row factors -------------------
    float c_one = 1.f;  // the one-pass stored column scale c'_j (kept for the refit)
    if (!pivot) {
        // x = sum_i w_i S'_ij^2 / (sum_i w_i c_j^2) (times sigma_j^2), so c'_j = c_j sqrt(x) / sigma_j
        // and the factor taking y to S'_ij / c'_j is 1 / sqrt(x)
        const float E = sum4(sm.red + D + cpos<FIT>(j), 2 * RS);
        const float wsum = sm.rsum[pb][0][0] + sm.rsum[pb][1][0] + sm.rsum[pb][2][0] + sm.rsum[pb][3][0];
        const float x = E * fast_rcp(wsum);
        float b = rsqrtf(x);
        float c = (cj * inv_sig) * (x * b);
        if (x == 0.f) {  // zero column: scale 1 (a NaN stays NaN)
            c = 1.f;
            b = 0.f;
        } else if (sb16) {  // the codes follow the stored (rounded) scale
            c = round_scale(c, 1);
            b = (cj * inv_sig) * fast_rcp(c);
        }
        c_one = c;
        if (!FIT) store_scale(reinterpret_cast<uint8_t *>(sm.meta[n & 3].gblock + W.soff), D + j, c, sb16);
        if (!isfinite(c) || c == 0.f) flag(p.status, kFlagNonfinite);
        sm.colB[cpos<FIT>(j)] = b;
    }
    const bool ok = precompute_rows<BITS, GATE, IN_BF16, FIT, SB16>(sm, smem, n + 1, my_count);
    if (__syncthreads_or(!ok)) return false;  // B4: new column scales and next row factors ready
    if constexpr (pivot) return true;

    // ---- Sweep C: z = y * c_j / c'_j and the per-row maxima of |z| ---------------------------
    tmem_wait_st();
    {
        float2 bb[4];
        load_cols<FIT>(sm.colB, cg, bb);
        float *rm = sm.red + rb * RS + cg;
        float2 cha[8], chb[8];
        tmem_ld16_async(tcol, cha);
        tmem_wait_ld(cha);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            float2 (&ch)[8] = (k & 1) ? chb : cha;
            float2 (&nx)[8] = (k & 1) ? cha : chb;
            if (k + 1 < 8) tmem_ld16_async(tcol + 16 * (k + 1), nx);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) ch[4 * r + pp] = __fmul2_rn(ch[4 * r + pp], bb[pp]);
                const float2 *z = ch + 4 * r;
                rm[(2 * k + r) * RM] = max3(max3(fabsf(z[0].x), fabsf(z[0].y), fabsf(z[1].x)),
                                            max3(fabsf(z[1].y), fabsf(z[2].x), fabsf(z[2].y)),
                                            fmaxf(fabsf(z[3].x), fabsf(z[3].y)));
            }
            tmem_st16(tcol + 16 * k, ch);
            if (k + 1 < 8) tmem_wait_ld(nx);
        }
    }
    __syncwarp();
    float r_one = 1.f, s_one = 0.f;  // this lane's row (i = 8 cg + rb): one-pass stored r_i and its factor
    {
        // lane cg of this half finishes its row m = cg (i = 8 cg + rb) from the 16 partials
        const float4 *src = reinterpret_cast<const float4 *>(sm.red + rb * RS + cg * RM);
        const float4 a = src[0], b = src[1], c = src[2], d = src[3];
        const float v = max3(max3(max3(a.x, a.y, a.z), max3(a.w, b.x, b.y), max3(b.z, b.w, c.x)),
                             max3(c.y, c.z, c.w), max3(d.x, d.y, fmaxf(d.z, d.w)));
        const int i = 8 * cg + rb;
        // v = max_j |sqrt(w_i) S'_ij / c'_j|: r'_i = v / (sqrt(w_i) qmax), and the factor taking
        // z to the code is 1 / (sqrt(w_i) r'_i) = qmax / v
        float r = v * sm.rowRq[pb][i];
        float s = W.qmax * fast_rcp(v);
        if (v == 0.f) {  // zero row: scale 1
            r = 1.f;
            s = 0.f;
        } else if (sb16) {  // the codes follow the stored (rounded) scale: s = 1 / (sqrt(w_i) r~_i)
            r = round_scale(r, 1);
            s = (sm.rowRq[pb][i] * W.qmax) * fast_rcp(r);
        }
        sm.rowS[rpos<FIT>(i)] = make_float2(s, s);
        if constexpr (FIT) {
            r_one = r;
            s_one = s;
            fitmem<BITS, GATE, IN_BF16, FIT, SB16>(smem).rowRho[i] = r * fast_rcp(sm.rowRq[pb][i] * W.qmax);  // sqrt(w_i) r_i
        } else {
            store_scale(reinterpret_cast<uint8_t *>(sm.meta[n & 3].gblock + W.soff), i, r, sb16);
        }
        if (!isfinite(r) || r == 0.f) flag(p.status, kFlagNonfinite);
    }
    __syncwarp();
    if constexpr (FIT) {
        if (!refit_scales<BITS, GATE, IN_BF16, FIT, SB16>(p, sm, smem, n, tcol, W, c_one, r_one, s_one)) return false;
    }

    // ---- Sweep D: x = z s rounded half to even by the 2^23 + offset FFMA, packed, stored ----
    tmem_wait_st();
    {
        uint8_t *gblock = reinterpret_cast<uint8_t *>(sm.meta[n & 3].gblock);
        if constexpr (BITS != 0) {
            sweep_pack<BITS, FIT>(gblock, sm, tcol, rb, cg);
        } else if (bits == 4) {
            sweep_pack<4, FIT>(gblock, sm, tcol, rb, cg);
        } else if (bits == 6) {
            sweep_pack<6, FIT>(gblock, sm, tcol, rb, cg);
        } else {
            sweep_pack<8, FIT>(gblock, sm, tcol, rb, cg);
        }
    }
    return true;
}

template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
__global__ void __launch_bounds__(NT, 4) decode_d128_kernel(const __grid_constant__ TileParams p)
{
    using C = Cfg<BITS, GATE, IN_BF16, FIT, SB16>;
    extern __shared__ __align__(128) uint8_t smem[];
    SmemFixed &sm = *reinterpret_cast<SmemFixed *>(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int G = (int)gridDim.x;
    const int my_count = (p.ntiles - (int)blockIdx.x + G - 1) / G;
    // A launch that follows this one in the same call (another width or request group: disjoint
    // tiles) may start as its CTAs find room; see launch_t.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {  // Tensor Memory for this CTA's tile (released below on every path)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    if (tid == 0) {
        for (int i = 0; i < C::NS; ++i) mbar_init(smem_u32(&sm.bars[i]), 2);
        fence_mbar_init();
        sm.magic = MAGIC;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // this thread's lane 32 * warp + lane, columns 0..127
    const uint32_t tcol = sm.tmem_base + ((uint32_t)(32 * warp) << 16);

    if (tid == 0) {
        Issuer &it = sm.iss;
        it.n = 0;
        it.pos = (int)blockIdx.x / p.B;
        it.b = (int)blockIdx.x - it.pos * p.B;
        it.qG = G / p.B;
        it.rG = G - it.qG * p.B;
        it.next_slot = my_count > 0 ? p.slots[it.b] : 0;
        for (int k = 0; k < C::NS; ++k) issue_next<BITS, GATE, IN_BF16, FIT, SB16>(p, sm, smem, it, my_count);
    }
    bool failed = __syncthreads_or(!precompute_rows<BITS, GATE, IN_BF16, FIT, SB16>(sm, smem, 0, my_count));

    int n = 0;
    for (; n < my_count && !failed; ++n) {
        // every thread observes the tile's completion itself (already complete: all waited)
        const bool got = mbar_wait_bounded(smem_u32(&sm.bars[n % C::NS]), (uint32_t)(n / C::NS) & 1u);
        if (sm.meta[n & 3].skip) {  // out-of-range slot: nothing loaded, nothing to do
            __syncthreads();
            if (tid == 0) issue_next<BITS, GATE, IN_BF16, FIT, SB16>(p, sm, smem, sm.iss, my_count);
            const bool ok = precompute_rows<BITS, GATE, IN_BF16, FIT, SB16>(sm, smem, n + 1, my_count);
            failed = __syncthreads_or(!ok || !got);
        } else {
            failed = !process_tile<BITS, GATE, IN_BF16, FIT, SB16>(p, sm, smem, n, my_count, tcol);
        }
    }
    if (failed && tid == 0) {
        flag(p.status, kFlagTimeout);
        // let every copy in flight (tiles n .. iss.n - 1) land before the CTA's shared memory is released
        for (int m = n; m < sm.iss.n; ++m)
            mbar_wait_bounded(smem_u32(&sm.bars[m % C::NS]), (uint32_t)((m / C::NS) & 1));
    }
    // release Tensor Memory once every thread's accesses have completed
    tmem_wait_st();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sm.tmem_base), "r"(TMEM_COLS));
    }
    // A launch that went out with programmatic dependent launch may have started before the launch
    // ahead of it finished; it completes only after that one has (a no-op for a launch in plain
    // stream order). Completion of a call's last launch therefore implies completion of the whole
    // call, which is what the work after it on the stream relies on.
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// pdl: this launch follows another launch of the same stq_decode_step call. Those touch disjoint
// tiles, so it may start while the earlier one drains (programmatic dependent launch); the first
// launch of a call is ordered normally after all earlier work on the stream, so every launch of a
// call starts after the previous call has finished.
template <int BITS, int GATE, int IN_BF16, int FIT, int SB16>
cudaError_t launch_t(const TileParams &p, cudaStream_t s, bool pdl)
{
    using C = Cfg<BITS, GATE, IN_BF16, FIT, SB16>;
    auto kernel = decode_d128_kernel<BITS, GATE, IN_BF16, FIT, SB16>;
    const int smem = (int)C::SMEM;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    // The launch geometry of this instance on this device, worked out on its first launch there
    // (per host thread) and reused: resident CTAs per SM from shared memory (+1 KB reserved per
    // CTA), registers and the SM's 512 Tensor Memory columns (TMEM_COLS per CTA). The runtime's
    // occupancy query does not model Tensor Memory and reports 1 for kernels that allocate it.
    static thread_local int cached_dev = -1, cached_cap = 0;
    if (cached_dev != dev) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err != cudaSuccess) return err;
        int sms = 0, smem_sm = 0, regs_sm = 0;
        err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
        if (err != cudaSuccess) return err;
        cudaFuncAttributes fa;
        err = cudaFuncGetAttributes(&fa, kernel);
        if (err != cudaSuccess) return err;
        int per_sm = smem_sm / (smem + 1024);
        const int by_regs = regs_sm / (NT * (fa.numRegs > 0 ? fa.numRegs : 64));
        if (by_regs < per_sm) per_sm = by_regs;
        if (per_sm > (int)(512 / TMEM_COLS)) per_sm = (int)(512 / TMEM_COLS);
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        cached_cap = sms * per_sm;
        cached_dev = dev;
    }
    const int grid = p.ntiles < cached_cap ? p.ntiles : cached_cap;
    if (!pdl) {
        kernel<<<grid, NT, smem, s>>>(p);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <int BITS, int FIT, int SB16>
cudaError_t launch_bits(const TileParams &p, int in_bf16, cudaStream_t s, bool pdl)
{
    switch (p.gate * 2 + (in_bf16 ? 1 : 0)) {
    case 0: return launch_t<BITS, 0, 0, FIT, SB16>(p, s, pdl);
    case 1: return launch_t<BITS, 0, 1, FIT, SB16>(p, s, pdl);
    case 2: return launch_t<BITS, 1, 0, FIT, SB16>(p, s, pdl);
    case 3: return launch_t<BITS, 1, 1, FIT, SB16>(p, s, pdl);
    case 4: return launch_t<BITS, 2, 0, FIT, SB16>(p, s, pdl);
    default: return launch_t<BITS, 2, 1, FIT, SB16>(p, s, pdl);
    }
}

// the refit and the scale format as compile-time parameters of the tuned kernel
template <int BITS>
cudaError_t launch_modes(const TileParams &p, int in_bf16, cudaStream_t s, bool pdl)
{
    const bool fit = p.fit_rounds > 0, sb16 = p.scale_bf16 != 0;
    if (fit) return sb16 ? launch_bits<BITS, 1, 1>(p, in_bf16, s, pdl) : launch_bits<BITS, 1, 0>(p, in_bf16, s, pdl);
    return sb16 ? launch_bits<BITS, 0, 1>(p, in_bf16, s, pdl) : launch_bits<BITS, 0, 0>(p, in_bf16, s, pdl);
}

}  // namespace

// bits = 4, 6, 8: every entry of p.table has that width; bits = 0: any mix of 4, 6 and 8 bits;
// bits = 16: FP16 pivot heads. p.fit_rounds is 0 or 1 (one round of the joint scale refinement;
// FP16 pivot heads have no scales and ignore it).
cudaError_t launch_decode_d128(const TileParams &p, int bits, int in_bf16, cudaStream_t s, bool pdl)
{
    switch (bits) {
    case 0: return launch_modes<0>(p, in_bf16, s, pdl);
    case 4: return launch_modes<4>(p, in_bf16, s, pdl);
    case 6: return launch_modes<6>(p, in_bf16, s, pdl);
    case 8: return launch_modes<8>(p, in_bf16, s, pdl);
    default: return launch_bits<16, 0, 0>(p, in_bf16, s, pdl);  // pivots: no scales
    }
}

}  // namespace stq
