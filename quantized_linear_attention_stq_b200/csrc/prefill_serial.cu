// prefill_serial.cu -- chunked prefill of 128 x 128 heads token by token with the state held in
// registers: every gate (scalar, channel, channel decay-first), any chunk length, fp32 or bf16
// inputs, 4/6/8-bit heads with row x column scales (one plain requantization per chunk end) and
// FP16 pivot heads.
//
// Method: the gated delta rule token by token, requantized at every chunk end exactly like a
// decode step ("K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), section 方法; "线性注意力状态
// 量化难题" (aitest123.com/news/n1kj09), sections 工程落地 and 空间维度):
//   u_j = sum_i k_i a_i S_ij (a_i = alpha_i for decay-first, else 1)
//   S_ij <- alpha_i (S_ij - beta k_i u_j) + beta k_i v_j        (scalar and channel gates)
//   S_ij <- alpha_i S_ij - beta k_i u_j + beta k_i v_j           (decay-first)
//   o_j = sum_i q_i S_ij
// and at every chunk end c_j = sqrt(sum_i w_i S_ij^2 / sum_i w_i), r_i = max_j |S_ij / c_j| / qmax
// (stored values), Q_ij = RNE(S_ij / c_j / r_i), after which the recurrence continues from
// S_ij = fp32(r_i c_j) Q_ij (an FP16 pivot head rounds S to fp16 instead).
//
// Design: one CTA of 512 threads per (request, head) tile. Thread (column j = tid / 4, quarter
// h = tid % 4) keeps rows 32 h .. 32 h + 31 of column j in registers, so that both sums over i per
// token are 16 paired FMAs plus two shuffles among the column's four threads, and the update is
// one or two paired FMAs per pair of elements with per-column coefficients; no CTA barrier runs
// per token. (Two rows of 64 per thread do not fit: the passes then need ~200 registers.) The token inputs are
// staged 16 tokens at a time by asynchronous copies into a double buffer (k and q converted to
// fp32 once per block, each 32-row quarter padded so that a warp's reads hit distinct banks). A chunk end computes the column scales from thread-pair sums, the row
// maxima by warp shuffles and shared-memory atomic max, and the codes in registers. The pool block is read once at
// the start and written once after the last token.
#include "stq_internal.cuh"

namespace stq {
namespace {

constexpr int NTS = 512;    // threads per CTA
constexpr int DS = 128;     // d_k = d_v
constexpr int TB = 16;      // tokens per staged block
constexpr int RS = DS / 4;  // rows per thread
// k, q and channel alpha of one token as f32 with each 32-row quarter padded by 4 floats, so that
// the 16-byte reads of a warp (four quarters at once) hit distinct banks
constexpr int QST = RS + 4;     // floats from one quarter to the next
constexpr int VST = 4 * QST;    // floats per token
__device__ __forceinline__ int vidx(int i) { return (i >> 5) * QST + (i & 31); }

// Shared memory (bytes). Two staging buffers, each: raw k, q, v (bf16 or f32), beta, alpha (one per
// token or d_k per token), then k and q as f32.
template <int IN_BF16>
struct SerialSmem {
    static constexpr uint32_t ISZ = IN_BF16 ? 2 : 4;
    static constexpr uint32_t RAW_K = 0;
    static constexpr uint32_t RAW_Q = RAW_K + TB * DS * ISZ;
    static constexpr uint32_t RAW_V = RAW_Q + TB * DS * ISZ;
    static constexpr uint32_t BETA = RAW_V + TB * DS * ISZ;
    static constexpr uint32_t ALPHA = BETA + TB * 4;
    static constexpr uint32_t KF = ALPHA + TB * VST * 4;
    static constexpr uint32_t QF = KF + TB * VST * 4;
    static constexpr uint32_t BUF = QF + TB * VST * 4;  // one staging buffer
    static constexpr uint32_t W = 2 * BUF;             // impact weights [128]
    static constexpr uint32_t RMAX = W + DS * 4;       // row maxima [128] (as unsigned bit patterns)
    static constexpr uint32_t MISC = RMAX + DS * 4;    // [0] sum w
    static constexpr uint32_t BYTES = MISC + 16;
    static_assert(BUF % 16 == 0 && KF % 16 == 0 && ALPHA % 16 == 0, "16-byte copies and float4 reads");
};

__device__ __forceinline__ float4 lds4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

template <int IN_BF16>
__device__ __forceinline__ float in_at(const uint8_t *raw, int idx)
{
    if constexpr (IN_BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(raw)[idx]);
    else
        return reinterpret_cast<const float *>(raw)[idx];
}

// Start copying tokens [t0, t0 + n) of one tile into staging buffer `buf` (n <= TB; the rest of
// the block is not read).
template <int IN_BF16>
__device__ __forceinline__ void stage_block(uint8_t *sm, int buf, const TileParams &p, uint64_t trow, int T, int t0,
                                            int n, bool channel)
{
    using L = SerialSmem<IN_BF16>;
    uint8_t *b = sm + buf * L::BUF;
    const int tid = threadIdx.x;
    const uint64_t base = trow * (uint64_t)T + (uint64_t)t0;
    // k, q, v: n rows of DS elements, 16-byte pieces
    constexpr int PER_ROW = DS * L::ISZ / 16;
    const int pieces = n * PER_ROW;
    const uint8_t *gk = reinterpret_cast<const uint8_t *>(p.k) + base * DS * L::ISZ;
    const uint8_t *gq = reinterpret_cast<const uint8_t *>(p.q) + base * DS * L::ISZ;
    const uint8_t *gv = reinterpret_cast<const uint8_t *>(p.v) + base * DS * L::ISZ;
    for (int e = tid; e < pieces; e += NTS) {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(b + L::RAW_K + 16 * e)), "l"(gk + 16 * e)
                     : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(b + L::RAW_Q + 16 * e)), "l"(gq + 16 * e)
                     : "memory");
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(b + L::RAW_V + 16 * e)), "l"(gv + 16 * e)
                     : "memory");
    }
    if (tid < n) cp_async4(smem_u32(b + L::BETA + 4 * tid), p.beta + base + tid);
    if (channel) {  // alpha is only 4-byte aligned: 4-byte copies
        const float *ga = p.alpha + base * DS;
        for (int e = tid; e < n * DS; e += NTS)
            cp_async4(smem_u32(b + L::ALPHA + 4 * ((e / DS) * VST + vidx(e % DS))), ga + e);
    } else if (tid < n) {
        cp_async4(smem_u32(b + L::ALPHA + 4 * tid), p.alpha + base + tid);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int IN_BF16, int GATE>
__global__ void __launch_bounds__(NTS, 1) prefill_serial_kernel(const __grid_constant__ TileParams p, const int T,
                                                                  const int chunk)
{
    using L = SerialSmem<IN_BF16>;
    extern __shared__ __align__(16) uint8_t sm[];
    const int tid = threadIdx.x, j = tid >> 2, h = tid & 3, i0 = RS * h;
    const int b = blockIdx.x % p.B, pos = blockIdx.x / p.B;
    const TileEntry ent = p.table[pos];
    const int head = entry_head(ent), bits = entry_bits(ent);
    const int slot = p.slots[b];
    if (slot < 0 || slot >= p.pool_slots) {
        if (tid == 0) flag(p.status, kFlagBounds);
        return;
    }
    uint8_t *gblock = p.pool + (uint64_t)slot * p.req_bytes + ent.off;
    const uint64_t trow = (uint64_t)b * (uint64_t)p.head_count + (uint64_t)head;
    constexpr bool channel = GATE != 0;
    float *sW = reinterpret_cast<float *>(sm + L::W);
    uint32_t *sRmax = reinterpret_cast<uint32_t *>(sm + L::RMAX);
    float *miscf = reinterpret_cast<float *>(sm + L::MISC);
    const bool pivot = bits == 16;
    const int qmax = (1 << (bits - 1)) - 1;
    const uint32_t soff = scale_offset(bits, DS, DS);

    stage_block<IN_BF16>(sm, 0, p, trow, T, 0, T < TB ? T : TB, channel);
    if (tid < DS) sW[tid] = p.w[(size_t)head * DS + tid];

    // ---- the start state of column j, rows i0 .. i0 + 63 ----------------------------------------
    float S[RS];
    float cj = 1.f;  // this column's stored scale
    if (pivot) {
        const __half *hs = reinterpret_cast<const __half *>(gblock);
#pragma unroll
        for (int r = 0; r < RS; ++r) S[r] = __half2float(hs[(size_t)(i0 + r) * DS + j]);
    } else {
        cj = load_scale(gblock + soff, DS + j, p.scale_bf16);
        const uint32_t *words = reinterpret_cast<const uint32_t *>(gblock);
        const int off = 1 << (bits - 1);
#pragma unroll
        for (int r = 0; r < RS; ++r) {
            const int i = i0 + r;
            const uint32_t bit = (uint32_t)bits * (uint32_t)(i * DS + j), wi = bit >> 5, sh = bit & 31;
            uint32_t u = words[wi] >> sh;
            if (sh + bits > 32) u |= words[wi + 1] << (32 - sh);
            u &= (1u << bits) - 1u;
            const float ri = load_scale(gblock + soff, i, p.scale_bf16);
            S[r] = (ri * cj) * (float)((int)u - off);
        }
    }
    __syncthreads();
    if (tid < 32) {
        float s = sW[tid] + sW[tid + 32] + sW[tid + 64] + sW[tid + 96];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (tid == 0) miscf[0] = s;
    }

    bool bad = false;
    int left = chunk;  // tokens to the next chunk end
    const int nblk = (T + TB - 1) / TB;
    for (int blk = 0; blk < nblk; ++blk) {
        const int buf = blk & 1, t0 = blk * TB, n = (T - t0) < TB ? (T - t0) : TB;
        uint8_t *bb = sm + buf * L::BUF;
        // this block's copies have landed; k and q to f32 once for every thread
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        for (int e = tid; e < n * DS; e += NTS) {
            const int x = (e / DS) * VST + vidx(e % DS);
            reinterpret_cast<float *>(bb + L::KF)[x] = in_at<IN_BF16>(bb + L::RAW_K, e);
            reinterpret_cast<float *>(bb + L::QF)[x] = in_at<IN_BF16>(bb + L::RAW_Q, e);
        }
        __syncthreads();
        if (blk + 1 < nblk) {
            const int t1 = t0 + TB, n1 = (T - t1) < TB ? (T - t1) : TB;
            stage_block<IN_BF16>(sm, buf ^ 1, p, trow, T, t1, n1, channel);
        }
        const float *kf = reinterpret_cast<const float *>(bb + L::KF);
        const float *qf = reinterpret_cast<const float *>(bb + L::QF);
        const float *af = reinterpret_cast<const float *>(bb + L::ALPHA);
        const float *bf = reinterpret_cast<const float *>(bb + L::BETA);
        for (int tt = 0; tt < n; ++tt) {
            const int tok = t0 + tt;
            const float *kt = kf + tt * VST + h * QST, *qt = qf + tt * VST + h * QST;
            const float *at = channel ? af + tt * VST + h * QST : af + tt;
            const float beta = bf[tt];
            const float vj = in_at<IN_BF16>(bb + L::RAW_V, tt * DS + j);
            // u_j = sum_i k_i a_i S_ij over this thread's rows (two chains), then the column's others
            float2 acc = make_float2(0.f, 0.f), acc2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < RS; r += 4) {
                const float4 k4 = lds4(kt + r);
                float2 ka = make_float2(k4.x, k4.y), kb = make_float2(k4.z, k4.w);
                if constexpr (GATE == 2) {
                    const float4 a4 = lds4(at + r);
                    ka = __fmul2_rn(ka, make_float2(a4.x, a4.y));
                    kb = __fmul2_rn(kb, make_float2(a4.z, a4.w));
                }
                acc = __ffma2_rn(ka, make_float2(S[r], S[r + 1]), acc);
                acc2 = __ffma2_rn(kb, make_float2(S[r + 2], S[r + 3]), acc2);
            }
            float u = (acc.x + acc.y) + (acc2.x + acc2.y);
            u += __shfl_xor_sync(0xffffffffu, u, 1);
            u += __shfl_xor_sync(0xffffffffu, u, 2);
            // the update, two rows at a time
            const float bu = beta * u, bv = beta * vj;
            if constexpr (GATE == 0) {
                // alpha (S - beta k u) + beta k v = alpha S + k (beta v - alpha beta u)
                const float al = at[0];
                const float cf = fmaf(-al, bu, bv);
                const float2 al2 = make_float2(al, al), cf2 = make_float2(cf, cf);
#pragma unroll
                for (int r = 0; r < RS; r += 4) {
                    const float4 k4 = lds4(kt + r);
                    const float2 s01 = __ffma2_rn(make_float2(k4.x, k4.y), cf2, __fmul2_rn(al2, make_float2(S[r], S[r + 1])));
                    const float2 s23 = __ffma2_rn(make_float2(k4.z, k4.w), cf2, __fmul2_rn(al2, make_float2(S[r + 2], S[r + 3])));
                    S[r] = s01.x; S[r + 1] = s01.y; S[r + 2] = s23.x; S[r + 3] = s23.y;
                }
            } else if constexpr (GATE == 1) {
                // alpha_i (S - beta k_i u) + beta k_i v
                const float2 nbu = make_float2(-bu, -bu), bv2 = make_float2(bv, bv);
#pragma unroll
                for (int r = 0; r < RS; r += 4) {
                    const float4 k4 = lds4(kt + r);
                    const float4 a4 = lds4(at + r);
                    const float2 ka = make_float2(k4.x, k4.y), kb = make_float2(k4.z, k4.w);
                    const float2 t01 = __ffma2_rn(ka, nbu, make_float2(S[r], S[r + 1]));
                    const float2 t23 = __ffma2_rn(kb, nbu, make_float2(S[r + 2], S[r + 3]));
                    const float2 s01 = __ffma2_rn(make_float2(a4.x, a4.y), t01, __fmul2_rn(ka, bv2));
                    const float2 s23 = __ffma2_rn(make_float2(a4.z, a4.w), t23, __fmul2_rn(kb, bv2));
                    S[r] = s01.x; S[r + 1] = s01.y; S[r + 2] = s23.x; S[r + 3] = s23.y;
                }
            } else {
                // alpha_i S - beta k_i u + beta k_i v = alpha_i S + k_i (beta v - beta u)
                const float cf = bv - bu;
                const float2 cf2 = make_float2(cf, cf);
#pragma unroll
                for (int r = 0; r < RS; r += 4) {
                    const float4 k4 = lds4(kt + r);
                    const float4 a4 = lds4(at + r);
                    const float2 s01 = __ffma2_rn(make_float2(k4.x, k4.y), cf2, __fmul2_rn(make_float2(a4.x, a4.y), make_float2(S[r], S[r + 1])));
                    const float2 s23 = __ffma2_rn(make_float2(k4.z, k4.w), cf2, __fmul2_rn(make_float2(a4.z, a4.w), make_float2(S[r + 2], S[r + 3])));
                    S[r] = s01.x; S[r + 1] = s01.y; S[r + 2] = s23.x; S[r + 3] = s23.y;
                }
            }
            // o_j = sum_i q_i S_ij
            acc = make_float2(0.f, 0.f);
            acc2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < RS; r += 4) {
                const float4 q4 = lds4(qt + r);
                acc = __ffma2_rn(make_float2(q4.x, q4.y), make_float2(S[r], S[r + 1]), acc);
                acc2 = __ffma2_rn(make_float2(q4.z, q4.w), make_float2(S[r + 2], S[r + 3]), acc2);
            }
            float o = (acc.x + acc.y) + (acc2.x + acc2.y);
            o += __shfl_xor_sync(0xffffffffu, o, 1);
            o += __shfl_xor_sync(0xffffffffu, o, 2);
            if (h == 0) {
                p.o[(trow * (uint64_t)T + (uint64_t)tok) * DS + j] = o;
                bad |= !isfinite(o);
            }

            // ---- chunk end: requantize (or round a pivot to fp16), then go on from the stored state
            if (--left == 0 || tok == T - 1) {
                left = chunk;
                if (pivot) {
#pragma unroll
                    for (int r = 0; r < RS; ++r) {
                        bad |= !(fabsf(S[r]) < 65520.0f);  // overflows fp16 (or is NaN)
                        S[r] = __half2float(__float2half_rn(S[r]));
                    }
                } else {
                    // column scale: impact-weighted RMS over the 128 rows (the column's four threads)
                    float e = 0.f;
#pragma unroll
                    for (int r = 0; r < RS; ++r) e = fmaf(sW[i0 + r] * S[r], S[r], e);
                    e += __shfl_xor_sync(0xffffffffu, e, 1);
                    e += __shfl_xor_sync(0xffffffffu, e, 2);
                    float c = sqrtf(e / miscf[0]);
                    if (c == 0.f) c = 1.f;
                    c = round_scale(c, p.scale_bf16);
                    bad |= !isfinite(c);
                    cj = c;
                    const float rc = __frcp_rn(c);
                    if (tid < DS) sRmax[tid] = 0u;
                    __syncthreads();
                    // t = S / c; the row maxima over a warp's 8 columns by shuffles among the lanes
                    // of one row quarter, then across warps by atomic max on the (non-negative) bit
                    // patterns
                    const int lane = tid & 31;
#pragma unroll
                    for (int r = 0; r < RS; ++r) {
                        S[r] *= rc;
                        float m = fabsf(S[r]);
#pragma unroll
                        for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                        if (lane < 4) atomicMax(&sRmax[i0 + r], __float_as_uint(m));
                    }
                    __syncthreads();
                    const float qm = (float)qmax;
#pragma unroll
                    for (int r = 0; r < RS; ++r) {
                        float ri = __uint_as_float(sRmax[i0 + r]) / qm;
                        if (ri == 0.f) ri = 1.f;
                        ri = round_scale(ri, p.scale_bf16);
                        bad |= !isfinite(ri);
                        const float x = fminf(fmaxf(S[r] * __frcp_rn(ri), -qm), qm);
                        const float code = __fadd_rn(__fadd_rn(x, 12582912.0f), -12582912.0f);
                        // the state the recurrence continues from, and the code for the pool
                        S[r] = (ri * c) * code;
                        if (tok == T - 1) reinterpret_cast<int8_t *>(sm)[(i0 + r) * DS + j] = (int8_t)code;
                    }
                    if (tok == T - 1) {
                        // scales to the pool; the codes go out below, row by row
                        if (h == 0) store_scale(gblock + soff, DS + j, c, p.scale_bf16);
                        if (tid < DS) {
                            float ri = __uint_as_float(sRmax[tid]) / qm;
                            if (ri == 0.f) ri = 1.f;
                            store_scale(gblock + soff, tid, round_scale(ri, p.scale_bf16), p.scale_bf16);
                        }
                    }
                    __syncthreads();  // the row maxima are read before the next chunk end rewrites them
                }
            }
        }
        __syncthreads();  // every thread is done with this buffer before it is restaged
    }

    // ---- the final state to the pool -----------------------------------------------------------
    if (pivot) {
        __half *hs = reinterpret_cast<__half *>(gblock);
#pragma unroll
        for (int r = 0; r < RS; ++r) hs[(size_t)(i0 + r) * DS + j] = __float2half_rn(S[r]);
    } else {
        // codes were parked as int8 [i][j] over the first staging buffer (its last block was
        // consumed): thread (row i = tid / 4, quarter) packs columns 32 quarter .. +31 of row i
        __syncthreads();
        const int i = tid >> 2, c0 = RS * (tid & 3);
        const int8_t *qrow = reinterpret_cast<const int8_t *>(sm) + i * DS + c0;
        const int off = 1 << (bits - 1);
        // 32 codes of `bits` bits = `bits` words, starting at bit bits * (128 i + c0) (a multiple of 32)
        uint32_t *dst = reinterpret_cast<uint32_t *>(gblock) + ((uint32_t)bits * (uint32_t)(i * DS + c0) >> 5);
        uint32_t word = 0u;
        int filled = 0, wo = 0;
        for (int x = 0; x < RS; ++x) {
            const uint32_t u = (uint32_t)((int)qrow[x] + off);
            word |= u << filled;
            filled += bits;
            if (filled >= 32) {
                dst[wo++] = word;
                filled -= 32;
                word = filled > 0 ? u >> (bits - filled) : 0u;
            }
        }
    }
    if (bad) flag(p.status, kFlagNonfinite);
}

template <int IN_BF16, int GATE>
cudaError_t launch_s(const TileParams &p, int T, int chunk, cudaStream_t s)
{
    auto kernel = prefill_serial_kernel<IN_BF16, GATE>;
    constexpr uint32_t smem = SerialSmem<IN_BF16>::BYTES;
    static_assert(SerialSmem<IN_BF16>::BUF >= DS * DS, "the int8 code park fits one staging buffer");
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    kernel<<<p.ntiles, NTS, smem, s>>>(p, T, chunk);
    return cudaGetLastError();
}

}  // namespace

// Token-by-token prefill of 128 x 128 heads with the state in registers (any gate, chunk length
// and width of p.table; row x column scales, no refit round).
cudaError_t launch_prefill_serial(const TileParams &p, int in_bf16, int T, int chunk, cudaStream_t s)
{
    switch (p.gate * 2 + (in_bf16 ? 1 : 0)) {
    case 0: return launch_s<0, 0>(p, T, chunk, s);
    case 1: return launch_s<1, 0>(p, T, chunk, s);
    case 2: return launch_s<0, 1>(p, T, chunk, s);
    case 3: return launch_s<1, 1>(p, T, chunk, s);
    case 4: return launch_s<0, 2>(p, T, chunk, s);
    default: return launch_s<1, 2>(p, T, chunk, s);
    }
}

}  // namespace stq
