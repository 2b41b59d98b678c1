// prefill_wy.cu -- chunked prefill of 128 x 128 quantized states in the WY / UT form, with the
// dense contractions on the fifth-generation tensor cores (tcgen05, bf16 operands, fp32
// accumulation in Tensor Memory).
//
// Method: the prompt is consumed in chunks; inside a chunk the state is carried unquantized and
// at every chunk end it is refitted and requantized exactly like a decode step ("K1 論文詳解"
// (k1-news.pages.dev/paper/2026-10-09), section 方法: chunked prefill writes the same quantized
// state; "线性注意力状态量化难题" (aitest123.com/news/n1kj09), section 工程落地). The chunk algebra
// is the standard UT transform of the gated delta rule S_t = a_t (S_{t-1} - b_t k_t k_t^T S_{t-1})
// + b_t k_t v_t^T, o_t = S_t^T q_t. With gamma_t = prod_{s<=t} a_s (chunk-relative) and the chunk
// start state S0 = diag(r) Q diag(c):
//   L_ts = b_t (gamma_t / gamma_s) k_t.k_s            (s < t)      T = (I + L)^-1
//   R'_t = b_t (v_t - gamma_t S0^T k_t)                             U = T R'
//   P_ts = (gamma_t / gamma_s) q_t.k_s                 (s <= t)
//   o_t  = gamma_t S0^T q_t + sum_s P_ts U_s
//   S_C  = gamma_C S0 + K^T diag(gamma_C / gamma) U
// Unrolling the per-token recurrence gives exactly these sums; inside a chunk nothing is rounded
// to the state's codes.
//
// Design (B200, one persistent CTA of 512 threads per SM, 512 Tensor Memory columns):
//  * bf16 inputs are exact bf16 MMA operands. fp32 quantities that enter a contraction (K r, Q r,
//    T, R', U, decayed U) are split into three bf16 terms carrying all 24 significand bits; the
//    products keep the terms whose order is at most 2^-24 of the result (P U, which only feeds the
//    readout, uses two terms each). The codes themselves (|Q| <= 127) are exact in bf16.
//  * Five MMA groups per chunk: D1 = [K;Q] K^T, D2 = [K r;Q r] Qcodes, DU = T R', DP = P U and
//    D3 = K^T (decayed U); 64-row operands sit in rows 64..127 of an M = 128 instruction so that
//    every accumulator row is its Tensor Memory lane.
//  * The 64 x 64 unit lower-triangular inverse T is formed on the CUDA cores by 16 x 16 blocks.
//  * K and Q of the next chunk stream in by cp.async while the current chunk finishes; the state
//    stays on chip (codes as bf16 in the B-operand layout, scales in shared memory) between chunks
//    and is packed to HBM once, after the last chunk.
#include "prefill_common.cuh"

namespace stq {
namespace {

using namespace pf;

constexpr int NT = 512;

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t XY_BYTES = 34816;           // one K/Q buffer (32 KB) or the L/T work area
constexpr uint32_t OFF_XY0 = 0;
constexpr uint32_t OFF_XY1 = XY_BYTES;
constexpr uint32_t OFF_QC = 2 * XY_BYTES;      // 69632: codes, bf16, B operand (MN-major), 32 KB
constexpr uint32_t OFF_BIG = OFF_QC + 32768;   // 102400: 96 KB of split operands
constexpr uint32_t OFF_RT = OFF_BIG + 98304;   // 200704: T in three bf16 terms, 24 KB
constexpr uint32_t OFF_SMALL = OFF_RT + 24576; // 225280
// small area
constexpr uint32_t S_BETA = 0;                 // [2][64] f32 (per buffer)
constexpr uint32_t S_ALPHA = 512;              // [2][64] f32
constexpr uint32_t S_LG = 1024;                // [64] f64: log alpha
constexpr uint32_t S_G = 1536;                 // [64] f64: cumulative log decay
constexpr uint32_t S_GAM = 2048;               // [64] f32: gamma_t
constexpr uint32_t S_DC = 2304;                // [64] f32: gamma_C / gamma_t
constexpr uint32_t S_R = 2560;                 // [128] f32 row scales
constexpr uint32_t S_C = 3072;                 // [128] f32 column scales
constexpr uint32_t S_W = 3584;                 // [128] f32 impact weights
constexpr uint32_t S_BAR = 4096;               // 4 mbarriers
constexpr uint32_t S_MISC = 4128;              // tmem base, W sum, gamma_C
constexpr uint32_t SMALL_BYTES = 4224;
constexpr uint32_t SMEM_BYTES = OFF_SMALL + SMALL_BYTES + 1024;  // + alignment slack

// Within the K/Q buffer: [K d0..63 | Q d0..63 | K d64..127 | Q d64..127], 64 rows x 128 B each.
constexpr uint32_t KQ_K0 = 0, KQ_Q0 = 8192, KQ_K1 = 16384, KQ_Q1 = 24576;
// Within BIG: phase 1 = three 32 KB A tiles of D2; phase 2 = R' terms + P terms; phase 3 = U,
// decayed-U and P terms.
constexpr uint32_t BIG_R0 = 0, BIG_R1 = 16384, BIG_R2 = 32768;            // R' terms (MN-major)
constexpr uint32_t BIG_P0 = 49152, BIG_P1 = 57344;                        // P terms (K-major)
constexpr uint32_t BIG_U0 = 0, BIG_U1 = 16384;                            // U terms
constexpr uint32_t BIG_Y0 = 32768, BIG_Y1 = 65536, BIG_Y2 = 81920;        // decayed U terms
// requantization scratch in BIG (after the last MMA of the chunk has completed)
constexpr int LDSQ = 132;                     // row stride (floats) of the weighted squares
constexpr uint32_t BIG_SQ = 0;                // [128][LDSQ] f32 w_i S_ij^2
constexpr uint32_t BIG_RED = 128 * LDSQ * 4;  // [4][128] f32 column-energy partials (per row quarter)
constexpr uint32_t BIG_RMAX = BIG_RED + 2048; // [4][128] f32 row-max partials (per column quarter)

// Tensor Memory columns
constexpr uint32_t TM_D1 = 0, TM_D3 = 0, TM_D2 = 128, TM_DU = 256, TM_DP = 384;

struct PrefillArgs {
    int T;       // tokens of this call
};


// Start loading the K and Q rows of one chunk into a K/Q buffer (rows past the prompt are zero
// filled), and its beta / alpha into ring `buf` of the small area (padding: beta 0, alpha 1).
__device__ __forceinline__ void load_chunk_async(uint8_t *sm, uint32_t kq_off, int buf, const __nv_bfloat16 *kbase,
                                                 const __nv_bfloat16 *qbase, const float *bbase, const float *abase,
                                                 int Lc)
{
    const int tid = threadIdx.x;
    // 2 tensors x 64 rows x 16 chunks of 16 B = 2048 copies, 4 per thread
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int e = tid + NT * k;
        const int tensor = e >> 10, row = (e >> 4) & 63, ch = e & 15;
        const __nv_bfloat16 *src = (tensor ? qbase : kbase) + (size_t)(row < Lc ? row : 0) * D + ch * 8;
        const uint32_t box = (ch >> 3) ? (tensor ? KQ_Q1 : KQ_K1) : (tensor ? KQ_Q0 : KQ_K0);
        const uint32_t dst = smem_u32(sm + kq_off + box + sw128_chunk(row, ch & 7));
        cp_async16(dst, src, row < Lc ? 16u : 0u);
    }
    if (tid < C) {
        float *bb = smf(sm, OFF_SMALL + S_BETA) + buf * C;
        float *aa = smf(sm, OFF_SMALL + S_ALPHA) + buf * C;
        if (tid < Lc) {
            cp_async4(smem_u32(bb + tid), bbase + tid);
            cp_async4(smem_u32(aa + tid), abase + tid);
        } else {
            bb[tid] = 0.f;
            aa[tid] = 1.f;
        }
    }
    cp_async_commit();
}


constexpr int INV_WARP0 = 12;  // warps 12..15 form T while warps 0..11 build the D2 operand
constexpr int MMA_TID = 64;    // issues every MMA group (lane quarter 2: it loads no v rows)

// ---------------------------------------------------------------------------------------------
// The kernel: persistent CTAs over (request, head) tiles of one code width; the chunks of a tile
// run in order. Warp w reads Tensor Memory lane quarter q4 = w % 4 and column quarter cq = w / 4.
// ---------------------------------------------------------------------------------------------
// FIT: one round of the impact-weighted joint refit at every chunk end (a separate instance, so
// that the plain requantization keeps its registers).
template <int BITS, int FIT>
__global__ void __launch_bounds__(NT, 1) prefill_wy_kernel(const __grid_constant__ TileParams p, const int T_tok)
{
    using P = PCfg<BITS>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, derived from the shared array so that accesses stay shared-space
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, cq = warp >> 2;
    float *sR = smf(sm, OFF_SMALL + S_R), *sC = smf(sm, OFF_SMALL + S_C), *sW = smf(sm, OFF_SMALL + S_W);
    double *sLG = smd(sm, OFF_SMALL + S_LG), *sG = smd(sm, OFF_SMALL + S_G);
    float *sGam = smf(sm, OFF_SMALL + S_GAM), *sDC = smf(sm, OFF_SMALL + S_DC);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_SMALL + S_BAR);
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + OFF_SMALL + S_MISC);  // [0] Tensor Memory base
    float *miscf = reinterpret_cast<float *>(misc + 1);                     // [0] sum w, [1] gamma_C
    uint8_t *big = sm + OFF_BIG;

    if (warp == 0) umma::tmem_alloc(smem_u32(misc), 512);
    if (tid == 0) {
        for (int k = 0; k < 4; ++k) mbar_init(smem_u32(&bars[k]), 1);
        fence_mbar_init();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = misc[0];
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);  // this warp's lane quarter
    const int nch = (T_tok + C - 1) / C;
    uint32_t parity = 0;
    bool ok = true;

    for (int n = blockIdx.x; n < p.ntiles && ok; n += gridDim.x) {
        const int b = n % p.B, pos = n / p.B;
        const TileEntry ent = p.table[pos];
        const int head = entry_head(ent);
        const int slot = p.slots[b];
        if (slot < 0 || slot >= p.pool_slots) {
            if (tid == 0) flag(p.status, kFlagBounds);
            continue;
        }
        uint8_t *gblock = p.pool + (uint64_t)slot * p.req_bytes + ent.off;
        const uint64_t trow = (uint64_t)b * (uint64_t)p.head_count + (uint64_t)head;
        const __nv_bfloat16 *kg = reinterpret_cast<const __nv_bfloat16 *>(p.k) + trow * (uint64_t)T_tok * D;
        const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(p.q) + trow * (uint64_t)T_tok * D;
        const __nv_bfloat16 *vg = reinterpret_cast<const __nv_bfloat16 *>(p.v) + trow * (uint64_t)T_tok * D;
        const float *bg = p.beta + trow * (uint64_t)T_tok, *ag = p.alpha + trow * (uint64_t)T_tok;
        float *og = p.o + trow * (uint64_t)T_tok * D;

        // ---- the tile's state onto the chip ----------------------------------------------
        __syncthreads();  // the previous tile is completely done with shared memory
        load_codes_row<BITS>(gblock, sm + OFF_QC, tid >> 2, tid & 3);
        if (tid < D) {
            sR[tid] = load_scale(gblock + P::SOFF, tid, p.scale_bf16);
            sC[tid] = load_scale(gblock + P::SOFF, D + tid, p.scale_bf16);
            sW[tid] = p.w[(size_t)head * D + tid];
        }
        load_chunk_async(sm, OFF_XY0, 0, kg, qg, bg, ag, T_tok < C ? T_tok : C);
        __syncthreads();
        if (warp == 0) {
            float s = sW[lane] + sW[lane + 32] + sW[lane + 64] + sW[lane + 96];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) miscf[0] = s;
        }

#pragma unroll 1
        for (int c = 0; c < nch && ok; ++c, parity ^= 1u) {
            const int t0 = c * C, Lc = (T_tok - t0) < C ? (T_tok - t0) : C;
            const uint32_t kq = (c & 1) ? OFF_XY1 : OFF_XY0;  // this chunk's K / Q
            const uint32_t lt = (c & 1) ? OFF_XY0 : OFF_XY1;  // L / T work, then the next chunk's K / Q
            const int buf = c & 1;
            const float *sBeta = smf(sm, OFF_SMALL + S_BETA) + buf * C;
            const float *sAlpha = smf(sm, OFF_SMALL + S_ALPHA) + buf * C;
            float *Lm = smf(sm, lt), *Tm = smf(sm, lt + 64 * LDL * 4);

            // v rows for R' (lane quarters 0, 1: row t, columns 32 cq .. +31), in flight early
            uint4 vraw[4];
            if (q4 < 2) {
                const int t = 32 * q4 + lane;
                const uint4 *vs = reinterpret_cast<const uint4 *>(vg + (size_t)(t0 + (t < Lc ? t : 0)) * D + 32 * cq);
#pragma unroll
                for (int k = 0; k < 4; ++k) vraw[k] = t < Lc ? vs[k] : make_uint4(0u, 0u, 0u, 0u);
            }
            cp_async_wait_all();
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();

            // ---- D1 = [K;Q] K^T (M 128, N 64) ------------------------------------------
            if (tid == MMA_TID) {
                umma::fence_after_sync();
                const uint32_t base = smem_u32(sm + kq);
                const uint32_t id = umma::idesc_bf16(128, 64, 0, 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma::mma_bf16(tmem + TM_D1, umma::smem_desc(base + o, 16, 1024), umma::smem_desc(base + o, 16, 1024),
                                   id, kk > 0);
                }
                umma::mma_commit(smem_u32(&bars[0]));
            }
            // ---- cumulative log decay of the chunk (fp64), warps 0 and 1 -------------------
            if (tid < C) {
                double g = tid < Lc ? log((double)sAlpha[tid]) : 0.0;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const double y = __shfl_up_sync(0xffffffffu, g, o);
                    if (lane >= o) g += y;
                }
                sLG[tid] = g;  // within-warp inclusive prefix
            }
            __syncthreads();
            if (tid < C) sG[tid] = sLG[tid] + (tid >= 32 ? sLG[31] : 0.0);
            __syncthreads();
            if (tid < C) {
                const double gl = sG[C - 1], g = sG[tid];
                sGam[tid] = (float)exp(g);
                sDC[tid] = (float)exp(gl - g);
                if (tid == 0) miscf[1] = (float)exp(gl);
            }

            // ---- L (lane quarters 0, 1; stored transposed) and P (quarters 2, 3) from D1 ----
            ok = wait_bar(smem_u32(&bars[0]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();
            float pv[16];
            {
                float v[16];
                tmem_ld16(tl + TM_D1 + 16 * cq, v);
                const int t = 32 * (q4 & 1) + lane;
                const double gt = sG[t];
                if (q4 < 2) {
                    const float bt = sBeta[t];
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int s = 16 * cq + u;
                        Lm[s * LDL + t] = s < t ? bt * expf((float)(gt - sG[s])) * v[u] : 0.f;
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int s = 16 * cq + u;
                        pv[u] = s <= t ? expf((float)(gt - sG[s])) * v[u] : 0.f;
                    }
                }
            }
            umma::fence_before_sync();
            __syncthreads();

            if (warp < INV_WARP0) {
                // ---- warps 0..11: A operand of D2, three bf16 terms of [K r; Q r] ------------
                for (int unit = tid; unit < 4 * D; unit += 32 * INV_WARP0) {
                    // the 8 lanes of a load phase take one part of 8 rows: one address of r, and 8
                    // bank quads in the swizzled K / Q boxes and term tiles
                    const int m = (unit & 7) + 8 * (unit >> 5), part = (unit >> 3) & 3, row = m & 63,
                              hb = part >> 1;
                    const uint8_t *xb = sm + kq + (m < 64 ? (hb ? KQ_K1 : KQ_K0) : (hb ? KQ_Q1 : KQ_Q0));
                    uint8_t *a0 = big + hb * 16384, *a1 = a0 + 32768, *a2 = a0 + 65536;
                    const float *rr = sR + 32 * part;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int c8 = 4 * (part & 1) + k;
                        float x[8];
                        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(xb + sw128_chunk(row, c8)), x);
                        const float4 ra = *reinterpret_cast<const float4 *>(rr + 8 * k);
                        const float4 rb = *reinterpret_cast<const float4 *>(rr + 8 * k + 4);
                        x[0] *= ra.x; x[1] *= ra.y; x[2] *= ra.z; x[3] *= ra.w;
                        x[4] *= rb.x; x[5] *= rb.y; x[6] *= rb.z; x[7] *= rb.w;
                        store_split3(a0, a1, a2, sw128_chunk(m, c8), x);
                    }
                }
                umma::fence_proxy_async();
                named_bar(1, 32 * INV_WARP0);
                if (tid == MMA_TID) {
                    umma::fence_after_sync();
                    const uint32_t abase = smem_u32(big), bbase = smem_u32(sm + OFF_QC);
                    const uint32_t id = umma::idesc_bf16(128, 128, 0, 1);
#pragma unroll 1
                    for (int term = 0; term < 3; ++term)
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma::mma_bf16(tmem + TM_D2,
                                           umma::smem_desc(abase + term * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32, 16,
                                                           1024),
                                           umma::smem_desc(bbase + kk * 2048, 16384, 1024), id, (term | kk) != 0);
                    umma::mma_commit(smem_u32(&bars[1]));
                }
            } else {
                // ---- warps 12..15: T = (I + L)^-1 ------------------------------------------
                invert_unit_lower<INV_WARP0>(Lm, Tm);
            }
            __syncthreads();  // T is complete
            {
                // its three bf16 terms, one 8-column unit of one row per thread (all 16 warps)
                static_assert(NT == 64 * 8, "one T unit per thread");
                uint8_t *r0 = sm + OFF_RT;
                // the 8 lanes of a load phase take one unit of 8 rows: 8 bank quads on Tm (row
                // stride 68 floats) and in the swizzled term tiles
                const int t = (tid & 7) + 8 * (tid >> 6), c8 = (tid >> 3) & 7;
                float x[8];
                const float4 xa = *reinterpret_cast<const float4 *>(Tm + t * LDL + 8 * c8);
                const float4 xb4 = *reinterpret_cast<const float4 *>(Tm + t * LDL + 8 * c8 + 4);
                x[0] = xa.x; x[1] = xa.y; x[2] = xa.z; x[3] = xa.w;
                x[4] = xb4.x; x[5] = xb4.y; x[6] = xb4.z; x[7] = xb4.w;
                store_split3(r0, r0 + 8192, r0 + 16384, sw128_chunk(t, c8), x);
                umma::fence_proxy_async();
            }
            __syncthreads();  // L / T are dead: the area takes the next chunk's K / Q
            if (c + 1 < nch) {
                const int t1 = t0 + C, L1 = (T_tok - t1) < C ? (T_tok - t1) : C;
                load_chunk_async(sm, lt, buf ^ 1, kg + (size_t)t1 * D, qg + (size_t)t1 * D, bg + t1, ag + t1, L1);
            }

            // ---- R' (quarters 0, 1) and P terms (quarters 2, 3) once D2 is complete -------
            ok = wait_bar(smem_u32(&bars[1]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();
            if (q4 < 2) {
                const int t = 32 * q4 + lane;
                const float bt = sBeta[t], gt = sGam[t];
                const uint32_t aoff = (cq >> 1) * 8192;
                float v[32];
                umma::tmem_ld32(tl + TM_D2 + 32 * cq, v);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float vv[8], x[8];
                    bf16x8_to_f32(vraw[k], vv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = bt * (vv[e] - gt * (sC[32 * cq + 8 * k + e] * v[8 * k + e]));
                    store_split3(big + BIG_R0, big + BIG_R1, big + BIG_R2, aoff + sw128_chunk(t, 4 * (cq & 1) + k), x);
                }
            } else {
                const int t = 32 * (q4 - 2) + lane;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = pv[8 * k + e];
                    store_split2(big + BIG_P0, big + BIG_P1, sw128_chunk(t, 2 * cq + k), x);
                }
            }
            umma::fence_proxy_async();
            __syncthreads();
            // ---- DU = T R' (rows 64..127 of an M 128 instruction) ---------------------------
            if (tid == MMA_TID) {
                umma::fence_after_sync();
                const uint32_t ta = smem_u32(sm + OFF_RT) - 8192, rb = smem_u32(big);
                const uint32_t id = umma::idesc_bf16(128, 128, 0, 1);
                constexpr int A_T[6] = {0, 0, 1, 0, 1, 2}, B_T[6] = {0, 1, 0, 2, 1, 0};
#pragma unroll
                for (int cmb = 0; cmb < 6; ++cmb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma::mma_bf16(tmem + TM_DU, umma::smem_desc(ta + A_T[cmb] * 8192 + kk * 32, 16, 1024),
                                       umma::smem_desc(rb + B_T[cmb] * 16384 + kk * 2048, 8192, 1024), id,
                                       (cmb | kk) != 0);
                umma::mma_commit(smem_u32(&bars[2]));
            }
            ok = wait_bar(smem_u32(&bars[2]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();
            // ---- U terms and decayed-U terms (quarters 2, 3: row t = lane - 64) --------------
            if (q4 >= 2) {
                const int t = 32 * (q4 - 2) + lane;
                const float dc = sDC[t];
                const uint32_t aoff = (cq >> 1) * 8192;
                float v[32];
                umma::tmem_ld32(tl + TM_DU + 32 * cq, v);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t off = aoff + sw128_chunk(t, 4 * (cq & 1) + k);
                    float x[8], y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        x[e] = v[8 * k + e];
                        y[e] = dc * x[e];
                    }
                    store_split2(big + BIG_U0, big + BIG_U1, off, x);
                    store_split3(big + BIG_Y0, big + BIG_Y1, big + BIG_Y2, off, y);
                }
            }
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();
            // ---- DP = P U (rows 64..127) and D3 = K^T (decayed U) ----------------------------
            if (tid == MMA_TID) {
                umma::fence_after_sync();
                const uint32_t bb = smem_u32(big);
                const uint32_t id = umma::idesc_bf16(128, 128, 0, 1);
                constexpr uint32_t PA[3] = {BIG_P0, BIG_P0, BIG_P1}, UB[3] = {BIG_U0, BIG_U1, BIG_U0};
#pragma unroll
                for (int cmb = 0; cmb < 3; ++cmb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma::mma_bf16(tmem + TM_DP, umma::smem_desc(bb + PA[cmb] - 8192 + kk * 32, 16, 1024),
                                       umma::smem_desc(bb + UB[cmb] + kk * 2048, 8192, 1024), id, (cmb | kk) != 0);
                const uint32_t ka = smem_u32(sm + kq + KQ_K0);
                const uint32_t id3 = umma::idesc_bf16(128, 128, 1, 1);
                constexpr uint32_t YB[3] = {BIG_Y0, BIG_Y1, BIG_Y2};
#pragma unroll
                for (int y = 0; y < 3; ++y)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma::mma_bf16(tmem + TM_D3, umma::smem_desc(ka + kk * 2048, 16384, 1024),
                                       umma::smem_desc(bb + YB[y] + kk * 2048, 8192, 1024), id3, (y | kk) != 0);
                umma::mma_commit(smem_u32(&bars[3]));
            }
            ok = wait_bar(smem_u32(&bars[3]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();

            // ---- readout o_t = gamma_t S0^T q_t + (P U)_t (quarters 2, 3) -------------------
            bool bad = false;
            if (q4 >= 2) {
                const int t = 32 * (q4 - 2) + lane;
                const float gt = sGam[t];
                float a[32], d[32];
                umma::tmem_ld32(tl + TM_D2 + 32 * cq, a);
                umma::tmem_ld32(tl + TM_DP + 32 * cq, d);
                if (t < Lc) {
                    float4 *dst = reinterpret_cast<float4 *>(og + (size_t)(t0 + t) * D + 32 * cq);
                    const float2 gt2 = make_float2(gt, gt);
#pragma unroll
                    for (int u = 0; u < 32; u += 4) {
                        const float4 c4 = *reinterpret_cast<const float4 *>(sC + 32 * cq + u);
                        // gt (c a) + d per element, two at a time
                        const float2 o01 = __ffma2_rn(gt2, __fmul2_rn(make_float2(c4.x, c4.y), make_float2(a[u], a[u + 1])),
                                                      make_float2(d[u], d[u + 1]));
                        const float2 o23 = __ffma2_rn(gt2, __fmul2_rn(make_float2(c4.z, c4.w), make_float2(a[u + 2], a[u + 3])),
                                                      make_float2(d[u + 2], d[u + 3]));
                        const float4 o4 = make_float4(o01.x, o01.y, o23.x, o23.y);
                        bad |= !isfinite(o4.x) || !isfinite(o4.y) || !isfinite(o4.z) || !isfinite(o4.w);
                        dst[u >> 2] = o4;
                    }
                }
            }
            // ---- chunk-end state S_C = gamma_C S0 + D3 (row i, columns 32 cq .. +31) -------
            const int i = 32 * q4 + lane;
            float S[32];
            {
                const float gC = miscf[1], ri = sR[i];
                const uint8_t *qrow = sm + OFF_QC + (cq >> 1) * 16384;
                float v[32];
                umma::tmem_ld32(tl + TM_D3 + 32 * cq, v);
                const float2 gC2 = make_float2(gC, gC), ri2 = make_float2(ri, ri);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float qv[8];
                    bf16x8_to_f32(*reinterpret_cast<const uint4 *>(qrow + sw128_chunk(i, 4 * (cq & 1) + k)), qv);
                    // gC ((ri c_j) Q_ij) + D3_ij per element, two at a time
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const float2 c2 = make_float2(sC[32 * cq + 8 * k + e], sC[32 * cq + 8 * k + e + 1]);
                        const float2 s2 = __ffma2_rn(gC2, __fmul2_rn(__fmul2_rn(ri2, c2), make_float2(qv[e], qv[e + 1])),
                                                     make_float2(v[8 * k + e], v[8 * k + e + 1]));
                        S[8 * k + e] = s2.x;
                        S[8 * k + e + 1] = s2.y;
                    }
                }
            }
            umma::fence_before_sync();
            __syncthreads();  // every use of the chunk-start scales is done

            // ---- requantize: column scales (impact-weighted RMS), row scales, codes -----------
            {
                float *red = smf(big, BIG_RED), *rmax = smf(big, BIG_RMAX), *sq = smf(big, BIG_SQ);
                const float wi = sW[i];
                const float2 wi2 = make_float2(wi, wi);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    // (w_i S) S per element, two at a time
                    const float2 a01 = make_float2(S[4 * k], S[4 * k + 1]), a23 = make_float2(S[4 * k + 2], S[4 * k + 3]);
                    const float2 e01 = __fmul2_rn(__fmul2_rn(wi2, a01), a01), e23 = __fmul2_rn(__fmul2_rn(wi2, a23), a23);
                    *reinterpret_cast<float4 *>(sq + i * LDSQ + 32 * cq + 4 * k) = make_float4(e01.x, e01.y, e23.x, e23.y);
                }
                __syncthreads();
                {
                    // column j = tid % 128 summed over the 32 rows of quarter tid / 128
                    const int j = tid & (D - 1), r0 = 32 * (tid >> 7);
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                    for (int r = 0; r < 32; r += 4) {
                        a0 += sq[(r0 + r) * LDSQ + j];
                        a1 += sq[(r0 + r + 1) * LDSQ + j];
                        a2 += sq[(r0 + r + 2) * LDSQ + j];
                        a3 += sq[(r0 + r + 3) * LDSQ + j];
                    }
                    red[(tid >> 7) * D + j] = (a0 + a1) + (a2 + a3);
                }
                __syncthreads();
                if (tid < D) {
                    const float E = (red[tid] + red[D + tid]) + (red[2 * D + tid] + red[3 * D + tid]);
                    float cj = sqrtf(E / miscf[0]);
                    if (cj == 0.f) cj = 1.f;
                    cj = round_scale(cj, p.scale_bf16);  // the codes follow the stored scale
                    bad |= !isfinite(cj);
                    sC[tid] = cj;
                    red[tid] = __frcp_rn(cj);  // this column's partials have been read
                }
                __syncthreads();
                float m = 0.f;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float2 t = __fmul2_rn(make_float2(S[j], S[j + 1]), make_float2(red[32 * cq + j], red[32 * cq + j + 1]));
                    S[j] = t.x;
                    S[j + 1] = t.y;
                    m = fmaxf(m, fmaxf(fabsf(t.x), fabsf(t.y)));
                }
                rmax[cq * D + i] = m;
                __syncthreads();
                m = fmaxf(fmaxf(rmax[i], rmax[D + i]), fmaxf(rmax[2 * D + i], rmax[3 * D + i]));
                float ri = m / (float)P::QMAX;
                if (ri == 0.f) ri = 1.f;
                ri = round_scale(ri, p.scale_bf16);
                bad |= !isfinite(ri);
                const float rri = __frcp_rn(ri);
                // the codes as exact small integers in fp32: clamped, then rounded half to even by
                // adding and subtracting 1.5 * 2^23 (the same value as rounding, then clamping)
                constexpr float RND = 12582912.0f;
                const float2 rri2 = make_float2(rri, rri), rnd2 = make_float2(RND, RND), nrnd2 = make_float2(-RND, -RND);
                float qc[32];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    float2 x = __fmul2_rn(make_float2(S[j], S[j + 1]), rri2);
                    x.x = fminf(fmaxf(x.x, -(float)P::QMAX), (float)P::QMAX);
                    x.y = fminf(fmaxf(x.y, -(float)P::QMAX), (float)P::QMAX);
                    const float2 q = __fadd2_rn(__fadd2_rn(x, rnd2), nrnd2);
                    qc[j] = q.x;
                    qc[j + 1] = q.y;
                }
                if constexpr (FIT) {
                    // One round of the impact-weighted joint refit (the same round as the decode
                    // kernel's): S[j] holds t_ij = S'_ij / c~_j, qc the one-pass codes.
                    //   c_j <- c~_j sum_i w_i r~_i Q_ij t_ij / sum_i w_i (r~_i Q_ij)^2
                    //   r_i <- sum_j c~new_j c~_j Q_ij t_ij / sum_j (c~new_j Q_ij)^2
                    // each stored (rounded) and kept only if finite and positive.
                    float *red2 = rmax;  // free once the row scales are formed
                    const float wr = wi * ri;
#pragma unroll 1
                    for (int pass = 0; pass < 2; ++pass) {
                        __syncthreads();  // the previous readers of sq / red are done
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            float e[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const float qv = qc[4 * k + u];
                                e[u] = pass == 0 ? wr * qv * S[4 * k + u] : (wr * ri) * (qv * qv);
                            }
                            *reinterpret_cast<float4 *>(sq + i * LDSQ + 32 * cq + 4 * k) = make_float4(e[0], e[1], e[2], e[3]);
                        }
                        __syncthreads();
                        const int j = tid & (D - 1), r0 = 32 * (tid >> 7);
                        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                        for (int r = 0; r < 32; r += 4) {
                            a0 += sq[(r0 + r) * LDSQ + j];
                            a1 += sq[(r0 + r + 1) * LDSQ + j];
                            a2 += sq[(r0 + r + 2) * LDSQ + j];
                            a3 += sq[(r0 + r + 3) * LDSQ + j];
                        }
                        (pass == 0 ? red : red2)[(tid >> 7) * D + j] = (a0 + a1) + (a2 + a3);
                    }
                    __syncthreads();
                    if (tid < D) {
                        const float N = (red[tid] + red[D + tid]) + (red[2 * D + tid] + red[3 * D + tid]);
                        const float Dn = (red2[tid] + red2[D + tid]) + (red2[2 * D + tid] + red2[3 * D + tid]);
                        const float co = sC[tid];
                        float cn = co;
                        if (Dn > 0.f) {
                            const float cr = round_scale(co * (N / Dn), p.scale_bf16);
                            if (isfinite(cr) && cr > 0.f) cn = cr;
                        }
                        red[tid] = cn * co;             // row-step factor of the numerator
                        red2[tid] = cn * cn;            // and of the denominator
                        red[2 * D + tid] = co / cn;     // t -> S' / c~new
                        sC[tid] = cn;
                    }
                    __syncthreads();
                    float pn = 0.f, pd = 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float qv = qc[j];
                        pn += red[32 * cq + j] * qv * S[j];
                        pd += red2[32 * cq + j] * (qv * qv);
                    }
                    sq[cq * D + i] = pn;
                    sq[4 * D + cq * D + i] = pd;
                    __syncthreads();
                    const float num = (sq[i] + sq[D + i]) + (sq[2 * D + i] + sq[3 * D + i]);
                    const float den = (sq[4 * D + i] + sq[5 * D + i]) + (sq[6 * D + i] + sq[7 * D + i]);
                    if (den > 0.f) {
                        const float rn = round_scale(num / den, p.scale_bf16);
                        if (isfinite(rn) && rn > 0.f) ri = rn;
                    }
                    const float rrn = __frcp_rn(ri);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float x =
                            fminf(fmaxf(S[j] * red[2 * D + 32 * cq + j] * rrn, -(float)P::QMAX), (float)P::QMAX);
                        qc[j] = __fadd_rn(__fadd_rn(x, RND), -RND);
                    }
                }
                // next chunk's B operand (row i, columns 32 cq ..) and scales
                uint8_t *qrow = sm + OFF_QC + (cq >> 1) * 16384;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w4[e] = bf2_bits(__floats2bfloat162_rn(qc[8 * k + 2 * e], qc[8 * k + 2 * e + 1]));
                    *reinterpret_cast<uint4 *>(qrow + sw128_chunk(i, 4 * (cq & 1) + k)) =
                        make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
                if (cq == 0) sR[i] = ri;
                if (c + 1 == nch) {  // the last chunk of the call: the state goes back to HBM
                    store_codes_row<BITS>(gblock, i, cq, qc);
                    if (cq == 0) store_scale(gblock + P::SOFF, i, ri, p.scale_bf16);
                    if (tid < D) store_scale(gblock + P::SOFF, D + tid, sC[tid], p.scale_bf16);
                }
            }
            if (bad) flag(p.status, kFlagNonfinite);
            umma::fence_before_sync();
            __syncthreads();
        }
    }
    // release Tensor Memory once every thread's accesses have completed
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 512);
    }
}

template <int BITS, int FIT>
cudaError_t launch_w(const TileParams &p, int T, cudaStream_t s)
{
    auto kernel = prefill_wy_kernel<BITS, FIT>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    int dev = 0, sms = 0;
    err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    const int grid = p.ntiles < sms ? p.ntiles : sms;
    kernel<<<grid, NT, SMEM_BYTES, s>>>(p, T);
    return cudaGetLastError();
}

}  // namespace

// Chunked prefill of 128 x 128 tiles with bf16 inputs and the scalar gate; every entry of
// p.table has width `bits` (4, 6 or 8).
cudaError_t launch_prefill_wy(const TileParams &p, int bits, int T, cudaStream_t s)
{
    const bool fit = p.fit_rounds > 0;  // 0 or 1 here
    switch (bits) {
    case 4: return fit ? launch_w<4, 1>(p, T, s) : launch_w<4, 0>(p, T, s);
    case 6: return fit ? launch_w<6, 1>(p, T, s) : launch_w<6, 0>(p, T, s);
    case 8: return fit ? launch_w<8, 1>(p, T, s) : launch_w<8, 0>(p, T, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace stq
