// prefill_ut.cu -- chunked prefill of 128 x 128 quantized states split into three kernels around a
// device workspace: the parts of a chunk that do not depend on the state run in parallel over all
// chunks, and only the state recurrence runs chunk after chunk.
//
// Method: the same chunk algebra as the one-kernel form (the UT transform of the gated delta rule,
// chunk-end requantization exactly like a decode step: "K1 論文詳解" (k1-news.pages.dev/paper/
// 2026-10-09), section 方法; "线性注意力状态量化难题" (aitest123.com/news/n1kj09), section 工程落地),
// with the state-free factors taken out of U = T R':
//   R'_t = b_t (v_t - gamma_t S0^T k_t)  =>  U = U_v - W S0,  U_v = T diag(b) V,  W = T diag(b gamma) K
// and S0 = diag(r) Q diag(c), so that W S0 = ((W diag(r)) Q) diag(c). Per chunk:
//   inputs kernel   gamma, L and P from [K;Q] K^T, T = (I + L)^-1, W and U_v        (all chunks at once)
//   state kernel    D2 = Q^T (W r)^T, U = U_v - c D2, D3 = K^T (decayed U),
//                   S_C = gamma_C S0 + D3, requantization                          (chunk after chunk)
//   readout kernel  o_t = gamma_t c (Q^T (q r))_t + (P U)_t                         (all chunks at once)
// The contractions run on the tensor cores exactly as in the one-kernel form: bf16 operands, fp32
// accumulation in Tensor Memory, fp32 factors split into three bf16 terms (two for P U). Inside a
// chunk nothing is rounded to the state's codes; at every chunk end the state is requantized.
//
// Each kernel fits two CTAs per SM (256 threads, at most 256 Tensor Memory columns and ~105 KB of
// shared memory each), so that the recurrence runs every (request, head) tile of a launch at once
// and two tiles share an SM's latency. The call is cut into segments of kUtSegmentChunks chunks;
// the workspace holds one record per (tile, chunk of a segment) and the state goes back to the
// pool at every segment end (the state between chunks is the quantized state, so segment ends
// change nothing in the arithmetic).
#include "prefill_common.cuh"

namespace stq {
namespace {

using namespace pf;

constexpr int NT3 = 256;

// One workspace record (per tile and chunk of the segment), byte offsets. The bf16 images are the
// shared-memory operand layouts of the kernels that read them (128-byte swizzle), so that they
// move by plain 16-byte copies.
constexpr uint32_t REC_W = 0;          // [64 t][128 i] f32: W; then two bf16 terms of U^T (K-major image, rows j)
constexpr uint32_t REC_UV = 32768;     // [128 j][64 t] f32: U_v^T
constexpr uint32_t REC_PT = 65536;     // two bf16 terms of P, 8 KB each (K-major image, rows t)
constexpr uint32_t REC_G = 81920;      // [64] gamma_t, [64] gamma_C / gamma_t, gamma_C, 3 pad
constexpr uint32_t REC_ST = 82944;     // the chunk-start state: codes as bf16 (MN-major image, 32 KB),
constexpr uint32_t REC_SC = REC_ST + 32768;  // then r[128] and c[128] as f32 (the stored values)
constexpr uint32_t G_BYTES = 528;      // gamma, decay-to-end, gamma_C and padding
static_assert(REC_SC + 1024 == kUtRecordBytes, "record layout");

// Within a K/Q buffer: [K d0..63 | Q d0..63 | K d64..127 | Q d64..127], 64 rows x 128 B each.
constexpr uint32_t KQ_K0 = 0, KQ_Q0 = 8192, KQ_K1 = 16384, KQ_Q1 = 24576;

struct UtArgs {
    uint8_t *ws;  // workspace, 256-byte aligned
    int T;        // tokens of the call
    int c0;       // first chunk of the segment
    int nsc;      // chunks of the segment
};

__device__ __forceinline__ uint8_t *ut_record(const UtArgs &a, int n, int cc)
{
    return a.ws + ((uint64_t)n * (uint64_t)a.nsc + (uint64_t)cc) * (uint64_t)kUtRecordBytes;
}

__device__ __forceinline__ uint8_t *aligned_smem(uint8_t *raw)
{
    return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

// Bring `bytes` (a multiple of 16 is taken; the rest is left) from global memory into L2.
__device__ __forceinline__ void l2_prefetch(const void *src, uint32_t bytes)
{
    bytes &= ~15u;
    if (bytes) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 64 rows of a bf16 [T][128] input into two swizzled boxes (d 0..63 at box0, 64..127 at box1);
// rows past the prompt are zero filled. 1024 copies of 16 B over NT3 threads.
__device__ __forceinline__ void load_rows_async(uint8_t *box0, uint8_t *box1, const __nv_bfloat16 *src, int Lc)
{
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int e = threadIdx.x + NT3 * k;
        const int row = e >> 4, ch = e & 15;
        const __nv_bfloat16 *g = src + (size_t)(row < Lc ? row : 0) * D + ch * 8;
        cp_async16(smem_u32((ch >> 3 ? box1 : box0) + sw128_chunk(row, ch & 7)), g, row < Lc ? 16u : 0u);
    }
}

// =============================================================================================
// Inputs kernel: per (tile, chunk) unit, gamma, P (two bf16 terms), W and U_v^T.
// =============================================================================================
constexpr uint32_t P1_KQ = 0;                  // K / Q boxes (V replaces Q once D1 is done)
constexpr uint32_t P1_L = 32768;               // f32 L (transposed), then split boxes 0 and 1
constexpr uint32_t P1_T = P1_L + 64 * LDL * 4; // f32 T
constexpr uint32_t P1_SPL = P1_T + 64 * LDL * 4;  // split boxes 2..5
constexpr uint32_t P1_SMALL = P1_SPL + 4 * 8192;
constexpr uint32_t P1S_BETA = 0, P1S_ALPHA = 256, P1S_GAM = 512, P1S_INV = 768, P1S_PW = 1024, P1S_BAR = 1280,
                   P1S_MISC = 1296;
constexpr uint32_t P1_SMEM = P1_SMALL + 1312 + 1024;
static_assert(P1_SPL % 1024 == 0 && P1_L % 1024 == 0, "swizzle atoms");

// Split box b (8 KB, 64 rows t x 64 columns s): T'' term x is box 2x, T' term x is box 2x + 1.
__device__ __forceinline__ uint8_t *p1_box(uint8_t *sm, int b)
{
    return b < 2 ? sm + P1_L + 8192 * b : sm + P1_SPL + 8192 * (b - 2);
}

// W^T and U_v^T of a finished unit (Tensor Memory columns 64..191) to its record: lane li = i for
// W and j for U_v, tokens [t0, t0 + 32 * nq) in nq blocks of 32. W leaves row-major [t][i] (a
// warp writes whole 128-byte rows), U_v^T row-major [j][t].
__device__ __forceinline__ void inputs_readback(uint8_t *rec, uint32_t tl, int li, int t0, int nq)
{
    float *wg = reinterpret_cast<float *>(rec + REC_W);
    for (int b = 0; b < nq; ++b) {
        const int tb = t0 + 32 * b;
        float v[32];
        umma::tmem_ld32(tl + 64 + tb, v);  // W^T[i][t = tb + e]
#pragma unroll
        for (int e = 0; e < 32; ++e) wg[(tb + e) * D + li] = v[e];
        umma::tmem_ld32(tl + 128 + tb, v);  // U_v^T[j][t]
        float4 *ug = reinterpret_cast<float4 *>(rec + REC_UV + (size_t)(li * C + tb) * 4);
#pragma unroll
        for (int k = 0; k < 8; ++k) ug[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    }
}

// The inputs work of one CTA: units first, first + stride, ... of the segment. A unit's W and U_v
// stay in Tensor Memory until the next unit's inverse, during which warps 0..3 (idle then) write
// them out; the last unit's go out after the loop.
__device__ __forceinline__ void inputs_run(const TileParams &p, const UtArgs &a, uint8_t *sm, const int first,
                                           const int stride)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, cq = warp >> 2;
    float *sBeta = smf(sm, P1_SMALL + P1S_BETA), *sAlpha = smf(sm, P1_SMALL + P1S_ALPHA);
    float *sGam = smf(sm, P1_SMALL + P1S_GAM), *sInv = smf(sm, P1_SMALL + P1S_INV);
    double *sPW = smd(sm, P1_SMALL + P1S_PW);  // the two warp-wide partial products of the decay
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + P1_SMALL + P1S_BAR);
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + P1_SMALL + P1S_MISC);
    float *Lm = smf(sm, P1_L), *Tm = smf(sm, P1_T);

    if (warp == 0) umma::tmem_alloc(smem_u32(misc), 256);
    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        fence_mbar_init();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = misc[0];
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
    uint32_t parity = 0;
    bool ok = true;
    const int units = p.ntiles * a.nsc;

    // K, Q, beta and alpha of unit u go into shared memory by asynchronous copies: for the first
    // unit at the top of the loop, for the next ones as soon as the previous unit's last MMA is done
    auto issue_inputs = [&](int uu) {
        const int n1 = uu / a.nsc, cc1 = uu - n1 * a.nsc;
        const uint64_t tr1 = (uint64_t)(n1 % p.B) * (uint64_t)p.head_count + (uint64_t)entry_head(p.table[n1 / p.B]);
        const int t1 = (a.c0 + cc1) * C, L1 = (a.T - t1) < C ? (a.T - t1) : C;
        const uint64_t rb1 = tr1 * (uint64_t)a.T + (uint64_t)t1;
        load_rows_async(sm + P1_KQ + KQ_K0, sm + P1_KQ + KQ_K1, reinterpret_cast<const __nv_bfloat16 *>(p.k) + rb1 * D, L1);
        load_rows_async(sm + P1_KQ + KQ_Q0, sm + P1_KQ + KQ_Q1, reinterpret_cast<const __nv_bfloat16 *>(p.q) + rb1 * D, L1);
        if (tid < C) {
            if (tid < L1) {
                cp_async4(smem_u32(sBeta + tid), p.beta + rb1 + tid);
                cp_async4(smem_u32(sAlpha + tid), p.alpha + rb1 + tid);
            } else {
                sBeta[tid] = 0.f;
                sAlpha[tid] = 1.f;
            }
        }
        cp_async_commit();
    };
    int issued = -1;           // the unit whose inputs are in flight
    uint8_t *pending = nullptr;  // the record whose W / U_v still sit in Tensor Memory

    for (int u = first; u < units && ok; u += stride) {
        const int n = u / a.nsc, cc = u - n * a.nsc;
        const int b = n % p.B, pos = n / p.B;
        const int slot = p.slots[b];
        if (slot < 0 || slot >= p.pool_slots) continue;  // flagged by the state kernel
        const int head = entry_head(p.table[pos]);
        const uint64_t trow = (uint64_t)b * (uint64_t)p.head_count + (uint64_t)head;
        const int t0 = (a.c0 + cc) * C, Lc = (a.T - t0) < C ? (a.T - t0) : C;
        const uint64_t rowbase = trow * (uint64_t)a.T + (uint64_t)t0;
        const __nv_bfloat16 *vg = reinterpret_cast<const __nv_bfloat16 *>(p.v) + rowbase * D;
        uint8_t *rec = ut_record(a, n, cc);

        if (tid == 0 && u + stride < units) {
            // the next unit's V rows into L2 while this one computes
            const int u1 = u + stride, n1 = u1 / a.nsc, cc1 = u1 - n1 * a.nsc;
            const uint64_t tr1 = (uint64_t)(n1 % p.B) * (uint64_t)p.head_count + (uint64_t)entry_head(p.table[n1 / p.B]);
            const int t1 = (a.c0 + cc1) * C, L1 = (a.T - t1) < C ? (a.T - t1) : C;
            l2_prefetch(reinterpret_cast<const __nv_bfloat16 *>(p.v) + (tr1 * (uint64_t)a.T + (uint64_t)t1) * D,
                        (uint32_t)L1 * 256u);
        }
        __syncthreads();  // the previous unit is done with shared memory and Tensor Memory
        if (issued != u) {
            cp_async_wait_all();  // copies for a unit that was skipped
            __syncthreads();
            issue_inputs(u);
        }
        cp_async_wait_all();
        umma::fence_proxy_async();
        umma::fence_before_sync();
        __syncthreads();

        // ---- D1 = [K;Q] K^T (M 128, N 64) -> columns 0..63 ------------------------------
        if (tid == 0) {
            umma::fence_after_sync();
            const uint32_t base = smem_u32(sm + P1_KQ);
            const uint32_t id = umma::idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
                umma::mma_bf16(tmem, umma::smem_desc(base + o, 16, 1024), umma::smem_desc(base + o, 16, 1024), id,
                               kk > 0);
            }
            umma::mma_commit(smem_u32(&bars[0]));
        }
        // ---- cumulative decay of the chunk gamma_t = prod_{s<=t} alpha_s (fp64 products) -----
        double gam_t = 1.0;
        if (tid < C) {
            gam_t = tid < Lc ? (double)sAlpha[tid] : 1.0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double y = __shfl_up_sync(0xffffffffu, gam_t, o);
                if (lane >= o) gam_t *= y;
            }
            if (lane == 31) sPW[warp] = gam_t;
        }
        __syncthreads();
        if (tid < C) {
            if (tid >= 32) gam_t *= sPW[0];
            const double gl = sPW[0] * sPW[1];
            float *gr = reinterpret_cast<float *>(rec + REC_G);
            const float gam = (float)gam_t;
            sGam[tid] = gam;
            sInv[tid] = (float)(1.0 / gam_t);
            gr[tid] = gam;
            gr[C + tid] = (float)(gl / gam_t);
            if (tid == 0) gr[2 * C] = (float)gl;
        }

        // ---- L (lanes 0..63, stored transposed) and the P terms (lanes 64..127) ------------
        ok = wait_bar(smem_u32(&bars[0]), parity, p.status);
        if (!__syncthreads_and(ok)) break;
        umma::fence_after_sync();
        {
            float v[32];
            umma::tmem_ld32(tl + 32 * cq, v);  // columns s = 32 cq + u
            // the decay from token s to token t, gamma_t / gamma_s, as gamma_t * (1 / gamma_s)
            const int t = 32 * (q4 & 1) + lane;
            const float gt = sGam[t];
            if (q4 < 2) {
                const float bt = sBeta[t];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int s = 32 * cq + e;
                    Lm[s * LDL + t] = s < t ? bt * (gt * sInv[s]) * v[e] : 0.f;
                }
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int s = 32 * cq + 8 * k + e;
                        x[e] = s <= t ? (gt * sInv[s]) * v[8 * k + e] : 0.f;
                    }
                    store_split2(rec + REC_PT, rec + REC_PT + 8192, sw128_chunk(t, 4 * cq + k), x);
                }
            }
        }
        umma::fence_before_sync();
        __syncthreads();  // D1 is consumed: the Q boxes take V

        load_rows_async(sm + P1_KQ + KQ_Q0, sm + P1_KQ + KQ_Q1, vg, Lc);
        cp_async_commit();
        if (warp >= 4) {
            invert_unit_lower<4>(Lm, Tm);
        } else if (pending) {
            inputs_readback(pending, tl, 32 * q4 + lane, 0, 2);  // the previous unit, all 64 tokens
            umma::fence_before_sync();
        }
        pending = nullptr;
        cp_async_wait_all();
        umma::fence_proxy_async();
        __syncthreads();  // T is complete and V has landed

        // ---- T' = T diag(beta) and T'' = T diag(beta gamma), three bf16 terms each ----------
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            // the 8 lanes of a load phase take one unit c8 of 8 rows: 8 bank quads on Tm (row
            // stride 68 floats), one broadcast address on beta and gamma
            const int unit = tid + NT3 * k, t = (unit & 7) + 8 * (unit >> 6), c8 = (unit >> 3) & 7;
            float x[8], y[8];
            const float4 xa = *reinterpret_cast<const float4 *>(Tm + t * LDL + 8 * c8);
            const float4 xb = *reinterpret_cast<const float4 *>(Tm + t * LDL + 8 * c8 + 4);
            x[0] = xa.x; x[1] = xa.y; x[2] = xa.z; x[3] = xa.w;
            x[4] = xb.x; x[5] = xb.y; x[6] = xb.z; x[7] = xb.w;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                x[e] *= sBeta[8 * c8 + e];
                y[e] = x[e] * sGam[8 * c8 + e];
            }
            const uint32_t off = sw128_chunk(t, c8);
            store_split3(p1_box(sm, 0), p1_box(sm, 2), p1_box(sm, 4), off, y);
            store_split3(p1_box(sm, 1), p1_box(sm, 3), p1_box(sm, 5), off, x);
        }
        umma::fence_proxy_async();
        umma::fence_before_sync();
        __syncthreads();

        // ---- W^T = K^T T''^T -> columns 64..127, U_v^T = V^T T'^T -> columns 128..191 -------
        if (tid == 0) {
            umma::fence_after_sync();
            const uint32_t kq = smem_u32(sm + P1_KQ);
            const uint32_t id = umma::idesc_bf16(128, 64, 1, 0);
#pragma unroll
            for (int x = 0; x < 3; ++x)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma::mma_bf16(tmem + 64, umma::smem_desc(kq + KQ_K0 + kk * 2048, 16384, 1024),
                                   umma::smem_desc(smem_u32(p1_box(sm, 2 * x)) + kk * 32, 16, 1024), id, (x | kk) != 0);
#pragma unroll
            for (int x = 0; x < 3; ++x)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma::mma_bf16(tmem + 128, umma::smem_desc(kq + KQ_Q0 + kk * 2048, 16384, 1024),
                                   umma::smem_desc(smem_u32(p1_box(sm, 2 * x + 1)) + kk * 32, 16, 1024), id,
                                   (x | kk) != 0);
            umma::mma_commit(smem_u32(&bars[1]));
        }
        ok = wait_bar(smem_u32(&bars[1]), parity, p.status);
        if (!__syncthreads_and(ok)) break;
        umma::fence_after_sync();
        if (u + stride < units) {
            issue_inputs(u + stride);  // K / Q and beta / alpha are free once the MMAs are done
            issued = u + stride;
        }
        pending = rec;
        parity ^= 1u;
    }
    if (ok && pending) {  // the last unit's W / U_v, on all eight warps
        inputs_readback(pending, tl, 32 * q4 + lane, 32 * cq, 1);
        umma::fence_before_sync();
    }
    cp_async_wait_all();
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 256);
    }
}

__global__ void __launch_bounds__(NT3, 2) ut_inputs_kernel(const __grid_constant__ TileParams p, const UtArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    inputs_run(p, a, aligned_smem(smem_raw), blockIdx.x, gridDim.x);
}

// =============================================================================================
// State kernel: per tile, the chunks of the segment in order. The next chunk's W, gamma and K are
// staged into shared memory by asynchronous copies while this chunk requantizes.
// =============================================================================================
constexpr uint32_t P2_QC = 0;       // codes, bf16, A operand of D2 (MN-major, atom columns j 0..63 / 64..127)
constexpr uint32_t P2_BY = 32768;   // staged W (f32, row stride WST floats); (W r) terms; then Y terms (48 KB)
constexpr uint32_t P2_K = 81920;    // K of the chunk, boxes d 0..63 / 64..127 (8 KB each)
constexpr uint32_t P2_SMALL = 98304;
constexpr uint32_t P2S_R = 0, P2S_C = 512, P2S_W = 1024, P2S_RC = 1536, P2S_RED = 2048, P2S_RMAX = 4096,
                   P2S_G = 5120, P2S_BAR = 5664, P2S_MISC = 5680;
constexpr uint32_t P2_SMEM = P2_SMALL + 5696 + 1024;
constexpr int WST = 132;  // row stride (floats) of the staged W: the 8-float reads of a warp hit distinct banks
static_assert(64 * WST * 4 <= 49152, "staged W fits the term area");

// Codes 64 half .. 64 half + 63 of row i (q holds them as exact small integers) into the packed
// rows of a head block.
template <int BITS>
__device__ __forceinline__ void store_codes_half(uint8_t *gblock, int i, int half, const float (&q)[64])
{
    using P = PCfg<BITS>;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
        uint32_t wv[BITS];
#pragma unroll
        for (int k = 0; k < BITS; ++k) wv[k] = 0u;
#pragma unroll
        for (int col = 0; col < 32; ++col) {
            const uint32_t u = (uint32_t)((int)q[32 * part + col] + P::OFFS);
            const int bit = BITS * col, wi = bit >> 5, sh = bit & 31;
            wv[wi] |= u << sh;
            if (sh + BITS > 32) wv[wi + 1] |= u >> (32 - sh);
        }
        uint2 *dst = reinterpret_cast<uint2 *>(gblock + (size_t)i * P::ROWB + (2 * half + part) * (4 * BITS));
#pragma unroll
        for (int k = 0; k < BITS / 2; ++k) dst[k] = make_uint2(wv[2 * k], wv[2 * k + 1]);
    }
}

// Asynchronous copies of a chunk's W (f32 rows of 512 B into rows of WST floats), its gamma block
// and its K rows (zero filled past the prompt).
__device__ __forceinline__ void p2_stage(uint8_t *sm, const uint8_t *rec, const __nv_bfloat16 *krows, int Lc)
{
    const int tid = threadIdx.x;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int e = tid + NT3 * k, t = e >> 5, c4 = e & 31;
        cp_async16(smem_u32(sm + P2_BY + t * (WST * 4) + 16 * c4), rec + REC_W + 16 * e, 16u);
    }
    if (tid < G_BYTES / 16) cp_async16(smem_u32(sm + P2_SMALL + P2S_G + 16 * tid), rec + REC_G + 16 * tid, 16u);
    load_rows_async(sm + P2_K, sm + P2_K + 8192, krows, Lc);
    cp_async_commit();
}

template <int BITS>
__global__ void __launch_bounds__(NT3, 2) ut_state_kernel(const __grid_constant__ TileParams p, const UtArgs a)
{
    using P = PCfg<BITS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_smem(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, cq = warp >> 2;
    float *sR = smf(sm, P2_SMALL + P2S_R), *sC = smf(sm, P2_SMALL + P2S_C), *sW = smf(sm, P2_SMALL + P2S_W);
    float *sRC = smf(sm, P2_SMALL + P2S_RC), *red = smf(sm, P2_SMALL + P2S_RED), *rmax = smf(sm, P2_SMALL + P2S_RMAX);
    const float *sDC = smf(sm, P2_SMALL + P2S_G) + C, *sGC = sDC + C;  // the gamma block as in the record
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + P2_SMALL + P2S_BAR);
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + P2_SMALL + P2S_MISC);  // [0] Tensor Memory base
    float *miscf = reinterpret_cast<float *>(misc + 1);                      // [0] sum w

    if (warp == 0) umma::tmem_alloc(smem_u32(misc), 128);
    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        fence_mbar_init();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = misc[0];
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
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
        const __nv_bfloat16 *kg = reinterpret_cast<const __nv_bfloat16 *>(p.k) + trow * (uint64_t)a.T * D;

        // ---- the tile's state onto the chip; it is the first chunk's start state ---------------
        __syncthreads();  // the previous tile is done with shared memory
        {
            const int t0 = a.c0 * C, Lc = (a.T - t0) < C ? (a.T - t0) : C;
            p2_stage(sm, ut_record(a, n, 0), kg + (size_t)t0 * D, Lc);
        }
        load_codes_row<BITS>(gblock, sm + P2_QC, tid >> 1, 2 * (tid & 1));
        load_codes_row<BITS>(gblock, sm + P2_QC, tid >> 1, 2 * (tid & 1) + 1);
        if (tid < D) {
            sR[tid] = load_scale(gblock + P::SOFF, tid, p.scale_bf16);
            sC[tid] = load_scale(gblock + P::SOFF, D + tid, p.scale_bf16);
            sW[tid] = p.w[(size_t)head * D + tid];
        }
        __syncthreads();
        {
            uint8_t *st = ut_record(a, n, 0) + REC_ST;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int e = tid + NT3 * k;
                *reinterpret_cast<uint4 *>(st + 16 * e) = *reinterpret_cast<const uint4 *>(sm + P2_QC + 16 * e);
            }
            float *sc = reinterpret_cast<float *>(st + 32768);
            sc[tid] = tid < D ? sR[tid] : sC[tid - D];
        }
        if (warp == 0) {
            float s = sW[lane] + sW[lane + 32] + sW[lane + 64] + sW[lane + 96];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) miscf[0] = s;
        }

#pragma unroll 1
        for (int cc = 0; cc < a.nsc && ok; ++cc, parity ^= 1u) {
            uint8_t *rec = ut_record(a, n, cc);
            cp_async_wait_all();  // this chunk's W, gamma and K
            umma::fence_proxy_async();
            __syncthreads();
            // U_v^T [j][32 cq ..] in flight while the D2 operand is built
            const int j = 32 * q4 + lane;
            float uv[32];
            {
                const float4 *ug = reinterpret_cast<const float4 *>(rec + REC_UV + (size_t)(j * C + 32 * cq) * 4);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 x = ug[k];
                    uv[4 * k] = x.x; uv[4 * k + 1] = x.y; uv[4 * k + 2] = x.z; uv[4 * k + 3] = x.w;
                }
            }
            // ---- B operand of D2: three bf16 terms of (W r) [t][i] ----------------------------
            {
                // thread (t, part): 8-float units c8 = part + 4 k of row t, read before any term is
                // written over the staged rows; the 8 lanes of a phase take one unit of 8 rows (8
                // bank quads on the 132-float rows and in the swizzled boxes, one address of r)
                const int t = (tid & 7) + 8 * (tid >> 5), part = (tid >> 3) & 3;
                float x[4][8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float *src = smf(sm, P2_BY + t * (WST * 4) + 32 * (part + 4 * k));
                    const float4 w0 = *reinterpret_cast<const float4 *>(src);
                    const float4 w1 = *reinterpret_cast<const float4 *>(src + 4);
                    x[k][0] = w0.x; x[k][1] = w0.y; x[k][2] = w0.z; x[k][3] = w0.w;
                    x[k][4] = w1.x; x[k][5] = w1.y; x[k][6] = w1.z; x[k][7] = w1.w;
                }
                __syncthreads();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int c8 = part + 4 * k;
                    const float4 r0 = *reinterpret_cast<const float4 *>(sR + 8 * c8);
                    const float4 r1 = *reinterpret_cast<const float4 *>(sR + 8 * c8 + 4);
                    x[k][0] *= r0.x; x[k][1] *= r0.y; x[k][2] *= r0.z; x[k][3] *= r0.w;
                    x[k][4] *= r1.x; x[k][5] *= r1.y; x[k][6] *= r1.z; x[k][7] *= r1.w;
                    uint8_t *box = sm + P2_BY + (c8 >> 3) * 8192;
                    store_split3(box, box + 16384, box + 32768, sw128_chunk(t, c8 & 7), x[k]);
                }
            }
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();
            // ---- D2^T = Q^T (W r)^T (M 128 = j, N 64 = t) -> columns 0..63 ---------------------
            if (tid == 0) {
                umma::fence_after_sync();
                const uint32_t qc = smem_u32(sm + P2_QC), by = smem_u32(sm + P2_BY);
                const uint32_t id = umma::idesc_bf16(128, 64, 1, 0);
#pragma unroll
                for (int x = 0; x < 3; ++x)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma::mma_bf16(tmem, umma::smem_desc(qc + kk * 2048, 16384, 1024),
                                       umma::smem_desc(by + x * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                       id, (x | kk) != 0);
                umma::mma_commit(smem_u32(&bars[0]));
            }
            ok = wait_bar(smem_u32(&bars[0]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();
            // ---- U^T = U_v^T - c D2^T: two bf16 terms to the record (over W, K-major image, rows j);
            //      decayed U as three bf16 terms for D3 ------------------------------------------------
            {
                float d[32];
                umma::tmem_ld32(tl + 32 * cq, d);
                const float ncj = -sC[j];
#pragma unroll
                for (int e = 0; e < 32; ++e) uv[e] = fmaf(ncj, d[e], uv[e]);
                uint8_t *by = sm + P2_BY;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float x[8], y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        x[e] = uv[8 * k + e];
                        y[e] = sDC[32 * cq + 8 * k + e] * x[e];
                    }
                    const uint32_t off = sw128_chunk(j, 4 * cq + k);
                    store_split2(rec + REC_W, rec + REC_W + 16384, off, x);
                    store_split3(by, by + 16384, by + 32768, off, y);
                }
            }
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();
            // ---- D3 = K^T (decayed U) (M 128 = i, N 128 = j) -> columns 0..127 -----------------
            if (tid == 0) {
                umma::fence_after_sync();
                const uint32_t kb = smem_u32(sm + P2_K), by = smem_u32(sm + P2_BY);
                const uint32_t id = umma::idesc_bf16(128, 128, 1, 0);
#pragma unroll
                for (int x = 0; x < 3; ++x)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma::mma_bf16(tmem, umma::smem_desc(kb + kk * 2048, 8192, 1024),
                                       umma::smem_desc(by + x * 16384 + kk * 32, 16, 1024), id, (x | kk) != 0);
                umma::mma_commit(smem_u32(&bars[1]));
            }
            ok = wait_bar(smem_u32(&bars[1]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();

            // ---- chunk-end state S_C = gamma_C S0 + D3 (row i, columns 64 cq .. +63) -----------
            const int i = 32 * q4 + lane;
            float S[64];
            {
                const float gC = sGC[0], ri = sR[i];
                const float2 gC2 = make_float2(gC, gC), ri2 = make_float2(ri, ri);
                const uint8_t *qrow = sm + P2_QC + cq * 16384;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    umma::tmem_ld32(tl + 64 * cq + 32 * hh, v);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float qv[8];
                        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(qrow + sw128_chunk(i, 4 * hh + k)), qv);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const int m = 32 * hh + 8 * k + e;
                            const float2 c2 = make_float2(sC[64 * cq + m], sC[64 * cq + m + 1]);
                            const float2 s2 = __ffma2_rn(gC2, __fmul2_rn(__fmul2_rn(ri2, c2), make_float2(qv[e], qv[e + 1])),
                                                         make_float2(v[8 * k + e], v[8 * k + e + 1]));
                            S[m] = s2.x;
                            S[m + 1] = s2.y;
                        }
                    }
                }
            }
            umma::fence_before_sync();
            __syncthreads();  // the chunk-start codes and scales, gamma, K and the term area are free
            if (cc + 1 < a.nsc) {
                const int t1 = (a.c0 + cc + 1) * C, L1 = (a.T - t1) < C ? (a.T - t1) : C;
                const uint8_t *nrec = ut_record(a, n, cc + 1);
                p2_stage(sm, nrec, kg + (size_t)t1 * D, L1);
                if (tid == 0) l2_prefetch(nrec + REC_UV, 32768u);
            }

            // ---- requantize: column scales (impact-weighted RMS), row scales, codes -------------
            bool bad = false;
            {
                // w_i S_ij^2 summed over the warp's 32 rows by a butterfly that leaves lane l with
                // columns 2l and 2l + 1 of this thread's 64
                const float wi = sW[i];
                const float2 wi2 = make_float2(wi, wi);
                float a1[32];
                {
                    const bool up = (lane & 16) != 0;
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        // (w_i S) S per element, two at a time
                        const float2 s_lo = make_float2(S[e], S[e + 1]), s_hi = make_float2(S[e + 32], S[e + 33]);
                        const float2 lo = __fmul2_rn(__fmul2_rn(wi2, s_lo), s_lo);
                        const float2 hi = __fmul2_rn(__fmul2_rn(wi2, s_hi), s_hi);
                        a1[e] = (up ? hi.x : lo.x) + __shfl_xor_sync(0xffffffffu, up ? lo.x : hi.x, 16);
                        a1[e + 1] = (up ? hi.y : lo.y) + __shfl_xor_sync(0xffffffffu, up ? lo.y : hi.y, 16);
                    }
                }
                float a2[16];
                {
                    const bool up = (lane & 8) != 0;
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        a2[e] = (up ? a1[e + 16] : a1[e]) + __shfl_xor_sync(0xffffffffu, up ? a1[e] : a1[e + 16], 8);
                }
                float a3[8];
                {
                    const bool up = (lane & 4) != 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        a3[e] = (up ? a2[e + 8] : a2[e]) + __shfl_xor_sync(0xffffffffu, up ? a2[e] : a2[e + 8], 4);
                }
                float a4[4];
                {
                    const bool up = (lane & 2) != 0;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        a4[e] = (up ? a3[e + 4] : a3[e]) + __shfl_xor_sync(0xffffffffu, up ? a3[e] : a3[e + 4], 2);
                }
                float a5[2];
                {
                    const bool up = (lane & 1) != 0;
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        a5[e] = (up ? a4[e + 2] : a4[e]) + __shfl_xor_sync(0xffffffffu, up ? a4[e] : a4[e + 2], 1);
                }
                *reinterpret_cast<float2 *>(red + q4 * D + 64 * cq + 2 * lane) = make_float2(a5[0], a5[1]);
            }
            __syncthreads();
            if (tid < D) {
                const float E = (red[tid] + red[D + tid]) + (red[2 * D + tid] + red[3 * D + tid]);
                float cj = sqrtf(E / miscf[0]);
                if (cj == 0.f) cj = 1.f;
                cj = round_scale(cj, p.scale_bf16);  // the codes follow the stored scale
                bad |= !isfinite(cj);
                sC[tid] = cj;
                sRC[tid] = __frcp_rn(cj);
            }
            __syncthreads();
            float m = 0.f;
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
                const float2 t = __fmul2_rn(make_float2(S[e], S[e + 1]),
                                            make_float2(sRC[64 * cq + e], sRC[64 * cq + e + 1]));
                S[e] = t.x;
                S[e + 1] = t.y;
                m = fmaxf(m, fmaxf(fabsf(t.x), fabsf(t.y)));
            }
            rmax[cq * D + i] = m;
            __syncthreads();
            m = fmaxf(rmax[i], rmax[D + i]);
            float ri = m / (float)P::QMAX;
            if (ri == 0.f) ri = 1.f;
            ri = round_scale(ri, p.scale_bf16);
            bad |= !isfinite(ri);
            {
                const float rri = __frcp_rn(ri);
                // the codes as exact small integers in fp32, rounded half to even by adding and
                // subtracting 1.5 * 2^23. With an fp32 r_i that is a normal number no clamp is needed:
                // |S'_ij / c_j| <= m_i and r_i = m_i / qmax, so after the three fp32 roundings
                // |x| <= qmax (1 + 3 * 2^-24) < qmax + 1/2. A bf16 r_i may be up to 2^-8 (relative)
                // below m_i / qmax, which leaves under 0.01 of margin at qmax = 127, and a subnormal
                // r_i has an inexact reciprocal, so there the value is clamped first (the same as
                // rounding, then clamping).
                constexpr float RND = 12582912.0f;
                const float2 rri2 = make_float2(rri, rri), rnd2 = make_float2(RND, RND), nrnd2 = make_float2(-RND, -RND);
                if (p.scale_bf16 || !(ri >= 1.17549435e-38f)) {
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        float2 x = __fmul2_rn(make_float2(S[e], S[e + 1]), rri2);
                        x.x = fminf(fmaxf(x.x, -(float)P::QMAX), (float)P::QMAX);
                        x.y = fminf(fmaxf(x.y, -(float)P::QMAX), (float)P::QMAX);
                        const float2 q = __fadd2_rn(__fadd2_rn(x, rnd2), nrnd2);
                        S[e] = q.x;
                        S[e + 1] = q.y;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const float2 q = __fadd2_rn(__fadd2_rn(__fmul2_rn(make_float2(S[e], S[e + 1]), rri2), rnd2), nrnd2);
                        S[e] = q.x;
                        S[e + 1] = q.y;
                    }
                }
            }
            // next chunk's A operand (row i, columns 64 cq ..) and scales; the same bytes and the
            // stored scales are the next chunk's start state in the workspace, and after the
            // segment's last chunk the packed state goes to the pool
            {
                const bool last = cc + 1 == a.nsc;
                uint8_t *st = last ? nullptr : ut_record(a, n, cc + 1) + REC_ST;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    uint32_t w4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w4[e] = bf2_bits(__floats2bfloat162_rn(S[8 * k + 2 * e], S[8 * k + 2 * e + 1]));
                    const uint4 v4 = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    const uint32_t off = cq * 16384 + sw128_chunk(i, k);
                    *reinterpret_cast<uint4 *>(sm + P2_QC + off) = v4;
                    if (!last) *reinterpret_cast<uint4 *>(st + off) = v4;
                }
                if (cq == 0) sR[i] = ri;
                if (last) {
                    store_codes_half<BITS>(gblock, i, cq, S);
                    if (cq == 0) store_scale(gblock + P::SOFF, i, ri, p.scale_bf16);
                    if (tid < D) store_scale(gblock + P::SOFF, D + tid, sC[tid], p.scale_bf16);
                } else {
                    float *sc = reinterpret_cast<float *>(st + 32768);
                    if (cq == 0) sc[i] = ri;
                    if (tid < D) sc[D + tid] = sC[tid];
                }
            }
            if (bad) flag(p.status, kFlagNonfinite);
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();
        }
    }
    cp_async_wait_all();
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 128);
    }
}

// =============================================================================================
// State kernel of an FP16 pivot head: the state is fp16 (exact as an fp16 MMA operand), W goes in
// as three fp16 terms after an exact power-of-two scaling that keeps its largest magnitude in
// [2^14, 2^15), and the chunk end rounds the state to fp16 (no scales, no codes).
// =============================================================================================
template <int DUMMY = 0>
__global__ void __launch_bounds__(NT3, 2) ut_state_pivot_kernel(const __grid_constant__ TileParams p, const UtArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_smem(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, cq = warp >> 2;
    float *red = smf(sm, P2_SMALL + P2S_RED);
    const float *sDC = smf(sm, P2_SMALL + P2S_G) + C, *sGC = sDC + C;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + P2_SMALL + P2S_BAR);
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + P2_SMALL + P2S_MISC);

    if (warp == 0) umma::tmem_alloc(smem_u32(misc), 128);
    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        fence_mbar_init();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = misc[0];
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
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
        const __nv_bfloat16 *kg = reinterpret_cast<const __nv_bfloat16 *>(p.k) + trow * (uint64_t)a.T * D;
        // thread (row i, columns 64 cq .. +63) owns 8 16-byte pieces of the state, in the pool
        // (row-major fp16) and in the MMA image (atom column cq, row i, swizzled)
        const int i = 32 * q4 + lane;

        // ---- the tile's fp16 state into the A-operand image; it is the first chunk's start state --
        __syncthreads();  // the previous tile is done with shared memory
        {
            const int t0 = a.c0 * C, Lc = (a.T - t0) < C ? (a.T - t0) : C;
            p2_stage(sm, ut_record(a, n, 0), kg + (size_t)t0 * D, Lc);
        }
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(gblock + (size_t)i * (2 * D) + 128 * cq);
            uint8_t *st = ut_record(a, n, 0) + REC_ST;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint4 v4 = src[k];
                const uint32_t off = cq * 16384 + sw128_chunk(i, k);
                *reinterpret_cast<uint4 *>(sm + P2_QC + off) = v4;
                *reinterpret_cast<uint4 *>(st + off) = v4;
            }
        }

#pragma unroll 1
        for (int cc = 0; cc < a.nsc && ok; ++cc, parity ^= 1u) {
            uint8_t *rec = ut_record(a, n, cc);
            cp_async_wait_all();  // this chunk's W, gamma and K
            umma::fence_proxy_async();
            __syncthreads();
            const int j = 32 * q4 + lane;
            float uv[32];
            {
                const float4 *ug = reinterpret_cast<const float4 *>(rec + REC_UV + (size_t)(j * C + 32 * cq) * 4);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 x = ug[k];
                    uv[4 * k] = x.x; uv[4 * k + 1] = x.y; uv[4 * k + 2] = x.z; uv[4 * k + 3] = x.w;
                }
            }
            // ---- B operand of D2: W [t][i] times 2^-e, three fp16 terms ------------------------
            int e2;
            {
                // the 8 lanes of a phase take one unit of 8 rows, as in the coded kernel
                const int t = (tid & 7) + 8 * (tid >> 5), part = (tid >> 3) & 3;
                float x[4][8];
                float mx = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float *src = smf(sm, P2_BY + t * (WST * 4) + 32 * (part + 4 * k));
                    const float4 w0 = *reinterpret_cast<const float4 *>(src);
                    const float4 w1 = *reinterpret_cast<const float4 *>(src + 4);
                    x[k][0] = w0.x; x[k][1] = w0.y; x[k][2] = w0.z; x[k][3] = w0.w;
                    x[k][4] = w1.x; x[k][5] = w1.y; x[k][6] = w1.z; x[k][7] = w1.w;
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(x[k][e]));
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) red[warp] = mx;
                __syncthreads();  // every staged row is read; the maxima are in
                mx = red[0];
#pragma unroll
                for (int w = 1; w < NT3 / 32; ++w) mx = fmaxf(mx, red[w]);
                // e with max |W| 2^-e in [2^14, 2^15) (0 for an all-zero W; a non-finite W gives a
                // non-finite state below, which is flagged)
                e2 = (mx > 0.f && isfinite(mx)) ? ilogbf(mx) - 14 : 0;
                const float down = ldexpf(1.f, -e2);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int c8 = part + 4 * k;
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[k][e] *= down;
                    uint8_t *box = sm + P2_BY + (c8 >> 3) * 8192;
                    store_split3_h(box, box + 16384, box + 32768, sw128_chunk(t, c8 & 7), x[k]);
                }
            }
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();
            // ---- D2^T 2^-e = S0^T (W 2^-e)^T (fp16 operands, M 128 = j, N 64 = t) -> columns 0..63
            if (tid == 0) {
                umma::fence_after_sync();
                const uint32_t qc = smem_u32(sm + P2_QC), by = smem_u32(sm + P2_BY);
                const uint32_t id = umma::idesc_f16(128, 64, 1, 0);
#pragma unroll
                for (int x = 0; x < 3; ++x)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma::mma_bf16(tmem, umma::smem_desc(qc + kk * 2048, 16384, 1024),
                                       umma::smem_desc(by + x * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                       id, (x | kk) != 0);
                umma::mma_commit(smem_u32(&bars[0]));
            }
            ok = wait_bar(smem_u32(&bars[0]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();
            // ---- U^T = U_v^T - D2^T: two bf16 terms to the record; decayed U in three bf16 terms -
            {
                float d[32];
                umma::tmem_ld32(tl + 32 * cq, d);
                const float up = -ldexpf(1.f, e2);
#pragma unroll
                for (int e = 0; e < 32; ++e) uv[e] = fmaf(up, d[e], uv[e]);
                uint8_t *by = sm + P2_BY;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float x[8], y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        x[e] = uv[8 * k + e];
                        y[e] = sDC[32 * cq + 8 * k + e] * x[e];
                    }
                    const uint32_t off = sw128_chunk(j, 4 * cq + k);
                    store_split2(rec + REC_W, rec + REC_W + 16384, off, x);
                    store_split3(by, by + 16384, by + 32768, off, y);
                }
            }
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();
            // ---- D3 = K^T (decayed U) -> columns 0..127 -----------------------------------------
            if (tid == 0) {
                umma::fence_after_sync();
                const uint32_t kb = smem_u32(sm + P2_K), by = smem_u32(sm + P2_BY);
                const uint32_t id = umma::idesc_bf16(128, 128, 1, 0);
#pragma unroll
                for (int x = 0; x < 3; ++x)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma::mma_bf16(tmem, umma::smem_desc(kb + kk * 2048, 8192, 1024),
                                       umma::smem_desc(by + x * 16384 + kk * 32, 16, 1024), id, (x | kk) != 0);
                umma::mma_commit(smem_u32(&bars[1]));
            }
            ok = wait_bar(smem_u32(&bars[1]), parity, p.status);
            if (!__syncthreads_and(ok)) break;
            umma::fence_after_sync();

            // ---- chunk end: S_C = gamma_C S0 + D3, rounded to fp16 (row i, columns 64 cq .. +63) --
            uint4 out[8];
            bool bad = false;
            {
                const float gC = sGC[0];
                const uint8_t *srow = sm + P2_QC + cq * 16384;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float v[32];
                    umma::tmem_ld32(tl + 64 * cq + 32 * hh, v);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float s0[8];
                        f16x8_to_f32(*reinterpret_cast<const uint4 *>(srow + sw128_chunk(i, 4 * hh + k)), s0);
                        uint32_t w4[4];
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const float x0 = fmaf(gC, s0[e], v[8 * k + e]);
                            const float x1 = fmaf(gC, s0[e + 1], v[8 * k + e + 1]);
                            bad |= !(fabsf(x0) < 65520.0f) || !(fabsf(x1) < 65520.0f);  // overflows fp16 (or NaN)
                            const __half2 h = __floats2half2_rn(x0, x1);
                            w4[e >> 1] = *reinterpret_cast<const uint32_t *>(&h);
                        }
                        out[4 * hh + k] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            umma::fence_before_sync();
            __syncthreads();  // the chunk-start state, gamma, K and the term area are free
            if (cc + 1 < a.nsc) {
                const int t1 = (a.c0 + cc + 1) * C, L1 = (a.T - t1) < C ? (a.T - t1) : C;
                const uint8_t *nrec = ut_record(a, n, cc + 1);
                p2_stage(sm, nrec, kg + (size_t)t1 * D, L1);
                if (tid == 0) l2_prefetch(nrec + REC_UV, 32768u);
            }
            {
                // the next chunk's A operand; the same bytes are its start state in the workspace,
                // and after the segment's last chunk the state goes to the pool (row-major fp16)
                const bool last = cc + 1 == a.nsc;
                uint8_t *st = last ? nullptr : ut_record(a, n, cc + 1) + REC_ST;
                uint4 *prow = reinterpret_cast<uint4 *>(gblock + (size_t)i * (2 * D) + 128 * cq);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t off = cq * 16384 + sw128_chunk(i, k);
                    *reinterpret_cast<uint4 *>(sm + P2_QC + off) = out[k];
                    if (last) prow[k] = out[k];
                    else *reinterpret_cast<uint4 *>(st + off) = out[k];
                }
            }
            if (bad) flag(p.status, kFlagNonfinite);
            umma::fence_proxy_async();
            umma::fence_before_sync();
            __syncthreads();
        }
    }
    cp_async_wait_all();
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 128);
    }
}

// =============================================================================================
// Readout kernel: per (tile, chunk) unit, o_t = gamma_t c (Q^T (q r))_t + (P U)_t. The chunk-start
// codes, the U and P terms and the scales arrive as images by asynchronous copies.
// =============================================================================================
constexpr uint32_t P3_QC = 0;       // chunk-start codes, bf16 (A operand of D_a, MN-major)
constexpr uint32_t P3_X = 32768;    // U^T terms (2 x 16 KB) and P terms (2 x 8 KB); then (q r) terms (3 x 16 KB)
constexpr uint32_t P3_SMALL = 81920;
// r is kept as four 32-float parts at a 36-float stride (RPS): the parts that a warp's lanes read
// at once sit on different banks
constexpr int RPS = 36;
constexpr uint32_t P3S_R = 0, P3S_C = 4 * RPS * 4, P3S_GAM = P3S_C + 512, P3S_BAR = P3S_GAM + 256,
                   P3S_MISC = P3S_BAR + 16;
constexpr uint32_t P3_SMEM = P3_SMALL + P3S_MISC + 16 + 1024;
constexpr int OST = 132;  // row stride (floats) of the readout staged over the term area
static_assert(64 * OST * 4 <= 49152, "readout rows fit the term area");

// The readout work of one CTA: units first, first + stride, ... of the segment. For FP16 pivot
// heads (`pivot`) the chunk-start state image is fp16 and unscaled (r = c = 1): D_a takes q as one
// fp16 term (q has |q_i| <= 1; below 2^-17 fp16 keeps it to 2^-25).
__device__ __forceinline__ void readout_run(const TileParams &p, const UtArgs &a, uint8_t *sm, const int first,
                                            const int stride, const bool pivot)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, cq = warp >> 2;
    float *sR = smf(sm, P3_SMALL + P3S_R), *sC = smf(sm, P3_SMALL + P3S_C), *sGam = smf(sm, P3_SMALL + P3S_GAM);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + P3_SMALL + P3S_BAR);
    uint32_t *misc = reinterpret_cast<uint32_t *>(sm + P3_SMALL + P3S_MISC);
    uint8_t *X = sm + P3_X;

    if (warp == 0) umma::tmem_alloc(smem_u32(misc), 128);
    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        fence_mbar_init();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = misc[0];
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);
    uint32_t parity = 0;
    bool ok = true;
    const int units = p.ntiles * a.nsc;

    for (int u = first; u < units && ok; u += stride) {
        const int n = u / a.nsc, cc = u - n * a.nsc;
        const int b = n % p.B, pos = n / p.B;
        const int slot = p.slots[b];
        if (slot < 0 || slot >= p.pool_slots) continue;  // flagged by the state kernel
        const int head = entry_head(p.table[pos]);
        const uint64_t trow = (uint64_t)b * (uint64_t)p.head_count + (uint64_t)head;
        const int t0 = (a.c0 + cc) * C, Lc = (a.T - t0) < C ? (a.T - t0) : C;
        const uint64_t rowbase = trow * (uint64_t)a.T + (uint64_t)t0;
        const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(p.q) + rowbase * D;
        float *og = p.o + rowbase * D;
        const uint8_t *rec = ut_record(a, n, cc);

        __syncthreads();  // the previous unit is done with shared memory and Tensor Memory
        // codes (32 KB), U terms (32 KB), P terms (16 KB), r and c (1 KB), gamma (256 B)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int e = tid + NT3 * k;
            cp_async16(smem_u32(sm + P3_QC + 16 * e), rec + REC_ST + 16 * e, 16u);
            cp_async16(smem_u32(X + 16 * e), rec + REC_W + 16 * e, 16u);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int e = tid + NT3 * k;
            cp_async16(smem_u32(X + 32768 + 16 * e), rec + REC_PT + 16 * e, 16u);
        }
        if (tid < 64) {
            // r (chunks 0..31: part tid / 8 of the padded parts) and c (chunks 32..63)
            uint8_t *dst = tid < 32 ? reinterpret_cast<uint8_t *>(sR) + 4 * RPS * (tid >> 3) + 16 * (tid & 7)
                                    : reinterpret_cast<uint8_t *>(sC) + 16 * (tid - 32);
            if (!pivot) cp_async16(smem_u32(dst), rec + REC_SC + 16 * tid, 16u);
        } else if (tid < 80) {
            cp_async16(smem_u32(reinterpret_cast<uint8_t *>(sGam) + 16 * (tid - 64)), rec + REC_G + 16 * (tid - 64), 16u);
        }
        cp_async_commit();
        // q row t, columns 32 part .. +31, in registers for the (q r) terms; the 8 lanes of a
        // phase take one part of 8 rows, so that their term stores fall in 8 bank quads
        const int t = (tid & 7) + 8 * (tid >> 5), part = (tid >> 3) & 3;
        uint4 qraw[4];
        {
            const uint4 *qs = reinterpret_cast<const uint4 *>(qg + (size_t)(t < Lc ? t : 0) * D + 32 * part);
#pragma unroll
            for (int k = 0; k < 4; ++k) qraw[k] = t < Lc ? qs[k] : make_uint4(0u, 0u, 0u, 0u);
        }
        if (tid == 0 && u + stride < units) {
            // the next unit's record and q rows into L2
            const int u1 = u + stride, n1 = u1 / a.nsc, cc1 = u1 - n1 * a.nsc;
            const uint64_t tr1 = (uint64_t)(n1 % p.B) * (uint64_t)p.head_count + (uint64_t)entry_head(p.table[n1 / p.B]);
            const int t1 = (a.c0 + cc1) * C, L1 = (a.T - t1) < C ? (a.T - t1) : C;
            const uint8_t *r1 = ut_record(a, n1, cc1);
            l2_prefetch(r1 + REC_W, 32768u);
            l2_prefetch(r1 + REC_PT, 16384u + 1024u);
            l2_prefetch(r1 + REC_ST, 32768u + 1024u);
            l2_prefetch(reinterpret_cast<const __nv_bfloat16 *>(p.q) + (tr1 * (uint64_t)a.T + (uint64_t)t1) * D,
                        (uint32_t)L1 * 256u);
        }
        cp_async_wait_all();
        umma::fence_proxy_async();
        umma::fence_before_sync();
        __syncthreads();
        // ---- D_b = U^T P^T (M 128 = j, N 64 = t) -> columns 64..127 ----------------------------
        if (tid == 0) {
            umma::fence_after_sync();
            const uint32_t x0 = smem_u32(X);
            const uint32_t id = umma::idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t UA[3] = {0, 16384, 0}, PB[3] = {32768, 32768, 40960};
#pragma unroll
            for (int cmb = 0; cmb < 3; ++cmb)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma::mma_bf16(tmem + 64, umma::smem_desc(x0 + UA[cmb] + kk * 32, 16, 1024),
                                   umma::smem_desc(x0 + PB[cmb] + kk * 32, 16, 1024), id, (cmb | kk) != 0);
            umma::mma_commit(smem_u32(&bars[0]));
        }
        ok = wait_bar(smem_u32(&bars[0]), parity, p.status);
        if (!__syncthreads_and(ok)) break;
        // ---- three bf16 terms of (q r) [t][i] over the same area (K-major B, rows t); for a
        //      pivot, q as one fp16 term -----------------------------------------------------------
        if (pivot) {
            uint8_t *box = X + (part >> 1) * 8192;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float x[8];
                bf16x8_to_f32(qraw[k], x);
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half2 h = __floats2half2_rn(x[2 * e], x[2 * e + 1]);
                    w4[e] = *reinterpret_cast<const uint32_t *>(&h);
                }
                *reinterpret_cast<uint4 *>(box + sw128_chunk(t, 4 * (part & 1) + k)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        } else {
            uint8_t *box = X + (part >> 1) * 8192;
            const float *rr = sR + RPS * part;  // r_i, i = 32 part + m, at m
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float x[8];
                bf16x8_to_f32(qraw[k], x);
                const float4 r0 = *reinterpret_cast<const float4 *>(rr + 8 * k);
                const float4 r1 = *reinterpret_cast<const float4 *>(rr + 8 * k + 4);
                x[0] *= r0.x; x[1] *= r0.y; x[2] *= r0.z; x[3] *= r0.w;
                x[4] *= r1.x; x[5] *= r1.y; x[6] *= r1.z; x[7] *= r1.w;
                store_split3(box, box + 16384, box + 32768, sw128_chunk(t, 4 * (part & 1) + k), x);
            }
        }
        umma::fence_proxy_async();
        umma::fence_before_sync();
        __syncthreads();
        // ---- D_a = Q^T (q r)^T (M 128 = j, N 64 = t) -> columns 0..63 -------------------------
        if (tid == 0) {
            umma::fence_after_sync();
            const uint32_t qc = smem_u32(sm + P3_QC), x0 = smem_u32(X);
            const uint32_t id = pivot ? umma::idesc_f16(128, 64, 1, 0) : umma::idesc_bf16(128, 64, 1, 0);
            const int terms = pivot ? 1 : 3;
            for (int x = 0; x < terms; ++x)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma::mma_bf16(tmem, umma::smem_desc(qc + kk * 2048, 16384, 1024),
                                   umma::smem_desc(x0 + x * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id,
                                   (x | kk) != 0);
            umma::mma_commit(smem_u32(&bars[1]));
        }
        ok = wait_bar(smem_u32(&bars[1]), parity, p.status);
        if (!__syncthreads_and(ok)) break;
        umma::fence_after_sync();
        {
            // o[t][j] = gamma_t (c_j a) + d (lane j, t = 32 cq + e) into rows of OST floats over the
            // term area, then out in 16-byte pieces of whole rows
            const int j = 32 * q4 + lane;
            float av[32], dv[32];
            umma::tmem_ld32(tl + 32 * cq, av);
            umma::tmem_ld32(tl + 64 + 32 * cq, dv);
            const float cj = pivot ? 1.f : sC[j];
            float *ob = reinterpret_cast<float *>(X);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int tt = 32 * cq + e;
                ob[tt * OST + j] = fmaf(sGam[tt], cj * av[e], dv[e]);
            }
        }
        umma::fence_before_sync();
        __syncthreads();
        {
            // piece e = 16 bytes c of row tt: a warp moves one whole row
            const float *ob = reinterpret_cast<const float *>(X);
            bool bad = false;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int e = tid + NT3 * k, tt = e >> 5, c = e & 31;
                if (tt < Lc) {
                    const float4 o4 = *reinterpret_cast<const float4 *>(ob + tt * OST + 4 * c);
                    bad |= !isfinite(o4.x) || !isfinite(o4.y) || !isfinite(o4.z) || !isfinite(o4.w);
                    reinterpret_cast<float4 *>(og + (size_t)tt * D)[c] = o4;
                }
            }
            if (bad) flag(p.status, kFlagNonfinite);
        }
        parity ^= 1u;
    }
    cp_async_wait_all();
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 128);
    }
}

__global__ void __launch_bounds__(NT3, 2) ut_readout_kernel(const __grid_constant__ TileParams p, const UtArgs a,
                                                            const int pivot)
{
    extern __shared__ uint8_t smem_raw[];
    readout_run(p, a, aligned_smem(smem_raw), blockIdx.x, gridDim.x, pivot != 0);
}

template <typename K, typename... X>
cudaError_t launch_one(K kernel, uint32_t smem, int work, int sms, const TileParams &p, const UtArgs &a, cudaStream_t s,
                       X... extra)
{
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    // the whole carveout as shared memory, so that two CTAs fit on an SM
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess) return err;
    const int grid = work < 2 * sms ? work : 2 * sms;
    kernel<<<grid, NT3, smem, s>>>(p, a, extra...);
    return cudaGetLastError();
}

// Segments of at most `seg` chunks: the workspace holds ntiles * seg records.
template <int BITS>
cudaError_t launch_ut_seg(const TileParams &p, int T, uint8_t *ws, int seg, cudaStream_t s)
{
    int dev = 0, sms = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    const int nch = (T + C - 1) / C;
    for (int c0 = 0; c0 < nch; c0 += seg) {
        const int nsc = nch - c0 < seg ? nch - c0 : seg;
        const UtArgs a{ws, T, c0, nsc};
        if ((err = launch_one(ut_inputs_kernel, P1_SMEM, p.ntiles * nsc, sms, p, a, s)) != cudaSuccess) return err;
        if constexpr (BITS == 16)
            err = launch_one(ut_state_pivot_kernel<0>, P2_SMEM, p.ntiles, sms, p, a, s);
        else
            err = launch_one(ut_state_kernel<BITS>, P2_SMEM, p.ntiles, sms, p, a, s);
        if (err != cudaSuccess) return err;
        if ((err = launch_one(ut_readout_kernel, P3_SMEM, p.ntiles * nsc, sms, p, a, s, (int)(BITS == 16))) !=
            cudaSuccess)
            return err;
    }
    return cudaSuccess;
}

template <int BITS>
cudaError_t launch_ut(const TileParams &p, int T, uint8_t *ws, cudaStream_t s)
{
    return launch_ut_seg<BITS>(p, T, ws, kUtSegmentChunks, s);
}

}  // namespace

cudaError_t launch_prefill_ut_seg(const TileParams &p, int bits, int T, void *ws, int seg, cudaStream_t s)
{
    uint8_t *w = static_cast<uint8_t *>(ws);
    if (seg < 1) return cudaErrorInvalidValue;
    switch (bits) {
    case 4: return launch_ut_seg<4>(p, T, w, seg, s);
    case 6: return launch_ut_seg<6>(p, T, w, seg, s);
    case 8: return launch_ut_seg<8>(p, T, w, seg, s);
    case 16: return launch_ut_seg<16>(p, T, w, seg, s);
    default: return cudaErrorInvalidValue;
    }
}

// Chunked prefill of 128 x 128 tiles (bf16 inputs, scalar gate, 64-token chunks, one plain
// requantization per chunk end) through the workspace; every entry of p.table has width `bits`
// (4, 6, 8, or 16 for FP16 pivot heads).
cudaError_t launch_prefill_ut(const TileParams &p, int bits, int T, void *ws, cudaStream_t s)
{
    uint8_t *w = static_cast<uint8_t *>(ws);
    switch (bits) {
    case 4: return launch_ut<4>(p, T, w, s);
    case 6: return launch_ut<6>(p, T, w, s);
    case 8: return launch_ut<8>(p, T, w, s);
    case 16: return launch_ut<16>(p, T, w, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace stq
