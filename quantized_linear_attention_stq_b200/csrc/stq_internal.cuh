// stq_internal.cuh -- internal declarations shared by the host code and the kernels of the
// quantized-state library (not part of the public ABI; see include/stq.h for the contract).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace stq {

// ------------------------------------------------------------------------------------------
// Status bits OR-ed into the caller's device status word: (1 << stq_status code).
// ------------------------------------------------------------------------------------------
constexpr int32_t kFlagNonfinite = 1 << 4;
constexpr int32_t kFlagTimeout = 1 << 5;
constexpr int32_t kFlagBounds = 1 << 6;

// A bounded wait gives up after this many SM clock cycles (~2 s at 2 GHz).
constexpr long long kWaitTimeoutCycles = 4000000000LL;

// ------------------------------------------------------------------------------------------
// Head-block layout (independent restatement of the byte layout in include/stq.h).
// ------------------------------------------------------------------------------------------
__host__ __device__ constexpr uint32_t round_up_u32(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }
__host__ __device__ constexpr uint32_t codes_bytes(int bits, int dk, int dv)
{
    return (uint32_t)(((uint64_t)bits * dk * dv + 7) / 8);
}
__host__ __device__ constexpr uint32_t scale_offset(int bits, int dk, int dv)
{
    return round_up_u32(codes_bytes(bits, dk, dv), 16);
}
__host__ __device__ constexpr uint32_t head_block_bytes(int bits, int dk, int dv)
{
    return bits == 16 ? round_up_u32(2u * dk * dv, 128)
                      : round_up_u32(scale_offset(bits, dk, dv) + 4u * dk + 4u * dv, 128);
}
// The same block with its row and column scales stored as bf16 (the 16-bit scale format).
__host__ __device__ constexpr uint32_t head_block_bytes_bf16s(int bits, int dk, int dv)
{
    return bits == 16 ? round_up_u32(2u * dk * dv, 128)
                      : round_up_u32(scale_offset(bits, dk, dv) + 2u * dk + 2u * dv, 128);
}

// One entry of the per-launch head table, in processing order (largest blocks first).
struct TileEntry {
    uint32_t off;   // byte offset of the head block inside a request block
    uint32_t info;  // bits 0..15: head index relative to the call's head_begin; 16..23: width
};
__host__ __device__ inline int entry_head(const TileEntry &e) { return (int)(e.info & 0xffffu); }
__host__ __device__ inline int entry_bits(const TileEntry &e) { return (int)((e.info >> 16) & 0xffu); }
// bit 24: the head uses one uniform scale (the baseline quantizer) instead of row x column scales
__host__ __device__ inline bool entry_uniform(const TileEntry &e) { return ((e.info >> 24) & 1u) != 0; }
__host__ __device__ constexpr uint32_t uniform_block_bytes(int bits, int dk, int dv)
{
    return round_up_u32(scale_offset(bits, dk, dv) + 4u, 128);
}

// Head table capacity of one launch; larger head ranges are split into several launches.
constexpr int kMaxTable = 3072;

struct TileParams {
    uint8_t *pool;
    const int32_t *slots;
    int32_t *status;
    uint64_t req_bytes;
    int32_t pool_slots;
    int32_t B;           // requests of this launch
    int32_t npos;        // heads of this launch (entries of the table)
    int32_t ntiles;      // B * npos
    int32_t head_count;  // heads of the call (row stride of the per-head input arrays)
    int32_t dk, dv;
    int32_t gate;
    int32_t scale_bf16;  // 1: row and column scales stored as bf16 (else fp32)
    int32_t fit_rounds;  // rounds of the impact-weighted joint refinement of the scales
    // decode / prefill inputs (indexed by request and call-relative head)
    const void *q, *k, *v;
    const float *beta, *alpha, *w;
    float *o;
    // init / dequantize
    const float *S0;
    float *S_out;
    TileEntry table[kMaxTable];
};

// ------------------------------------------------------------------------------------------
// Kernel launchers (host side; defined next to their kernels). Each returns a cudaError_t.
// ------------------------------------------------------------------------------------------
cudaError_t launch_init_generic(const TileParams &p, cudaStream_t s);
cudaError_t launch_dequant_generic(const TileParams &p, cudaStream_t s);
cudaError_t launch_decode_generic(const TileParams &p, int in_bf16, cudaStream_t s);
// bits: the width of every head of the table (4, 6, 8; 16 for FP16 pivots) or 0 for any mix of 4, 6
// and 8; pdl: a later launch of the same call (disjoint tiles) that may overlap the earlier ones
cudaError_t launch_decode_d128(const TileParams &p, int bits, int in_bf16, cudaStream_t s, bool pdl);
cudaError_t launch_prefill_seq(const TileParams &p, int in_bf16, int T, int chunk, cudaStream_t s);
// 128 x 128 heads token by token with the state in registers: any gate, chunk length and width of
// p.table (4/6/8 with row x column scales and no refit round, or 16)
cudaError_t launch_prefill_serial(const TileParams &p, int in_bf16, int T, int chunk, cudaStream_t s);
cudaError_t launch_prefill_wy(const TileParams &p, int bits, int T, cudaStream_t s);  // one width per launch
// The same chunk form as three kernels around a workspace of ntiles * min(chunks, kUtSegmentChunks)
// records of kUtRecordBytes (one plain requantization per chunk end; one width per launch).
constexpr uint64_t kUtRecordBytes = 116736;
constexpr int kUtSegmentChunks = 32;
cudaError_t launch_prefill_ut(const TileParams &p, int bits, int T, void *ws, cudaStream_t s);
// ... with segments of at most `seg` chunks (a workspace of ntiles * seg records)
cudaError_t launch_prefill_ut_seg(const TileParams &p, int bits, int T, void *ws, int seg, cudaStream_t s);

// ------------------------------------------------------------------------------------------
// Device helpers
// ------------------------------------------------------------------------------------------
#ifdef __CUDACC__

template <int IN_BF16>
__device__ __forceinline__ float load_in(const void *base, size_t idx)
{
    if constexpr (IN_BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(base)[idx]);
    else
        return reinterpret_cast<const float *>(base)[idx];
}

// Scale n of a head block's scale array (r[0..dk) then c[0..dv)) in the layout's storage format;
// a stored bf16 scale is rounded half to even from the fp32 value.
__device__ __forceinline__ float load_scale(const uint8_t *scales, int n, int bf16)
{
    return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(scales)[n])
                : reinterpret_cast<const float *>(scales)[n];
}
__device__ __forceinline__ float round_scale(float v, int bf16)
{
    return bf16 ? __bfloat162float(__float2bfloat16_rn(v)) : v;
}
__device__ __forceinline__ void store_scale(uint8_t *scales, int n, float v, int bf16)
{
    if (bf16)
        reinterpret_cast<__nv_bfloat16 *>(scales)[n] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float *>(scales)[n] = v;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for phase `parity` of an mbarrier, giving up after kWaitTimeoutCycles. Returns false on
// timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - start > kWaitTimeoutCycles) return false;
    }
}

// 4-byte asynchronous copy global -> shared (tracked with cp_async_arrive on an mbarrier).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// The mbarrier receives one arrival when all of this thread's prior cp.async copies have landed
// (no pending-count increment: the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Bulk copy global -> this CTA's shared memory, completing `bytes` on the mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void flag(int32_t *status, int32_t bits)
{
    if (status) atomicOr(status, bits);
}

#endif  // __CUDACC__

}  // namespace stq
