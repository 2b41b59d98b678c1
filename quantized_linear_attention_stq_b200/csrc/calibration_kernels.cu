// calibration_kernels.cu -- offline calibration statistics computed on the GPU (declared in
// include/stq.h).
//
// Key-row impact ("线性注意力状态量化难题" (aitest123.com/news/n1kj09), section 空间维度): the
// output error is a sum over key rows of each row's accumulated error times a weight set by the
// current key, query and gate, and the row impact score is the mean square of that weight. One
// update carries a state error E to E' and the next readout error is E'^T q = E^T g:
//   scalar gate g = a (q - b (k.q) k); channel (literal) g = a*q - b (k.(a*q)) k;
//   channel, decay first g = a * (q - b (k.q) k).
// One CTA per head, one thread per key row; the tokens are walked in order.
#include "../../include/stq.h"
#include "stq_internal.cuh"

namespace stq {
namespace {

template <int IN_BF16>
__global__ void row_impact_kernel(int T, int H, int d, int gate, const void *q, const void *k, const float *beta,
                                  const float *alpha, float *w_out)
{
    __shared__ float part[4];
    const int h = blockIdx.x, i = threadIdx.x, lane = i & 31, warp = i >> 5, nw = (d + 31) >> 5;
    float acc = 0.f;
    for (int t = 0; t < T; ++t) {
        const size_t row = (size_t)t * H + h;
        float qi = 0.f, ki = 0.f, ai = 0.f;
        if (i < d) {
            qi = load_in<IN_BF16>(q, row * d + i);
            ki = load_in<IN_BF16>(k, row * d + i);
            ai = gate == 0 ? alpha[row] : alpha[row * d + i];
        }
        // gate 1 projects the decayed query, the others the query itself
        float s = ki * (gate == 1 ? ai * qi : qi);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) part[warp] = s;
        __syncthreads();
        float kq = 0.f;
        for (int w = 0; w < nw; ++w) kq += part[w];
        __syncthreads();
        const float b = beta[row];
        const float g = gate == 1 ? ai * qi - b * kq * ki : ai * (qi - b * kq * ki);
        acc = fmaf(g, g, acc);
    }
    if (i < d) w_out[(size_t)h * d + i] = acc / (float)T;
}

}  // namespace
}  // namespace stq

extern "C" stq_status stq_row_impact(int32_t T, int32_t H, int32_t d, int32_t gate, int32_t in_dtype, const void *q,
                                     const void *k, const float *beta, const float *alpha, float *w_out, void *stream)
{
    if (T < 1 || H < 1 || !q || !k || !beta || !alpha || !w_out) return STQ_ERR_INVALID_ARG;
    if (!(d == 16 || d == 32 || d == 64 || d == 128)) return STQ_ERR_UNSUPPORTED;
    if (gate < STQ_GATE_SCALAR || gate > STQ_GATE_CHANNEL_DECAY_FIRST) return STQ_ERR_INVALID_ARG;
    if (in_dtype != STQ_F32 && in_dtype != STQ_BF16) return STQ_ERR_INVALID_ARG;
    const int threads = d < 32 ? 32 : d;
    cudaStream_t s = (cudaStream_t)stream;
    if (in_dtype == STQ_BF16)
        stq::row_impact_kernel<1><<<H, threads, 0, s>>>(T, H, d, gate, q, k, beta, alpha, w_out);
    else
        stq::row_impact_kernel<0><<<H, threads, 0, s>>>(T, H, d, gate, q, k, beta, alpha, w_out);
    return cudaGetLastError() == cudaSuccess ? STQ_OK : STQ_ERR_CUDA;
}
