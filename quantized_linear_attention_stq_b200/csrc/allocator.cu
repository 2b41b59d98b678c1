// allocator.cu -- lifetime-aware width allocation (host code; declared in include/stq.h).
//
// The time dimension of the method ("线性注意力状态量化难题" (aitest123.com/news/n1kj09), section
// 时间维度; "K1 論文詳解" (k1-news.pages.dev/paper/2026-10-09), section 方法): errors of a state
// unit accumulate over its memory lifetime, so the budget goes to heads whose distortion and
// lifetime are both large, and the highest-risk heads stay FP16. Risk R_h(b) = D_h(b) / (1 - e^l_h);
// pivots are the largest R_h(8); the other heads climb 4 -> 6 -> 8 one step at a time, always the
// step of largest risk reduction per byte, while the request's bytes stay within budget (a heap of
// each head's next step; ties go to the lower head index).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <queue>
#include <vector>

#include "../../include/stq.h"
#include "stq_internal.cuh"

namespace {

struct Step {
    double gain;  // risk reduction per extra byte of the head's next width step
    int32_t head;
};

struct StepLess {
    // priority: larger gain first, then lower head index
    bool operator()(const Step &a, const Step &b) const
    {
        if (a.gain != b.gain) return a.gain < b.gain;
        return a.head > b.head;
    }
};

constexpr int kWidths[3] = {4, 6, 8};

}  // namespace

extern "C" stq_status stq_allocate_widths(int32_t H, int32_t d, const double *distortion,
                                          const double *mean_log_retention, int32_t num_pivots,
                                          uint64_t budget_bytes, uint8_t *widths_out)
{
    if (H < 1 || !distortion || !mean_log_retention || !widths_out) return STQ_ERR_INVALID_ARG;
    if (!(d == 16 || d == 32 || d == 64 || d == 128)) return STQ_ERR_INVALID_ARG;
    if (num_pivots < 0 || num_pivots > H) return STQ_ERR_INVALID_ARG;
    std::vector<double> R((size_t)H * 3);
    for (int32_t h = 0; h < H; ++h) {
        const double l = mean_log_retention[h];
        if (!std::isfinite(l) || l > 0.0) return STQ_ERR_INVALID_ARG;
        double forget = -std::expm1(l);
        if (forget < 1e-12) forget = 1e-12;
        const double lam = 1.0 / forget;
        for (int k = 0; k < 3; ++k) {
            const double D = distortion[(size_t)h * 3 + k];
            if (!std::isfinite(D) || D < 0.0) return STQ_ERR_INVALID_ARG;
            R[(size_t)h * 3 + k] = D == 0.0 ? 0.0 : lam * D;
        }
    }
    uint64_t bytes[3];
    for (int k = 0; k < 3; ++k) bytes[k] = stq::head_block_bytes(kWidths[k], d, d);
    const uint64_t pivot_bytes = stq::head_block_bytes(16, d, d);

    // pivots: largest 8-bit risk, lower head index first on ties
    std::vector<int32_t> order(H);
    for (int32_t h = 0; h < H; ++h) order[h] = h;
    std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return R[(size_t)a * 3 + 2] > R[(size_t)b * 3 + 2]; });
    std::vector<int8_t> level(H, 0);  // -1: pivot, else index into kWidths
    for (int32_t i = 0; i < num_pivots; ++i) level[order[i]] = -1;
    uint64_t total = 0;
    for (int32_t h = 0; h < H; ++h) total += level[h] < 0 ? pivot_bytes : bytes[0];
    total = (total + 127) / 128 * 128;
    if (total > budget_bytes) return STQ_ERR_INVALID_ARG;

    std::priority_queue<Step, std::vector<Step>, StepLess> heap;
    auto push_next = [&](int32_t h) {
        const int k = level[h];
        if (k < 0 || k >= 2) return;
        const double extra = (double)(bytes[k + 1] - bytes[k]);
        heap.push(Step{(R[(size_t)h * 3 + k] - R[(size_t)h * 3 + k + 1]) / extra, h});
    };
    for (int32_t h = 0; h < H; ++h) push_next(h);
    while (!heap.empty()) {
        const Step s = heap.top();
        heap.pop();
        const int k = level[s.head];
        const uint64_t extra = bytes[k + 1] - bytes[k];
        if (total + extra <= budget_bytes) {
            level[s.head] = (int8_t)(k + 1);
            total += extra;
            push_next(s.head);
        }
    }
    for (int32_t h = 0; h < H; ++h) widths_out[h] = (uint8_t)(level[h] < 0 ? 16 : kWidths[level[h]]);
    return STQ_OK;
}
