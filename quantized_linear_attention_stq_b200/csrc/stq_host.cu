// stq_host.cu -- host side of the C ABI declared in include/stq.h: layout objects, argument
// checks, per-launch head tables and kernel dispatch. No device memory is allocated here and no
// call synchronizes; every launch goes to the caller's stream.
#include <algorithm>
#include <cstddef>
#include <cstdlib>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "../../include/stq.h"
#include "stq_internal.cuh"

namespace stq {
// Persistent streaming init of 128 x 128 row x column heads (init_d128.cu).
cudaError_t launch_init_d128(const TileParams &p, cudaStream_t s);
}  // namespace stq

namespace {
// The head tables of one decode call (a head range of a layout), built on its first call and
// reused: the FP16 pivot heads, and the other heads grouped by width.
struct CallPlan {
    std::vector<stq::TileEntry> pivots;
    std::vector<stq::TileEntry> coded;  // the 4/6/8-bit heads, 8-bit first, then 6, then 4
    int start[3], count[3];             // the 8-, 6- and 4-bit runs of `coded`
};
}  // namespace

struct stq_layout {
    int32_t H, dk, dv, gate, in_dtype;
    bool uniform;  // STQ_SCALES_UNIFORM
    bool sb16;     // row and column scales stored as bf16
    int fit_rounds;  // rounds of the impact-weighted joint refinement of the scales
    std::vector<uint8_t> bits;
    std::vector<uint64_t> offset;
    std::vector<uint64_t> bytes;
    uint64_t req_bytes;
    // decode plans by (head_begin, head_count); the layout is otherwise immutable and may be
    // shared between threads, so the cache has its own lock
    mutable std::mutex plan_mu;
    mutable std::map<std::pair<int, int>, std::shared_ptr<const CallPlan>> plans;
};

namespace {

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Processing order of a launch: largest blocks first (FP16 pivots, then 8-, 6-, 4-bit), head
// index order inside a width, so that round-robin CTAs see the same mix of tile sizes.
std::vector<int> order_by_size(const stq_layout *L, int h0, int count)
{
    std::vector<int> ord(count);
    for (int i = 0; i < count; ++i) ord[i] = h0 + i;
    std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return L->bits[a] > L->bits[b]; });
    return ord;
}

// Prefill shapes that take the tensor-core chunk form: 128 x 128 heads, bf16 inputs, the scalar
// gate and 64-token chunks (the FP16 pivot heads of such a layout take the token-by-token kernel).
bool wy_form(const stq_layout *L, int chunk)
{
    return L->dk == 128 && L->gate == STQ_GATE_SCALAR && L->in_dtype == STQ_BF16 && chunk == 64 && !L->uniform &&
           L->fit_rounds <= 1;
}
// ... of which those with one plain requantization per chunk end run as the three workspace
// kernels, every head (FP16 pivots included) in the chunk form.
bool ut_form(const stq_layout *L, int chunk) { return wy_form(L, chunk) && L->fit_rounds == 0; }

// Fill the common fields of a TileParams for heads ord[first .. first+n) of a call.
void fill_table(stq::TileParams &p, const stq_layout *L, const std::vector<int> &ord, int first, int n, int h0)
{
    p.npos = n;
    p.scale_bf16 = L->sb16 ? 1 : 0;
    p.fit_rounds = L->fit_rounds;
    for (int e = 0; e < n; ++e) {
        const int h = ord[first + e];
        p.table[e].off = (uint32_t)L->offset[h];
        p.table[e].info = (uint32_t)(h - h0) | ((uint32_t)L->bits[h] << 16) |
                          ((L->uniform && L->bits[h] != 16) ? (1u << 24) : 0u);
    }
}

stq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? STQ_OK : STQ_ERR_CUDA; }

// The parameter block is ~24 KB; keep it off the (small) thread stack.
std::unique_ptr<stq::TileParams> new_params()
{
    std::unique_ptr<stq::TileParams> p(new (std::nothrow) stq::TileParams);
    if (p) std::memset(p.get(), 0, sizeof(stq::TileParams));
    return p;
}

// The decode path's parameter block: one per host thread, reused across calls (a launch copies
// its parameters when it is enqueued). Only the fields before the table are cleared.
stq::TileParams &thread_params()
{
    static thread_local stq::TileParams tp;
    std::memset(&tp, 0, offsetof(stq::TileParams, table));
    return tp;
}

stq::TileEntry entry_of(const stq_layout *L, int h, int h0)
{
    stq::TileEntry e;
    e.off = (uint32_t)L->offset[h];
    e.info = (uint32_t)(h - h0) | ((uint32_t)L->bits[h] << 16);
    return e;
}

// Tables of the tuned decode path for heads [h0, h0 + count): the pivots, and the other heads
// sorted by width (largest blocks first, head order inside a width).
std::shared_ptr<const CallPlan> call_plan(const stq_layout *L, int h0, int count)
{
    std::lock_guard<std::mutex> lock(L->plan_mu);
    auto it = L->plans.find({h0, count});
    if (it != L->plans.end()) return it->second;
    auto plan = std::make_shared<CallPlan>();
    static const int widths[3] = {8, 6, 4};
    for (int h = h0; h < h0 + count; ++h)
        if (L->bits[h] == 16) plan->pivots.push_back(entry_of(L, h, h0));
    for (int c = 0; c < 3; ++c) {
        plan->start[c] = (int)plan->coded.size();
        for (int h = h0; h < h0 + count; ++h)
            if (L->bits[h] == widths[c]) plan->coded.push_back(entry_of(L, h, h0));
        plan->count[c] = (int)plan->coded.size() - plan->start[c];
    }
    if (L->plans.size() > 4096) L->plans.clear();  // bounded: head ranges of one model are few
    L->plans[{h0, count}] = plan;
    return plan;
}

}  // namespace

// The workspace of stq_prefill_chunk_noalloc: one fixed array per device, part of this library's
// module. The host-side name is only a handle; its device address comes from cudaGetSymbolAddress.
constexpr size_t kNoallocScratchBytes = (size_t)32 << 20;
static __device__ __align__(256) uint8_t stq_noalloc_scratch[kNoallocScratchBytes];

namespace {
// The array's device address on the current device, looked up on the first call per device and
// kept (no allocation: a fixed table for the first 64 device ordinals).
void *noalloc_scratch()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    static std::mutex mu;
    static void *addr[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && addr[dev]) return addr[dev];
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, stq_noalloc_scratch) != cudaSuccess) return nullptr;
    if (dev >= 0 && dev < 64) addr[dev] = ptr;
    return ptr;
}
}  // namespace

extern "C" {

int32_t stq_abi_version(void) { return STQ_ABI_VERSION; }

const char *stq_status_string(int32_t status)
{
    switch (status) {
    case STQ_OK: return "ok";
    case STQ_ERR_INVALID_ARG: return "invalid argument";
    case STQ_ERR_UNSUPPORTED: return "unsupported shape, width or mode";
    case STQ_ERR_CUDA: return "CUDA launch error";
    case STQ_ERR_NONFINITE: return "non-finite state, scale or output";
    case STQ_ERR_TIMEOUT: return "bounded wait timed out";
    case STQ_ERR_BOUNDS: return "slot out of range";
    default: return "unknown status";
    }
}

stq_status stq_layout_create(const stq_layout_desc *desc, stq_layout **out)
{
    if (!desc || !out || !desc->head_bits) return STQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (desc->num_heads < 1 || desc->d_k < 1 || desc->d_v < 1) return STQ_ERR_INVALID_ARG;
    if (desc->gate < STQ_GATE_SCALAR || desc->gate > STQ_GATE_CHANNEL_DECAY_FIRST) return STQ_ERR_INVALID_ARG;
    if (desc->in_dtype != STQ_F32 && desc->in_dtype != STQ_BF16) return STQ_ERR_INVALID_ARG;
    if (desc->scale_mode != STQ_SCALES_ROW_COLUMN && desc->scale_mode != STQ_SCALES_UNIFORM) return STQ_ERR_INVALID_ARG;
    if (desc->scale_dtype != STQ_F32 && desc->scale_dtype != STQ_BF16) return STQ_ERR_INVALID_ARG;
    if (desc->scale_dtype == STQ_BF16 && desc->scale_mode == STQ_SCALES_UNIFORM) return STQ_ERR_UNSUPPORTED;
    if (desc->scale_fit_rounds < 0 || desc->scale_fit_rounds > 8) return STQ_ERR_INVALID_ARG;
    if (desc->scale_fit_rounds > 0 && desc->scale_mode == STQ_SCALES_UNIFORM) return STQ_ERR_UNSUPPORTED;
    const int d = desc->d_k;
    if (desc->d_v != d || !(d == 16 || d == 32 || d == 64 || d == 128)) return STQ_ERR_UNSUPPORTED;
    if (desc->num_heads > 65535) return STQ_ERR_UNSUPPORTED;
    std::unique_ptr<stq_layout> L(new (std::nothrow) stq_layout);
    if (!L) return STQ_ERR_INVALID_ARG;
    L->H = desc->num_heads;
    L->dk = desc->d_k;
    L->dv = desc->d_v;
    L->gate = desc->gate;
    L->in_dtype = desc->in_dtype;
    L->uniform = desc->scale_mode == STQ_SCALES_UNIFORM;
    L->sb16 = desc->scale_dtype == STQ_BF16;
    L->fit_rounds = desc->scale_fit_rounds;
    uint64_t pos = 0;
    for (int h = 0; h < L->H; ++h) {
        const int b = desc->head_bits[h];
        if (b != 4 && b != 6 && b != 8 && b != 16) return STQ_ERR_UNSUPPORTED;
        L->bits.push_back((uint8_t)b);
        L->offset.push_back(pos);
        const uint64_t nb = (L->uniform && b != 16) ? stq::uniform_block_bytes(b, L->dk, L->dv)
                            : L->sb16               ? stq::head_block_bytes_bf16s(b, L->dk, L->dv)
                                                    : stq::head_block_bytes(b, L->dk, L->dv);
        L->bytes.push_back(nb);
        pos += nb;
    }
    L->req_bytes = (pos + 127) / 128 * 128;
    if (L->req_bytes > 0xFFFFFFFFull) return STQ_ERR_UNSUPPORTED;  // head offsets are 32-bit
    *out = L.release();
    return STQ_OK;
}

void stq_layout_destroy(stq_layout *layout) { delete layout; }

size_t stq_layout_bytes_per_request(const stq_layout *L) { return L ? (size_t)L->req_bytes : 0; }

size_t stq_layout_head_offset(const stq_layout *L, int32_t h)
{
    return (L && h >= 0 && h < L->H) ? (size_t)L->offset[h] : 0;
}

size_t stq_layout_head_bytes(const stq_layout *L, int32_t h)
{
    return (L && h >= 0 && h < L->H) ? (size_t)L->bytes[h] : 0;
}

int32_t stq_layout_head_bits(const stq_layout *L, int32_t h) { return (L && h >= 0 && h < L->H) ? L->bits[h] : 0; }

stq_status stq_init_state(const stq_layout *L, void *pool, int32_t pool_slots, const int32_t *slots, int32_t B,
                          const float *S0, const float *w, int32_t *dev_status, void *stream)
{
    if (!L || B < 0 || pool_slots < 0) return STQ_ERR_INVALID_ARG;
    if (B == 0) return STQ_OK;
    if (!pool || !slots || !S0 || !w || !aligned(pool, 128) || !aligned(S0, 4) || !aligned(w, 4))
        return STQ_ERR_INVALID_ARG;
    if (B > 2147483647 / L->H) return STQ_ERR_UNSUPPORTED;
    auto p = new_params();
    if (!p) return STQ_ERR_INVALID_ARG;
    p->pool = static_cast<uint8_t *>(pool);
    p->slots = slots;
    p->status = dev_status;
    p->req_bytes = L->req_bytes;
    p->pool_slots = pool_slots;
    p->B = B;
    p->head_count = L->H;
    p->dk = L->dk;
    p->dv = L->dv;
    p->gate = L->gate;
    p->S0 = S0;
    p->w = w;
    const std::vector<int> ord = order_by_size(L, 0, L->H);
    // 128 x 128 row x column heads without refinement rounds go to the persistent streaming
    // kernel when S0 and w allow 16-byte copies; FP16 pivots and everything else to the plain one
    const bool streamed = L->dk == 128 && L->dv == 128 && !L->uniform && L->fit_rounds == 0 && aligned(S0, 16) &&
                          aligned(w, 16);
    std::vector<int> plain, tuned;
    for (int h : ord) (streamed && L->bits[h] != 16 ? tuned : plain).push_back(h);
    for (int pass = 0; pass < 2; ++pass) {
        const std::vector<int> &heads = pass == 0 ? plain : tuned;
        const int nh = (int)heads.size();
        for (int first = 0; first < nh; first += stq::kMaxTable) {
            const int n = std::min(stq::kMaxTable, nh - first);
            fill_table(*p, L, heads, first, n, 0);
            p->ntiles = B * n;
            const cudaError_t e = pass == 0 ? stq::launch_init_generic(*p, (cudaStream_t)stream)
                                            : stq::launch_init_d128(*p, (cudaStream_t)stream);
            const stq_status st = from_cuda(e);
            if (st != STQ_OK) return st;
        }
    }
    return STQ_OK;
}

stq_status stq_dequantize(const stq_layout *L, const void *pool, int32_t pool_slots, const int32_t *slots, int32_t B,
                          float *S_out, int32_t *dev_status, void *stream)
{
    if (!L || B < 0 || pool_slots < 0) return STQ_ERR_INVALID_ARG;
    if (B == 0) return STQ_OK;
    if (!pool || !slots || !S_out || !aligned(pool, 128) || !aligned(S_out, 4)) return STQ_ERR_INVALID_ARG;
    auto p = new_params();
    if (!p) return STQ_ERR_INVALID_ARG;
    p->pool = static_cast<uint8_t *>(const_cast<void *>(pool));
    p->slots = slots;
    p->status = dev_status;
    p->req_bytes = L->req_bytes;
    p->pool_slots = pool_slots;
    p->B = B;
    p->head_count = L->H;
    p->dk = L->dk;
    p->dv = L->dv;
    p->S_out = S_out;
    const std::vector<int> ord = order_by_size(L, 0, L->H);
    for (int first = 0; first < L->H; first += stq::kMaxTable) {
        const int n = std::min(stq::kMaxTable, L->H - first);
        fill_table(*p, L, ord, first, n, 0);
        p->ntiles = B * n;
        const stq_status st = from_cuda(stq::launch_dequant_generic(*p, (cudaStream_t)stream));
        if (st != STQ_OK) return st;
    }
    return STQ_OK;
}

stq_status stq_decode_step(const stq_layout *L, void *pool, int32_t pool_slots, const int32_t *slots, int32_t B,
                           int32_t head_begin, int32_t head_count, const void *q, const void *k, const void *v,
                           const float *beta, const float *alpha, const float *w, float *o, int32_t *dev_status,
                           void *stream)
{
    if (!L || B < 0 || pool_slots < 0 || head_begin < 0 || head_count < 0 || head_begin > L->H ||
        head_count > L->H - head_begin)
        return STQ_ERR_INVALID_ARG;
    if (B == 0 || head_count == 0) return STQ_OK;
    if (!pool || !slots || !q || !k || !v || !beta || !alpha || !w || !o) return STQ_ERR_INVALID_ARG;
    if (!aligned(pool, 128) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(alpha, 16) ||
        !aligned(w, 16) || !aligned(beta, 4) || !aligned(o, 16))
        return STQ_ERR_INVALID_ARG;
    if (B > 2147483647 / head_count) return STQ_ERR_UNSUPPORTED;
    const int in_bf16 = L->in_dtype == STQ_BF16;
    const size_t in_sz = in_bf16 ? 2 : 4;
    const int na = L->gate == STQ_GATE_SCALAR ? 1 : L->dk;
    if (L->dk == 128 && !L->uniform && L->fit_rounds <= 1) {
        // the tuned kernel (one refit round included): the call's FP16 pivot heads in one launch,
        // then all its other heads, any mix of widths, in one more (tables of at most kMaxTable
        // heads each); a launch after the first may overlap the ones before it (disjoint tiles)
        const std::shared_ptr<const CallPlan> plan = call_plan(L, head_begin, head_count);
        stq::TileParams &tp = thread_params();
        tp.pool = static_cast<uint8_t *>(pool);
        tp.slots = slots;
        tp.status = dev_status;
        tp.req_bytes = L->req_bytes;
        tp.pool_slots = pool_slots;
        tp.B = B;
        tp.head_count = head_count;
        tp.dk = L->dk;
        tp.dv = L->dv;
        tp.gate = L->gate;
        tp.scale_bf16 = L->sb16 ? 1 : 0;
        tp.fit_rounds = L->fit_rounds;
        tp.q = q;
        tp.k = k;
        tp.v = v;
        tp.beta = beta;
        tp.alpha = alpha;
        tp.w = w;
        tp.o = o;
        bool later = false;
        // Launch the table entries [first, first + n) with width `bits` (0: any mix of 4/6/8).
        auto launch = [&](const std::vector<stq::TileEntry> &tab, int first0, int n0, int bits) -> bool {
            for (int first = first0; first < first0 + n0; first += stq::kMaxTable) {
                const int n = std::min(stq::kMaxTable, first0 + n0 - first);
                std::memcpy(tp.table, tab.data() + first, sizeof(stq::TileEntry) * (size_t)n);
                tp.npos = n;
                tp.ntiles = B * n;
                if (stq::launch_decode_d128(tp, bits, in_bf16, (cudaStream_t)stream, later) != cudaSuccess)
                    return false;
                later = true;
            }
            return true;
        };
        // A launch per width keeps each width's compile-time ring (three slots for 4-bit tiles) but
        // pays the ring's start and the tail per launch: worth it when every width present has
        // enough tiles to fill the GPU several times over. Otherwise (the serving shape: one call
        // per layer) one launch takes every width.
        static const int widths[3] = {8, 6, 4};
        constexpr long long kPerWidthTiles = 8192;
        int present = 0;
        bool big = true;
        for (int c = 0; c < 3; ++c)
            if (plan->count[c] > 0) {
                ++present;
                big = big && (long long)plan->count[c] * B >= kPerWidthTiles;
            }
        if (present == 1 || big) {
            for (int c = 0; c < 3; ++c)
                if (plan->count[c] > 0 && !launch(plan->coded, plan->start[c], plan->count[c], widths[c]))
                    return STQ_ERR_CUDA;
        } else if (!launch(plan->coded, 0, (int)plan->coded.size(), 0)) {
            return STQ_ERR_CUDA;
        }
        // The FP16 pivots last: their few CTAs fill SMs as the coded launch drains, instead of
        // holding SMs while it starts.
        if (!launch(plan->pivots, 0, (int)plan->pivots.size(), 16)) return STQ_ERR_CUDA;
        return STQ_OK;
    }
    // the plain kernel: the same per-thread parameter block (the table entries are filled below)
    stq::TileParams *p = &thread_params();
    p->pool = static_cast<uint8_t *>(pool);
    p->status = dev_status;
    p->req_bytes = L->req_bytes;
    p->pool_slots = pool_slots;
    p->head_count = head_count;
    p->dk = L->dk;
    p->dv = L->dv;
    p->gate = L->gate;
    p->w = w;
    // the plain kernel (uniform scales, d < 128, two or more refit rounds): any mix of widths
    const int maxb = 65535;
    const std::vector<int> ord = order_by_size(L, head_begin, head_count);
    for (int b0 = 0; b0 < B; b0 += maxb) {
        const int nb = std::min(maxb, B - b0);
        // requests [b0, b0+nb): shift every per-request array
        const size_t rq = (size_t)b0 * head_count;
        p->slots = slots + b0;
        p->B = nb;
        p->q = static_cast<const uint8_t *>(q) + rq * L->dk * in_sz;
        p->k = static_cast<const uint8_t *>(k) + rq * L->dk * in_sz;
        p->v = static_cast<const uint8_t *>(v) + rq * L->dv * in_sz;
        p->beta = beta + rq;
        p->alpha = alpha + rq * na;
        p->o = o + rq * L->dv;
        for (int first = 0; first < head_count; first += stq::kMaxTable) {
            const int n = std::min(stq::kMaxTable, head_count - first);
            fill_table(*p, L, ord, first, n, head_begin);
            p->ntiles = nb * n;
            if (stq::launch_decode_generic(*p, in_bf16, (cudaStream_t)stream) != cudaSuccess) return STQ_ERR_CUDA;
        }
    }
    return STQ_OK;
}

size_t stq_prefill_workspace_bytes(const stq_layout *L, int32_t B, int32_t T, int32_t chunk)
{
    if (!L || B < 0 || T < 0 || chunk < 1) return 0;
    if (!ut_form(L, chunk)) return 0;  // the other kernels carry everything on chip
    // one record per (request, head, chunk of a segment); the widths run one after another
    const int64_t nch = ((int64_t)T + 63) / 64;
    const int64_t seg = nch < stq::kUtSegmentChunks ? nch : stq::kUtSegmentChunks;
    return (size_t)B * (size_t)L->H * (size_t)seg * (size_t)stq::kUtRecordBytes;
}

stq_status stq_prefill_chunk(const stq_layout *L, void *pool, int32_t pool_slots, const int32_t *slots, int32_t B,
                             int32_t T, int32_t chunk, const void *q, const void *k, const void *v, const float *beta,
                             const float *alpha, const float *w, float *o, void *workspace, size_t workspace_bytes,
                             int32_t *dev_status, void *stream)
{
    if (!L || B < 0 || T < 0 || chunk < 1 || pool_slots < 0) return STQ_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return STQ_OK;
    if (!pool || !slots || !q || !k || !v || !beta || !alpha || !w || !o) return STQ_ERR_INVALID_ARG;
    // a workspace, when given, must hold stq_prefill_workspace_bytes; without one the chunk form
    // runs as a single kernel
    const size_t need = stq_prefill_workspace_bytes(L, B, T, chunk);
    if (need > 0 && workspace && (workspace_bytes < need || !aligned(workspace, 256))) return STQ_ERR_INVALID_ARG;
    const bool use_ws = need > 0 && workspace != nullptr;
    if (B > 2147483647 / L->H) return STQ_ERR_UNSUPPORTED;
    if (!aligned(pool, 128) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(w, 16) ||
        !aligned(o, 16) || !aligned(beta, 4) || !aligned(alpha, 4))
        return STQ_ERR_INVALID_ARG;
    if (L->H > stq::kMaxTable) return STQ_ERR_UNSUPPORTED;
    auto p = new_params();
    if (!p) return STQ_ERR_INVALID_ARG;
    p->pool = static_cast<uint8_t *>(pool);
    p->slots = slots;
    p->status = dev_status;
    p->req_bytes = L->req_bytes;
    p->pool_slots = pool_slots;
    p->B = B;
    p->head_count = L->H;
    p->dk = L->dk;
    p->dv = L->dv;
    p->gate = L->gate;
    p->q = q;
    p->k = k;
    p->v = v;
    p->beta = beta;
    p->alpha = alpha;
    p->w = w;
    p->o = o;
    // 128 x 128 heads with bf16 inputs, the scalar gate and 64-token chunks take the tensor-core
    // chunk form, one width at a time (three kernels around the workspace, or one kernel); FP16
    // pivot heads and every other configuration take the sequential kernel.
    const bool wy = wy_form(L, chunk);
    const int in_bf16 = L->in_dtype == STQ_BF16;
    if (!wy) {
        std::vector<int> ord(L->H);
        for (int h = 0; h < L->H; ++h) ord[h] = h;
        fill_table(*p, L, ord, 0, L->H, 0);
        p->ntiles = B * L->H;
        // 128 x 128 heads with row x column scales and no refit round: the state in registers;
        // the others (smaller heads, the uniform baseline, refit rounds): the general kernel
        const bool serial = L->dk == 128 && !L->uniform && L->fit_rounds == 0;
        return from_cuda(serial ? stq::launch_prefill_serial(*p, in_bf16, T, chunk, (cudaStream_t)stream)
                                : stq::launch_prefill_seq(*p, in_bf16, T, chunk, (cudaStream_t)stream));
    }
    const std::vector<int> ord = order_by_size(L, 0, L->H);
    for (int first = 0; first < L->H;) {
        const int bits = L->bits[ord[first]];
        int n = 0;
        while (first + n < L->H && L->bits[ord[first + n]] == bits) ++n;
        fill_table(*p, L, ord, first, n, 0);
        p->ntiles = B * n;
        const cudaError_t e = use_ws       ? stq::launch_prefill_ut(*p, bits, T, workspace, (cudaStream_t)stream)
                              : bits == 16 ? stq::launch_prefill_serial(*p, 1, T, chunk, (cudaStream_t)stream)
                                           : stq::launch_prefill_wy(*p, bits, T, (cudaStream_t)stream);
        if (e != cudaSuccess) return STQ_ERR_CUDA;
        first += n;
    }
    return STQ_OK;
}

stq_status stq_prefill_chunk_noalloc(const stq_layout *L, void *pool, int32_t pool_slots, const int32_t *slots,
                                     int32_t B, int32_t T, int32_t chunk, const void *q, const void *k,
                                     const void *v, const float *beta, const float *alpha, const float *w, float *o,
                                     int32_t *dev_status, void *stream)
{
    if (!L || B < 0 || T < 0 || chunk < 1 || pool_slots < 0) return STQ_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return STQ_OK;
    if (!ut_form(L, chunk))  // these shapes keep everything on chip: nothing to stage
        return stq_prefill_chunk(L, pool, pool_slots, slots, B, T, chunk, q, k, v, beta, alpha, w, o, nullptr, 0,
                                 dev_status, stream);
    if (!pool || !slots || !q || !k || !v || !beta || !alpha || !w || !o) return STQ_ERR_INVALID_ARG;
    if (B > 2147483647 / L->H) return STQ_ERR_UNSUPPORTED;
    if (!aligned(pool, 128) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(w, 16) ||
        !aligned(o, 16) || !aligned(beta, 4) || !aligned(alpha, 4))
        return STQ_ERR_INVALID_ARG;
    if (L->H > stq::kMaxTable) return STQ_ERR_UNSUPPORTED;
    // one width at a time: the largest class sets how many chunks a segment of records can hold
    int count[4] = {0, 0, 0, 0};
    static const int widths[4] = {16, 8, 6, 4};
    for (int h = 0; h < L->H; ++h)
        for (int c = 0; c < 4; ++c) count[c] += L->bits[h] == widths[c];
    const uint64_t most = (uint64_t)std::max(std::max(count[0], count[1]), std::max(count[2], count[3]));
    const uint64_t per_chunk = (uint64_t)B * most * stq::kUtRecordBytes;
    if (per_chunk > kNoallocScratchBytes) return STQ_ERR_UNSUPPORTED;
    const uint64_t fit = kNoallocScratchBytes / per_chunk;
    const int seg = fit < (uint64_t)stq::kUtSegmentChunks ? (int)fit : stq::kUtSegmentChunks;
    void *scratch = noalloc_scratch();
    if (!scratch) return STQ_ERR_CUDA;

    stq::TileParams &tp = thread_params();
    tp.pool = static_cast<uint8_t *>(pool);
    tp.slots = slots;
    tp.status = dev_status;
    tp.req_bytes = L->req_bytes;
    tp.pool_slots = pool_slots;
    tp.B = B;
    tp.head_count = L->H;
    tp.dk = L->dk;
    tp.dv = L->dv;
    tp.gate = L->gate;
    tp.scale_bf16 = L->sb16 ? 1 : 0;
    tp.fit_rounds = L->fit_rounds;
    tp.q = q;
    tp.k = k;
    tp.v = v;
    tp.beta = beta;
    tp.alpha = alpha;
    tp.w = w;
    tp.o = o;
    // FP16 pivots first, then the 8-, 6- and 4-bit heads, head index order inside a width
    for (int c = 0; c < 4; ++c) {
        int n = 0;
        for (int h = 0; h < L->H; ++h)
            if (L->bits[h] == widths[c]) tp.table[n++] = entry_of(L, h, 0);
        if (n == 0) continue;
        tp.npos = n;
        tp.ntiles = B * n;
        if (stq::launch_prefill_ut_seg(tp, widths[c], T, scratch, seg, (cudaStream_t)stream) != cudaSuccess)
            return STQ_ERR_CUDA;
    }
    return STQ_OK;
}

}  // extern "C"
