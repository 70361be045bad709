// onebit_adam.cu -- host side of the C ABI declared in include/onebit_adam.h: argument checks,
// the workspace layout, the launch sequence of one step and the state/timing helpers.
//
// One compressed step is five launches on the caller's stream, ordered by the stream alone
// (no kernel waits on another, so nothing can spin or hang):
//   k_worker  -> k_scales (worker)  -> k_server -> k_scales (server) -> k_apply
// The boundary between k_worker/k_scales and k_server is where the compressed allreduce of the
// method crosses the network ("1-bit Adam" index page, Abstract: communication is the
// bottleneck; LIT-278 note: the compressed allreduce is a custom collective); here the W
// workers live in one GPU's memory, so the "network" is the packed planes in HBM.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>  // header-only; ranges are free unless a profiler is attached

#include "onebit_adam.h"
#include "kernels.cuh"

using namespace onebit;

namespace {

thread_local std::string g_last_error;

constexpr int32_t kMaxWorkers = 256;
constexpr int kLaunchesPerStep = 5;
constexpr int kEventsPerStep = kLaunchesPerStep + 1;

enum Phase { kUnbound = 0, kWarmup = 1, kCompressed = 2 };

int cuda_fail(cudaError_t e) {
    g_last_error = cudaGetErrorString(e);
    return ONEBIT_ERR_CUDA;
}

#define ONEBIT_CUDA(call)                                 \
    do {                                                  \
        cudaError_t e_ = (call);                          \
        if (e_ != cudaSuccess) return cuda_fail(e_);      \
    } while (0)

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Workspace regions, each 256-byte aligned.
struct Layout {
    uint64_t m, v, es, ew, bits_w, bits_s, s_out, s_lazy, S_out, S_lazy, part_w, part_s, status;
    uint64_t total;
};

}  // namespace

struct onebit_adam_s {
    Geometry geo;
    int64_t nw;  // words per plane, ceil(d / 32)
    float beta1, beta2, eps;
    int phase = kUnbound;
    int64_t steps = 0;
    bool m_explicit = true;  // m in the fp32 buffer; else m = +-S_out by the server plane
    int32_t gtype = -1;
    char* ws = nullptr;
    Layout lay{};
    // region pointers (valid once bound)
    float *m = nullptr, *v = nullptr, *es = nullptr, *ew = nullptr;
    float *s_out = nullptr, *s_lazy = nullptr, *S_out = nullptr, *S_lazy = nullptr;
    uint32_t *bits_w = nullptr, *bits_s = nullptr, *status = nullptr;
    double *part_w = nullptr, *part_s = nullptr;
    // per-kernel timing
    std::vector<cudaEvent_t> ev;
    int32_t tmax = 0, tcount = 0;
    // host-buffer steps: the read-back of x runs on its own stream so that it overlaps the
    // next step's gradient upload (created on the first host-buffer step)
    cudaStream_t d2h = nullptr;
    cudaEvent_t step_done = nullptr, d2h_done = nullptr;
    bool d2h_pending = false;
};

namespace {

Layout make_layout(const onebit_adam_s& h) {
    const Geometry& g = h.geo;
    Layout L{};
    uint64_t off = 0;
    auto take = [&](uint64_t bytes) {
        const uint64_t at = off;
        off = (uint64_t)round_up((int64_t)(off + bytes), 256);
        return at;
    };
    const uint64_t f = sizeof(float);
    L.m = take(g.ld * f);
    L.v = take(g.ld * f);
    L.es = take(g.ld * f);
    L.ew = take((uint64_t)g.W * g.ld * f);
    L.bits_w = take((uint64_t)g.W * g.ldw * sizeof(uint32_t));
    L.bits_s = take(g.ldw * sizeof(uint32_t));
    L.s_out = take((uint64_t)g.W * g.nch * f);
    L.s_lazy = take((uint64_t)g.W * g.nch * f);
    L.S_out = take(g.nch * f);
    L.S_lazy = take(g.nch * f);
    L.part_w = take((uint64_t)g.W * g.nch * g.nseg * sizeof(double));
    L.part_s = take((uint64_t)g.nch * g.nseg_s * sizeof(double));
    L.status = take(4 * sizeof(uint32_t));
    L.total = off;
    return L;
}

bool valid_handle(onebit_adam_t h) { return h != nullptr; }

int64_t step_blocks(const Geometry& g) { return g.nch * g.nseg; }
int64_t server_blocks_per_chunk(const Geometry& g) {
    return ceil_div(g.nseg_s, kSrvSegsPerBlock);
}
int64_t server_blocks(const Geometry& g) { return g.nch * server_blocks_per_chunk(g); }

// The k_server instantiation for W workers: exact scaling for power-of-two W, residuals staged
// by TMA for narrow W.
using ServerKernel = void (*)(ServerArgs);
ServerKernel server_kernel(int W) {
    const bool pow2 = (W & (W - 1)) == 0, staged = server_stage_residuals(W);
    if (pow2) return staged ? k_server<true, true> : k_server<true, false>;
    return staged ? k_server<false, true> : k_server<false, false>;
}

// Launch the chunk-scale reduction (nseg partials of seg elements per row) with the thread
// count that fits the partial count.
int launch_scales(const Geometry& g, const double* part, int64_t rows, int64_t nseg, int seg,
                  float* out, float* lazy, cudaStream_t st) {
    if (rows == 0) return ONEBIT_OK;
    if (nseg <= 8) {
        k_scales<1><<<(unsigned)ceil_div(rows, kThreads), kThreads, 0, st>>>(
            part, rows, g.nch, nseg, seg, g.C, g.d, out, lazy);
    } else if (nseg <= 1024) {
        k_scales<32><<<(unsigned)ceil_div(rows, kWarps), kThreads, 0, st>>>(
            part, rows, g.nch, nseg, seg, g.C, g.d, out, lazy);
    } else {
        k_scales<kThreads><<<(unsigned)rows, kThreads, 0, st>>>(part, rows, g.nch, nseg, seg,
                                                                g.C, g.d, out, lazy);
    }
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

// Vector width of the worker kernel: 8 elements per thread (16-byte loads of 8 bf16 values)
// when bf16 gradient rows are 16-byte aligned, 4 (16-byte loads of 4 fp32 values, or 8-byte
// loads of 4 bf16 values) when rows are 16- or 8-byte aligned, element by element otherwise.
template <typename GT, bool LAZY_M>
void launch_worker_t(onebit_adam_s* h, const WorkerArgs& a, unsigned blocks, size_t smem,
                     cudaStream_t st) {
    const int64_t d = h->geo.d;
    if constexpr (sizeof(GT) == 2) {
        if (d % 8 == 0) {
            k_worker<GT, true, LAZY_M, 8><<<blocks, kThreads, smem, st>>>(a);
            return;
        }
    }
    if (d % kVec == 0)
        k_worker<GT, true, LAZY_M, 4><<<blocks, kThreads, smem, st>>>(a);
    else
        k_worker<GT, false, LAZY_M, 4><<<blocks, kThreads, smem, st>>>(a);
}

template <typename GT>
int launch_worker(onebit_adam_s* h, const void* grads, cudaStream_t st) {
    WorkerArgs a{h->geo, h->beta1, 1.0f - h->beta1, h->m, h->bits_s, h->S_out, grads, h->ew,
                 h->s_lazy, h->bits_w, h->part_w, h->status};
    const size_t smem = (size_t)h->geo.W * kWarps * sizeof(double);
    const unsigned blocks = (unsigned)step_blocks(h->geo);
    if (h->m_explicit)
        launch_worker_t<GT, false>(h, a, blocks, smem, st);
    else
        launch_worker_t<GT, true>(h, a, blocks, smem, st);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

// m = +-S_out by the server plane, for elements [i0, i0 + n) (chunk-aligned i0), into dst.
int launch_materialize_m(onebit_adam_s* h, int64_t i0, int64_t n, float* dst, cudaStream_t st) {
    if (n == 0) return ONEBIT_OK;
    const Geometry& g = h->geo;
    k_unpack<<<(unsigned)ceil_div(n, kSeg), kThreads, 0, st>>>(h->bits_s + i0 / 32,
                                                               h->S_out + i0 / g.C, n, g.C, dst);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

template <typename GT>
int launch_warmup(onebit_adam_s* h, float* x, const void* grads, float lr, cudaStream_t st) {
    WarmupArgs a{h->geo, h->beta1, 1.0f - h->beta1, h->beta2, 1.0f - h->beta2, h->eps, lr,
                 grads, h->m, h->v, x};
    const unsigned blocks = (unsigned)step_blocks(h->geo);
    const int64_t d = h->geo.d;
    if constexpr (sizeof(GT) == 2) {
        if (d % 8 == 0) {
            k_warmup<GT, true, 8><<<blocks, kThreads, 0, st>>>(a);
            ONEBIT_CUDA(cudaGetLastError());
            return ONEBIT_OK;
        }
    }
    if (d % kVec == 0)
        k_warmup<GT, true, 4><<<blocks, kThreads, 0, st>>>(a);
    else
        k_warmup<GT, false, 4><<<blocks, kThreads, 0, st>>>(a);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

void record(onebit_adam_s* h, int slot, cudaStream_t st) {
    if (h->tcount < h->tmax) cudaEventRecord(h->ev[(size_t)h->tcount * kEventsPerStep + slot], st);
}

void free_events(onebit_adam_s* h) {
    for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
    h->ev.clear();
    h->tmax = h->tcount = 0;
}

uint64_t grad_elem_bytes(int32_t gtype) { return gtype == ONEBIT_BF16 ? 2 : 4; }

// Explicit residuals of elements [i0, i0 + n) of every row (W rows for the workers, 1 for the
// server) into dst[rows][n].
int launch_materialize(onebit_adam_s* h, bool workers, int64_t i0, int64_t n, float* dst,
                       cudaStream_t st) {
    const Geometry& g = h->geo;
    const int64_t rows = workers ? g.W : 1;
    const int64_t total = rows * n;
    if (total == 0) return ONEBIT_OK;
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(total, kThreads), 148 * 32);
    k_materialize<<<blocks, kThreads, 0, st>>>(workers ? h->ew : h->es, g.ld,
                                               workers ? h->s_lazy : h->S_lazy, g.nch, g.C, i0,
                                               n, rows, dst);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

}  // namespace

extern "C" {

const char* onebit_strerror(int32_t code) {
    switch (code) {
        case ONEBIT_OK: return "ok";
        case ONEBIT_ERR_ARG: return "invalid argument";
        case ONEBIT_ERR_ALIGN: return "misaligned pointer or chunk length not a multiple of 32";
        case ONEBIT_ERR_PHASE: return "call not allowed in the handle's current phase";
        case ONEBIT_ERR_CUDA: return "CUDA error";
        case ONEBIT_ERR_SPACE: return "workspace too small";
        default: return "unknown status";
    }
}

const char* onebit_last_error(void) { return g_last_error.c_str(); }

int onebit_adam_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1,
                     float beta2, float eps) {
    if (out == nullptr) return ONEBIT_ERR_ARG;
    *out = nullptr;
    if (d < 0 || W < 1 || W > kMaxWorkers || C <= 0) return ONEBIT_ERR_ARG;
    if (C % 32 != 0) return ONEBIT_ERR_ALIGN;
    if (!std::isfinite(beta1) || !std::isfinite(beta2) || !std::isfinite(eps)) return ONEBIT_ERR_ARG;
    if (beta1 < 0.0f || beta1 >= 1.0f || beta2 < 0.0f || beta2 >= 1.0f || eps < 0.0f)
        return ONEBIT_ERR_ARG;
    // sizes must stay far from int64 overflow: W * ld * 8 bytes < 2^62
    if (d > ((int64_t)1 << 46)) return ONEBIT_ERR_ARG;
    onebit_adam_s* h = new (std::nothrow) onebit_adam_s();
    if (h == nullptr) return ONEBIT_ERR_ARG;
    Geometry& g = h->geo;
    g.d = d;
    g.W = W;
    g.C = C;
    g.nch = ceil_div(d, C);
    g.nseg = ceil_div(C > d ? (d > 0 ? d : 1) : C, kSeg);
    g.nseg_s = ceil_div(C > d ? (d > 0 ? d : 1) : C, kSegS);
    g.ld = round_up(d > 0 ? d : 1, 64);
    h->nw = ceil_div(d, 32);
    g.ldw = round_up(h->nw > 0 ? h->nw : 1, 4);
    h->beta1 = beta1;
    h->beta2 = beta2;
    h->eps = eps;
    if (g.nch * g.nseg > (int64_t)INT32_MAX) {  // one block per segment must fit the grid
        delete h;
        return ONEBIT_ERR_ARG;
    }
    *out = h;
    return ONEBIT_OK;
}

int onebit_adam_workspace_bytes(onebit_adam_t h, int32_t grad_dtype, uint64_t* bytes) {
    if (!valid_handle(h) || bytes == nullptr) return ONEBIT_ERR_ARG;
    if (grad_dtype != ONEBIT_F32 && grad_dtype != ONEBIT_BF16) return ONEBIT_ERR_ARG;
    *bytes = make_layout(*h).total;
    return ONEBIT_OK;
}

int onebit_adam_bind(onebit_adam_t h, void* workspace, uint64_t bytes, int32_t grad_dtype,
                     void* stream) {
    if (!valid_handle(h) || workspace == nullptr) return ONEBIT_ERR_ARG;
    if (grad_dtype != ONEBIT_F32 && grad_dtype != ONEBIT_BF16) return ONEBIT_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ONEBIT_ERR_ALIGN;
    const Layout L = make_layout(*h);
    if (bytes < L.total) return ONEBIT_ERR_SPACE;
    char* b = static_cast<char*>(workspace);
    h->ws = b;
    h->lay = L;
    h->m = reinterpret_cast<float*>(b + L.m);
    h->v = reinterpret_cast<float*>(b + L.v);
    h->es = reinterpret_cast<float*>(b + L.es);
    h->ew = reinterpret_cast<float*>(b + L.ew);
    h->bits_w = reinterpret_cast<uint32_t*>(b + L.bits_w);
    h->bits_s = reinterpret_cast<uint32_t*>(b + L.bits_s);
    h->s_out = reinterpret_cast<float*>(b + L.s_out);
    h->s_lazy = reinterpret_cast<float*>(b + L.s_lazy);
    h->S_out = reinterpret_cast<float*>(b + L.S_out);
    h->S_lazy = reinterpret_cast<float*>(b + L.S_lazy);
    h->part_w = reinterpret_cast<double*>(b + L.part_w);
    h->part_s = reinterpret_cast<double*>(b + L.part_s);
    h->status = reinterpret_cast<uint32_t*>(b + L.status);
    h->gtype = grad_dtype;
    const int ssm = (int)server_smem_bytes(h->geo.W, server_stages(h->geo.W, h->geo.nseg_s));
    ONEBIT_CUDA(cudaFuncSetAttribute(server_kernel(h->geo.W),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, ssm));
    cudaStream_t st = as_stream(stream);
    // m and v start at zero (Adam); the rest is cleared too so padding is deterministic.
    ONEBIT_CUDA(cudaMemsetAsync(b, 0, L.total, st));
    h->phase = kWarmup;
    h->steps = 0;
    h->m_explicit = true;
    return ONEBIT_OK;
}

int onebit_adam_warmup_step(onebit_adam_t h, float* x, const void* grads, float lr,
                            void* stream) {
    if (!valid_handle(h) || !std::isfinite(lr)) return ONEBIT_ERR_ARG;
    if (h->phase != kWarmup) return ONEBIT_ERR_PHASE;
    if (h->geo.d == 0) return ONEBIT_OK;
    if (x == nullptr || grads == nullptr) return ONEBIT_ERR_ARG;
    if (!aligned16(x) || !aligned16(grads)) return ONEBIT_ERR_ALIGN;
    cudaStream_t st = as_stream(stream);
    return h->gtype == ONEBIT_BF16 ? launch_warmup<uint16_t>(h, x, grads, lr, st)
                                   : launch_warmup<float>(h, x, grads, lr, st);
}

int onebit_adam_freeze_variance(onebit_adam_t h, void* stream) {
    if (!valid_handle(h)) return ONEBIT_ERR_ARG;
    if (h->phase != kWarmup) return ONEBIT_ERR_PHASE;
    cudaStream_t st = as_stream(stream);
    const Layout& L = h->lay;
    // residuals (lazy form: stored 0 with scale 0 rebuilds e = 0), planes, scales, partials
    ONEBIT_CUDA(cudaMemsetAsync(h->ws + L.es, 0, L.total - L.es, st));
    h->phase = kCompressed;
    h->steps = 0;
    return ONEBIT_OK;
}

int onebit_adam_compressed_step(onebit_adam_t h, float* x, const void* grads, float lr,
                                void* stream) {
    if (!valid_handle(h) || !std::isfinite(lr)) return ONEBIT_ERR_ARG;
    if (h->phase != kCompressed) return ONEBIT_ERR_PHASE;
    if (h->geo.d == 0) {
        ++h->steps;
        return ONEBIT_OK;
    }
    if (x == nullptr || grads == nullptr) return ONEBIT_ERR_ARG;
    if (!aligned16(x) || !aligned16(grads)) return ONEBIT_ERR_ALIGN;
    cudaStream_t st = as_stream(stream);
    const Geometry& g = h->geo;
    const unsigned blocks = (unsigned)step_blocks(g);
    int rc;
    // one profiler range per step (NVTX; a no-op without a tool attached)
    struct Range {
        Range() { nvtxRangePushA("onebit_adam_compressed_step"); }
        ~Range() { nvtxRangePop(); }
    } range;

    record(h, 0, st);
    rc = h->gtype == ONEBIT_BF16 ? launch_worker<uint16_t>(h, grads, st)
                                 : launch_worker<float>(h, grads, st);
    if (rc != ONEBIT_OK) return rc;
    record(h, 1, st);
    rc = launch_scales(g, h->part_w, (int64_t)g.W * g.nch, g.nseg, kSeg, h->s_out, h->s_lazy, st);
    if (rc != ONEBIT_OK) return rc;
    record(h, 2, st);
    ServerArgs sa{g, h->bits_w, h->s_out, h->es, h->S_lazy, h->bits_s, h->part_s, h->status};
    const size_t ssm = server_smem_bytes(g.W, server_stages(g.W, g.nseg_s));
    const unsigned sblocks = (unsigned)server_blocks(g);
    server_kernel(g.W)<<<sblocks, kThreads, ssm, st>>>(sa);
    ONEBIT_CUDA(cudaGetLastError());
    record(h, 3, st);
    rc = launch_scales(g, h->part_s, g.nch, server_blocks_per_chunk(g),
                       kSegS * kSrvSegsPerBlock, h->S_out, h->S_lazy, st);
    if (rc != ONEBIT_OK) return rc;
    record(h, 4, st);
    ApplyArgs pa{g, h->eps, lr, h->bits_s, h->S_out, h->v, x};
    k_apply<<<blocks, kThreads, 0, st>>>(pa);
    ONEBIT_CUDA(cudaGetLastError());
    record(h, 5, st);
    if (h->tcount < h->tmax) ++h->tcount;
    ++h->steps;
    h->m_explicit = false;  // m is now the server message of this step
    return ONEBIT_OK;
}

int onebit_adam_compressed_step_host(onebit_adam_t h, float* x_dev, void* grads_dev,
                                     const void* grads_host, float* x_host, float lr,
                                     void* stream) {
    if (!valid_handle(h)) return ONEBIT_ERR_ARG;
    if (h->phase != kCompressed) return ONEBIT_ERR_PHASE;
    if (h->geo.d == 0) return onebit_adam_compressed_step(h, x_dev, grads_dev, lr, stream);
    if (grads_host == nullptr || x_host == nullptr || grads_dev == nullptr || x_dev == nullptr)
        return ONEBIT_ERR_ARG;
    cudaStream_t st = as_stream(stream);
    if (h->d2h == nullptr) {
        ONEBIT_CUDA(cudaStreamCreateWithFlags(&h->d2h, cudaStreamNonBlocking));
        ONEBIT_CUDA(cudaEventCreateWithFlags(&h->step_done, cudaEventDisableTiming));
        ONEBIT_CUDA(cudaEventCreateWithFlags(&h->d2h_done, cudaEventDisableTiming));
    }
    const uint64_t gbytes = (uint64_t)h->geo.W * h->geo.d * grad_elem_bytes(h->gtype);
    // the upload is queued first, so it overlaps the previous step's read-back of x; the step
    // itself (which rewrites x) waits for that read-back
    ONEBIT_CUDA(cudaMemcpyAsync(grads_dev, grads_host, gbytes, cudaMemcpyHostToDevice, st));
    if (h->d2h_pending) ONEBIT_CUDA(cudaStreamWaitEvent(st, h->d2h_done, 0));
    const int rc = onebit_adam_compressed_step(h, x_dev, grads_dev, lr, stream);
    if (rc != ONEBIT_OK) return rc;
    ONEBIT_CUDA(cudaEventRecord(h->step_done, st));
    ONEBIT_CUDA(cudaStreamWaitEvent(h->d2h, h->step_done, 0));
    ONEBIT_CUDA(cudaMemcpyAsync(x_host, x_dev, (uint64_t)h->geo.d * sizeof(float),
                                cudaMemcpyDeviceToHost, h->d2h));
    ONEBIT_CUDA(cudaEventRecord(h->d2h_done, h->d2h));
    h->d2h_pending = true;
    return ONEBIT_OK;
}

int onebit_adam_host_wait(onebit_adam_t h, void* stream) {
    if (!valid_handle(h)) return ONEBIT_ERR_ARG;
    if (h->d2h_pending) ONEBIT_CUDA(cudaStreamWaitEvent(as_stream(stream), h->d2h_done, 0));
    return ONEBIT_OK;
}

int onebit_adam_state_bytes(onebit_adam_t h, int32_t which, uint64_t* bytes) {
    if (!valid_handle(h) || bytes == nullptr) return ONEBIT_ERR_ARG;
    const Geometry& g = h->geo;
    const uint64_t f = sizeof(float);
    switch (which) {
        case ONEBIT_STATE_M:
        case ONEBIT_STATE_V:
        case ONEBIT_STATE_ES: *bytes = g.d * f; break;
        case ONEBIT_STATE_EW: *bytes = (uint64_t)g.W * g.d * f; break;
        case ONEBIT_STATE_SW: *bytes = (uint64_t)g.W * g.nch * f; break;
        case ONEBIT_STATE_SS: *bytes = g.nch * f; break;
        case ONEBIT_STATE_BITSW: *bytes = (uint64_t)g.W * h->nw * sizeof(uint32_t); break;
        case ONEBIT_STATE_BITSS: *bytes = h->nw * sizeof(uint32_t); break;
        default: return ONEBIT_ERR_ARG;
    }
    return ONEBIT_OK;
}

int onebit_adam_get_state(onebit_adam_t h, int32_t which, void* dst, void* stream) {
    uint64_t bytes = 0;
    int rc = onebit_adam_state_bytes(h, which, &bytes);
    if (rc != ONEBIT_OK) return rc;
    if (h->phase == kUnbound) return ONEBIT_ERR_PHASE;
    if (bytes == 0) return ONEBIT_OK;
    if (dst == nullptr) return ONEBIT_ERR_ARG;
    cudaStream_t st = as_stream(stream);
    const Geometry& g = h->geo;
    const auto D2D = cudaMemcpyDeviceToDevice;
    switch (which) {
        case ONEBIT_STATE_M:
            if (!h->m_explicit) return launch_materialize_m(h, 0, g.d, static_cast<float*>(dst), st);
            ONEBIT_CUDA(cudaMemcpyAsync(dst, h->m, bytes, D2D, st));
            break;
        case ONEBIT_STATE_V: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->v, bytes, D2D, st)); break;
        case ONEBIT_STATE_SW: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->s_out, bytes, D2D, st)); break;
        case ONEBIT_STATE_SS: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->S_out, bytes, D2D, st)); break;
        case ONEBIT_STATE_BITSW:
            ONEBIT_CUDA(cudaMemcpy2DAsync(dst, h->nw * sizeof(uint32_t), h->bits_w,
                                          g.ldw * sizeof(uint32_t), h->nw * sizeof(uint32_t),
                                          g.W, D2D, st));
            break;
        case ONEBIT_STATE_BITSS: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->bits_s, bytes, D2D, st)); break;
        case ONEBIT_STATE_EW:
        case ONEBIT_STATE_ES: {
            const bool wk = which == ONEBIT_STATE_EW;
            const int rc2 = launch_materialize(h, wk, 0, g.d, static_cast<float*>(dst), st);
            if (rc2 != ONEBIT_OK) return rc2;
            break;
        }
        default: return ONEBIT_ERR_ARG;
    }
    return ONEBIT_OK;
}

int onebit_adam_get_chunk_state(onebit_adam_t h, int32_t which, int64_t k, void* dst,
                                void* stream) {
    if (!valid_handle(h)) return ONEBIT_ERR_ARG;
    if (h->phase == kUnbound) return ONEBIT_ERR_PHASE;
    const Geometry& g = h->geo;
    if (k < 0 || k >= g.nch || dst == nullptr) return ONEBIT_ERR_ARG;
    cudaStream_t st = as_stream(stream);
    const int64_t i0 = k * g.C, n = std::min(g.C, g.d - i0);
    const int64_t w0 = i0 / 32, nwk = ceil_div(n, 32);
    const uint64_t f = sizeof(float), u = sizeof(uint32_t);
    const auto D2D = cudaMemcpyDeviceToDevice;
    switch (which) {
        case ONEBIT_STATE_M:
            if (!h->m_explicit) return launch_materialize_m(h, i0, n, static_cast<float*>(dst), st);
            ONEBIT_CUDA(cudaMemcpyAsync(dst, h->m + i0, n * f, D2D, st));
            break;
        case ONEBIT_STATE_V: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->v + i0, n * f, D2D, st)); break;
        case ONEBIT_STATE_EW:
        case ONEBIT_STATE_ES:
            return launch_materialize(h, which == ONEBIT_STATE_EW, i0, n,
                                      static_cast<float*>(dst), st);
        case ONEBIT_STATE_SW:
            ONEBIT_CUDA(cudaMemcpy2DAsync(dst, f, h->s_out + k, g.nch * f, f, g.W, D2D, st));
            break;
        case ONEBIT_STATE_SS: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->S_out + k, f, D2D, st)); break;
        case ONEBIT_STATE_BITSW:
            ONEBIT_CUDA(cudaMemcpy2DAsync(dst, nwk * u, h->bits_w + w0, g.ldw * u, nwk * u, g.W,
                                          D2D, st));
            break;
        case ONEBIT_STATE_BITSS:
            ONEBIT_CUDA(cudaMemcpyAsync(dst, h->bits_s + w0, nwk * u, D2D, st));
            break;
        default: return ONEBIT_ERR_ARG;
    }
    return ONEBIT_OK;
}

int onebit_adam_set_state(onebit_adam_t h, int32_t which, const void* src, void* stream) {
    uint64_t bytes = 0;
    int rc = onebit_adam_state_bytes(h, which, &bytes);
    if (rc != ONEBIT_OK) return rc;
    if (h->phase == kUnbound) return ONEBIT_ERR_PHASE;
    if (which != ONEBIT_STATE_M && which != ONEBIT_STATE_V && which != ONEBIT_STATE_EW &&
        which != ONEBIT_STATE_ES)
        return ONEBIT_ERR_ARG;
    if (bytes == 0) return ONEBIT_OK;
    if (src == nullptr) return ONEBIT_ERR_ARG;
    cudaStream_t st = as_stream(stream);
    const Geometry& g = h->geo;
    const auto D2D = cudaMemcpyDeviceToDevice;
    const uint64_t f = sizeof(float);
    switch (which) {
        case ONEBIT_STATE_M:
            ONEBIT_CUDA(cudaMemcpyAsync(h->m, src, bytes, D2D, st));
            h->m_explicit = true;
            break;
        case ONEBIT_STATE_V: ONEBIT_CUDA(cudaMemcpyAsync(h->v, src, bytes, D2D, st)); break;
        case ONEBIT_STATE_EW:
            // explicit residual with a zero rebuild scale: e = stored - (+-0) = stored exactly
            ONEBIT_CUDA(cudaMemcpy2DAsync(h->ew, g.ld * f, src, g.d * f, g.d * f, g.W, D2D, st));
            ONEBIT_CUDA(cudaMemsetAsync(h->s_lazy, 0, (uint64_t)g.W * g.nch * f, st));
            ONEBIT_CUDA(cudaMemsetAsync(h->s_out, 0, (uint64_t)g.W * g.nch * f, st));
            break;
        case ONEBIT_STATE_ES:
            if (!h->m_explicit) {
                // m lives in S_out, which is about to be cleared: make it explicit first
                const int rc2 = launch_materialize_m(h, 0, g.d, h->m, st);
                if (rc2 != ONEBIT_OK) return rc2;
                h->m_explicit = true;
            }
            ONEBIT_CUDA(cudaMemcpyAsync(h->es, src, bytes, D2D, st));
            ONEBIT_CUDA(cudaMemsetAsync(h->S_lazy, 0, g.nch * f, st));
            ONEBIT_CUDA(cudaMemsetAsync(h->S_out, 0, g.nch * f, st));
            break;
        default: return ONEBIT_ERR_ARG;
    }
    return ONEBIT_OK;
}

int onebit_adam_status(onebit_adam_t h, void* stream, uint32_t* flags) {
    if (!valid_handle(h) || flags == nullptr) return ONEBIT_ERR_ARG;
    *flags = 0;
    if (h->phase == kUnbound) return ONEBIT_ERR_PHASE;
    cudaStream_t st = as_stream(stream);
    uint32_t hostv = 0;
    ONEBIT_CUDA(cudaMemcpyAsync(&hostv, h->status, sizeof hostv, cudaMemcpyDeviceToHost, st));
    ONEBIT_CUDA(cudaMemsetAsync(h->status, 0, sizeof hostv, st));
    ONEBIT_CUDA(cudaStreamSynchronize(st));
    *flags = hostv;
    return ONEBIT_OK;
}

int onebit_adam_info(onebit_adam_t h, int64_t out[8]) {
    if (!valid_handle(h) || out == nullptr) return ONEBIT_ERR_ARG;
    out[0] = h->geo.d;
    out[1] = h->geo.W;
    out[2] = h->geo.C;
    out[3] = h->geo.nch;
    out[4] = h->phase;
    out[5] = h->steps;
    out[6] = h->gtype;
    out[7] = kLaunchesPerStep;
    return ONEBIT_OK;
}

int onebit_adam_timing(onebit_adam_t h, int32_t max_steps) {
    if (!valid_handle(h) || max_steps < 0 || max_steps > (1 << 20)) return ONEBIT_ERR_ARG;
    free_events(h);
    if (max_steps == 0) return ONEBIT_OK;
    h->ev.resize((size_t)max_steps * kEventsPerStep, nullptr);
    for (auto& e : h->ev) {
        const cudaError_t rc = cudaEventCreate(&e);
        if (rc != cudaSuccess) {
            e = nullptr;
            for (auto& f : h->ev)
                if (f) cudaEventDestroy(f);
            h->ev.clear();
            return cuda_fail(rc);
        }
    }
    h->tmax = max_steps;
    h->tcount = 0;
    return ONEBIT_OK;
}

int onebit_adam_timing_read(onebit_adam_t h, double ms_out[5], int32_t* steps) {
    if (!valid_handle(h) || ms_out == nullptr || steps == nullptr) return ONEBIT_ERR_ARG;
    for (int i = 0; i < kLaunchesPerStep; ++i) ms_out[i] = 0.0;
    *steps = h->tcount;
    if (h->tcount == 0) return ONEBIT_OK;
    ONEBIT_CUDA(cudaEventSynchronize(h->ev[(size_t)h->tcount * kEventsPerStep - 1]));
    for (int32_t s = 0; s < h->tcount; ++s) {
        for (int i = 0; i < kLaunchesPerStep; ++i) {
            float ms = 0.0f;
            ONEBIT_CUDA(cudaEventElapsedTime(&ms, h->ev[(size_t)s * kEventsPerStep + i],
                                             h->ev[(size_t)s * kEventsPerStep + i + 1]));
            ms_out[i] += ms;
        }
    }
    h->tcount = 0;
    return ONEBIT_OK;
}

void onebit_adam_destroy(onebit_adam_t h) {
    if (h == nullptr) return;
    free_events(h);
    if (h->d2h != nullptr) {
        cudaStreamSynchronize(h->d2h);
        cudaStreamDestroy(h->d2h);
        cudaEventDestroy(h->step_done);
        cudaEventDestroy(h->d2h_done);
    }
    delete h;
}

int onebit_selftest_bounded_wait(int32_t polls, uint32_t* timed_out, void* stream) {
    if (polls < 1 || polls > kSpinLimit || timed_out == nullptr) return ONEBIT_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(timed_out) & 3u) return ONEBIT_ERR_ALIGN;
    k_selftest_wait<<<1, 32, 0, as_stream(stream)>>>(polls, timed_out);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

int onebit_pack(const float* x, int64_t n, uint32_t* words, void* stream) {
    if (n < 0) return ONEBIT_ERR_ARG;
    if (n == 0) return ONEBIT_OK;
    if (x == nullptr || words == nullptr) return ONEBIT_ERR_ARG;
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(words) & 3u)) return ONEBIT_ERR_ALIGN;
    if (n > ((int64_t)1 << 46)) return ONEBIT_ERR_ARG;
    k_pack<<<(unsigned)ceil_div(n, kSeg), kThreads, 0, as_stream(stream)>>>(x, n, words);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

int onebit_unpack(const uint32_t* words, const float* scales, int64_t n, int64_t C, float* out,
                  void* stream) {
    if (n < 0 || C < 1) return ONEBIT_ERR_ARG;
    if (n == 0) return ONEBIT_OK;
    if (words == nullptr || scales == nullptr || out == nullptr) return ONEBIT_ERR_ARG;
    if (!aligned16(out) || (reinterpret_cast<uintptr_t>(words) & 3u) ||
        (reinterpret_cast<uintptr_t>(scales) & 3u))
        return ONEBIT_ERR_ALIGN;
    if (n > ((int64_t)1 << 46)) return ONEBIT_ERR_ARG;
    k_unpack<<<(unsigned)ceil_div(n, kSeg), kThreads, 0, as_stream(stream)>>>(words, scales, n,
                                                                            C, out);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// One-vector compression whose scratch is a fixed array inside the library, so that neither the
// caller nor the library allocates device memory for it.

namespace {

// fp64 norm partials of onebit_compress_static: one slot per kSeg-element segment, 512 KiB.
// Every GPU that loads the library holds this array until the process exits.
constexpr int64_t kStaticSegs = 1 << 16;
static __device__ __align__(256) double g_static_partials[kStaticSegs];

constexpr int kMaxDevices = 64;
double* g_static_addr[kMaxDevices] = {};
std::mutex g_static_mu;

// Device address of g_static_partials on the current device, looked up once per device. In
// host code the array's name is only a host-side stand-in, never a device address.
int static_partials(double** out) {
    int dev = 0;
    ONEBIT_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return ONEBIT_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_addr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_partials);
        if (e != cudaSuccess) return cuda_fail(e);
        g_static_addr[dev] = static_cast<double*>(p);
    }
    *out = g_static_addr[dev];
    return ONEBIT_OK;
}

// Sign words and per-segment fp64 sums of squares of x, one kSeg segment per block; the
// per-thread, per-warp and per-block summation order is the worker kernel's, so the scales
// equal the compressed step's worker scales for the same values.
__global__ void __launch_bounds__(kThreads, 8) k_compress_partials(const float* x, int64_t n,
                                                                   int64_t C, int64_t nseg,
                                                                   uint32_t* words,
                                                                   double* part) {
    __shared__ double red[kWarps];
    const int64_t k = (int64_t)blockIdx.x / nseg;
    const int64_t j = (int64_t)blockIdx.x - k * nseg;
    const int64_t c0 = k * C;
    const int64_t clen = min(C, n - c0);
    const int64_t s0 = j * kSeg;
    if (s0 >= clen) return;
    const int64_t base = c0 + s0;
    const int64_t len = min((int64_t)kSeg, clen - s0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    double ss = 0.0;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * kVec;
        const int nv = valid_of(len, off);
        float xv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (nv > 0) ld4_caller(x + base + off, nv, xv);
        uint32_t nib = 0u;
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            const float v = c < nv ? xv[c] : 0.0f;
            nib |= (c < nv && v >= 0.0f) ? (1u << c) : 0u;
            ss = __fma_rn((double)v, (double)v, ss);
        }
        const uint32_t word = gather_word(nib, lane);
        if ((lane & 7) == 0 && nv > 0) words[(base >> 5) + (q >> 3)] = word;
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) part[k * nseg + j] = block_total(red);
}

}  // namespace

extern "C" int onebit_compress_static(const float* x, int64_t n, int64_t C, uint32_t* words,
                                      float* scales, void* stream) {
    if (n < 0 || C <= 0) return ONEBIT_ERR_ARG;
    if (C % 32 != 0) return ONEBIT_ERR_ALIGN;
    if (n == 0) return ONEBIT_OK;
    if (x == nullptr || words == nullptr || scales == nullptr) return ONEBIT_ERR_ARG;
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(words) & 3u) ||
        (reinterpret_cast<uintptr_t>(scales) & 3u))
        return ONEBIT_ERR_ALIGN;
    if (n > ((int64_t)1 << 46)) return ONEBIT_ERR_ARG;
    const int64_t nch = ceil_div(n, C);
    const int64_t nseg = ceil_div(std::min(C, n), kSeg);
    if (nch * nseg > kStaticSegs) {
        g_last_error = "onebit_compress_static: ceil(n/C) * ceil(min(C,n)/2048) = " +
                       std::to_string(nch * nseg) + " segments exceeds the fixed scratch of " +
                       std::to_string(kStaticSegs);
        return ONEBIT_ERR_SPACE;
    }
    double* part = nullptr;
    const int rc = static_partials(&part);
    if (rc != ONEBIT_OK) return rc;
    cudaStream_t st = as_stream(stream);
    k_compress_partials<<<(unsigned)(nch * nseg), kThreads, 0, st>>>(x, n, C, nseg, words, part);
    ONEBIT_CUDA(cudaGetLastError());
    Geometry g{};
    g.d = n;
    g.C = C;
    g.nch = nch;
    g.nseg = nseg;
    g.W = 1;
    // every slot read by the reduction was written by k_compress_partials in this same call,
    // so nothing in the shared array has to be cleared first
    return launch_scales(g, part, nch, nseg, kSeg, scales, scales, st);
}
