// onebit_adam.cu -- host side of the C ABI declared in include/onebit_adam.h: argument checks,
// the workspace layout, the launch sequence of one step and the state/timing helpers.
//
// One compressed step is five launches on the caller's stream (three for small buckets, whose
// chunk-scale reductions fold into the server and apply kernels), ordered by the stream alone
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
#include "kernels_dp.cuh"
#include "kernels_zero_one.cuh"

using namespace onebit;

namespace {

thread_local std::string g_last_error;

constexpr int32_t kMaxWorkers = 256;
constexpr int kLaunchesPerStep = 5;
constexpr int kLaunchesPerStepDp = 7;  // plus one barrier after each half of the exchange
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

// Workspace regions, each 256-byte aligned. For a data-parallel rank, m, v, bits_w, bits_s and
// S_out have no space here (m, v, the server plane and scales live in the exchange region, the
// worker planes at their servers) and `route` holds the device copy of the rank's route.
struct Layout {
    uint64_t route, m, v, es, ew, sbits, bits_s, s_out, s_lazy, S_out, S_lazy, part_w, part_s,
        status, mw, uw;
    uint64_t total;
};

// Exchange region of a data-parallel rank: the buffers that other ranks write (and, for the
// warm-up partial sums, read). Its layout depends only on (d, W, C, R), so it is the same on
// every rank and one base address per rank locates all of a peer's buffers.
struct XLayout {
    uint64_t flags, m, v, wpart, planes, rscales, bits_s, S;
    uint64_t total;
};

// The data-parallel part of a handle (R = 0: a single-GPU handle).
struct DpState {
    int32_t R = 0, rank = 0;
    int32_t Wg = 0;                    // workers over all ranks
    int64_t kb[kMaxRanks + 1] = {};    // chunk bounds of the ranks
    Geometry gs{};                     // this rank's chunks, all Wg workers
    int64_t e0 = 0;                    // first element of this rank's chunks
    XLayout xl{};
    char* xch = nullptr;               // this rank's exchange region (cudaMalloc)
    char* peer[kMaxRanks] = {};        // peers' exchange regions, addresses in this process
    bool ipc[kMaxRanks] = {};          // peer mapped by CUDA IPC (closed at destroy)
    DpRoute route{};                   // host copy of the route
    DpRoute* route_dev = nullptr;      // device copy (in the workspace)
    uint32_t* epoch_dev = nullptr;     // barriers signalled so far (device, after the route)
    bool connected = false;
    int next_phase = 0;                // phase-by-phase driving: the phase expected next
    int phase_kind = 0;                // 0 none in progress, 1 warm-up, 2 compressed
    uint64_t timeout_ns = 10000000000ull;
};

}  // namespace

// The 0/1 Adam variant's schedule and step state (zero_one false: a 1-bit Adam handle).
struct ZoState {
    bool on = false;
    int32_t H = 1, K = 0;      // a synchronisation every H steps, a refresh every K-th (0: never)
    int32_t t = 0;             // steps since the last synchronisation
    int64_t syncs = 0;
    float gamma = 0.0f;        // fp32 sum of the learning rates since the last synchronisation
    float gamma_prev = 0.0f;   // Gamma of the last synchronisation (mbar = ubar / gamma_prev)
    float lr_first = 0.0f;     // learning rate of the interval's first step (kZoMWorkerU1)
    int src = kZoMShared;      // where the next step's momentum comes from (ZoSource)
};

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
    uint8_t* sbits = nullptr;  // worker sign bits grouped by 8 workers (single GPU)
    uint32_t *bits_s = nullptr, *status = nullptr;
    double *part_w = nullptr, *part_s = nullptr;
    // per-kernel timing
    std::vector<cudaEvent_t> ev;
    int32_t tmax = 0, tcount = 0;
    // host-buffer steps: the read-back of x runs on its own stream so that it overlaps the
    // next step's gradient upload (created on the first host-buffer step)
    cudaStream_t d2h = nullptr;
    cudaEvent_t step_done = nullptr, d2h_done = nullptr;
    bool d2h_pending = false;
    DpState dp;
    ZoState zo;
    // optional bias-corrected warm-up: the fp64 products beta^t of the steps so far
    bool bc = false;
    int64_t wsteps = 0;
    double p1 = 1.0, p2 = 1.0;
    float *mw = nullptr, *uw = nullptr;  // the 0/1 variant's per-worker momentum and update
};

namespace {

Layout make_layout(const onebit_adam_s& h) {
    const Geometry& g = h.geo;
    const bool dp = h.dp.R > 0;
    const Geometry& gs = dp ? h.dp.gs : g;  // the server's chunks
    Layout L{};
    uint64_t off = 0;
    auto take = [&](uint64_t bytes) {
        const uint64_t at = off;
        off = (uint64_t)round_up((int64_t)(off + bytes), 256);
        return at;
    };
    const uint64_t f = sizeof(float), u = sizeof(uint32_t);
    // the route, then the rank's barrier count (kept across connects and freezes)
    L.route = take(dp ? sizeof(DpRoute) + sizeof(uint32_t) : 0);
    L.m = take(dp ? 0 : g.ld * f);
    L.v = take(dp ? 0 : g.ld * f);
    L.es = take(gs.ld * f);
    L.ew = take((uint64_t)g.W * g.ld * f);
    L.sbits = take(dp ? 0 : (uint64_t)((g.W + 7) / 8) * g.ld);
    L.bits_s = take(dp ? 0 : g.ldw * u);
    L.s_out = take((uint64_t)g.W * g.nch * f);
    L.s_lazy = take((uint64_t)g.W * g.nch * f);
    L.S_out = take(dp ? 0 : g.nch * f);
    L.S_lazy = take((uint64_t)std::max<int64_t>(gs.nch, 1) * f);
    L.part_w = take((uint64_t)g.W * g.nch * g.nseg * sizeof(double));
    L.part_s = take((uint64_t)std::max<int64_t>(gs.nch, 1) * g.nseg_s * sizeof(double));
    L.status = take(4 * sizeof(uint32_t));
    L.mw = take(h.zo.on ? (uint64_t)g.W * g.ld * f : 0);
    L.uw = take(h.zo.on ? (uint64_t)g.W * g.ld * f : 0);
    L.total = off;
    return L;
}

// Rank q's chunks of nch: [q * nch / R, (q + 1) * nch / R), contiguous and balanced.
void dp_range(int64_t nch, int32_t R, int32_t q, int64_t* k0, int64_t* k1) {
    *k0 = (int64_t)((__int128)nch * q / R);
    *k1 = (int64_t)((__int128)nch * (q + 1) / R);
}

// Elements and receive-plane row length (words, padded to 16 bytes) of rank q's chunks.
int64_t dp_elems(const onebit_adam_s& h, int32_t q) {
    const Geometry& g = h.geo;
    const int64_t* kb = h.dp.kb;
    return std::max<int64_t>(0, std::min(kb[q + 1] * g.C, g.d) - kb[q] * g.C);
}
int64_t dp_ldw(const onebit_adam_s& h, int32_t q) {
    return round_up(std::max<int64_t>(ceil_div(dp_elems(h, q), 32), 1), 4);
}

XLayout make_xlayout(const onebit_adam_s& h) {
    const Geometry& g = h.geo;
    const DpState& dp = h.dp;
    int64_t ldw_max = 4, nch_max = 1;
    for (int32_t q = 0; q < dp.R; ++q) {
        ldw_max = std::max(ldw_max, dp_ldw(h, q));
        nch_max = std::max(nch_max, dp.kb[q + 1] - dp.kb[q]);
    }
    XLayout X{};
    uint64_t off = 0;
    auto take = [&](uint64_t bytes) {
        const uint64_t at = off;
        off = (uint64_t)round_up((int64_t)(off + bytes), 256);
        return at;
    };
    const uint64_t f = sizeof(float), u = sizeof(uint32_t);
    X.flags = take(kMaxRanks * u);
    X.m = take(g.ld * f);
    X.v = take(g.ld * f);
    X.wpart = take(g.ld * sizeof(double));
    X.planes = take((uint64_t)dp.Wg * ldw_max * u);
    X.rscales = take((uint64_t)dp.Wg * nch_max * f);
    X.bits_s = take(g.ldw * u);
    X.S = take(g.nch * f);
    X.total = off;
    return X;
}

bool valid_handle(onebit_adam_t h) { return h != nullptr; }
bool is_dp(const onebit_adam_s* h) { return h->dp.R > 0; }

int64_t step_blocks(const Geometry& g) { return g.nch * g.nseg; }
int64_t server_blocks_per_chunk(const Geometry& g) {
    return ceil_div(g.nseg_s, g.spb);
}
int64_t server_blocks(const Geometry& g) { return g.nch * server_blocks_per_chunk(g); }

// Small chunk-scale reductions are folded into the kernel that consumes them (one launch less
// each, which is what small buckets pay for): the worker scales into the server kernel's
// prologue when a chunk has at most 8 server blocks and few partials (each of those blocks
// reduces them itself, in the order of the separate reduction), the server scale into the
// apply kernel when a chunk has at most 8 server partials.
bool fold_worker_scales(const Geometry& g) {
    return server_blocks_per_chunk(g) <= 8 && g.nseg <= 1024 && (int64_t)g.W * g.nseg <= 8192;
}
bool fold_server_scales(const Geometry& g) { return server_blocks_per_chunk(g) <= 8; }
int launches_per_step(const Geometry& g) {
    return kLaunchesPerStep - (fold_worker_scales(g) ? 1 : 0) - (fold_server_scales(g) ? 1 : 0);
}

// The k_server instantiation for a geometry: exact scaling for power-of-two W; bank-private
// int32 tables (unrolled over the 4 or 8 groups) where server_bank_private picks them, else
// single-copy tables with the residuals staged by TMA for W <= 32.
using ServerKernel = void (*)(ServerArgs);
template <bool POW2>
ServerKernel server_kernel_pow2(const Geometry& g) {
    const bool bp = server_bank_private(g.W, g.nseg_s, g.nch);
    if (bp) {
        const int ngroups = (g.W + 7) / 8;
        if (ngroups == 2)
            return server_stage_residuals(g.W, true) ? k_server<POW2, true, false, 2>
                                                     : k_server<POW2, false, false, 2>;
        return ngroups == 4 ? k_server<POW2, false, false, 4> : k_server<POW2, false, false, 8>;
    }
    return server_stage_residuals(g.W, false) ? k_server<POW2, true> : k_server<POW2, false>;
}
ServerKernel server_kernel(const Geometry& g) {
    return (g.W & (g.W - 1)) == 0 ? server_kernel_pow2<true>(g) : server_kernel_pow2<false>(g);
}

// Dynamic shared memory of the single-GPU server kernel of a geometry.
size_t server_smem(const Geometry& g) {
    return server_smem_bytes(g.W, server_stages(g.W, g.nseg_s),
                             server_bank_private(g.W, g.nseg_s, g.nch));
}

// The same for a data-parallel rank: the server plane is broadcast to every rank.
ServerKernel server_kernel_dp(int W) {
    const bool pow2 = (W & (W - 1)) == 0, staged = server_stage_residuals(W, false);
    if (pow2) return staged ? k_server<true, true, true> : k_server<true, false, true>;
    return staged ? k_server<false, true, true> : k_server<false, false, true>;
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

// Data-parallel scales (see k_scales_dp): geometry (nch, C, d) of the rows' chunks.
template <bool SERVER>
int launch_scales_dp(int64_t nch, int64_t C, int64_t d, const double* part, int64_t rows,
                     int64_t nseg, int64_t seg, float* out, float* lazy, const DpRoute* rt,
                     cudaStream_t st) {
    if (rows == 0) return ONEBIT_OK;
    if (nseg <= 8) {
        k_scales_dp<1, SERVER><<<(unsigned)ceil_div(rows, kThreads), kThreads, 0, st>>>(
            part, rows, nch, nseg, seg, C, d, out, lazy, rt);
    } else if (nseg <= 1024) {
        k_scales_dp<32, SERVER><<<(unsigned)ceil_div(rows, kWarps), kThreads, 0, st>>>(
            part, rows, nch, nseg, seg, C, d, out, lazy, rt);
    } else {
        k_scales_dp<kThreads, SERVER><<<(unsigned)rows, kThreads, 0, st>>>(
            part, rows, nch, nseg, seg, C, d, out, lazy, rt);
    }
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

// Vector width of the worker kernel: 8 elements per thread (16-byte loads of 8 bf16 values)
// when bf16 gradient rows are 16-byte aligned, 4 (16-byte loads of 4 fp32 values, or 8-byte
// loads of 4 bf16 values) when rows are 16- or 8-byte aligned, element by element otherwise.
template <typename GT, bool LAZY_M, bool DP>
void launch_worker_t(onebit_adam_s* h, const WorkerArgs& a, unsigned blocks, size_t smem,
                     cudaStream_t st) {
    const int64_t d = h->geo.d;
    if constexpr (sizeof(GT) == 2) {
        if (d % 8 == 0) {
            k_worker<GT, true, LAZY_M, 8, DP><<<blocks, kThreads, smem, st>>>(a);
            return;
        }
    }
    if (d % kVec == 0)
        k_worker<GT, true, LAZY_M, 4, DP><<<blocks, kThreads, smem, st>>>(a);
    else
        k_worker<GT, false, LAZY_M, 4, DP><<<blocks, kThreads, smem, st>>>(a);
}

template <typename GT>
int launch_worker(onebit_adam_s* h, const void* grads, cudaStream_t st) {
    WorkerArgs a{h->geo, h->beta1, 1.0f - h->beta1, h->m, h->bits_s, h->S_out, grads, h->ew,
                 h->s_lazy, h->sbits, h->part_w, h->status, h->dp.route_dev};
    const size_t smem = (size_t)h->geo.W * kWarps * sizeof(double);
    const unsigned blocks = (unsigned)step_blocks(h->geo);
    if (is_dp(h)) {
        if (h->m_explicit)
            launch_worker_t<GT, false, true>(h, a, blocks, smem, st);
        else
            launch_worker_t<GT, true, true>(h, a, blocks, smem, st);
    } else {
        if (h->m_explicit)
            launch_worker_t<GT, false, false>(h, a, blocks, smem, st);
        else
            launch_worker_t<GT, true, false>(h, a, blocks, smem, st);
    }
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

// c_t = fl32(1 - beta^t), beta^t the fp64 product of t factors beta (its fp32 value) in step
// order: the bias corrections of the optional bias-corrected warm-up (1 - beta2^t would lose
// most of its digits to cancellation in fp32).
float bias_correction(double p) { return (float)(1.0 - p); }

template <typename GT, bool BC>
void launch_warmup_t(onebit_adam_s* h, const WarmupArgs& a, cudaStream_t st) {
    const unsigned blocks = (unsigned)step_blocks(h->geo);
    const int64_t d = h->geo.d;
    if constexpr (sizeof(GT) == 2) {
        if (d % 8 == 0) {
            k_warmup<GT, true, 8, BC><<<blocks, kThreads, 0, st>>>(a);
            return;
        }
    }
    if (d % kVec == 0)
        k_warmup<GT, true, 4, BC><<<blocks, kThreads, 0, st>>>(a);
    else
        k_warmup<GT, false, 4, BC><<<blocks, kThreads, 0, st>>>(a);
}

template <typename GT>
int launch_warmup(onebit_adam_s* h, float* x, const void* grads, float lr, cudaStream_t st) {
    WarmupArgs a{h->geo, h->beta1, 1.0f - h->beta1, h->beta2, 1.0f - h->beta2, h->eps, lr,
                 1.0f, 1.0f, grads, h->m, h->v, x};
    if (h->bc) {
        a.c1 = bias_correction(h->p1 * (double)h->beta1);
        a.c2 = bias_correction(h->p2 * (double)h->beta2);
        launch_warmup_t<GT, true>(h, a, st);
    } else {
        launch_warmup_t<GT, false>(h, a, st);
    }
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
// For a data-parallel rank the server residual covers the rank's own chunks only, and i0 counts
// from their first element.
int launch_materialize(onebit_adam_s* h, bool workers, int64_t i0, int64_t n, float* dst,
                       cudaStream_t st) {
    const Geometry& g = workers || !is_dp(h) ? h->geo : h->dp.gs;
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

// Worker planes of a data-parallel rank, rebuilt from the stored x_w (bit = x_w >= 0): rows of
// elements [i0, i0 + n) into dst[W][ceil(n / 32)].
int launch_pack_rows(onebit_adam_s* h, int64_t i0, int64_t n, uint32_t* dst, cudaStream_t st) {
    const Geometry& g = h->geo;
    if (n == 0) return ONEBIT_OK;
    const int64_t nwk = ceil_div(n, 32);
    for (int32_t w = 0; w < g.W; ++w)
        k_pack<<<(unsigned)ceil_div(n, kSeg), kThreads, 0, st>>>(h->ew + (int64_t)w * g.ld + i0,
                                                                 n, dst + (int64_t)w * nwk);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

// ------------------------------------------------------------------------------------------
// Data-parallel step sequences. Phase p of a step runs on this rank alone up to the point
// where it needs the other ranks' stores; `sig` ends the phase with this rank's barrier signal
// and `wait` starts it with the wait for every rank's signal. A whole step fuses each signal
// with the following wait into one barrier launch.

int dp_barrier(onebit_adam_s* h, int mode, cudaStream_t st) {
    DpState& dp = h->dp;
    k_dp_barrier<<<1, 32, 0, st>>>(dp.route_dev, dp.epoch_dev, mode, dp.timeout_ns, h->status);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

template <typename GT>
int dp_warmup_partial(onebit_adam_s* h, const void* grads, cudaStream_t st) {
    const Geometry& g = h->geo;
    double* wpart = reinterpret_cast<double*>(h->dp.xch + h->dp.xl.wpart);
    const unsigned blocks = (unsigned)step_blocks(g);
    if constexpr (sizeof(GT) == 2) {
        if (g.d % 8 == 0) {
            k_warmup_partial<GT, true, 8><<<blocks, kThreads, 0, st>>>(g, grads, wpart);
            ONEBIT_CUDA(cudaGetLastError());
            return ONEBIT_OK;
        }
    }
    if (g.d % kVec == 0)
        k_warmup_partial<GT, true, 4><<<blocks, kThreads, 0, st>>>(g, grads, wpart);
    else
        k_warmup_partial<GT, false, 4><<<blocks, kThreads, 0, st>>>(g, grads, wpart);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

int dp_warmup_phase(onebit_adam_s* h, int phase, float* x, const void* grads, float lr,
                    int mode_in, int mode_out, cudaStream_t st) {
    DpState& dp = h->dp;
    int rc = ONEBIT_OK;
    if (mode_in) rc = dp_barrier(h, mode_in, st);
    if (rc != ONEBIT_OK) return rc;
    if (phase == 0) {
        rc = h->gtype == ONEBIT_BF16 ? dp_warmup_partial<uint16_t>(h, grads, st)
                                     : dp_warmup_partial<float>(h, grads, st);
    } else if (phase == 1) {
        if (dp.gs.d > 0) {
            WarmupDpArgs a{dp.gs, dp.e0, h->beta1, 1.0f - h->beta1, h->beta2, 1.0f - h->beta2,
                           dp.route_dev};
            k_warmup_reduce<<<(unsigned)step_blocks(dp.gs), kThreads, 0, st>>>(a);
            ONEBIT_CUDA(cudaGetLastError());
        }
    } else {
        WarmupApplyArgs a{h->geo, h->eps, lr, h->m, h->v, x};
        k_warmup_apply<<<(unsigned)step_blocks(h->geo), kThreads, 0, st>>>(a);
        ONEBIT_CUDA(cudaGetLastError());
    }
    if (rc != ONEBIT_OK) return rc;
    if (mode_out) rc = dp_barrier(h, mode_out, st);
    return rc;
}

int dp_compressed_phase(onebit_adam_s* h, int phase, float* x, const void* grads, float lr,
                        int mode_in, int mode_out, cudaStream_t st) {
    DpState& dp = h->dp;
    const Geometry& g = h->geo;
    int rc = ONEBIT_OK;
    if (mode_in) rc = dp_barrier(h, mode_in, st);
    if (rc != ONEBIT_OK) return rc;
    if (phase == 0) {
        record(h, 0, st);
        rc = h->gtype == ONEBIT_BF16 ? launch_worker<uint16_t>(h, grads, st)
                                     : launch_worker<float>(h, grads, st);
        if (rc != ONEBIT_OK) return rc;
        record(h, 1, st);
        rc = launch_scales_dp<false>(g.nch, g.C, g.d, h->part_w, (int64_t)g.W * g.nch, g.nseg,
                                     kSeg, h->s_out, h->s_lazy, dp.route_dev, st);
    } else if (phase == 1) {
        record(h, 2, st);
        const Geometry& gs = dp.gs;
        if (gs.d > 0) {
            uint32_t* planes = reinterpret_cast<uint32_t*>(dp.xch + dp.xl.planes);
            const float* rs = reinterpret_cast<const float*>(dp.xch + dp.xl.rscales);
            ServerArgs sa{gs, nullptr, planes, rs, h->es, h->S_lazy, h->bits_s + dp.e0 / 32,
                          h->part_s, h->status, dp.route_dev};
            const size_t ssm = server_smem_bytes(gs.W, server_stages(gs.W, gs.nseg_s), false);
            server_kernel_dp(gs.W)<<<(unsigned)server_blocks(gs), kThreads, ssm, st>>>(sa);
            ONEBIT_CUDA(cudaGetLastError());
        }
        record(h, 3, st);
        rc = launch_scales_dp<true>(gs.nch, gs.C, gs.d, h->part_s, gs.nch,
                                    server_blocks_per_chunk(gs), kSegS * gs.spb,
                                    nullptr, h->S_lazy, dp.route_dev, st);
    } else {
        record(h, 4, st);
        ApplyArgs pa{g, h->eps, lr, h->bits_s, h->S_out, h->v, x};
        k_apply<<<(unsigned)step_blocks(g), kThreads, 0, st>>>(pa);
        ONEBIT_CUDA(cudaGetLastError());
        record(h, 5, st);
    }
    if (rc != ONEBIT_OK) return rc;
    if (mode_out) rc = dp_barrier(h, mode_out, st);
    return rc;
}

// Checks shared by the step and phase entry points of a data-parallel rank.
int dp_ready(onebit_adam_s* h) {
    if (!h->dp.connected) return ONEBIT_ERR_PHASE;
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
    g.spb = server_segs_per_block(W, g.nseg_s, g.nch);
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
    h->sbits = reinterpret_cast<uint8_t*>(b + L.sbits);
    h->bits_s = reinterpret_cast<uint32_t*>(b + L.bits_s);
    h->s_out = reinterpret_cast<float*>(b + L.s_out);
    h->s_lazy = reinterpret_cast<float*>(b + L.s_lazy);
    h->S_out = reinterpret_cast<float*>(b + L.S_out);
    h->S_lazy = reinterpret_cast<float*>(b + L.S_lazy);
    h->part_w = reinterpret_cast<double*>(b + L.part_w);
    h->part_s = reinterpret_cast<double*>(b + L.part_s);
    h->status = reinterpret_cast<uint32_t*>(b + L.status);
    h->mw = h->zo.on ? reinterpret_cast<float*>(b + L.mw) : nullptr;
    h->uw = h->zo.on ? reinterpret_cast<float*>(b + L.uw) : nullptr;
    h->gtype = grad_dtype;
    cudaStream_t st = as_stream(stream);
    if (is_dp(h)) {
        DpState& dp = h->dp;
        if (dp.xch == nullptr) {
            // the exchange region is an allocation of its own so that CUDA IPC can map it
            void* p = nullptr;
            ONEBIT_CUDA(cudaMalloc(&p, dp.xl.total));
            dp.xch = static_cast<char*>(p);
        }
        char* x = dp.xch;
        h->m = reinterpret_cast<float*>(x + dp.xl.m);
        h->v = reinterpret_cast<float*>(x + dp.xl.v);
        h->bits_s = reinterpret_cast<uint32_t*>(x + dp.xl.bits_s);
        h->S_out = reinterpret_cast<float*>(x + dp.xl.S);
        h->sbits = nullptr;
        dp.route_dev = reinterpret_cast<DpRoute*>(b + L.route);
        dp.epoch_dev = reinterpret_cast<uint32_t*>(b + L.route + sizeof(DpRoute));
        dp.connected = false;
        dp.next_phase = 0;
        dp.phase_kind = 0;
        const int ssm = (int)server_smem_bytes(dp.Wg, server_stages(dp.Wg, dp.gs.nseg_s), false);
        ONEBIT_CUDA(cudaFuncSetAttribute(server_kernel_dp(dp.Wg),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, ssm));
        ONEBIT_CUDA(cudaMemsetAsync(dp.xch, 0, dp.xl.total, st));
    } else {
        const int ssm = (int)server_smem(h->geo);
        ONEBIT_CUDA(cudaFuncSetAttribute(server_kernel(h->geo),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, ssm));
    }
    // m and v start at zero (Adam); the rest is cleared too so padding is deterministic.
    ONEBIT_CUDA(cudaMemsetAsync(b, 0, L.total, st));
    h->phase = kWarmup;
    h->steps = 0;
    h->m_explicit = true;
    h->wsteps = 0;
    h->p1 = h->p2 = 1.0;
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
    if (is_dp(h)) {
        if (dp_ready(h) != ONEBIT_OK || h->dp.phase_kind != 0) return ONEBIT_ERR_PHASE;
        const int both = kBarrierSignal | kBarrierWait;
        int rc = dp_warmup_phase(h, 0, x, grads, lr, 0, both, st);
        if (rc == ONEBIT_OK) rc = dp_warmup_phase(h, 1, x, grads, lr, 0, both, st);
        if (rc == ONEBIT_OK) rc = dp_warmup_phase(h, 2, x, grads, lr, 0, 0, st);
        return rc;
    }
    const int rc = h->gtype == ONEBIT_BF16 ? launch_warmup<uint16_t>(h, x, grads, lr, st)
                                           : launch_warmup<float>(h, x, grads, lr, st);
    if (rc == ONEBIT_OK) {
        ++h->wsteps;
        h->p1 *= (double)h->beta1;
        h->p2 *= (double)h->beta2;
    }
    return rc;
}

int onebit_adam_set_bias_correction(onebit_adam_t h, int32_t on) {
    if (!valid_handle(h) || (on != 0 && on != 1)) return ONEBIT_ERR_ARG;
    if (is_dp(h)) return ONEBIT_ERR_ARG;
    if (h->phase == kCompressed || h->wsteps > 0) return ONEBIT_ERR_PHASE;
    h->bc = on != 0;
    return ONEBIT_OK;
}

int onebit_adam_freeze_variance(onebit_adam_t h, void* stream) {
    if (!valid_handle(h)) return ONEBIT_ERR_ARG;
    if (h->phase != kWarmup) return ONEBIT_ERR_PHASE;
    cudaStream_t st = as_stream(stream);
    const Layout& L = h->lay;
    if (is_dp(h) && h->dp.phase_kind != 0) return ONEBIT_ERR_PHASE;
    // after a bias-corrected warm-up the compression phase continues from the corrected moments
    if (h->bc && h->wsteps > 0 && h->geo.d > 0) {
        const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(h->geo.d, kThreads), 148 * 32);
        k_bc_freeze<<<blocks, kThreads, 0, st>>>(h->m, h->v, bias_correction(h->p1),
                                                 bias_correction(h->p2), h->geo.d);
        ONEBIT_CUDA(cudaGetLastError());
    }
    // residuals (lazy form: stored 0 with scale 0 rebuilds e = 0), planes, scales, partials
    ONEBIT_CUDA(cudaMemsetAsync(h->ws + L.es, 0, L.total - L.es, st));
    if (is_dp(h)) {
        // this rank's copy of the server plane and scales; not the receive planes and scales,
        // which the other ranks may already be filling for the first compressed step (every
        // word the server reads is written by its worker rank before the barrier)
        const XLayout& X = h->dp.xl;
        ONEBIT_CUDA(cudaMemsetAsync(h->dp.xch + X.bits_s, 0, X.total - X.bits_s, st));
    }
    h->phase = kCompressed;
    h->steps = 0;
    if (h->zo.on) {
        ZoState& z = h->zo;
        z.t = 0;
        z.syncs = 0;
        z.gamma = z.gamma_prev = 0.0f;
        z.src = kZoMShared;  // every worker starts from the warm-up momentum, u_w = 0
    }
    return ONEBIT_OK;
}

int onebit_adam_compressed_step(onebit_adam_t h, float* x, const void* grads, float lr,
                                void* stream) {
    if (!valid_handle(h) || !std::isfinite(lr)) return ONEBIT_ERR_ARG;
    if (h->phase != kCompressed || h->zo.on) return ONEBIT_ERR_PHASE;
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
    if (is_dp(h)) {
        if (dp_ready(h) != ONEBIT_OK || h->dp.phase_kind != 0) return ONEBIT_ERR_PHASE;
        const int both = kBarrierSignal | kBarrierWait;
        rc = dp_compressed_phase(h, 0, x, grads, lr, 0, both, st);
        if (rc == ONEBIT_OK) rc = dp_compressed_phase(h, 1, x, grads, lr, 0, both, st);
        if (rc == ONEBIT_OK) rc = dp_compressed_phase(h, 2, x, grads, lr, 0, 0, st);
        if (rc != ONEBIT_OK) return rc;
        if (h->tcount < h->tmax) ++h->tcount;
        ++h->steps;
        h->m_explicit = false;
        return ONEBIT_OK;
    }

    record(h, 0, st);
    rc = h->gtype == ONEBIT_BF16 ? launch_worker<uint16_t>(h, grads, st)
                                 : launch_worker<float>(h, grads, st);
    if (rc != ONEBIT_OK) return rc;
    record(h, 1, st);
    const bool fold_ws = fold_worker_scales(g), fold_ss = fold_server_scales(g);
    if (!fold_ws) {
        rc = launch_scales(g, h->part_w, (int64_t)g.W * g.nch, g.nseg, kSeg, h->s_out, h->s_lazy,
                           st);
        if (rc != ONEBIT_OK) return rc;
    }
    record(h, 2, st);
    ServerArgs sa{g, h->sbits, nullptr, h->s_out, h->es, h->S_lazy, h->bits_s, h->part_s,
                  h->status, nullptr, fold_ws ? h->part_w : nullptr, g.nseg <= 8 ? 1 : 32,
                  h->s_out, h->s_lazy};
    const size_t ssm = server_smem(g);
    const unsigned sblocks = (unsigned)server_blocks(g);
    server_kernel(g)<<<sblocks, kThreads, ssm, st>>>(sa);
    ONEBIT_CUDA(cudaGetLastError());
    record(h, 3, st);
    if (!fold_ss) {
        rc = launch_scales(g, h->part_s, g.nch, server_blocks_per_chunk(g),
                           kSegS * g.spb, h->S_out, h->S_lazy, st);
        if (rc != ONEBIT_OK) return rc;
    }
    record(h, 4, st);
    ApplyArgs pa{g, h->eps, lr, h->bits_s, h->S_out, h->v, x,
                 fold_ss ? h->part_s : nullptr, server_blocks_per_chunk(g), h->S_out, h->S_lazy};
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
    if (h->phase != kCompressed || h->zo.on) return ONEBIT_ERR_PHASE;
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
        case ONEBIT_STATE_V: *bytes = g.d * f; break;
        case ONEBIT_STATE_ES: *bytes = (is_dp(h) ? h->dp.gs.d : g.d) * f; break;
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
    if (h->zo.on && which == ONEBIT_STATE_M) return ONEBIT_ERR_ARG;  // per worker: onebit01_*
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
            // the signs of the stored x_w (the lazy residual holds x_w itself)
            return launch_pack_rows(h, 0, g.d, static_cast<uint32_t*>(dst), st);
        case ONEBIT_STATE_BITSS: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->bits_s, bytes, D2D, st)); break;
        case ONEBIT_STATE_EW:
        case ONEBIT_STATE_ES: {
            const bool wk = which == ONEBIT_STATE_EW;
            const int64_t n = wk || !is_dp(h) ? g.d : h->dp.gs.d;
            const int rc2 = launch_materialize(h, wk, 0, n, static_cast<float*>(dst), st);
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
    if (h->zo.on && which == ONEBIT_STATE_M) return ONEBIT_ERR_ARG;
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
            return launch_materialize(h, true, i0, n, static_cast<float*>(dst), st);
        case ONEBIT_STATE_ES:
            if (is_dp(h)) {
                // the server residual of a data-parallel rank covers its own chunks only
                const int64_t k0 = h->dp.kb[h->dp.rank], k1 = h->dp.kb[h->dp.rank + 1];
                if (k < k0 || k >= k1) return ONEBIT_ERR_ARG;
                return launch_materialize(h, false, (k - k0) * g.C, n, static_cast<float*>(dst),
                                          st);
            }
            return launch_materialize(h, false, i0, n, static_cast<float*>(dst), st);
        case ONEBIT_STATE_SW:
            ONEBIT_CUDA(cudaMemcpy2DAsync(dst, f, h->s_out + k, g.nch * f, f, g.W, D2D, st));
            break;
        case ONEBIT_STATE_SS: ONEBIT_CUDA(cudaMemcpyAsync(dst, h->S_out + k, f, D2D, st)); break;
        case ONEBIT_STATE_BITSW:
            return launch_pack_rows(h, i0, n, static_cast<uint32_t*>(dst), st);
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
    // a 0/1 handle's momenta are per worker (onebit01_set_worker_state)
    if (h->zo.on && which == ONEBIT_STATE_M) return ONEBIT_ERR_ARG;
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
            if (h->zo.on) {
                // explicit server residual; S_out and the server plane stay (the momentum
                // estimate of the last synchronisation is built from them)
                ONEBIT_CUDA(cudaMemcpyAsync(h->es, src, bytes, D2D, st));
                ONEBIT_CUDA(cudaMemsetAsync(h->S_lazy, 0,
                                            (is_dp(h) ? h->dp.gs.nch : g.nch) * f, st));
                break;
            }
            if (!h->m_explicit) {
                // m lives in S_out, which is about to be cleared: make it explicit first
                const int rc2 = launch_materialize_m(h, 0, g.d, h->m, st);
                if (rc2 != ONEBIT_OK) return rc2;
                h->m_explicit = true;
            }
            ONEBIT_CUDA(cudaMemcpyAsync(h->es, src, bytes, D2D, st));
            ONEBIT_CUDA(cudaMemsetAsync(h->S_lazy, 0, (is_dp(h) ? h->dp.gs.nch : g.nch) * f, st));
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
    out[7] = is_dp(h) ? kLaunchesPerStepDp : launches_per_step(h->geo);
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

int onebit_adam_timing_steps(onebit_adam_t h, double* step_ms, int32_t cap, int32_t* steps) {
    if (!valid_handle(h) || steps == nullptr || cap < 0 || (cap > 0 && step_ms == nullptr))
        return ONEBIT_ERR_ARG;
    *steps = h->tcount;
    if (h->tcount == 0 || cap == 0) return ONEBIT_OK;
    ONEBIT_CUDA(cudaEventSynchronize(h->ev[(size_t)h->tcount * kEventsPerStep - 1]));
    for (int32_t s = 0; s < h->tcount && s < cap; ++s) {
        float ms = 0.0f;
        ONEBIT_CUDA(cudaEventElapsedTime(&ms, h->ev[(size_t)s * kEventsPerStep],
                                         h->ev[(size_t)s * kEventsPerStep + kLaunchesPerStep]));
        step_ms[s] = ms;
    }
    return ONEBIT_OK;
}

void onebit_adam_destroy(onebit_adam_t h) {
    if (h == nullptr) return;
    free_events(h);
    for (int q = 0; q < kMaxRanks; ++q)
        if (h->dp.ipc[q]) cudaIpcCloseMemHandle(h->dp.peer[q]);
    if (h->dp.xch != nullptr) cudaFree(h->dp.xch);
    if (h->d2h != nullptr) {
        cudaStreamSynchronize(h->d2h);
        cudaStreamDestroy(h->d2h);
        cudaEventDestroy(h->step_done);
        cudaEventDestroy(h->d2h_done);
    }
    delete h;
}

// ------------------------------------------------------------------------------------------
// Data-parallel ranks

int onebit_server_layout(int64_t d, int32_t W, int64_t C, int64_t out[5]) {
    if (out == nullptr || d < 0 || W < 1 || W > kMaxWorkers || C <= 0) return ONEBIT_ERR_ARG;
    if (C % 32 != 0) return ONEBIT_ERR_ALIGN;
    if (d > ((int64_t)1 << 46)) return ONEBIT_ERR_ARG;
    Geometry g{};
    g.d = d;
    g.W = W;
    g.C = C;
    g.nch = ceil_div(d, C);
    g.nseg_s = ceil_div(C > d ? (d > 0 ? d : 1) : C, kSegS);
    g.spb = server_segs_per_block(W, g.nseg_s, g.nch);
    out[0] = server_bank_private(W, g.nseg_s, g.nch) ? 1 : 0;
    out[1] = g.spb;
    out[2] = (int64_t)server_smem(g);
    out[3] = (int64_t)server_smem_bytes(W, server_stages(W, g.nseg_s), false);
    out[4] = server_blocks(g);
    return ONEBIT_OK;
}

int onebit_dp_chunk_range(int64_t nch, int32_t R, int32_t q, int64_t* k0, int64_t* k1) {
    if (nch < 0 || R < 1 || R > kMaxRanks || q < 0 || q >= R || k0 == nullptr || k1 == nullptr)
        return ONEBIT_ERR_ARG;
    dp_range(nch, R, q, k0, k1);
    return ONEBIT_OK;
}

int onebit_dp_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1,
                   float beta2, float eps, int32_t R, int32_t rank) {
    if (out == nullptr) return ONEBIT_ERR_ARG;
    *out = nullptr;
    if (R < 1 || R > kMaxRanks || rank < 0 || rank >= R) return ONEBIT_ERR_ARG;
    if (W < 1 || W > kMaxWorkers || W % R != 0) return ONEBIT_ERR_ARG;
    const int rc = onebit_adam_init(out, d, W / R, C, beta1, beta2, eps);
    if (rc != ONEBIT_OK) return rc;
    onebit_adam_s* h = *out;
    const Geometry& g = h->geo;
    DpState& dp = h->dp;
    dp.R = R;
    dp.rank = rank;
    dp.Wg = W;
    for (int32_t q = 0; q < R; ++q) dp_range(g.nch, R, q, &dp.kb[q], &dp.kb[q + 1]);
    Geometry& gs = dp.gs;
    gs.d = dp_elems(*h, rank);
    gs.C = g.C;
    gs.nch = dp.kb[rank + 1] - dp.kb[rank];
    gs.nseg = g.nseg;      // the global segment counts: block partials and their reduction
    gs.nseg_s = g.nseg_s;  // order are those of the single-GPU step
    gs.spb = g.spb;
    gs.ld = round_up(std::max<int64_t>(gs.d, 1), 64);
    gs.ldw = dp_ldw(*h, rank);
    gs.W = W;
    dp.e0 = dp.kb[rank] * g.C;
    dp.xl = make_xlayout(*h);
    return ONEBIT_OK;
}

int onebit_dp_info(onebit_adam_t h, int64_t out[8]) {
    if (!valid_handle(h) || out == nullptr || !is_dp(h)) return ONEBIT_ERR_ARG;
    const DpState& dp = h->dp;
    out[0] = dp.R;
    out[1] = dp.rank;
    out[2] = dp.Wg;
    out[3] = dp.kb[dp.rank];
    out[4] = dp.kb[dp.rank + 1];
    out[5] = dp.e0;
    out[6] = dp.gs.d;
    out[7] = (int64_t)dp.xl.total;
    return ONEBIT_OK;
}

int onebit_dp_exchange(onebit_adam_t h, void** base, uint64_t* bytes) {
    if (!valid_handle(h) || base == nullptr || bytes == nullptr || !is_dp(h)) return ONEBIT_ERR_ARG;
    if (h->dp.xch == nullptr) return ONEBIT_ERR_PHASE;
    *base = h->dp.xch;
    *bytes = h->dp.xl.total;
    return ONEBIT_OK;
}

int onebit_dp_ipc_handle(onebit_adam_t h, void* out) {
    if (!valid_handle(h) || out == nullptr || !is_dp(h)) return ONEBIT_ERR_ARG;
    if (h->dp.xch == nullptr) return ONEBIT_ERR_PHASE;
    static_assert(sizeof(cudaIpcMemHandle_t) == ONEBIT_IPC_HANDLE_BYTES, "IPC handle size");
    cudaIpcMemHandle_t hd;
    ONEBIT_CUDA(cudaIpcGetMemHandle(&hd, h->dp.xch));
    std::memcpy(out, &hd, sizeof hd);
    return ONEBIT_OK;
}

int onebit_dp_open_peer(onebit_adam_t h, int32_t q, const void* handle) {
    if (!valid_handle(h) || handle == nullptr || !is_dp(h)) return ONEBIT_ERR_ARG;
    DpState& dp = h->dp;
    if (q < 0 || q >= dp.R || q == dp.rank) return ONEBIT_ERR_ARG;
    cudaIpcMemHandle_t hd;
    std::memcpy(&hd, handle, sizeof hd);
    void* p = nullptr;
    ONEBIT_CUDA(cudaIpcOpenMemHandle(&p, hd, cudaIpcMemLazyEnablePeerAccess));
    if (dp.ipc[q]) cudaIpcCloseMemHandle(dp.peer[q]);
    dp.peer[q] = static_cast<char*>(p);
    dp.ipc[q] = true;
    dp.connected = false;
    return ONEBIT_OK;
}

int onebit_dp_set_peer(onebit_adam_t h, int32_t q, void* base) {
    if (!valid_handle(h) || base == nullptr || !is_dp(h)) return ONEBIT_ERR_ARG;
    DpState& dp = h->dp;
    if (q < 0 || q >= dp.R || q == dp.rank) return ONEBIT_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(base) & 255u) != 0) return ONEBIT_ERR_ALIGN;
    if (dp.ipc[q]) cudaIpcCloseMemHandle(dp.peer[q]);
    dp.peer[q] = static_cast<char*>(base);
    dp.ipc[q] = false;
    dp.connected = false;
    return ONEBIT_OK;
}

int onebit_dp_connect(onebit_adam_t h, void* stream) {
    if (!valid_handle(h) || !is_dp(h)) return ONEBIT_ERR_ARG;
    DpState& dp = h->dp;
    if (h->phase == kUnbound || dp.xch == nullptr) return ONEBIT_ERR_PHASE;
    for (int32_t q = 0; q < dp.R; ++q)
        if (q != dp.rank && dp.peer[q] == nullptr) return ONEBIT_ERR_PHASE;
    DpRoute& r = dp.route;
    r = DpRoute{};
    r.R = dp.R;
    r.rank = dp.rank;
    r.w0 = dp.rank * h->geo.W;
    r.W = dp.Wg;
    const XLayout& X = dp.xl;
    for (int32_t q = 0; q <= dp.R; ++q) r.kb[q] = dp.kb[q];
    for (int32_t q = 0; q < dp.R; ++q) {
        char* b = q == dp.rank ? dp.xch : dp.peer[q];
        r.ldw[q] = dp_ldw(*h, q);
        r.planes[q] = reinterpret_cast<uint32_t*>(b + X.planes);
        r.scales[q] = reinterpret_cast<float*>(b + X.rscales);
        r.bits_s[q] = reinterpret_cast<uint32_t*>(b + X.bits_s);
        r.S[q] = reinterpret_cast<float*>(b + X.S);
        r.m[q] = reinterpret_cast<float*>(b + X.m);
        r.v[q] = reinterpret_cast<float*>(b + X.v);
        r.wpart[q] = reinterpret_cast<const double*>(b + X.wpart);
        r.flags[q] = reinterpret_cast<uint32_t*>(b + X.flags);
    }
    ONEBIT_CUDA(cudaMemcpyAsync(dp.route_dev, &r, sizeof r, cudaMemcpyHostToDevice,
                                as_stream(stream)));
    dp.connected = true;
    return ONEBIT_OK;
}

int onebit_dp_set_timeout(onebit_adam_t h, uint64_t timeout_us) {
    if (!valid_handle(h) || !is_dp(h)) return ONEBIT_ERR_ARG;
    if (timeout_us < 1 || timeout_us > 3600ull * 1000000ull) return ONEBIT_ERR_ARG;
    h->dp.timeout_ns = timeout_us * 1000ull;
    return ONEBIT_OK;
}

}  // extern "C"

namespace {

// Argument and order checks of one phase; kind 1 warm-up, 2 compressed.
int dp_phase_check(onebit_adam_t h, int kind, int32_t phase, const float* x, const void* grads,
                   float lr) {
    if (!valid_handle(h) || !is_dp(h) || !std::isfinite(lr)) return ONEBIT_ERR_ARG;
    if (phase < 0 || phase > 2) return ONEBIT_ERR_ARG;
    if (h->phase != (kind == 1 ? kWarmup : kCompressed)) return ONEBIT_ERR_PHASE;
    const DpState& dp = h->dp;
    if (!dp.connected || phase != dp.next_phase) return ONEBIT_ERR_PHASE;
    if (phase > 0 && dp.phase_kind != kind) return ONEBIT_ERR_PHASE;
    if (h->geo.d == 0) return ONEBIT_OK;
    if (phase == 0) {
        if (grads == nullptr) return ONEBIT_ERR_ARG;
        if (!aligned16(grads)) return ONEBIT_ERR_ALIGN;
    }
    if (phase == 2) {
        if (x == nullptr) return ONEBIT_ERR_ARG;
        if (!aligned16(x)) return ONEBIT_ERR_ALIGN;
    }
    return ONEBIT_OK;
}

void dp_phase_done(onebit_adam_t h, int kind, int32_t phase) {
    DpState& dp = h->dp;
    dp.next_phase = (phase + 1) % 3;
    dp.phase_kind = phase == 2 ? 0 : kind;
}

}  // namespace

extern "C" {

int onebit_dp_warmup_phase(onebit_adam_t h, int32_t phase, float* x, const void* grads,
                           float lr, void* stream) {
    int rc = dp_phase_check(h, 1, phase, x, grads, lr);
    if (rc != ONEBIT_OK) return rc;
    if (h->geo.d > 0) {
        rc = dp_warmup_phase(h, phase, x, grads, lr, phase > 0 ? kBarrierWait : 0,
                             phase < 2 ? kBarrierSignal : 0, as_stream(stream));
        if (rc != ONEBIT_OK) return rc;
    }
    dp_phase_done(h, 1, phase);
    return ONEBIT_OK;
}

int onebit_dp_compressed_phase(onebit_adam_t h, int32_t phase, float* x, const void* grads,
                               float lr, void* stream) {
    int rc = dp_phase_check(h, 2, phase, x, grads, lr);
    if (rc != ONEBIT_OK) return rc;
    if (h->zo.on) return ONEBIT_ERR_PHASE;  // a 0/1 rank steps with onebit01_dp_phase
    if (h->geo.d > 0) {
        rc = dp_compressed_phase(h, phase, x, grads, lr, phase > 0 ? kBarrierWait : 0,
                                 phase < 2 ? kBarrierSignal : 0, as_stream(stream));
        if (rc != ONEBIT_OK) return rc;
    }
    dp_phase_done(h, 2, phase);
    if (phase == 2) {
        if (h->tcount < h->tmax) ++h->tcount;
        ++h->steps;
        if (h->geo.d > 0) h->m_explicit = false;
    }
    return ONEBIT_OK;
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
// The 0/1 Adam variant (codewithpapers.app "0/1 Adam" page, abstract): local steps on each
// worker's own momentum and accumulated update, and every H-th step a synchronisation through
// the compressed allreduce of the accumulated updates.

namespace {

template <typename GT, bool SYNC, bool DP = false>
void launch_zo_worker_t(onebit_adam_s* h, const ZoArgs& a, unsigned blocks, size_t smem,
                        cudaStream_t st) {
    const int64_t d = h->geo.d;
    if constexpr (sizeof(GT) == 2) {
        if (d % 8 == 0) {
            k01_worker<GT, true, 8, SYNC, DP><<<blocks, kThreads, smem, st>>>(a);
            return;
        }
    }
    if (d % kVec == 0)
        k01_worker<GT, true, 4, SYNC, DP><<<blocks, kThreads, smem, st>>>(a);
    else
        k01_worker<GT, false, 4, SYNC, DP><<<blocks, kThreads, smem, st>>>(a);
}

ZoArgs zo_args(onebit_adam_s* h, const void* grads, float lr) {
    ZoArgs a{};
    a.geo = h->geo;
    a.beta1 = h->beta1;
    a.omb1 = 1.0f - h->beta1;
    a.lr = lr;
    a.src = h->zo.src;
    a.m = h->m;
    a.bits_s = h->bits_s;
    a.S = h->S_out;
    a.gamma_prev = h->zo.gamma_prev;
    a.lr_first = h->zo.lr_first;
    a.mw = h->mw;
    a.uw = h->uw;
    a.g = grads;
    a.ew = h->ew;
    a.s_lazy = h->s_lazy;
    a.sbits = h->sbits;
    a.part_w = h->part_w;
    a.status = h->status;
    a.route = is_dp(h) ? h->dp.route_dev : nullptr;
    return a;
}

int launch_zo_worker(onebit_adam_s* h, const void* grads, float lr, bool sync, cudaStream_t st) {
    const ZoArgs a = zo_args(h, grads, lr);
    const unsigned blocks = (unsigned)step_blocks(h->geo);
    const size_t smem = sync ? (size_t)h->geo.W * kWarps * sizeof(double) : 0;
    const bool dp = sync && is_dp(h);
    if (h->gtype == ONEBIT_BF16) {
        if (dp) launch_zo_worker_t<uint16_t, true, true>(h, a, blocks, smem, st);
        else if (sync) launch_zo_worker_t<uint16_t, true>(h, a, blocks, smem, st);
        else launch_zo_worker_t<uint16_t, false>(h, a, blocks, smem, st);
    } else {
        if (dp) launch_zo_worker_t<float, true, true>(h, a, blocks, smem, st);
        else if (sync) launch_zo_worker_t<float, true>(h, a, blocks, smem, st);
        else launch_zo_worker_t<float, false>(h, a, blocks, smem, st);
    }
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

// The kind of the coming 0/1 step: whether it synchronises, refreshes v, and its Gamma.
struct ZoStep {
    bool sync, refresh, gamma_ok;
    float gamma;
};
ZoStep zo_step_kind(const onebit_adam_s* h, float lr) {
    const ZoState& z = h->zo;
    ZoStep zs;
    zs.sync = z.t + 1 == z.H;
    zs.refresh = zs.sync && z.K > 0 && (z.syncs + 1) % z.K == 0;
    zs.gamma = z.gamma + lr;  // fp32, in step order
    zs.gamma_ok = zs.gamma != 0.0f && std::isfinite(zs.gamma);
    return zs;
}

// One phase of a 0/1 step. Phase 0: every worker's step (and, when it synchronises, the
// compression of u_w + e_w and the worker scales); phase 1: the server stage; phase 2: the
// synchronised step. A local step launches phase 0's kernel only. mode_in / mode_out: barrier
// modes of a data-parallel rank before and after the phase.
int zo_phase(onebit_adam_s* h, int phase, float* x, const void* grads, float lr,
             const ZoStep& zs, int mode_in, int mode_out, cudaStream_t st) {
    const Geometry& g = h->geo;
    const bool dp = is_dp(h);
    int rc = ONEBIT_OK;
    if (phase == 1 && zs.sync && dp)   // the server stage of a data-parallel rank, as 1-bit Adam's
        return dp_compressed_phase(h, 1, x, grads, lr, mode_in, mode_out, st);
    if (mode_in) rc = dp_barrier(h, mode_in, st);
    if (rc != ONEBIT_OK) return rc;
    if (phase == 0) {
        record(h, 0, st);
        rc = launch_zo_worker(h, grads, lr, zs.sync, st);
        if (rc != ONEBIT_OK) return rc;
        record(h, 1, st);
        if (zs.sync) {
            rc = dp ? launch_scales_dp<false>(g.nch, g.C, g.d, h->part_w, (int64_t)g.W * g.nch,
                                              g.nseg, kSeg, h->s_out, h->s_lazy,
                                              h->dp.route_dev, st)
                    : launch_scales(g, h->part_w, (int64_t)g.W * g.nch, g.nseg, kSeg, h->s_out,
                                    h->s_lazy, st);
            if (rc != ONEBIT_OK) return rc;
        }
    } else if (phase == 1) {
        record(h, 2, st);
        if (zs.sync) {
            ServerArgs sa{g, h->sbits, nullptr, h->s_out, h->es, h->S_lazy, h->bits_s,
                          h->part_s, h->status};
            const size_t ssm = server_smem(g);
            server_kernel(g)<<<(unsigned)server_blocks(g), kThreads, ssm, st>>>(sa);
            ONEBIT_CUDA(cudaGetLastError());
        }
        record(h, 3, st);
        if (zs.sync) {
            rc = launch_scales(g, h->part_s, g.nch, server_blocks_per_chunk(g),
                               kSegS * g.spb, h->S_out, h->S_lazy, st);
            if (rc != ONEBIT_OK) return rc;
        }
    } else {
        record(h, 4, st);
        if (zs.sync) {
            ZoApplyArgs pa{g, h->eps, zs.gamma, h->beta2, 1.0f - h->beta2, zs.refresh ? 1 : 0,
                           h->bits_s, h->S_out, h->v, x};
            k01_apply<<<(unsigned)step_blocks(g), kThreads, 0, st>>>(pa);
            ONEBIT_CUDA(cudaGetLastError());
        }
        record(h, 5, st);
    }
    if (mode_out) rc = dp_barrier(h, mode_out, st);
    return rc;
}

// The schedule after a step of learning rate lr.
void zo_advance(onebit_adam_s* h, float lr, bool sync) {
    ZoState& z = h->zo;
    const float gamma = z.gamma + lr;
    if (sync) {
        z.gamma_prev = gamma;
        z.gamma = 0.0f;
        z.t = 0;
        ++z.syncs;
        z.src = kZoMBar;
    } else {
        z.gamma = gamma;
        ++z.t;
        // the interval's first step stored m_w only; the next one rebuilds its u_w
        if (z.src == kZoMShared || z.src == kZoMBar) {
            z.src = kZoMWorkerU1;
            z.lr_first = lr;
        } else {
            z.src = kZoMWorker;
        }
    }
}

}  // namespace

extern "C" {

int onebit01_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1, float beta2,
                  float eps, int32_t H, int32_t K) {
    if (out == nullptr) return ONEBIT_ERR_ARG;
    *out = nullptr;
    if (H < 1 || H > (1 << 20) || K < 0 || K > (1 << 20)) return ONEBIT_ERR_ARG;
    const int rc = onebit_adam_init(out, d, W, C, beta1, beta2, eps);
    if (rc != ONEBIT_OK) return rc;
    (*out)->zo.on = true;
    (*out)->zo.H = H;
    (*out)->zo.K = K;
    return ONEBIT_OK;
}

int onebit01_step(onebit_adam_t h, float* x, const void* grads, float lr, void* stream) {
    if (!valid_handle(h) || !std::isfinite(lr)) return ONEBIT_ERR_ARG;
    if (!h->zo.on || h->phase != kCompressed) return ONEBIT_ERR_PHASE;
    const ZoStep zs = zo_step_kind(h, lr);
    if (h->geo.d > 0) {
        if (x == nullptr || grads == nullptr) return ONEBIT_ERR_ARG;
        if (!aligned16(x) || !aligned16(grads)) return ONEBIT_ERR_ALIGN;
        if (zs.sync && !zs.gamma_ok) return ONEBIT_ERR_ARG;
        if (is_dp(h) && (dp_ready(h) != ONEBIT_OK || h->dp.phase_kind != 0))
            return ONEBIT_ERR_PHASE;
        cudaStream_t st = as_stream(stream);
        struct Range {
            Range() { nvtxRangePushA("onebit01_step"); }
            ~Range() { nvtxRangePop(); }
        } range;
        // a data-parallel rank's synchronising step: each half of the exchange ends with this
        // rank's barrier signal and the wait for every other rank's
        const int both = zs.sync && is_dp(h) ? (kBarrierSignal | kBarrierWait) : 0;
        for (int p = 0; p < 3; ++p) {
            const int rc = zo_phase(h, p, x, grads, lr, zs, 0, p < 2 ? both : 0, st);
            if (rc != ONEBIT_OK) return rc;
        }
        if (h->tcount < h->tmax) ++h->tcount;
    }
    ++h->steps;
    zo_advance(h, lr, zs.sync);
    return ONEBIT_OK;
}

int onebit01_set_worker_state(onebit_adam_t h, int32_t which, const void* src, void* stream) {
    if (!valid_handle(h) || !h->zo.on) return ONEBIT_ERR_ARG;
    if (which != 0 && which != 1) return ONEBIT_ERR_ARG;
    if (h->phase != kCompressed) return ONEBIT_ERR_PHASE;
    const Geometry& g = h->geo;
    if (g.d > 0) {
        if (src == nullptr) return ONEBIT_ERR_ARG;
        const uint64_t f = sizeof(float);
        float* dst = which == 0 ? h->mw : h->uw;
        ONEBIT_CUDA(cudaMemcpy2DAsync(dst, g.ld * f, src, g.d * f, g.d * f, g.W,
                                      cudaMemcpyDeviceToDevice, as_stream(stream)));
    }
    // the next step starts from each worker's own (now explicit) momentum and update
    h->zo.src = kZoMWorker;
    return ONEBIT_OK;
}

int onebit01_get_schedule(onebit_adam_t h, int64_t ints[2], float floats[2]) {
    if (!valid_handle(h) || !h->zo.on || ints == nullptr || floats == nullptr)
        return ONEBIT_ERR_ARG;
    ints[0] = h->zo.t;
    ints[1] = h->zo.syncs;
    floats[0] = h->zo.gamma;
    floats[1] = h->zo.gamma_prev;
    return ONEBIT_OK;
}

int onebit01_set_schedule(onebit_adam_t h, const int64_t ints[2], const float floats[2]) {
    if (!valid_handle(h) || !h->zo.on || ints == nullptr || floats == nullptr)
        return ONEBIT_ERR_ARG;
    if (h->phase != kCompressed) return ONEBIT_ERR_PHASE;
    if (ints[0] < 0 || ints[0] >= h->zo.H || ints[1] < 0 || !std::isfinite(floats[0]) ||
        !std::isfinite(floats[1]))
        return ONEBIT_ERR_ARG;
    if (is_dp(h) && h->dp.phase_kind != 0) return ONEBIT_ERR_PHASE;
    h->zo.t = (int32_t)ints[0];
    h->zo.syncs = ints[1];
    h->zo.gamma = floats[0];
    h->zo.gamma_prev = floats[1];
    return ONEBIT_OK;
}

int onebit01_dp_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1,
                     float beta2, float eps, int32_t H, int32_t K, int32_t R, int32_t rank) {
    if (out == nullptr) return ONEBIT_ERR_ARG;
    *out = nullptr;
    if (H < 1 || H > (1 << 20) || K < 0 || K > (1 << 20)) return ONEBIT_ERR_ARG;
    const int rc = onebit_dp_init(out, d, W, C, beta1, beta2, eps, R, rank);
    if (rc != ONEBIT_OK) return rc;
    (*out)->zo.on = true;
    (*out)->zo.H = H;
    (*out)->zo.K = K;
    return ONEBIT_OK;
}

int onebit01_dp_phase(onebit_adam_t h, int32_t phase, float* x, const void* grads, float lr,
                      void* stream) {
    int rc = dp_phase_check(h, 3, phase, x, grads, lr);
    if (rc != ONEBIT_OK) return rc;
    if (!h->zo.on) return ONEBIT_ERR_PHASE;
    const ZoStep zs = zo_step_kind(h, lr);
    if (h->geo.d > 0) {
        if (phase == 0 && zs.sync && !zs.gamma_ok) return ONEBIT_ERR_ARG;
        // barriers only around the exchange of a synchronising step (every rank runs the same
        // schedule, so every rank takes the same ones)
        const int in = zs.sync && phase > 0 ? kBarrierWait : 0;
        const int out_mode = zs.sync && phase < 2 ? kBarrierSignal : 0;
        rc = zo_phase(h, phase, x, grads, lr, zs, in, out_mode, as_stream(stream));
        if (rc != ONEBIT_OK) return rc;
    }
    dp_phase_done(h, 3, phase);
    if (phase == 2) {
        if (h->geo.d > 0 && h->tcount < h->tmax) ++h->tcount;
        ++h->steps;
        zo_advance(h, lr, zs.sync);
    }
    return ONEBIT_OK;
}

int onebit01_info(onebit_adam_t h, int64_t out[6]) {
    if (!valid_handle(h) || out == nullptr || !h->zo.on) return ONEBIT_ERR_ARG;
    const ZoState& z = h->zo;
    out[0] = z.H;
    out[1] = z.K;
    out[2] = z.t;
    out[3] = z.syncs;
    out[4] = z.src;
    out[5] = z.t + 1 == z.H ? kLaunchesPerStep : 1;
    return ONEBIT_OK;
}

int onebit01_get_worker_state(onebit_adam_t h, int32_t which, int64_t k, void* dst,
                              void* stream) {
    if (!valid_handle(h) || !h->zo.on || dst == nullptr) return ONEBIT_ERR_ARG;
    if (which != 0 && which != 1) return ONEBIT_ERR_ARG;
    if (h->phase != kCompressed) return ONEBIT_ERR_PHASE;
    const Geometry& g = h->geo;
    if (k < -1 || k >= g.nch) return ONEBIT_ERR_ARG;
    const int64_t i0 = k < 0 ? 0 : k * g.C, n = k < 0 ? g.d : std::min(g.C, g.d - i0);
    const int64_t total = (int64_t)g.W * n;
    if (total == 0) return ONEBIT_OK;
    const ZoArgs a = zo_args(h, nullptr, 0.0f);
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(total, kThreads), 148 * 32);
    float* out = static_cast<float*>(dst);
    k01_export<<<blocks, kThreads, 0, as_stream(stream)>>>(a, i0, n, which == 0 ? out : nullptr,
                                                           which == 1 ? out : nullptr);
    ONEBIT_CUDA(cudaGetLastError());
    return ONEBIT_OK;
}

int onebit01_local_model(onebit_adam_t h, int32_t w, const float* x, float* out, void* stream) {
    if (!valid_handle(h) || !h->zo.on || x == nullptr || out == nullptr) return ONEBIT_ERR_ARG;
    const Geometry& g = h->geo;
    if (w < 0 || w >= g.W) return ONEBIT_ERR_ARG;
    if (h->phase != kCompressed) return ONEBIT_ERR_PHASE;
    if (g.d == 0) return ONEBIT_OK;
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(g.d, kThreads), 148 * 32);
    k01_local_model<<<blocks, kThreads, 0, as_stream(stream)>>>(
        x, h->mw + (int64_t)w * g.ld, h->uw + (int64_t)w * g.ld, h->zo.src, h->zo.lr_first,
        h->v, h->eps, g.d, out);
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
    g.spb = 8;
    // every slot read by the reduction was written by k_compress_partials in this same call,
    // so nothing in the shared array has to be cleared first
    return launch_scales(g, part, nch, nseg, kSeg, scales, scales, st);
}
