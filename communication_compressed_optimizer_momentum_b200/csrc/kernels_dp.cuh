// kernels_dp.cuh -- kernels that only data-parallel ranks use: the cross-rank barrier and the
// three warm-up kernels. The compressed step's kernels take their data-parallel form from
// kernels.cuh (k_worker<..., DP>, k_server<..., BCAST>, k_scales_dp).
//
// Cross-rank ordering. A thread that stored into another rank's memory ends with a
// system-scope fence, so those stores are complete everywhere before its kernel finishes;
// stores into the rank's own memory (read by peers later) are ordered by the kernel boundary.
// The barrier kernel that follows on the stream then publishes the rank's epoch into every
// rank's flag array with a system-scope release store, and waits (acquire loads, bounded) until
// every rank's flag in its own array has reached the epoch. Kernels after the barrier
// therefore see everything that every rank stored before its signal. Each wait has a deadline:
// when it passes, the barrier sets the kWaitTimeout status bit and returns, so a missing rank
// shows up as a status flag on the host instead of a hung GPU.
#pragma once

#include "kernels.cuh"

namespace onebit {

constexpr int kBarrierSignal = 1;
constexpr int kBarrierWait = 2;
constexpr int kBarrierPolls = 1 << 28;  // hard cap on the polls of one wait

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// One warp. The rank's barrier count lives in device memory (*epoch_p), so that a captured and
// replayed step synchronizes like an eager one. Signal: the count goes up by one and thread
// q < R stores it into rank q's flag of this rank. Wait: thread q < R polls this rank's flag of
// rank q until it reaches the count (wrap-safe compare), for at most timeout_ns and
// kBarrierPolls polls.
__global__ void k_dp_barrier(const DpRoute* rt, uint32_t* epoch_p, int mode, uint64_t timeout_ns,
                             uint32_t* status) {
    const int t = threadIdx.x;
    const int R = rt->R, me = rt->rank;
    uint32_t epoch = *epoch_p;
    if (mode & kBarrierSignal) {
        ++epoch;
        __syncwarp();
        if (t == 0) *epoch_p = epoch;
        if (t < R) {
            __threadfence_system();
            st_release_sys(rt->flags[t] + me, epoch);
        }
    }
    if (mode & kBarrierWait) {
        bool ok = true;
        if (t < R) {
            const uint32_t* f = rt->flags[me] + t;
            const uint64_t t0 = globaltimer_ns();
            ok = false;
            for (int i = 0; i < kBarrierPolls; ++i) {
                if ((int32_t)(ld_acquire_sys(f) - epoch) >= 0) {
                    ok = true;
                    break;
                }
                if (globaltimer_ns() - t0 > timeout_ns) break;
                __nanosleep(256);
            }
        }
        if (!ok) atomicOr(status, kWaitTimeout);
        __syncwarp();
    }
}

// ------------------------------------------------------------------------------------------
// Data-parallel warm-up (full-precision Adam on the average over all W workers). Three kernels
// with a barrier after the first two:
//   k_warmup_partial  every rank: fp64 sum of its own workers' gradients, in worker order;
//   k_warmup_reduce   rank q, its chunks: the R partial sums in rank order, the fp32 average,
//                     the Adam moments, stored into every rank's m and v;
//   k_warmup_apply    every rank, all elements: x -= lr * (m / (sqrt(v) + eps)).
// With one rank this is the single-GPU warm-up exactly; with several, the fp64 sum is grouped
// by rank, which equals the in-order sum whenever the fp64 partial sums are exact.

template <typename GT, bool VEC, int EPT>
__global__ void __launch_bounds__(kThreads, 4) k_warmup_partial(const Geometry geo,
                                                                const void* g, double* wpart) {
    constexpr int ITEMS = kSeg / (kThreads * EPT);
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(geo, geo.nseg, k, j, base, len)) return;
    const int tid = threadIdx.x;
    const GT* g0 = static_cast<const GT*>(g) + base;
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int64_t off = (int64_t)(it * kThreads + tid) * EPT;
        const int64_t r = len - off;
        const int nv = r <= 0 ? 0 : (r >= EPT ? EPT : (int)r);
        if (nv == 0) continue;
        double acc[EPT];
        worker_grad_sum<GT, VEC, EPT>(g0, geo.d, geo.W, off, nv, acc);
        double* dst = wpart + base + off;
#pragma unroll
        for (int h = 0; h < EPT / 2; ++h)
            *reinterpret_cast<double2*>(dst + 2 * h) = make_double2(acc[2 * h], acc[2 * h + 1]);
    }
}

struct WarmupDpArgs {
    Geometry gs;     // this rank's chunks (elements e0 .. e0 + gs.d)
    int64_t e0;
    float beta1, omb1, beta2, omb2;
    const DpRoute* rt;
};

__global__ void __launch_bounds__(kThreads) k_warmup_reduce(const WarmupDpArgs a) {
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(a.gs, a.gs.nseg, k, j, base, len)) return;
    const DpRoute* rt = a.rt;
    const int tid = threadIdx.x, R = rt->R, me = rt->rank;
    const double dW = (double)rt->W;
    const int64_t gbase = a.e0 + base;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int64_t off = (int64_t)(it * kThreads + tid) * kVec;
        const int nv = valid_of(len, off);
        if (nv == 0) continue;
        const int64_t i = gbase + off;
        double acc[4];
        {
            const double2 p0 = *reinterpret_cast<const double2*>(rt->wpart[0] + i);
            const double2 p1 = *reinterpret_cast<const double2*>(rt->wpart[0] + i + 2);
            acc[0] = p0.x; acc[1] = p0.y; acc[2] = p1.x; acc[3] = p1.y;
        }
        for (int p = 1; p < R; ++p) {
            const double2 p0 = *reinterpret_cast<const double2*>(rt->wpart[p] + i);
            const double2 p1 = *reinterpret_cast<const double2*>(rt->wpart[p] + i + 2);
            acc[0] = __dadd_rn(acc[0], p0.x);
            acc[1] = __dadd_rn(acc[1], p0.y);
            acc[2] = __dadd_rn(acc[2], p1.x);
            acc[3] = __dadd_rn(acc[3], p1.y);
        }
        float m[4], v[4];
        ld4(rt->m[me] + i, m);
        ld4(rt->v[me] + i, v);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float gbar = __double2float_rn(__ddiv_rn(acc[c], dW));
            m[c] = __fadd_rn(__fmul_rn(a.beta1, m[c]), __fmul_rn(a.omb1, gbar));
            v[c] = __fadd_rn(__fmul_rn(a.beta2, v[c]), __fmul_rn(a.omb2, __fmul_rn(gbar, gbar)));
        }
        for (int p = 0; p < R; ++p) {
            st4(rt->m[p] + i, m);
            st4(rt->v[p] + i, v);
        }
    }
    if (R > 1) __threadfence_system();  // peer stores before the barrier signal
}

struct WarmupApplyArgs {
    Geometry geo;
    float eps, lr;
    const float* m;  // [ld]
    const float* v;  // [ld]
    float* x;        // [d] caller-owned
};

__global__ void __launch_bounds__(kThreads) k_warmup_apply(const WarmupApplyArgs a) {
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(a.geo, a.geo.nseg, k, j, base, len)) return;
    const int tid = threadIdx.x;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int64_t off = (int64_t)(it * kThreads + tid) * kVec;
        const int nv = valid_of(len, off);
        if (nv == 0) continue;
        float m[4], v[4], x[4];
        ld4(a.m + base + off, m);
        ld4(a.v + base + off, v);
        ld4_caller(a.x + base + off, nv, x);
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            const float den = __fadd_rn(__fsqrt_rn(v[c]), a.eps);
            x[c] = __fsub_rn(x[c], __fmul_rn(a.lr, __fdiv_rn(m[c], den)));
        }
        st4_caller(a.x + base + off, nv, x);
    }
}

}  // namespace onebit
