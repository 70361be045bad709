// kernels_zero_one.cuh -- the 0/1 Adam variant's own kernels (codewithpapers.app "0/1 Adam"
// page, abstract: each Adam step linearised through stale state estimates and their linear
// correlation, so that 1-bit compression and local steps work together). The compressed
// allreduce's server stage and the chunk-scale reductions are 1-bit Adam's (kernels.cuh).
//
// State per worker w: its momentum m_w and its accumulated update u_w = sum of lr_t * m_w over
// the steps since the last synchronisation ([W][ld] each), next to the lazy residual of
// kernels.cuh. Every H-th step ends with a synchronisation, which compresses u_w + e_w with
// error feedback, runs the server stage and takes the synchronised step
// x -= ubar / (sqrt(v) + eps); the momentum estimate mbar = ubar / Gamma (Gamma = the sum of
// the interval's learning rates) becomes every worker's momentum, and u_w restarts at zero.
// Neither is written: the next step rebuilds mbar = +-fl(S_k / Gamma) from the server plane
// and takes u_w = 0 (kZoMBar), as the first step after the freeze takes the warm-up momentum
// (kZoMShared). That first step of an interval stores m_w only: its u_w = fl(0 + fl(lr * m_w))
// is rebuilt from the stored m_w by the next step and by the exports, with the same two
// roundings (kZoMWorkerU1). The steps after it read and write both buffers (kZoMWorker).
#pragma once

#include "kernels.cuh"

namespace onebit {

// where the momentum a step starts from comes from (and whether u_w starts at zero)
enum ZoSource : int {
    kZoMShared = 0,  // the shared fp32 momentum (the warm-up m, first step after the freeze);
                     // u_w = 0
    kZoMBar = 1,     // mbar = +-fl(S_k / Gamma) by the last synchronisation's server plane; u_w = 0
    kZoMWorker = 2,  // each worker's own m_w and u_w (steps after a local step)
    kZoMWorkerU1 = 3,  // each worker's own m_w; u_w = fl(0 + fl(lr_first * m_w)), not stored
                       // (the step after the interval's first step)
};

struct ZoArgs {
    Geometry geo;
    float beta1, omb1, lr;
    int src;                 // ZoSource
    const float* m;          // [ld] shared momentum (kZoMShared)
    const uint32_t* bits_s;  // [ldw] last synchronisation's server plane (kZoMBar)
    const float* S;          // [nch] its server scales (kZoMBar)
    float gamma_prev;        // its Gamma (kZoMBar)
    float lr_first;          // the learning rate of the interval's first step (kZoMWorkerU1)
    float* mw;               // [W][ld] per-worker momentum
    float* uw;               // [W][ld] per-worker accumulated update
    const void* g;           // [W][d] caller-owned, GT
    float* ew;               // [W][ld] lazy residual: holds the last synchronisation's x_w
    const float* s_lazy;     // [W][nch] scale that rebuilds the residual
    uint8_t* sbits;          // [ceil(W/8)][ld] sign bits grouped by 8 workers (single GPU)
    double* part_w;          // [W][nch][nseg]
    uint32_t* status;
    const DpRoute* route;    // data-parallel ranks: where each chunk's plane words go
};

// One step of every worker for one segment (a block owns a kSeg segment and loops over the W
// workers, like k_worker). Local step: m_w = b1 m + (1-b1) g_w; u_w += lr m_w, stored (u_w only
// when it did not start at zero: the first step's is rebuilt, kZoMWorkerU1). SYNC
// (the step that ends with a synchronisation): the same m_w and u_w, then x_w = u_w + e_w
// compressed as in k_worker (sign bits grouped by 8 workers, lazy residual, fp64 partials of the
// chunk norm); m_w and u_w are not stored, since the synchronisation replaces them.
// DP (synchronising step of a data-parallel rank): the rows are this rank's W / R workers, and
// the plane words of chunk k go to row (w0 + w) of the receive planes of the rank that serves
// chunk k, as in k_worker's data-parallel form.
// No blocks-per-SM bound: with the three per-worker streams of a step (and the residual of the
// synchronising one) the bound of k_worker made the compiler spill, which cost up to 16% of a
// step (measured); at the registers it picks (32-60) the kernel runs without spills.
template <typename GT, bool VEC, int EPT, bool SYNC, bool DP = false>
__global__ void __launch_bounds__(kThreads) k01_worker(const ZoArgs a) {
    static_assert(SYNC || !DP, "only the synchronising step exchanges");
    constexpr int ITEMS = kSeg / (kThreads * EPT);
    constexpr int LPW = 32 / EPT;  // lanes that share one 32-element word of the server plane
    extern __shared__ double red_w[];  // [W][kWarps] (SYNC)
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(a.geo, a.geo.nseg, k, j, base, len)) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = a.geo.W;
    const int sub = lane & (LPW - 1);
    const int src = a.src;

    // the shared momentum of the block's elements (kZoMShared, kZoMBar), kept in registers
    float ms[ITEMS][EPT];
    int nv[ITEMS];
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * EPT;
        const int64_t r = len - off;
        nv[it] = r <= 0 ? 0 : (r >= EPT ? EPT : (int)r);
#pragma unroll
        for (int c = 0; c < EPT; ++c) ms[it][c] = 0.0f;
        if (nv[it] > 0 && src == kZoMBar) {
            const float mb = __fdiv_rn(a.S[k], a.gamma_prev);
            const uint32_t bits = a.bits_s[(base >> 5) + q / LPW] >> (EPT * sub);
#pragma unroll
            for (int c = 0; c < EPT; ++c) ms[it][c] = ((bits >> c) & 1u) ? mb : -mb;
        } else if (nv[it] > 0 && src == kZoMShared) {
#pragma unroll
            for (int h = 0; h < EPT / 4; ++h) {
                float t4[4];
                ld4(a.m + base + off + 4 * h, t4);
#pragma unroll
                for (int c = 0; c < 4; ++c) ms[it][4 * h + c] = t4[c];
            }
        }
    }
    const float b1 = a.beta1, omb1 = a.omb1, lr = a.lr;
    const GT* g0 = static_cast<const GT*>(a.g) + base;
    // DP: this block's destination row start and row length, and whether the destination is
    // another rank's memory
    __shared__ uint32_t* dp_bw0[1];
    __shared__ int64_t dp_bld[1];
    __shared__ int dp_remote[1];
    if constexpr (DP) {
        if (tid == 0) {
            const DpRoute* rt = a.route;
            const int q = dp_owner(rt, k);
            dp_bld[0] = rt->ldw[q];
            dp_bw0[0] = rt->planes[q] + (int64_t)rt->w0 * rt->ldw[q] +
                        ((base - rt->kb[q] * a.geo.C) >> 5);
            dp_remote[0] = q != rt->rank;
        }
        __syncthreads();
    }
    uint32_t glo[ITEMS], ghi[ITEMS];   // SYNC: sign bits of the current group of 8 workers
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) glo[it] = ghi[it] = 0u;
    for (int w = 0; w < W; ++w) {
        const float sp = SYNC ? a.s_lazy[(int64_t)w * a.geo.nch + k] : 0.0f;
        const GT* gw = g0 + (int64_t)w * a.geo.d;
        float* mwp = a.mw + (int64_t)w * a.geo.ld + base;
        float* uwp = a.uw + (int64_t)w * a.geo.ld + base;
        float* ew = a.ew + (int64_t)w * a.geo.ld + base;
        uint32_t* bw = DP ? dp_bw0[0] + (int64_t)w * dp_bld[0] : nullptr;
        double ss = 0.0;
#pragma unroll
        for (int it = 0; it < ITEMS; ++it) {
            const int q = it * kThreads + tid;
            const int64_t off = (int64_t)q * EPT;
            float gf[EPT], m0[EPT], u0[EPT], xp[EPT];
#pragma unroll
            for (int c = 0; c < EPT; ++c) {
                gf[c] = 0.0f;
                m0[c] = ms[it][c];
                u0[c] = 0.0f;
                xp[c] = 0.0f;
            }
            if (nv[it] > 0) {
                GradLoadN<GT, VEC, EPT>::load(gw + off, nv[it], gf);
#pragma unroll
                for (int h = 0; h < EPT / 4; ++h) {
                    float t4[4];
                    if (src == kZoMWorker) {
                        ld4(mwp + off + 4 * h, t4);
#pragma unroll
                        for (int c = 0; c < 4; ++c) m0[4 * h + c] = t4[c];
                        ld4(uwp + off + 4 * h, t4);
#pragma unroll
                        for (int c = 0; c < 4; ++c) u0[4 * h + c] = t4[c];
                    } else if (src == kZoMWorkerU1) {
                        ld4(mwp + off + 4 * h, t4);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            m0[4 * h + c] = t4[c];
                            u0[4 * h + c] = __fadd_rn(0.0f, __fmul_rn(a.lr_first, t4[c]));
                        }
                    }
                    if (SYNC) {
                        ld4(ew + off + 4 * h, t4);
#pragma unroll
                        for (int c = 0; c < 4; ++c) xp[4 * h + c] = t4[c];
                    }
                }
            }
            float mn[EPT], un[EPT];
#pragma unroll
            for (int c = 0; c < EPT; ++c) {
                const bool ok = c < nv[it];
                mn[c] = ok ? __fadd_rn(__fmul_rn(b1, m0[c]), __fmul_rn(omb1, gf[c])) : 0.0f;
                un[c] = ok ? __fadd_rn(u0[c], __fmul_rn(lr, mn[c])) : 0.0f;
            }
            if constexpr (!SYNC) {
                if (nv[it] > 0) {
#pragma unroll
                    for (int h = 0; h < EPT / 4; ++h) {
                        const float tm[4] = {mn[4 * h], mn[4 * h + 1], mn[4 * h + 2], mn[4 * h + 3]};
                        const float tu[4] = {un[4 * h], un[4 * h + 1], un[4 * h + 2], un[4 * h + 3]};
                        st4(mwp + off + 4 * h, tm);
                        if (src >= kZoMWorker) st4(uwp + off + 4 * h, tu);
                    }
                }
            } else {
                float x[EPT];
                uint32_t bits = 0u;
#pragma unroll
                for (int c = 0; c < EPT; ++c) {
                    const float e = __fsub_rn(xp[c], xp[c] >= 0.0f ? sp : -sp);
                    const float xv = c < nv[it] ? __fadd_rn(un[c], e) : 0.0f;
                    x[c] = xv;
                    bits |= (c < nv[it] && xv >= 0.0f) ? (1u << c) : 0u;
                    ss = __fma_rn((double)xv, (double)xv, ss);   // NaN here marks a NaN x_w
                }
                if (nv[it] > 0) {
#pragma unroll
                    for (int h = 0; h < EPT / 4; ++h) {
                        const float t4[4] = {x[4 * h], x[4 * h + 1], x[4 * h + 2], x[4 * h + 3]};
                        st4(ew + off + 4 * h, t4);
                    }
                }
                if constexpr (DP) {
                    // OR the LPW lanes' bit groups of one 32-element word together (LSB-first)
                    uint32_t word = bits << (EPT * sub);
#pragma unroll
                    for (int o = 1; o < LPW; o <<= 1) word |= __shfl_xor_sync(kFull, word, o);
                    if (sub == 0 && nv[it] > 0) bw[q / LPW] = word;
                } else {
                    const int wi = w & 7;
                    if (EPT == 8) {
                        if (wi < 4) glo[it] |= bits << (8 * wi);
                        else ghi[it] |= bits << (8 * (wi - 4));
                    } else {
                        glo[it] |= bits << (4 * wi);
                    }
                    if ((wi == 7 || w == W - 1) && nv[it] > 0)
                        flush_group_bits<EPT>(glo[it], ghi[it],
                                              a.sbits + (int64_t)(w >> 3) * a.geo.ld + base + off);
                    if (wi == 7) glo[it] = ghi[it] = 0u;
                }
            }
        }
        if constexpr (SYNC) {
            ss = warp_sum(ss);
            if (lane == 0) red_w[w * kWarps + warp] = ss;
        }
    }
    if constexpr (SYNC) {
        // stores into another rank's memory are complete at system scope before this rank's
        // barrier signal
        if constexpr (DP) {
            if (dp_remote[0]) __threadfence_system();
        }
        __syncthreads();
        bool nan_seen = false;
        for (int w = tid; w < W; w += kThreads) {
            const double tot = block_total(red_w + w * kWarps);
            a.part_w[((int64_t)w * a.geo.nch + k) * a.geo.nseg + j] = tot;
            nan_seen |= (tot != tot);
        }
        if (nan_seen) atomicOr(a.status, kNanWorker);
    }
}

// The synchronised step from the server message of the accumulated updates:
//   ubar = (bit ? S_k : -S_k);  x -= ubar / (sqrt(v) + eps);
//   refresh:  mbar = ubar / Gamma;  v = b2 v + (1-b2) mbar^2   (after the step, which used the
//   old v).
struct ZoApplyArgs {
    Geometry geo;
    float eps, gamma, beta2, omb2;
    int refresh;
    const uint32_t* bits_s;  // [ldw]
    const float* S;          // [nch]
    float* v;                // [ld]
    float* x;                // [d] caller-owned
};

__global__ void __launch_bounds__(kThreads) k01_apply(const ZoApplyArgs a) {
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(a.geo, a.geo.nseg, k, j, base, len)) return;
    const int tid = threadIdx.x, lane = tid & 31;
    const float S = a.S[k];
    const int sh = 4 * (lane & 7);
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * kVec;
        const int nv = valid_of(len, off);
        if (nv == 0) continue;
        const uint32_t nib = a.bits_s[(base >> 5) + (q >> 3)] >> sh;
        float v[4], x[4];
        ld4(a.v + base + off, v);
        ld4_caller(a.x + base + off, nv, x);
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            const float ub = c < nv ? (((nib >> c) & 1u) ? S : -S) : 0.0f;
            const float den = __fadd_rn(__fsqrt_rn(v[c]), a.eps);
            x[c] = __fsub_rn(x[c], __fdiv_rn(ub, den));
            if (a.refresh) {
                const float mb = __fdiv_rn(ub, a.gamma);
                v[c] = __fadd_rn(__fmul_rn(a.beta2, v[c]), __fmul_rn(a.omb2, __fmul_rn(mb, mb)));
            }
        }
        st4_caller(a.x + base + off, nv, x);
        if (a.refresh) st4(a.v + base + off, v);
    }
}

// State export: each worker's momentum and accumulated update for elements [i0, i0 + n),
// rows r < W, into mw_out[W][n] / uw_out[W][n] (either may be null), from whichever form the
// state is in (src as in ZoArgs).
__global__ void k01_export(const ZoArgs a, int64_t i0, int64_t n, float* mw_out, float* uw_out) {
    const int64_t total = (int64_t)a.geo.W * n;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = t / n, i = i0 + (t - r * n);
        float m, u;
        if (a.src == kZoMWorker) {
            m = a.mw[r * a.geo.ld + i];
            u = a.uw[r * a.geo.ld + i];
        } else if (a.src == kZoMWorkerU1) {
            m = a.mw[r * a.geo.ld + i];
            u = __fadd_rn(0.0f, __fmul_rn(a.lr_first, m));
        } else {
            u = 0.0f;
            if (a.src == kZoMShared) {
                m = a.m[i];
            } else {
                const float mb = __fdiv_rn(a.S[i / a.geo.C], a.gamma_prev);
                m = ((a.bits_s[i >> 5] >> (i & 31)) & 1u) ? mb : -mb;
            }
        }
        if (mw_out) mw_out[t] = m;
        if (uw_out) uw_out[t] = u;
    }
}

// Worker w's local model, out[i] = x[i] - u_w[i] / (sqrt(v[i]) + eps), for i < d, with u_w
// as the state holds it (src as in ZoArgs; mw, uw the worker's rows).
__global__ void k01_local_model(const float* x, const float* mw, const float* uw, int src,
                                float lr_first, const float* v, float eps, int64_t d,
                                float* out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < d;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float den = __fadd_rn(__fsqrt_rn(v[i]), eps);
        const float u = src == kZoMWorker     ? uw[i]
                        : src == kZoMWorkerU1 ? __fadd_rn(0.0f, __fmul_rn(lr_first, mw[i]))
                                              : 0.0f;
        out[i] = __fsub_rn(x[i], __fdiv_rn(u, den));
    }
}

}  // namespace onebit
