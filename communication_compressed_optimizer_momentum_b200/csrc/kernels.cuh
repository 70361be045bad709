// kernels.cuh -- device kernels of the 1-bit Adam compression phase for B200 (sm_100a).
//
// Every kernel here streams HBM: there is no dense contraction in the method, so the tensor
// cores play no part and the design goal is bytes moved once, coalesced, with enough loads in
// flight. The work unit is a SEGMENT: kSeg = 4096 consecutive elements that never cross a chunk
// boundary (chunk k = elements [kC, kC + C_k), LIT-278 note, Key takeaways: per-chunk scaling).
// A block owns one segment; thread t owns kItems groups of kVec = 4 consecutive elements at
// offsets (it * kThreads + t) * 4, so each warp-wide access is one contiguous 512-byte run.
//
// Determinism: chunk norms are fp64 sums in a fixed tree (thread -> warp butterfly -> block in
// warp order -> segments in order), so a run is bit-reproducible; no float atomics anywhere.
//
// Lazy residuals: the worker kernel stores x_w itself in the residual buffer; the next step
// rebuilds e_w = x_w - (x_w >= 0 ? s : -s) with one IEEE subtraction, which is bit-identical to
// storing e_w explicitly and saves a second pass over W x d floats. The server residual is kept
// the same way.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace onebit {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kVec = 4;
constexpr int kItems = 4;
constexpr int kSeg = kThreads * kVec * kItems;  // 4096 elements per segment
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kNanWorker = 1u;
constexpr uint32_t kNanServer = 2u;

// Shape of the problem and of the library's own buffers.
struct Geometry {
    int64_t d;     // parameters
    int64_t C;     // chunk length (multiple of 32)
    int64_t nch;   // chunks, ceil(d / C)
    int64_t nseg;  // segments per full chunk, ceil(C / kSeg)
    int64_t ld;    // row length (elements) of the library's fp32 [W][ld] residual buffer
    int64_t ldw;   // row length (words) of a packed sign plane
    int32_t W;     // workers
};

// ------------------------------------------------------------------------------------------
// small helpers

__device__ __forceinline__ double warp_sum(double v) {
    // Butterfly: lane l adds v_l + v_{l^o}; commutativity makes every lane's result identical.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Segment of this block: chunk k, segment j within it, global start `base`, length `len`.
__device__ __forceinline__ bool block_segment(const Geometry& g, int64_t& k, int64_t& j,
                                              int64_t& base, int64_t& len) {
    k = (int64_t)blockIdx.x / g.nseg;
    j = (int64_t)blockIdx.x - k * g.nseg;
    const int64_t c0 = k * g.C;
    const int64_t clen = min(g.C, g.d - c0);
    const int64_t s0 = j * kSeg;
    if (s0 >= clen) return false;
    base = c0 + s0;
    len = min((int64_t)kSeg, clen - s0);
    return true;
}

__device__ __forceinline__ int valid_of(int64_t len, int64_t off) {
    const int64_t r = len - off;
    return r <= 0 ? 0 : (r >= kVec ? kVec : (int)r);
}

__device__ __forceinline__ void ld4(const float* p, float (&o)[4]) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
}

__device__ __forceinline__ void st4(float* p, const float (&o)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
}

// Caller-owned fp32 vector (no padding): vector access only for a full group of 4.
__device__ __forceinline__ void ld4_caller(const float* p, int nv, float (&o)[4]) {
    if (nv == kVec) { ld4(p, o); return; }
#pragma unroll
    for (int c = 0; c < kVec; ++c) o[c] = c < nv ? p[c] : 0.0f;
}

__device__ __forceinline__ void st4_caller(float* p, int nv, const float (&o)[4]) {
    if (nv == kVec) { st4(p, o); return; }
#pragma unroll
    for (int c = 0; c < kVec; ++c)
        if (c < nv) p[c] = o[c];
}

// Gradient element types: fp32, or bf16 bit patterns (uint16_t) that widen exactly.
template <typename GT, bool VEC> struct GradLoad;

template <bool VEC> struct GradLoad<float, VEC> {
    static __device__ __forceinline__ void load4(const float* p, int nv, float (&o)[4]) {
        if (VEC && nv == kVec) { ld4(p, o); return; }
#pragma unroll
        for (int c = 0; c < kVec; ++c) o[c] = c < nv ? p[c] : 0.0f;
    }
};

template <bool VEC> struct GradLoad<uint16_t, VEC> {
    static __device__ __forceinline__ void load4(const uint16_t* p, int nv, float (&o)[4]) {
        if (VEC && nv == kVec) {
            const uint2 t = *reinterpret_cast<const uint2*>(p);
            o[0] = __uint_as_float(t.x << 16);
            o[1] = __uint_as_float(t.x & 0xffff0000u);
            o[2] = __uint_as_float(t.y << 16);
            o[3] = __uint_as_float(t.y & 0xffff0000u);
            return;
        }
#pragma unroll
        for (int c = 0; c < kVec; ++c) o[c] = c < nv ? __uint_as_float((uint32_t)p[c] << 16) : 0.0f;
    }
};

// OR together the nibbles of the 8 lanes that share one 32-element word; lane l contributes
// elements 4(l%8)..4(l%8)+3 of the word (LSB-first).
__device__ __forceinline__ uint32_t gather_word(uint32_t nib, int lane) {
    uint32_t w = nib << (4 * (lane & 7));
    w |= __shfl_xor_sync(kFull, w, 1);
    w |= __shfl_xor_sync(kFull, w, 2);
    w |= __shfl_xor_sync(kFull, w, 4);
    return w;
}

// Block-wide fixed-order sum of one double per warp held by lane 0 in red[warp].
__device__ __forceinline__ double block_total(const double* red) {
    double t = 0.0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) t += red[i];
    return t;
}

// ------------------------------------------------------------------------------------------
// K1: worker compression for all W workers of one segment.
//   m_w = b1 m + (1-b1) g_w;  x_w = m_w + e_w;  bit = x_w >= 0;  store x_w (lazy residual);
//   fp64 partial of sum x_w^2 for the chunk scale.
// LIT-278 note, Key takeaways (momentum SGD, error-compensated 1-bit compression, per-chunk
// scaling); tag list (compress the momentum with error feedback, not the update).

struct WorkerArgs {
    Geometry geo;
    float beta1, omb1;
    const float* m;       // [ld] library-owned
    const void* g;        // [W][d] caller-owned, GT
    float* ew;            // [W][ld] lazy residual: holds last step's x_w
    const float* s_lazy;  // [W][nch] scale that rebuilds the residual
    uint32_t* bits_w;     // [W][ldw]
    double* part_w;       // [W][nch][nseg]
    uint32_t* status;
};

template <typename GT, bool VEC>
__global__ void __launch_bounds__(kThreads) k_worker(const WorkerArgs a) {
    extern __shared__ double red_w[];  // [W][kWarps]
    int64_t k, j, base, len;
    if (!block_segment(a.geo, k, j, base, len)) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = a.geo.W;

    float mr[kItems][4];
    int nv[kItems];
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int64_t off = (int64_t)(it * kThreads + tid) * kVec;
        nv[it] = valid_of(len, off);
        if (nv[it] > 0) ld4(a.m + base + off, mr[it]);
        else { mr[it][0] = mr[it][1] = mr[it][2] = mr[it][3] = 0.0f; }
    }
    const float b1 = a.beta1, omb1 = a.omb1;
    bool nan_seen = false;
    const GT* g0 = static_cast<const GT*>(a.g) + base;
    for (int w = 0; w < W; ++w) {
        const float sp = a.s_lazy[(int64_t)w * a.geo.nch + k];
        const GT* gw = g0 + (int64_t)w * a.geo.d;
        float* ew = a.ew + (int64_t)w * a.geo.ld + base;
        uint32_t* bw = a.bits_w + (int64_t)w * a.geo.ldw + (base >> 5);
        double ss = 0.0;
#pragma unroll
        for (int it = 0; it < kItems; ++it) {
            const int q = it * kThreads + tid;
            const int64_t off = (int64_t)q * kVec;
            float xp[4] = {0.0f, 0.0f, 0.0f, 0.0f}, gf[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            if (nv[it] > 0) {
                ld4(ew + off, xp);
                GradLoad<GT, VEC>::load4(gw + off, nv[it], gf);
            }
            float x[4];
            uint32_t nib = 0u;
#pragma unroll
            for (int c = 0; c < kVec; ++c) {
                const float e = __fsub_rn(xp[c], xp[c] >= 0.0f ? sp : -sp);
                const float mw = __fadd_rn(__fmul_rn(b1, mr[it][c]), __fmul_rn(omb1, gf[c]));
                const float xv = c < nv[it] ? __fadd_rn(mw, e) : 0.0f;
                x[c] = xv;
                nib |= (c < nv[it] && xv >= 0.0f) ? (1u << c) : 0u;
                nan_seen |= (xv != xv);
                ss = __fma_rn((double)xv, (double)xv, ss);
            }
            if (nv[it] > 0) st4(ew + off, x);
            const uint32_t word = gather_word(nib, lane);
            if ((lane & 7) == 0 && nv[it] > 0) bw[q >> 3] = word;
        }
        ss = warp_sum(ss);
        if (lane == 0) red_w[w * kWarps + warp] = ss;
    }
    __syncthreads();
    for (int w = tid; w < W; w += kThreads)
        a.part_w[((int64_t)w * a.geo.nch + k) * a.geo.nseg + j] = block_total(red_w + w * kWarps);
    if (__syncthreads_or(nan_seen) && tid == 0) atomicOr(a.status, kNanWorker);
}

// ------------------------------------------------------------------------------------------
// Chunk scales from the per-segment fp64 partials: s = fl32(sqrt(sum / C_k)). TPR threads
// reduce one row (row = w * nch + k for the workers, k for the server). Writes the reported
// scale and the scale that rebuilds the lazy residual next step.

template <int TPR>
__global__ void __launch_bounds__(kThreads) k_scales(const double* part, int64_t rows,
                                                     int64_t nch, int64_t nseg, int64_t C,
                                                     int64_t d, float* out, float* lazy) {
    __shared__ double red[kWarps];
    const int64_t r = (int64_t)blockIdx.x * (kThreads / TPR) + threadIdx.x / TPR;
    const int sub = threadIdx.x % TPR;
    const bool active = r < rows;
    int64_t clen = 1;
    double acc = 0.0;
    if (active) {
        const int64_t k = r % nch;
        clen = min(C, d - k * C);
        const int64_t nsk = (clen + kSeg - 1) / kSeg;
        const double* p = part + r * nseg;
        for (int64_t jj = sub; jj < nsk; jj += TPR) acc += p[jj];
    }
    if (TPR >= 32) acc = warp_sum(acc);
    if (TPR == kThreads) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
        __syncthreads();
        acc = block_total(red);
    }
    if (active && sub == 0) {
        const float s = __double2float_rn(__dsqrt_rn(__ddiv_rn(acc, (double)clen)));
        out[r] = s;
        lazy[r] = s;
    }
}

// ------------------------------------------------------------------------------------------
// K2: the server side of the compressed allreduce for one segment of chunk k.
//   y = fl32(fp64 sum_w (+-s_w,k) / W) with the workers taken in order 0..W-1;
//   z = y + e_s;  bit = z >= 0;  store z (lazy server residual);  fp64 partial of sum z^2.
// LIT-278 note, Key takeaways and "What the evidence does not cover" (the compressed allreduce).

struct ServerArgs {
    Geometry geo;
    const uint32_t* bits_w;  // [W][ldw]
    const float* s;          // [W][nch] this step's worker scales
    float* es;               // [ld] lazy server residual: holds last step's z
    const float* S_lazy;     // [nch]
    uint32_t* bits_s;        // [ldw]
    double* part_s;          // [nch][nseg]
    uint32_t* status;
};

__global__ void __launch_bounds__(kThreads) k_server(const ServerArgs a) {
    extern __shared__ double sm_s[];  // sw[W], then red[kWarps]
    int64_t k, j, base, len;
    if (!block_segment(a.geo, k, j, base, len)) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = a.geo.W;
    double* sw = sm_s;
    double* red = sm_s + W;
    for (int w = tid; w < W; w += kThreads) sw[w] = (double)a.s[(int64_t)w * a.geo.nch + k];
    __syncthreads();
    const float Sp = a.S_lazy[k];
    const double dW = (double)W;
    const uint32_t* b0 = a.bits_w + (base >> 5);
    const int sh = 4 * (lane & 7);
    double ss = 0.0;
    bool nan_seen = false;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * kVec;
        const int nv = valid_of(len, off);
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        float zp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (nv > 0) {
            ld4(a.es + base + off, zp);
            const uint32_t* bw = b0 + (q >> 3);
            for (int w = 0; w < W; ++w) {
                const uint32_t nib = bw[(int64_t)w * a.geo.ldw] >> sh;
                const double s = sw[w];
#pragma unroll
                for (int c = 0; c < kVec; ++c) acc[c] = __dadd_rn(acc[c], ((nib >> c) & 1u) ? s : -s);
            }
        }
        float z[4];
        uint32_t nib = 0u;
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            const float y = __double2float_rn(__ddiv_rn(acc[c], dW));
            const float e = __fsub_rn(zp[c], zp[c] >= 0.0f ? Sp : -Sp);
            const float zv = c < nv ? __fadd_rn(y, e) : 0.0f;
            z[c] = zv;
            nib |= (c < nv && zv >= 0.0f) ? (1u << c) : 0u;
            nan_seen |= (zv != zv);
            ss = __fma_rn((double)zv, (double)zv, ss);
        }
        if (nv > 0) st4(a.es + base + off, z);
        const uint32_t word = gather_word(nib, lane);
        if ((lane & 7) == 0 && nv > 0) a.bits_s[(base >> 5) + (q >> 3)] = word;
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) a.part_s[k * a.geo.nseg + j] = block_total(red);
    if (__syncthreads_or(nan_seen) && tid == 0) atomicOr(a.status, kNanServer);
}

// ------------------------------------------------------------------------------------------
// K3: every worker decompresses the server message into the shared momentum and steps with
// the frozen variance: m = (bit ? S_k : -S_k);  x -= lr * (m / (sqrt(v) + eps)).
// "1-bit Adam" index page, Abstract (variance as a fixed preconditioner); LIT-278 note, Key
// takeaways.

struct ApplyArgs {
    Geometry geo;
    float eps, lr;
    const uint32_t* bits_s;  // [ldw]
    const float* S;          // [nch]
    const float* v;          // [ld]
    float* m;                // [ld]
    float* x;                // [d] caller-owned
};

__global__ void __launch_bounds__(kThreads) k_apply(const ApplyArgs a) {
    int64_t k, j, base, len;
    if (!block_segment(a.geo, k, j, base, len)) return;
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
        float v[4], x[4], m[4];
        ld4(a.v + base + off, v);
        ld4_caller(a.x + base + off, nv, x);
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            m[c] = c < nv ? (((nib >> c) & 1u) ? S : -S) : 0.0f;
            const float den = __fadd_rn(__fsqrt_rn(v[c]), a.eps);
            const float upd = __fmul_rn(a.lr, __fdiv_rn(m[c], den));
            x[c] = __fsub_rn(x[c], upd);
        }
        st4(a.m + base + off, m);
        st4_caller(a.x + base + off, nv, x);
    }
}

// ------------------------------------------------------------------------------------------
// Warm-up: one full-precision Adam step on the fp64 worker average (LIT-278 note, "What the
// evidence does not cover": the warm-up phase is plain Adam). No bias correction.

struct WarmupArgs {
    Geometry geo;
    float beta1, omb1, beta2, omb2, eps, lr;
    const void* g;  // [W][d] caller-owned
    float* m;       // [ld]
    float* v;       // [ld]
    float* x;       // [d] caller-owned
};

template <typename GT, bool VEC>
__global__ void __launch_bounds__(kThreads) k_warmup(const WarmupArgs a) {
    int64_t k, j, base, len;
    if (!block_segment(a.geo, k, j, base, len)) return;
    const int tid = threadIdx.x;
    const GT* g0 = static_cast<const GT*>(a.g) + base;
    const double dW = (double)a.geo.W;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int64_t off = (int64_t)(it * kThreads + tid) * kVec;
        const int nv = valid_of(len, off);
        if (nv == 0) continue;
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        for (int w = 0; w < a.geo.W; ++w) {
            float gf[4];
            GradLoad<GT, VEC>::load4(g0 + (int64_t)w * a.geo.d + off, nv, gf);
#pragma unroll
            for (int c = 0; c < kVec; ++c) acc[c] = __dadd_rn(acc[c], (double)gf[c]);
        }
        float m[4], v[4], x[4];
        ld4(a.m + base + off, m);
        ld4(a.v + base + off, v);
        ld4_caller(a.x + base + off, nv, x);
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            if (c >= nv) continue;
            const float gbar = __double2float_rn(__ddiv_rn(acc[c], dW));
            m[c] = __fadd_rn(__fmul_rn(a.beta1, m[c]), __fmul_rn(a.omb1, gbar));
            v[c] = __fadd_rn(__fmul_rn(a.beta2, v[c]), __fmul_rn(a.omb2, __fmul_rn(gbar, gbar)));
            const float den = __fadd_rn(__fsqrt_rn(v[c]), a.eps);
            x[c] = __fsub_rn(x[c], __fmul_rn(a.lr, __fdiv_rn(m[c], den)));
        }
        st4(a.m + base + off, m);
        st4(a.v + base + off, v);
        st4_caller(a.x + base + off, nv, x);
    }
}

// ------------------------------------------------------------------------------------------
// State export: explicit residual out[r][i] = stored[r][i0 + i] - (stored >= 0 ? s : -s), with
// s the rebuild scale of element i0 + i's chunk, for rows r < rows and i < n.

__global__ void k_materialize(const float* stored, int64_t ld_in, const float* lazy,
                              int64_t nch, int64_t C, int64_t i0, int64_t n, int64_t rows,
                              float* out) {
    const int64_t total = rows * n;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = t / n, i = i0 + (t - r * n);
        const float v = stored[r * ld_in + i];
        const float s = lazy[r * nch + i / C];
        out[t] = __fsub_rn(v, v >= 0.0f ? s : -s);
    }
}

// ------------------------------------------------------------------------------------------
// Test boundary: sign packing and decompression of one flat plane (segments of kSeg elements).

__global__ void __launch_bounds__(kThreads) k_pack(const float* x, int64_t n, uint32_t* words) {
    const int64_t base = (int64_t)blockIdx.x * kSeg;
    const int64_t len = min((int64_t)kSeg, n - base);
    const int tid = threadIdx.x, lane = tid & 31;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * kVec;
        const int nv = valid_of(len, off);
        float xv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if (nv > 0) ld4_caller(x + base + off, nv, xv);
        uint32_t nib = 0u;
#pragma unroll
        for (int c = 0; c < kVec; ++c) nib |= (c < nv && xv[c] >= 0.0f) ? (1u << c) : 0u;
        const uint32_t word = gather_word(nib, lane);
        if ((lane & 7) == 0 && nv > 0) words[(base >> 5) + (q >> 3)] = word;
    }
}

__global__ void __launch_bounds__(kThreads) k_unpack(const uint32_t* words, const float* scales,
                                                     int64_t n, int64_t C, float* out) {
    const int64_t base = (int64_t)blockIdx.x * kSeg;
    const int64_t len = min((int64_t)kSeg, n - base);
    const int tid = threadIdx.x, lane = tid & 31;
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * kVec;
        const int nv = valid_of(len, off);
        if (nv == 0) continue;
        const uint32_t nib = words[(base >> 5) + (q >> 3)] >> (4 * (lane & 7));
        float o[4];
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            const float s = c < nv ? scales[(base + off + c) / C] : 0.0f;
            o[c] = ((nib >> c) & 1u) ? s : -s;
        }
        st4_caller(out + base + off, nv, o);
    }
}

}  // namespace onebit
