// kernels.cuh -- device kernels of the 1-bit Adam compression phase for B200 (sm_100a).
//
// Every kernel here streams HBM: there is no dense contraction in the method, so the tensor
// cores play no part and the design goal is bytes moved once, coalesced, with enough loads in
// flight. The work unit is a SEGMENT of consecutive elements that never crosses a chunk
// boundary (chunk k = elements [kC, kC + C_k), LIT-278 note, Key takeaways: per-chunk scaling):
// kSeg = 2048 elements for the worker, apply and warm-up kernels, kSegS = 4096 for the server
// kernel. A block owns one segment (the server kernel a run of up to 8 segments of one chunk);
// thread t owns groups of 4 or 8 consecutive elements at offsets (it * kThreads + t) * EPT, so
// each warp-wide access is one contiguous 512- or 1024-byte run of 16-byte accesses. Small
// per-thread state (32-40 registers) keeps 48-64 warps per SM in flight, which is what hides
// HBM latency here.
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
constexpr int kItems = 2;
constexpr int kSeg = kThreads * kVec * kItems;  // 2048 elements per segment
constexpr int kSrvVec = 8;                      // server kernel: elements per thread per item
constexpr int kSrvItems = 2;
constexpr int kSegS = kThreads * kSrvVec * kSrvItems;  // 4096 elements per server segment
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kNanWorker = 1u;
constexpr uint32_t kNanServer = 2u;
constexpr uint32_t kWaitTimeout = 4u;           // a bounded wait gave up (see k_server)
constexpr int kSpinLimit = 1 << 22;

// Shape of the problem and of the library's own buffers.
struct Geometry {
    int64_t d;     // parameters
    int64_t C;     // chunk length (multiple of 32)
    int64_t nch;   // chunks, ceil(d / C)
    int64_t nseg;    // kSeg segments per full chunk
    int64_t nseg_s;  // kSegS segments per full chunk
    int64_t ld;    // row length (elements) of the library's fp32 [W][ld] residual buffer
    int64_t ldw;   // row length (words) of a packed sign plane
    int32_t W;     // workers
    int32_t spb;   // server segments per block (server_segs_per_block)
};

// ------------------------------------------------------------------------------------------
// Data-parallel ranks. With R ranks (one per GPU), rank q holds W / R of the workers and serves
// the chunks [kb[q], kb[q + 1]): the compressed allreduce becomes an exchange of plane slices
// and scales (worker side -> the chunk's server) and a broadcast of the server plane and scales
// (server -> every rank), written by the kernels straight into the peers' memory. The route
// lists, per rank, the addresses (in this process: mapped peer memory, or this GPU's own
// memory when ranks are emulated on one GPU) of the buffers the peers write.

constexpr int kMaxRanks = 8;

struct DpRoute {
    int32_t R, rank;          // ranks, this rank
    int32_t w0;               // global index of this rank's first worker
    int32_t W;                // workers over all ranks
    int64_t kb[kMaxRanks + 1];      // chunk bounds of the ranks
    int64_t ldw[kMaxRanks];         // receive-plane row length (words) at rank q
    uint32_t* planes[kMaxRanks];    // rank q's receive planes [W][ldw[q]]
    float* scales[kMaxRanks];       // rank q's receive scales [W][kb[q+1] - kb[q]]
    uint32_t* bits_s[kMaxRanks];    // rank q's server plane over all chunks
    float* S[kMaxRanks];            // rank q's server scales over all chunks
    float* m[kMaxRanks];            // rank q's momentum
    float* v[kMaxRanks];            // rank q's variance
    const double* wpart[kMaxRanks];  // rank q's warm-up gradient sums over its workers
    uint32_t* flags[kMaxRanks];     // rank q's barrier flags, one per sending rank
};

// The rank that serves chunk k (ranks with an empty range are skipped).
__device__ __forceinline__ int dp_owner(const DpRoute* rt, int64_t k) {
    int q = 0;
    while (q + 1 < rt->R && k >= rt->kb[q + 1]) ++q;
    return q;
}

// ------------------------------------------------------------------------------------------
// small helpers

__device__ __forceinline__ double warp_sum(double v) {
    // Butterfly: lane l adds v_l + v_{l^o}; commutativity makes every lane's result identical.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Segment of this block (SEG elements, nseg of them per full chunk): chunk k, segment j within
// it, global start `base`, length `len`.
template <int SEG>
__device__ __forceinline__ bool block_segment(const Geometry& g, int64_t nseg, int64_t& k,
                                              int64_t& j, int64_t& base, int64_t& len) {
    k = (int64_t)blockIdx.x / nseg;
    j = (int64_t)blockIdx.x - k * nseg;
    const int64_t c0 = k * g.C;
    const int64_t clen = min(g.C, g.d - c0);
    const int64_t s0 = j * SEG;
    if (s0 >= clen) return false;
    base = c0 + s0;
    len = min((int64_t)SEG, clen - s0);
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

// OR together the nibbles of the 8 lanes that share one 32-element word; lane l contributes
// elements 4(l%8)..4(l%8)+3 of the word (LSB-first).
__device__ __forceinline__ uint32_t gather_word(uint32_t nib, int lane) {
    uint32_t w = nib << (4 * (lane & 7));
    w |= __shfl_xor_sync(kFull, w, 1);
    w |= __shfl_xor_sync(kFull, w, 2);
    w |= __shfl_xor_sync(kFull, w, 4);
    return w;
}

// byte i bit c  ->  byte c bit i, on (lo = bytes 0..3, hi = bytes 4..7): three delta swaps of
// the row/column index bits; the first two stay inside each 32-bit half.
__device__ __forceinline__ void transpose8x8(uint32_t& lo, uint32_t& hi) {
    uint32_t t;
    t = ((lo >> 7) ^ lo) & 0x00AA00AAu;  lo ^= t ^ (t << 7);
    t = ((hi >> 7) ^ hi) & 0x00AA00AAu;  hi ^= t ^ (t << 7);
    t = ((lo >> 14) ^ lo) & 0x0000CCCCu; lo ^= t ^ (t << 14);
    t = ((hi >> 14) ^ hi) & 0x0000CCCCu; hi ^= t ^ (t << 14);
    t = ((hi << 4) ^ lo) & 0xF0F0F0F0u;  lo ^= t;  hi ^= t >> 4;
}

// Byte `b` (0..3) of 8 words -> lo/hi whose byte i is word i's byte b.
__device__ __forceinline__ void gather_bytes(const uint32_t (&w)[8], int b, uint32_t& lo,
                                             uint32_t& hi) {
    const uint32_t sel = (uint32_t)b | ((uint32_t)(4 + b) << 4);
    const uint32_t p01 = __byte_perm(w[0], w[1], sel), p23 = __byte_perm(w[2], w[3], sel);
    const uint32_t p45 = __byte_perm(w[4], w[5], sel), p67 = __byte_perm(w[6], w[7], sel);
    lo = __byte_perm(p01, p23, 0x5410);
    hi = __byte_perm(p45, p67, 0x5410);
}

__device__ __forceinline__ uint32_t byte_of(uint32_t lo, uint32_t hi, int c) {
    return ((c < 4 ? lo : hi) >> (8 * (c & 3))) & 0xffu;
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
    const float* m;       // [ld] explicit momentum (first step after freeze or set_state)
    const uint32_t* bits_s;  // [ldw] previous step's server plane: m = +-S (later steps)
    const float* S;          // [nch] previous step's server scales
    const void* g;        // [W][d] caller-owned, GT
    float* ew;            // [W][ld] lazy residual: holds last step's x_w
    const float* s_lazy;  // [W][nch] scale that rebuilds the residual
    uint8_t* sbits;       // [ceil(W/8)][ld] sign bits grouped by 8 workers (single GPU)
    double* part_w;       // [W][nch][nseg]
    uint32_t* status;
    const DpRoute* route;  // data-parallel ranks only: where the plane words go
};

// Gradient loads of N consecutive elements (N = 4 or 8), fp32 or bf16 bit patterns (uint16_t,
// widened exactly by a 16-bit shift): one 16-byte access for 4 fp32 or 8 bf16 values, an 8-byte
// one for 4 bf16; element by element for a ragged group or when the caller's rows are not
// aligned for vector access (VEC false).
template <typename GT, bool VEC, int N> struct GradLoadN;

template <bool VEC, int N> struct GradLoadN<float, VEC, N> {
    static __device__ __forceinline__ void load(const float* p, int nv, float (&o)[N]) {
        if (VEC && nv == N) {
#pragma unroll
            for (int h = 0; h < N / 4; ++h) {
                const float4 t = *reinterpret_cast<const float4*>(p + 4 * h);
                o[4 * h] = t.x; o[4 * h + 1] = t.y; o[4 * h + 2] = t.z; o[4 * h + 3] = t.w;
            }
            return;
        }
#pragma unroll
        for (int c = 0; c < N; ++c) o[c] = c < nv ? p[c] : 0.0f;
    }
};

template <bool VEC> struct GradLoadN<uint16_t, VEC, 4> {
    static __device__ __forceinline__ void load(const uint16_t* p, int nv, float (&o)[4]) {
        if (VEC && nv == 4) {
            const uint2 t = *reinterpret_cast<const uint2*>(p);
            o[0] = __uint_as_float(t.x << 16);
            o[1] = __uint_as_float(t.x & 0xffff0000u);
            o[2] = __uint_as_float(t.y << 16);
            o[3] = __uint_as_float(t.y & 0xffff0000u);
            return;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) o[c] = c < nv ? __uint_as_float((uint32_t)p[c] << 16) : 0.0f;
    }
};

template <bool VEC> struct GradLoadN<uint16_t, VEC, 8> {
    static __device__ __forceinline__ void load(const uint16_t* p, int nv, float (&o)[8]) {
        if (VEC && nv == 8) {
            const uint4 t = *reinterpret_cast<const uint4*>(p);
            const uint32_t u[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                o[2 * h] = __uint_as_float(u[h] << 16);
                o[2 * h + 1] = __uint_as_float(u[h] & 0xffff0000u);
            }
            return;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) o[c] = c < nv ? __uint_as_float((uint32_t)p[c] << 16) : 0.0f;
    }
};

// Sign bits grouped by 8 workers: byte i of group row g holds the bits of workers 8g .. 8g+7 of
// element i (bit j = worker 8g + j), the layout the server kernel decodes without transposing.
// A thread collects, over 8 consecutive workers, its EPT elements' bits -- EPT = 8: byte j of
// (lo, hi) = worker 8g + j's 8 bits; EPT = 4: nibble j of lo = worker 8g + j's 4 bits -- and
// transposes them into one byte per element.
template <int EPT>
__device__ __forceinline__ void flush_group_bits(uint32_t lo, uint32_t hi, uint8_t* dst) {
    if constexpr (EPT == 8) {
        transpose8x8(lo, hi);
        *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
    } else {
        const uint32_t t = lo & 0x0f0f0f0fu, u = (lo >> 4) & 0x0f0f0f0fu;
        uint32_t a = __byte_perm(t, u, 0x5140), b = __byte_perm(t, u, 0x7362);
        transpose8x8(a, b);
        *reinterpret_cast<uint32_t*>(dst) = a;
    }
}

// The kernel is latency-bound on HBM: more warps in flight beat deeper per-thread prefetch
// (measured on B200). EPT: elements per thread per item, 4 (fp32 gradients: 16-byte loads; 8
// resident blocks per SM at 32 registers) or 8 (bf16 gradients: 16-byte loads of 8 values; 6
// blocks per SM at 40 registers, which measured faster than 8 blocks with spills or EPT 4 with
// 8-byte gradient loads); a 2048-element segment is kSeg / (256 * EPT) items.
// LAZY_M: the shared momentum is the decompressed server message of the previous step, m =
// (bit ? S_k : -S_k), rebuilt here from the server plane instead of read as fp32 (4 bytes per
// parameter fewer to read, and k_apply need not write it).
// Single GPU: the sign bits leave grouped by 8 workers (flush_group_bits), one byte per element
// and group, so that the server reads each element's 8-worker pattern directly.
// DP: the worker rows are this rank's W / R workers, and the plane words of chunk k go to row
// (w0 + w) of the receive planes of the rank that serves chunk k (a store to peer memory), so
// that the exchange of the compressed allreduce travels with the compression itself.
template <typename GT, bool VEC, bool LAZY_M, int EPT, bool DP = false>
__global__ void __launch_bounds__(kThreads, EPT == 8 ? 6 : 8) k_worker(const WorkerArgs a) {
    constexpr int ITEMS = kSeg / (kThreads * EPT);
    constexpr int LPW = 32 / EPT;  // lanes that share one 32-element sign word
    extern __shared__ double red_w[];  // [W][kWarps]
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(a.geo, a.geo.nseg, k, j, base, len)) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int W = a.geo.W;
    const int sub = lane & (LPW - 1);

    float mr[ITEMS][EPT];
    int nv[ITEMS];
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * EPT;
        const int64_t r = len - off;
        nv[it] = r <= 0 ? 0 : (r >= EPT ? EPT : (int)r);
        if (nv[it] > 0) {
            if (LAZY_M) {
                const float S = a.S[k];
                const uint32_t bits = a.bits_s[(base >> 5) + q / LPW] >> (EPT * sub);
#pragma unroll
                for (int c = 0; c < EPT; ++c) mr[it][c] = ((bits >> c) & 1u) ? S : -S;
            } else {
#pragma unroll
                for (int h = 0; h < EPT / 4; ++h) {
                    float t4[4];
                    ld4(a.m + base + off + 4 * h, t4);
#pragma unroll
                    for (int c = 0; c < 4; ++c) mr[it][4 * h + c] = t4[c];
                }
            }
        } else {
#pragma unroll
            for (int c = 0; c < EPT; ++c) mr[it][c] = 0.0f;
        }
    }
    const float b1 = a.beta1, omb1 = a.omb1;
    const GT* g0 = static_cast<const GT*>(a.g) + base;
    // DP: this block's destination row start and row length, kept in shared memory (the
    // kernel runs at its register limit), and whether the destination is another rank's
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
    uint32_t glo[ITEMS], ghi[ITEMS];   // sign bits of the current group of 8 workers
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) glo[it] = ghi[it] = 0u;
    for (int w = 0; w < W; ++w) {
        const float sp = a.s_lazy[(int64_t)w * a.geo.nch + k];
        const GT* gw = g0 + (int64_t)w * a.geo.d;
        float* ew = a.ew + (int64_t)w * a.geo.ld + base;
        uint32_t* bw = DP ? dp_bw0[0] + (int64_t)w * dp_bld[0] : nullptr;
        double ss = 0.0;
#pragma unroll
        for (int it = 0; it < ITEMS; ++it) {
            const int q = it * kThreads + tid;
            const int64_t off = (int64_t)q * EPT;
            float xp[EPT], gf[EPT];
            if (nv[it] > 0) {
#pragma unroll
                for (int h = 0; h < EPT / 4; ++h) {
                    float t4[4];
                    ld4(ew + off + 4 * h, t4);
#pragma unroll
                    for (int c = 0; c < 4; ++c) xp[4 * h + c] = t4[c];
                }
                GradLoadN<GT, VEC, EPT>::load(gw + off, nv[it], gf);
            } else {
#pragma unroll
                for (int c = 0; c < EPT; ++c) xp[c] = gf[c] = 0.0f;
            }
            float x[EPT];
            uint32_t bits = 0u;
#pragma unroll
            for (int c = 0; c < EPT; ++c) {
                const float e = __fsub_rn(xp[c], xp[c] >= 0.0f ? sp : -sp);
                const float mw = __fadd_rn(__fmul_rn(b1, mr[it][c]), __fmul_rn(omb1, gf[c]));
                const float xv = c < nv[it] ? __fadd_rn(mw, e) : 0.0f;
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
                if ((wi == 7 || w == W - 1) && nv[it] > 0) {
                    flush_group_bits<EPT>(glo[it], ghi[it],
                                          a.sbits + (int64_t)(w >> 3) * a.geo.ld + base + off);
                }
                if (wi == 7) glo[it] = ghi[it] = 0u;
            }
        }
        ss = warp_sum(ss);
        if (lane == 0) red_w[w * kWarps + warp] = ss;
    }
    // stores into another rank's memory are complete at system scope before this rank's
    // barrier signal (stores to this GPU's own memory are ordered by the kernel boundary)
    if constexpr (DP) {
        if (dp_remote[0]) __threadfence_system();
    }
    __syncthreads();
    bool nan_seen = false;
    for (int w = tid; w < W; w += kThreads) {
        const double tot = block_total(red_w + w * kWarps);
        a.part_w[((int64_t)w * a.geo.nch + k) * a.geo.nseg + j] = tot;
        nan_seen |= (tot != tot);                         // a NaN x_w makes its sum NaN
    }
    if (nan_seen) atomicOr(a.status, kNanWorker);
}

// ------------------------------------------------------------------------------------------
// Chunk scales from the per-segment fp64 partials: s = fl32(sqrt(sum / C_k)). TPR threads
// reduce one row (row = w * nch + k for the workers, k for the server). Writes the reported
// scale and the scale that rebuilds the lazy residual next step.

// The scale of row r (active rows only; every thread of the row returns it). The TPR threads of
// the row sum its nseg-strided partials in a fixed order.
template <int TPR>
__device__ __forceinline__ float row_scale(const double* part, int64_t r, bool active,
                                           int64_t nch, int64_t nseg, int64_t seg, int64_t C,
                                           int64_t d, double* red) {
    const int sub = threadIdx.x % TPR;
    int64_t clen = 1;
    double acc = 0.0;
    if (active) {
        const int64_t k = r % nch;
        clen = min(C, d - k * C);
        const int64_t nsk = (clen + seg - 1) / seg;
        const double* p = part + r * nseg;
        for (int64_t jj = sub; jj < nsk; jj += TPR) acc += p[jj];
    }
    if (TPR >= 32) acc = warp_sum(acc);
    if (TPR == kThreads) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
        __syncthreads();
        acc = block_total(red);
    }
    return __double2float_rn(__dsqrt_rn(__ddiv_rn(acc, (double)clen)));
}

template <int TPR>
__global__ void __launch_bounds__(kThreads) k_scales(const double* part, int64_t rows,
                                                     int64_t nch, int64_t nseg, int64_t seg,
                                                     int64_t C, int64_t d, float* out,
                                                     float* lazy) {
    __shared__ double red[kWarps];
    const int64_t r = (int64_t)blockIdx.x * (kThreads / TPR) + threadIdx.x / TPR;
    const bool active = r < rows;
    const float s = row_scale<TPR>(part, r, active, nch, nseg, seg, C, d, red);
    if (active && threadIdx.x % TPR == 0) {
        out[r] = s;
        lazy[r] = s;
    }
}

// Data-parallel scales. Workers (SERVER false; rows = this rank's workers x all chunks): the
// scale is also stored in the serving rank's receive scales, row w0 + w. Server (SERVER true;
// rows = this rank's chunks): the scale is broadcast into every rank's server scales; `out` is
// not used (the broadcast includes this rank's own copy).
template <int TPR, bool SERVER>
__global__ void __launch_bounds__(kThreads) k_scales_dp(const double* part, int64_t rows,
                                                        int64_t nch, int64_t nseg, int64_t seg,
                                                        int64_t C, int64_t d, float* out,
                                                        float* lazy, const DpRoute* rt) {
    __shared__ double red[kWarps];
    const int64_t r = (int64_t)blockIdx.x * (kThreads / TPR) + threadIdx.x / TPR;
    const bool active = r < rows;
    const float s = row_scale<TPR>(part, r, active, nch, nseg, seg, C, d, red);
    bool remote = false;
    if (active && threadIdx.x % TPR == 0) {
        lazy[r] = s;
        if constexpr (SERVER) {
            const int64_t kg = rt->kb[rt->rank] + r;
            for (int p = 0; p < rt->R; ++p) rt->S[p][kg] = s;
            remote = rt->R > 1;
        } else {
            out[r] = s;
            const int64_t w = r / nch, k = r - w * nch;
            const int q = dp_owner(rt, k);
            rt->scales[q][(rt->w0 + w) * (rt->kb[q + 1] - rt->kb[q]) + (k - rt->kb[q])] = s;
            remote = q != rt->rank;
        }
    }
    if (remote) __threadfence_system();  // peer stores before the barrier signal
}

// ------------------------------------------------------------------------------------------
// TMA bulk copies (global -> shared, completion counted on an mbarrier) and bounded waits.

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// 1-D bulk copy; dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// One plain arrival (no transaction bytes) on a barrier.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for phase `parity` of the barrier, giving up after `limit` polls.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  int limit = kSpinLimit) {
    for (int i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Self-test of the bounded wait: arm a barrier for 16 bytes that nothing will deliver and wait
// on it with the bound the server kernel uses (here `limit` polls). Nothing is copied, so the
// block can leave with the barrier still pending. *timed_out = 1 when the wait gave up.
__global__ void k_selftest_wait(int limit, uint32_t* timed_out) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_arrive_expect_tx(&bar, 16);
    }
    __syncthreads();
    const bool landed = mbar_wait_bounded(&bar, 0, limit);
    const int gave_up = __syncthreads_or(!landed);
    if (threadIdx.x == 0) *timed_out = gave_up ? 1u : 0u;
}

// ------------------------------------------------------------------------------------------
// K2: the server side of the compressed allreduce. Per element of chunk k:
//   y = fl32(fp64 sum_w (+-s_w,k) / W);  z = y + e_s;  bit = z >= 0;
//   store z (lazy server residual);  fp64 partial of sum z^2.
// LIT-278 note, Key takeaways and "What the evidence does not cover" (the compressed allreduce).
//
// Work split. A block owns up to spb (8 or 16) consecutive kSegS-element segments of one chunk:
// it reads the chunk's W scales, picks the decode mode and builds its lookup tables once, then
// streams its segments. Each segment's sign bits arrive in shared memory by TMA bulk copies
// counted on a per-stage mbarrier: on one GPU the ceil(W/8) rows of the grouped sign bytes
// (4096 bytes each), on a data-parallel rank the W per-worker plane rows (at most 528 bytes
// each). With two stages the copies of segment t + 2 are in flight while segment t is decoded.
// Each warp, done with a stage, arrives on the stage's second mbarrier; thread 0 waits for all
// eight arrivals before it refills the stage, so no block-wide barrier sits in the segment loop
// and a warp that is ahead goes straight on to the next stage. Residuals are staged with the
// sign bits or read into registers, and z is written with plain 16-byte accesses.
//
// Decoding. Thread t owns 8 consecutive elements. For each group of 8 workers it takes their
// 8-bit patterns of those elements -- one 8-byte shared load of the grouped sign bytes, or, from
// per-worker planes, a gather of 8 bytes (__byte_perm) and an 8x8 bit transpose -- and looks
// each pattern up in a per-block table of the sums of (+-s) over that group. Every partial sum
// of the W values +-s_w is exact in fp64 when sum |s_w| <= 2^53 * u (u = the smallest ulp among
// the nonzero s_w), so then the grouping cannot change the result. The block picks one of four
// decodes, all bit-identical to the in-order fp64 sum of the definition:
//   kModeY     W <= 8: one table of y itself (its entries are the in-order sums);
//   kModeInt   exact and sum |s_w| / u < 2^31: the +-s_w are integers in units of u, the tables
//              are int32 and a lookup costs one integer add; y = fl32(A * u / W);
//   kModeF64   exact: fp64 tables;
//   kModeSeq   otherwise (or NaN/inf scales): worker by worker in order 0..W-1.

enum ServerMode : int { kModeY = 0, kModeInt = 1, kModeF64 = 2, kModeSeq = 3 };

constexpr int kSegWords = kSegS / 32;      // sign words per worker per server segment
constexpr int kTileRow = kSegWords + 4;    // staged row: the segment's words plus up to 3 words
                                           // before them (copies start 16-byte aligned)

struct ServerArgs {
    Geometry geo;
    const uint8_t* sbits;    // [ceil(W/8)][ld] sign bits grouped by 8 workers (single GPU)
    const uint32_t* bits_w;  // [W][ldw] per-worker receive planes (data-parallel ranks)
    const float* s;          // [W][nch] this step's worker scales
    float* es;               // [ld] lazy server residual: holds last step's z
    const float* S_lazy;     // [nch]
    uint32_t* bits_s;        // [ldw]
    double* part_s;          // [nch][blocks per chunk]: one fp64 partial per block
    uint32_t* status;
    const DpRoute* route;    // data-parallel ranks only: where the server plane goes
    // Folded worker scales (single GPU, few partials per chunk): instead of reading s, every
    // block reduces the chunk's worker partials itself, in the order of k_scales<ws_tpr>, and
    // block 0 of the chunk stores them (s_out, s_lazy). part_w null: s is read.
    const double* part_w;    // [W][nch][nseg]
    int ws_tpr;              // 1 or 32: threads per row, as launch_scales would pick
    float* s_out;            // [W][nch]
    float* s_lazy;           // [W][nch]
};

// Pipeline depth of k_server: two stages while they fit next to the tables and a block has
// more than one segment to stream.
__host__ __device__ inline int server_stages(int W, int64_t nseg_s) {
    return (W <= 128 && nseg_s > 1) ? 2 : 1;
}

// Lookup tables. The 4-byte tables (int32 group sums, or the fp32 y table for W <= 8) are read
// at random entries by all 32 lanes of a warp at once; with one copy of a table several lanes
// land on the same shared-memory bank (about 3 wavefronts per lookup instead of 1).
//
// Bank-private tables cut that for 2, 4 or 8 groups (9 <= W <= 64): every bank holds a whole
// copy of one group's table. Entry i of the tables is row i of RW = NG * K words (NG groups, K
// copies each); word g * K + h of a row is copy h of group g's entry. In lookup slot s, lane l
// reads group (s + l) mod NG from copy (l / NG) mod K. With 4 or 8 groups K = 32 / NG and the
// lanes that read one group at once use K different banks: one wavefront per lookup (32 KB).
// With 2 groups K = 8 (16 KB, rows of 16 words): lanes l and l + 16 share a copy and meet in a
// bank when their entries have the same parity, so a lookup takes 2 wavefronts.
//
// The copies cost shared memory (fewer blocks per SM) and a longer table set-up, which pays
// where a block streams many segments and, for 2 groups (3 blocks per SM instead of 4), where
// the grid is long enough that its last wave matters little (at least 2048 x 8 segments).
// Otherwise (W <= 8, W > 64, short chunks, small grids) each group's table is one 1 KB copy
// (measured both ways). Partial
// replication with lane l reading copy l mod R does not help for R < 16: the cost of a warp's
// lookup is the busiest bank's load, and with R = 2, 4 or 8 that load stays at about 3. For 2
// groups, 16 copies (32 KB) with the residuals staged leave 2 blocks per SM, and with the
// residuals in registers or in one buffer of their own the stream stalls: both measured slower
// than 8 copies with staged residuals.
__host__ __device__ constexpr int server_copies(int ng) { return ng == 2 ? 8 : 32 / ng; }
__host__ __device__ inline bool server_bank_private(int W, int64_t nseg_s, int64_t nch) {
    const int ngroups = (W + 7) / 8;
    if (nseg_s < 8) return false;
    if (ngroups == 4 || ngroups == 8) return true;
    return ngroups == 2 && nch * ((nseg_s + 7) / 8) >= 2048;
}

// Server segments per block: 16 with bank-private tables and long chunks (their set-up is
// spread over more segments; measured 3-4% faster than 8 for 2 groups), else 8.
__host__ __device__ inline int server_segs_per_block(int W, int64_t nseg_s, int64_t nch) {
    return (server_bank_private(W, nseg_s, nch) && nseg_s >= 16) ? 16 : 8;
}

// Residuals staged by TMA next to the sign words (STAGE_RES) while the stages stay small enough
// for several blocks per SM (W <= 32, single-copy tables or the 16 KB tables of 2 groups);
// otherwise they are read into registers at the top of each segment (measured).
__host__ __device__ inline bool server_stage_residuals(int W, bool bank_private) {
    return W <= 32 && (!bank_private || (W + 7) / 8 == 2);
}

// Bytes of the table region: the bank-private int32 tables or, in the same place, the fp64
// tables of kModeF64 (one copy of [ngroups][256]); with single-copy tables, the fp64 tables and
// the int32 tables in the same place, then the y table (W <= 8).
__host__ __device__ inline size_t server_table_bytes(int W, bool bank_private) {
    const int ngroups = (W + 7) / 8;
    const size_t f64 = (size_t)ngroups * 256 * sizeof(double);
    if (!bank_private) return f64 + 256 * sizeof(float);
    const size_t tab = (size_t)256 * ngroups * server_copies(ngroups) * sizeof(int32_t);
    return f64 > tab ? f64 : tab;
}

// Words of one pipeline stage: wpad plane rows, then the segment's residuals when staged.
__host__ __device__ inline size_t server_stage_words(int W, bool stage_res) {
    return (size_t)((W + 7) & ~7) * kTileRow + (stage_res ? kSegS : 0);
}

// Dynamic shared memory of k_server for W workers, `nst` stages and the table layout (bytes).
__host__ __device__ inline size_t server_smem_bytes(int W, int nst, bool bank_private) {
    const int wpad = (W + 7) & ~7;
    return 64                                                   // mbarriers, mode, unit
         + (size_t)nst * server_stage_words(W, server_stage_residuals(W, bank_private)) *
               sizeof(uint32_t)
         + (size_t)wpad * sizeof(double)                        // scales
         + server_table_bytes(W, bank_private)                  // tables
         + kWarps * sizeof(double)                              // reduction
         + (size_t)wpad * sizeof(int32_t);                      // integer scales (kModeInt)
}

template <bool POW2>
__device__ __forceinline__ float server_average(double acc, double dW, double invW) {
    return __double2float_rn(POW2 ? acc * invW : __ddiv_rn(acc, dW));
}

// Start the bulk copies of segment j's sign bits -- grouped (ceil(W/8) rows of kSegS bytes at
// word offsets 0, kSegS/4, ...), or with PLANES the W per-worker plane rows (kTileRow words
// apart) -- and, with STAGE_RES, its residuals after wpad * kTileRow words, into one stage
// (thread 0 only). The grouped rows fit inside the space of the plane rows.
template <bool STAGE_RES, bool PLANES>
__device__ __forceinline__ void server_issue(const ServerArgs& a, uint32_t* stage, int wpad,
                                             uint64_t* bar, int64_t c0, int64_t clen,
                                             int64_t j) {
    const int64_t base = c0 + j * kSegS;
    const int64_t len = min((int64_t)kSegS, clen - j * kSegS);
    const uint32_t es_bytes = STAGE_RES ? (uint32_t)(((len + 3) / 4) * 16) : 0u;
    if constexpr (!PLANES) {
        // bytes [base, base + round_up(len, 16)) of each group row: base is a multiple of 32
        // and rows are ld (a multiple of 64) bytes long, so both ends are 16-byte aligned and
        // inside the row
        const uint32_t row_bytes = (uint32_t)(((len + 15) / 16) * 16);
        const int ngroups = wpad / 8;
        mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)ngroups + es_bytes);
        for (int g = 0; g < ngroups; ++g)
            bulk_load(stage + (size_t)g * (kSegS / 4), a.sbits + (int64_t)g * a.geo.ld + base,
                      row_bytes, bar);
        if (STAGE_RES) bulk_load(stage + (size_t)wpad * kTileRow, a.es + base, es_bytes, bar);
        return;
    }
    const int64_t wbase = base >> 5;
    // words [wbase & ~3, round_up(wbase + ceil(len / 32), 4)) of each row: both ends 16-byte
    // aligned and inside the row (plane rows are padded to a multiple of 4 words)
    const int lead = (int)(wbase & 3);
    const uint32_t row_bytes = (uint32_t)(((lead + (len + 31) / 32 + 3) / 4) * 16);
    // residuals [base, base + round_up(len, 4)): base is a multiple of 32 elements and the
    // buffer is padded to a multiple of 64, so the copy is 16-byte aligned and in bounds
    mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)a.geo.W + es_bytes);
    for (int w = 0; w < a.geo.W; ++w)
        bulk_load(stage + (size_t)w * kTileRow,
                  a.bits_w + (int64_t)w * a.geo.ldw + (wbase - lead), row_bytes, bar);
    if (STAGE_RES) bulk_load(stage + (size_t)wpad * kTileRow, a.es + base, es_bytes, bar);
}

// BCAST (data-parallel ranks): the geometry is this rank's range of chunks, the plane rows are
// the receive planes of all W workers, bits_s points at this rank's first chunk in its own copy
// of the server plane, and each block then stores its server words into every other rank's copy
// (the broadcast half of the compressed allreduce, to peer memory).
template <bool POW2, bool STAGE_RES, bool BCAST = false, int NG = 0>
__global__ void __launch_bounds__(kThreads, NG == 8 ? 2 : (NG == 4 || NG == 2 ? 3 : 4))
k_server(const ServerArgs a) {
    extern __shared__ __align__(16) unsigned char smem_srv[];
    const int W = a.geo.W;
    const int spb = a.geo.spb;
    const int64_t nsb = (a.geo.nseg_s + spb - 1) / spb;
    const int64_t k = (int64_t)blockIdx.x / nsb;
    const int64_t b = (int64_t)blockIdx.x - k * nsb;
    const int64_t c0 = k * a.geo.C;
    const int64_t clen = min(a.geo.C, a.geo.d - c0);
    const int64_t nseg_k = (clen + kSegS - 1) / kSegS;
    const int64_t j0 = b * spb;
    if (j0 >= nseg_k) return;
    const int nseg_blk = (int)min((int64_t)spb, nseg_k - j0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wpad = (W + 7) & ~7, ngroups = wpad / 8;
    const int nst = server_stages(W, a.geo.nseg_s);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_srv);             // [nst] (<= 2): full
    uint64_t* ebars = reinterpret_cast<uint64_t*>(smem_srv + 32);       // [nst]: stage read
    int* mode_p = reinterpret_cast<int*>(smem_srv + 16);
    int* emin_p = reinterpret_cast<int*>(smem_srv + 20);     // smallest effective exponent
    double* unit_p = reinterpret_cast<double*>(smem_srv + 24);
    // [nst][stage_words]: wpad plane rows (rows W..wpad-1 stay zero, so every group of 8 rows
    // is complete), then, with STAGE_RES, the segment's residuals
    const size_t stage_words = server_stage_words(W, STAGE_RES);
    uint32_t* stages = reinterpret_cast<uint32_t*>(smem_srv + 64);
    double* sw = reinterpret_cast<double*>(stages + (size_t)nst * stage_words);
    // one table region: the fp64 tables [ngroups][256] (kModeF64), and in the same place the
    // int32 tables (kModeInt): with NG > 0 bank-private, [256 rows][32 banks], else
    // [ngroups][256]; without NG the y table (kModeY) follows the fp64 tables
    constexpr bool BP = NG > 0;
    double* lut = sw + wpad;
    int32_t* ilut = reinterpret_cast<int32_t*>(lut);
    float* ylut = reinterpret_cast<float*>(lut + ngroups * 256);
    double* red = reinterpret_cast<double*>(reinterpret_cast<unsigned char*>(lut) +
                                            server_table_bytes(W, BP));
    int32_t* mint = reinterpret_cast<int32_t*>(red + kWarps);   // [wpad] (kModeInt)
    const double dW = (double)W, invW = 1.0 / (double)W;

    if (tid == 0) {
        for (int st = 0; st < nst; ++st) {
            mbar_init(&bars[st], 1);
            mbar_init(&ebars[st], kWarps);
        }
        for (int t = 0; t < nst && t < nseg_blk; ++t)
            server_issue<STAGE_RES, BCAST>(a, stages + (size_t)t * stage_words, wpad, &bars[t],
                                           c0, clen, j0 + t);
    }
    if (a.part_w == nullptr) {
        for (int w = tid; w < wpad; w += kThreads)
            sw[w] = w < W ? (double)a.s[(int64_t)w * a.geo.nch + k] : 0.0;
    } else if (a.ws_tpr == 1) {
        for (int w = tid; w < wpad; w += kThreads) {
            const bool on = w < W;
            const int64_t r = (int64_t)w * a.geo.nch + k;
            const float sv = row_scale<1>(a.part_w, r, on, a.geo.nch, a.geo.nseg, kSeg, a.geo.C,
                                          a.geo.d, nullptr);
            sw[w] = on ? (double)sv : 0.0;
            if (on && b == 0) { a.s_out[r] = sv; a.s_lazy[r] = sv; }
        }
    } else {
        for (int w = warp; w < wpad; w += kWarps) {
            const bool on = w < W;
            const int64_t r = (int64_t)w * a.geo.nch + k;
            const float sv = row_scale<32>(a.part_w, r, on, a.geo.nch, a.geo.nseg, kSeg, a.geo.C,
                                           a.geo.d, nullptr);
            if (lane == 0) {
                sw[w] = on ? (double)sv : 0.0;
                if (on && b == 0) { a.s_out[r] = sv; a.s_lazy[r] = sv; }
            }
        }
    }
    if constexpr (BCAST)
        for (int st = 0; st < nst; ++st)
            for (int e = W * kTileRow + tid; e < wpad * kTileRow; e += kThreads)
                stages[(size_t)st * stage_words + e] = 0u;
    // without STAGE_RES: the first segment's residuals, fetched while the tables are built
    float zp[kSrvItems][kSrvVec];
    int nvs[kSrvItems];
    auto load_residuals = [&](int64_t base, int64_t len) {
#pragma unroll
        for (int it = 0; it < kSrvItems; ++it) {
            const int64_t off = (int64_t)(it * kThreads + tid) * kSrvVec;
            const int64_t rem = len - off;
            nvs[it] = rem <= 0 ? 0 : (rem >= kSrvVec ? kSrvVec : (int)rem);
            if (nvs[it] > 0) {
                float h0[4], h1[4];
                ld4(a.es + base + off, h0);
                ld4(a.es + base + off + 4, h1);
#pragma unroll
                for (int c = 0; c < 4; ++c) { zp[it][c] = h0[c]; zp[it][c + 4] = h1[c]; }
            } else {
#pragma unroll
                for (int c = 0; c < kSrvVec; ++c) zp[it][c] = 0.0f;
            }
        }
    };
    if (!STAGE_RES) load_residuals(c0 + j0 * kSegS, min((int64_t)kSegS, clen - j0 * kSegS));
    __syncthreads();
    if (warp == 0) {
        // exactness bound over the W scales (warp-parallel, fixed reduction order)
        double umin = 0.0, tot = 0.0;
        int emin = 255;
        for (int w = lane; w < W; w += 32) {
            const float sv = (float)sw[w];
            if (sv == 0.0f) continue;
            const int eb = max((int)((__float_as_uint(sv) >> 23) & 0xff), 1);
            const double ulp = ldexp(1.0, eb - 150);
            umin = (umin == 0.0 || ulp < umin) ? ulp : umin;
            emin = min(emin, eb);
            tot += fabs((double)sv);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double u2 = __shfl_xor_sync(kFull, umin, o);
            umin = (umin == 0.0 || (u2 != 0.0 && u2 < umin)) ? u2 : umin;
            emin = min(emin, __shfl_xor_sync(kFull, emin, o));
            tot += __shfl_xor_sync(kFull, tot, o);
        }
        if (lane == 0) {
            int mode;
            const bool exact = tot == 0.0 || (tot / umin <= 9007199254740992.0);
            const int p2 = __ffs(W) - 1;                       // log2 W when W is a power of 2
            const int kexp = emin - 150 - p2;                  // y = fl32(A) * 2^kexp
            if (W <= 8) mode = kModeY;
            else if (!exact) mode = kModeSeq;
            else if (tot == 0.0 || (tot / umin <= 2147483647.0 && (!POW2 || (kexp >= -126 && kexp <= 96))))
                mode = kModeInt;
            else mode = kModeF64;
            *mode_p = mode;
            *emin_p = tot == 0.0 ? 1 : emin;
            *unit_p = tot == 0.0 ? 0x1p-149 : umin;
        }
    }
    __syncthreads();
    const int mode = *mode_p;
    if (mode == kModeInt) {
        // s_w as exact integers in units of u = 2^(emin - 150)
        const int emin = *emin_p;
        auto int_scale = [&](int w) {
            const uint32_t bits = __float_as_uint((float)sw[w]);
            const int eb = (int)((bits >> 23) & 0xff);
            const uint32_t mant = (bits & 0x7fffffu) | (eb > 0 ? 0x800000u : 0u);
            return bits == 0u ? 0 : (int32_t)(mant << (max(eb, 1) - emin));
        };
        if constexpr (BP) {
            // entry e: group e mod NG (= lane mod NG, the same for every entry of a thread),
            // index e / NG, so each thread keeps its group's 8 integers in registers. The K
            // copies of an entry go to banks g * K + (q + h) mod K at step q, h = lane / NG: a
            // warp's 32 lanes hold NG groups x K consecutive entries, so at every step they
            // store to 32 different banks.
            constexpr int K = server_copies(NG), RW = NG * K;
            const int g = lane % NG, h = (lane / NG) % K;
            int32_t M[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) M[i] = int_scale(g * 8 + i);
            for (int e = tid; e < NG * 256; e += kThreads) {
                const int idx = e / NG;
                int32_t v = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) v += ((idx >> i) & 1) ? M[i] : -M[i];
                int32_t* row = ilut + idx * RW + g * K;
#pragma unroll
                for (int q = 0; q < K; ++q) row[(q + h) % K] = v;
            }
        } else {
            // entry e: group e / 256, the same for a whole warp: the group's 8 integers once
            // per block in shared memory, read by broadcast
            for (int w = tid; w < wpad; w += kThreads) mint[w] = int_scale(w);
            __syncthreads();
            for (int e = tid; e < ngroups * 256; e += kThreads) {
                const int g = e >> 8, idx = e & 255;
                int32_t v = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int32_t M = mint[g * 8 + i];
                    v += ((idx >> i) & 1) ? M : -M;
                }
                ilut[e] = v;
            }
        }
    } else if (mode == kModeY) {
        // one group: y itself, from the in-order fp64 sum over the 8 (padded) workers
        for (int idx = tid; idx < 256; idx += kThreads) {
            double acc = 0.0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const double sv = sw[i];
                acc = __dadd_rn(acc, ((idx >> i) & 1) ? sv : -sv);
            }
            ylut[idx] = server_average<POW2>(acc, dW, invW);
        }
    } else if (mode == kModeF64) {
        // fp64 tables: entry idx of group g = sum over i of (bit i of idx ? s : -s), in order
        for (int e = tid; e < ngroups * 256; e += kThreads) {
            const int g = e >> 8, idx = e & 255;
            double acc = 0.0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const double sv = sw[g * 8 + i];
                acc = __dadd_rn(acc, ((idx >> i) & 1) ? sv : -sv);
            }
            lut[e] = acc;
        }
    }
    __syncthreads();
    const float ykscale = __int_as_float((min(max(*emin_p - 150 - (__ffs(W) - 1), -126), 127) + 127) << 23);
    const double unit = *unit_p;
    const float Sp = a.S_lazy[k];
    double ss = 0.0;
    int consumed = nseg_blk;                      // segments this warp waited for
    int issued = nst < nseg_blk ? nst : nseg_blk;  // segments whose copies were issued (thread 0)
    bool issuing = true;

    for (int t = 0; t < nseg_blk; ++t) {
        const int st = t % nst;
        const uint32_t parity = (uint32_t)((t / nst) & 1);
        const int64_t base = c0 + (j0 + t) * kSegS;
        const int64_t len = min((int64_t)kSegS, clen - (j0 + t) * kSegS);
        const int64_t wbase = base >> 5;
        const int lead = (int)(wbase & 3);
        // residuals first, so their latency overlaps the wait for the planes
        if (!STAGE_RES && t > 0) load_residuals(base, len);
        const bool landed = mbar_wait_bounded(&bars[st], parity);
        if (landed) {
            const uint32_t* tile = stages + (size_t)st * stage_words;
            if (STAGE_RES) {
                const float* res = reinterpret_cast<const float*>(tile + (size_t)wpad * kTileRow);
#pragma unroll
                for (int it = 0; it < kSrvItems; ++it) {
                    const int64_t off = (int64_t)(it * kThreads + tid) * kSrvVec;
                    const int64_t rem = len - off;
                    nvs[it] = rem <= 0 ? 0 : (rem >= kSrvVec ? kSrvVec : (int)rem);
                    float h0[4], h1[4];
                    ld4(res + off, h0);
                    ld4(res + off + 4, h1);
#pragma unroll
                    for (int c = 0; c < 4; ++c) { zp[it][c] = h0[c]; zp[it][c + 4] = h1[c]; }
                }
            }
#pragma unroll
            for (int it = 0; it < kSrvItems; ++it) {
                const int q = it * kThreads + tid;        // 8-element group index in the segment
                const int64_t off = (int64_t)q * kSrvVec;
                const int nv = nvs[it];
                const int wd = q >> 2, bsel = q & 3;       // word within the segment, byte in it
                const uint32_t* tw = tile + lead + wd;
                const uint8_t* gb = reinterpret_cast<const uint8_t*>(tile) + off;
                // group g's pattern: byte c of (lo, hi) = element c's bits of workers 8g .. 8g+7
                // (bit i = worker 8g + i): read as it is from the grouped rows, or gathered from
                // the 8 plane rows and transposed
                auto pattern = [&](int g, uint32_t& lo, uint32_t& hi) {
                    if constexpr (!BCAST) {
                        const uint2 u = *reinterpret_cast<const uint2*>(gb + (size_t)g * kSegS);
                        lo = u.x;
                        hi = u.y;
                    } else {
                        uint32_t wv[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) wv[i] = tw[(g * 8 + i) * kTileRow];
                        gather_bytes(wv, bsel, lo, hi);
                        transpose8x8(lo, hi);
                    }
                };
                float y[kSrvVec];
                if (mode == kModeY) {
                    uint32_t lo, hi;
                    pattern(0, lo, hi);
#pragma unroll
                    for (int c = 0; c < kSrvVec; ++c) y[c] = ylut[byte_of(lo, hi, c)];
                } else if (mode == kModeInt) {
                    int32_t acc[kSrvVec];
#pragma unroll
                    for (int c = 0; c < kSrvVec; ++c) acc[c] = 0;
                    if constexpr (BP) {
                        // slot sl: this lane's group (sl + lane) mod NG, from its own copy
                        // (integer sums: the order of the groups does not matter)
#pragma unroll
                        for (int sl = 0; sl < NG; ++sl) {
                            const int gs = (sl + lane) % NG;
                            uint32_t lo, hi;
                            pattern(gs, lo, hi);
                            constexpr int K = server_copies(NG), RW = NG * K;
                            const int32_t* L = ilut + gs * K + (lane / NG) % K;
#pragma unroll
                            for (int c = 0; c < kSrvVec; ++c) acc[c] += L[byte_of(lo, hi, c) * RW];
                        }
                    } else {
#pragma unroll 2
                        for (int g = 0; g < ngroups; ++g) {
                            uint32_t lo, hi;
                            pattern(g, lo, hi);
                            const int32_t* L = ilut + g * 256;
#pragma unroll
                            for (int c = 0; c < kSrvVec; ++c) acc[c] += L[byte_of(lo, hi, c)];
                        }
                    }
#pragma unroll
                    for (int c = 0; c < kSrvVec; ++c)
                        y[c] = POW2 ? __int2float_rn(acc[c]) * ykscale
                                    : __double2float_rn(__ddiv_rn((double)acc[c] * unit, dW));
                } else if (mode == kModeF64) {
                    double acc[kSrvVec];
#pragma unroll
                    for (int c = 0; c < kSrvVec; ++c) acc[c] = 0.0;
                    for (int g = 0; g < ngroups; ++g) {
                        uint32_t lo, hi;
                        pattern(g, lo, hi);
                        const double* L = lut + g * 256;
#pragma unroll
                        for (int c = 0; c < kSrvVec; ++c) acc[c] = __dadd_rn(acc[c], L[byte_of(lo, hi, c)]);
                    }
#pragma unroll
                    for (int c = 0; c < kSrvVec; ++c) y[c] = server_average<POW2>(acc[c], dW, invW);
                } else {
                    // worker by worker, in order 0 .. W-1
                    double acc[kSrvVec];
#pragma unroll
                    for (int c = 0; c < kSrvVec; ++c) acc[c] = 0.0;
                    for (int g = 0; g < ngroups; ++g) {
                        uint32_t lo, hi;
                        pattern(g, lo, hi);
                        for (int i = 0; i < 8 && 8 * g + i < W; ++i) {
                            const double sv = sw[8 * g + i];
#pragma unroll
                            for (int c = 0; c < kSrvVec; ++c)
                                acc[c] = __dadd_rn(acc[c], ((byte_of(lo, hi, c) >> i) & 1u) ? sv : -sv);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < kSrvVec; ++c) y[c] = server_average<POW2>(acc[c], dW, invW);
                }
                float z[kSrvVec];
                uint32_t byte = 0u;
#pragma unroll
                for (int c = 0; c < kSrvVec; ++c) {
                    const float e = __fsub_rn(zp[it][c], zp[it][c] >= 0.0f ? Sp : -Sp);
                    const float zv = c < nv ? __fadd_rn(y[c], e) : 0.0f;
                    z[c] = zv;
                    byte |= (c < nv && zv >= 0.0f) ? (1u << c) : 0u;
                    ss = __fma_rn((double)zv, (double)zv, ss);   // NaN here marks a NaN z
                }
                if (nv > 0) {
                    const float h0[4] = {z[0], z[1], z[2], z[3]}, h1[4] = {z[4], z[5], z[6], z[7]};
                    st4(a.es + base + off, h0);
                    st4(a.es + base + off + 4, h1);
                }
                uint32_t word = byte << (8 * (lane & 3));
                word |= __shfl_xor_sync(kFull, word, 1);
                word |= __shfl_xor_sync(kFull, word, 2);
                if ((lane & 3) == 0 && nv > 0) a.bits_s[wbase + wd] = word;
            }
        }
        // this warp is done with the stage: one arrival on its "read" barrier. A warp whose
        // wait expired does not arrive (the copy may still land), sets the flag and stops.
        if (!__all_sync(kFull, landed)) {
            if (lane == 0) atomicOr(a.status, kWaitTimeout);
            consumed = t;
            break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ebars[st]);
        // thread 0 refills the stage once all warps have read it (bounded wait; if it expires,
        // no further copies are issued and the warps waiting for them time out in turn)
        if (tid == 0 && t + nst < nseg_blk && issuing) {
            if (mbar_wait_bounded(&ebars[st], parity)) {
                server_issue<STAGE_RES, BCAST>(a, stages + (size_t)st * stage_words, wpad,
                                               &bars[st], c0, clen, j0 + t + nst);
                issued = t + nst + 1;
            } else {
                atomicOr(a.status, kWaitTimeout);
                issuing = false;
            }
        }
    }
    // copies that thread 0 issued and its warp never waited for (only after an expired wait)
    // must land before the block leaves: one more bounded wait on each, in order
    if (tid == 0)
        for (int u = consumed; u < issued; ++u)
            mbar_wait_bounded(&bars[u % nst], (uint32_t)((u / nst) & 1));
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
        const double tot = block_total(red);
        a.part_s[k * nsb + b] = tot;
        if (tot != tot) atomicOr(a.status, kNanServer);   // a NaN z makes the sum NaN
    }
    if constexpr (BCAST) {
        // the block's server words, written to this rank's copy above (visible to the block
        // after the barrier), go to every other rank's copy; word ranges of blocks are disjoint
        // because chunks start on word boundaries
        // (the block's element range is recomputed from k and b, so that nothing else has to
        // stay live through the main loop)
        const DpRoute* rt = a.route;
        const int64_t e_lo = k * a.geo.C + b * ((int64_t)spb * kSegS);
        const int64_t e_hi = min(min((k + 1) * a.geo.C, a.geo.d), e_lo + (int64_t)spb * kSegS);
        const int64_t w_lo = e_lo >> 5, w_hi = (e_hi + 31) >> 5;
        const int64_t gw0 = (rt->kb[rt->rank] * a.geo.C) >> 5;
        for (int p = 0; p < rt->R; ++p) {
            if (p == rt->rank) continue;
            uint32_t* dst = rt->bits_s[p] + gw0;
            for (int64_t i = w_lo + tid; i < w_hi; i += kThreads) dst[i] = __ldcg(a.bits_s + i);
        }
        if (rt->R > 1) __threadfence_system();  // peer stores before the barrier signal
    }
}

// ------------------------------------------------------------------------------------------
// K3: every worker decompresses the server message into the shared momentum and steps with
// the frozen variance: m = (bit ? S_k : -S_k);  x -= lr * (m / (sqrt(v) + eps)). The momentum
// is kept in its compressed form (the server plane and S), which is exactly m.
// "1-bit Adam" index page, Abstract (variance as a fixed preconditioner); LIT-278 note, Key
// takeaways.

struct ApplyArgs {
    Geometry geo;
    float eps, lr;
    const uint32_t* bits_s;  // [ldw]
    const float* S;          // [nch]
    const float* v;          // [ld]
    float* x;                // [d] caller-owned
    // Folded server scale (at most 8 server partials per chunk): every block sums the chunk's
    // partials itself in the order of k_scales<1>, and segment 0's block stores S_out, S_lazy.
    // part_s null: S is read.
    const double* part_s;    // [nch][nsb]
    int64_t nsb;             // server blocks per chunk
    float* S_out;            // [nch]
    float* S_lazy;           // [nch]
};

__global__ void __launch_bounds__(kThreads, 8) k_apply(const ApplyArgs a) {
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(a.geo, a.geo.nseg, k, j, base, len)) return;
    const int tid = threadIdx.x, lane = tid & 31;
    float S;
    if (a.part_s == nullptr) {
        S = a.S[k];
    } else {
        __shared__ float S_sh;
        if (tid == 0) {
            // the partial length as a constant (spb is 8 or 16): no 64-bit division
            S_sh = a.geo.spb == 16
                ? row_scale<1>(a.part_s, k, true, a.geo.nch, a.nsb, kSegS * 16, a.geo.C, a.geo.d,
                               nullptr)
                : row_scale<1>(a.part_s, k, true, a.geo.nch, a.nsb, kSegS * 8, a.geo.C, a.geo.d,
                               nullptr);
            if (j == 0) { a.S_out[k] = S_sh; a.S_lazy[k] = S_sh; }
        }
        __syncthreads();
        S = S_sh;
    }
    const int sh = 4 * (lane & 7);
#pragma unroll
    for (int it = 0; it < kItems; ++it) {
        const int q = it * kThreads + tid;
        const int64_t off = (int64_t)q * kVec;
        const int nv = valid_of(len, off);
        if (nv == 0) continue;
        const uint32_t nib = a.bits_s[(base >> 5) + (q >> 3)] >> sh;
        float v[4], x[4], m[4];  // m stays in registers: the next step rebuilds it from the plane
        ld4(a.v + base + off, v);
        ld4_caller(a.x + base + off, nv, x);
#pragma unroll
        for (int c = 0; c < kVec; ++c) {
            m[c] = c < nv ? (((nib >> c) & 1u) ? S : -S) : 0.0f;
            const float den = __fadd_rn(__fsqrt_rn(v[c]), a.eps);
            const float upd = __fmul_rn(a.lr, __fdiv_rn(m[c], den));
            x[c] = __fsub_rn(x[c], upd);
        }
        st4_caller(a.x + base + off, nv, x);
    }
}


// ------------------------------------------------------------------------------------------
// Warm-up: one full-precision Adam step on the fp64 worker average (LIT-278 note, "What the
// evidence does not cover": the warm-up phase is plain Adam). No bias correction.

struct WarmupArgs {
    Geometry geo;
    float beta1, omb1, beta2, omb2, eps, lr;
    float c1, c2;   // bias corrections 1 - beta^t of this step (BC only)
    const void* g;  // [W][d] caller-owned
    float* m;       // [ld]
    float* v;       // [ld]
    float* x;       // [d] caller-owned
};

// fp64 sum over the W gradient rows (row stride d) of EPT consecutive elements at offset off,
// nv of them valid, in worker order (bit-exact with the definition); the loads of UNR workers
// are issued together so that they are in flight at once. A bf16 value becomes fp32 by a 16-bit
// shift and fp64 by the hardware conversion, both exact for every pattern (measured on B200:
// this keeps the kernel at the copy bandwidth, where widening with integer operations made it
// issue-bound at 0.74 of it).
template <typename GT, bool VEC, int EPT>
__device__ __forceinline__ void worker_grad_sum(const GT* g0, int64_t d, int W, int64_t off,
                                                int nv, double (&acc)[EPT]) {
    constexpr int UNR = 4;
#pragma unroll
    for (int c = 0; c < EPT; ++c) acc[c] = 0.0;
    int w = 0;
    if constexpr (sizeof(GT) == 2 && VEC && EPT == 8) {
        for (; w + UNR <= W && nv == EPT; w += UNR) {
            uint4 raw[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u)
                raw[u] = *reinterpret_cast<const uint4*>(g0 + (int64_t)(w + u) * d + off);
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const uint32_t r[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    acc[2 * h] = __dadd_rn(acc[2 * h], (double)__uint_as_float(r[h] << 16));
                    acc[2 * h + 1] = __dadd_rn(acc[2 * h + 1],
                                               (double)__uint_as_float(r[h] & 0xffff0000u));
                }
            }
        }
    }
    for (; w + UNR <= W; w += UNR) {
        float gf[UNR][EPT];
#pragma unroll
        for (int u = 0; u < UNR; ++u)
            GradLoadN<GT, VEC, EPT>::load(g0 + (int64_t)(w + u) * d + off, nv, gf[u]);
#pragma unroll
        for (int u = 0; u < UNR; ++u)
#pragma unroll
            for (int c = 0; c < EPT; ++c) acc[c] = __dadd_rn(acc[c], (double)gf[u][c]);
    }
    for (; w < W; ++w) {
        float gf[EPT];
        GradLoadN<GT, VEC, EPT>::load(g0 + (int64_t)w * d + off, nv, gf);
#pragma unroll
        for (int c = 0; c < EPT; ++c) acc[c] = __dadd_rn(acc[c], (double)gf[c]);
    }
}

// EPT elements per thread as in k_worker (8 for bf16, 4 for fp32 gradients).
// BC: Adam's optional bias correction -- the step uses m / c1 and v / c2 (m and v are stored
// uncorrected); off by default, since the pages' step has none.
template <typename GT, bool VEC, int EPT, bool BC = false>
__global__ void __launch_bounds__(kThreads, 4) k_warmup(const WarmupArgs a) {
    constexpr int ITEMS = kSeg / (kThreads * EPT);
    int64_t k, j, base, len;
    if (!block_segment<kSeg>(a.geo, a.geo.nseg, k, j, base, len)) return;
    const int tid = threadIdx.x;
    const int W = a.geo.W;
    const GT* g0 = static_cast<const GT*>(a.g) + base;
    const double dW = (double)W;
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int64_t off = (int64_t)(it * kThreads + tid) * EPT;
        const int64_t r = len - off;
        const int nv = r <= 0 ? 0 : (r >= EPT ? EPT : (int)r);
        if (nv == 0) continue;
        double acc[EPT];
        worker_grad_sum<GT, VEC, EPT>(g0, a.geo.d, W, off, nv, acc);
#pragma unroll
        for (int h = 0; h < EPT / 4; ++h) {
            const int64_t o4 = off + 4 * h;
            const int nv4 = nv - 4 * h;
            if (nv4 <= 0) break;
            float m[4], v[4], x[4];
            ld4(a.m + base + o4, m);
            ld4(a.v + base + o4, v);
            ld4_caller(a.x + base + o4, nv4 >= 4 ? 4 : nv4, x);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (c >= nv4) continue;
                const float gbar = __double2float_rn(__ddiv_rn(acc[4 * h + c], dW));
                m[c] = __fadd_rn(__fmul_rn(a.beta1, m[c]), __fmul_rn(a.omb1, gbar));
                v[c] = __fadd_rn(__fmul_rn(a.beta2, v[c]), __fmul_rn(a.omb2, __fmul_rn(gbar, gbar)));
                const float mh = BC ? __fdiv_rn(m[c], a.c1) : m[c];
                const float vh = BC ? __fdiv_rn(v[c], a.c2) : v[c];
                const float den = __fadd_rn(__fsqrt_rn(vh), a.eps);
                x[c] = __fsub_rn(x[c], __fmul_rn(a.lr, __fdiv_rn(mh, den)));
            }
            st4(a.m + base + o4, m);
            st4(a.v + base + o4, v);
            st4_caller(a.x + base + o4, nv4 >= 4 ? 4 : nv4, x);
        }
    }
}

// The freeze after a bias-corrected warm-up: the compression phase continues from the moments
// the last warm-up step used, m = m / c1, v = v / c2 (i < n).
__global__ void k_bc_freeze(float* m, float* v, float c1, float c2, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        m[i] = __fdiv_rn(m[i], c1);
        v[i] = __fdiv_rn(v[i], c2);
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
