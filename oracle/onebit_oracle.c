/*
 * onebit_oracle.c -- plain, slow, single-threaded CPU oracle for the compression phase of
 * 1-bit Adam (Tang et al., "1-bit Adam: Communication Efficient Large-Scale Training with
 * Adam's Convergence Speed", arXiv 2102.02888).
 *
 * TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA path is checked against.
 * Only the test suite, the package's smoke check and the benchmark's CPU-baseline leg may load
 * it. The product path never calls it, and it shares no code, header, table or constant with
 * the CUDA library.
 *
 * What the pages fix (cited by page title and section):
 *   - "1-bit Adam" index page (mlsanity.com/paper/2102.02888), Abstract: after a full-precision
 *     Adam warm-up, Adam's variance is stable and is used as a fixed preconditioner for the rest
 *     of training (the compression phase); error-compensated 1-bit compression.
 *   - LIT-278 note (dmarx.github.io anthology), Key takeaways: the compression phase is 1-bit
 *     compressed momentum SGD with the frozen variance as preconditioner; Theorem 1's conditions
 *     name error-compensated 1-bit compression with per-chunk scaling.
 *   - LIT-278 note, tag list: freeze the variance before compressing, never compress the update
 *     directly; pair the compressor with error feedback on the momentum it is applied to.
 *   - LIT-278 note, "What the evidence does not cover": the warm-up runs full-precision Adam;
 *     the compressed allreduce is a custom collective, not a stock allreduce.
 *
 * Readings where the pages are silent (every one is restated in the design notes):
 *   R1  scale of a chunk of C_k elements = ||x_chunk||_2 / sqrt(C_k): the square root of the
 *       mean square, summed in fp64 in element order, rounded once to fp32. The tail chunk uses
 *       its true length.
 *   R2  chunks are contiguous runs of C elements of the flat parameter vector; the same
 *       partition for every worker and for the server; the last chunk may be shorter.
 *   R3  sign bit = (x >= 0.0f) in IEEE binary32: +0 and -0 give 1, NaN gives 0.
 *   R4  packed words are LSB-first: element i lives in word i/32, bit i%32; bits past n are 0.
 *   R5  the server average of the W decompressed slices is an fp64 sum in worker order,
 *       divided by W in fp64, rounded once to fp32. This sum is exact (so any order gives the
 *       same bits) whenever every partial sum fits 53 bits; oracle_server reports the chunks
 *       where that cannot be guaranteed.
 *   R6  no Adam bias correction in either phase; no weight decay.
 *   R7  every fp32 operation is one IEEE round-to-nearest-even operation; no fused
 *       multiply-add (compile with -ffp-contract=off), no flush-to-zero.
 *   R8  (1 - beta) is computed in fp32 as 1.0f - beta.
 *   R9  the update is x - lr * (m / (sqrt(v) + eps)), with sqrt the correctly rounded fp32
 *       square root.
 *   R10 one shared momentum m: the first compressed step uses the warm-up momentum; every
 *       later step uses the decompressed server result written back as m.
 *   R11 worker and server errors start at zero when the variance is frozen.
 *
 * Grads are passed as fp32 (gtype 0) or as raw bf16 bit patterns (gtype 1, uint16), which
 * widen to fp32 exactly.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

static float grad_at(const void* g, int gtype, int64_t idx) {
    if (gtype == ORACLE_BF16) {
        uint32_t bits = ((uint32_t)((const uint16_t*)g)[idx]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return f;
    }
    return ((const float*)g)[idx];
}

static int64_t chunk_count(int64_t d, int64_t C) { return (d + C - 1) / C; }

static int64_t chunk_len(int64_t d, int64_t C, int64_t k) {
    int64_t lo = k * C, hi = lo + C;
    if (hi > d) hi = d;
    return hi - lo;
}

/* R3 */
static int sign_bit(float x) { return x >= 0.0f; }

/* R1: sqrt of the fp64 mean square, rounded once to fp32. */
static float chunk_scale(const float* x, int64_t len) {
    double ss = 0.0;
    for (int64_t i = 0; i < len; ++i) ss += (double)x[i] * (double)x[i];
    return (float)sqrt(ss / (double)len);
}

/* R4: LSB-first packing of sign bits. */
void oracle_pack(const float* x, int64_t n, uint32_t* words) {
    int64_t nw = (n + 31) / 32;
    for (int64_t j = 0; j < nw; ++j) words[j] = 0u;
    for (int64_t i = 0; i < n; ++i)
        if (sign_bit(x[i])) words[i / 32] |= (1u << (i % 32));
}

/* Decompression of one packed plane: out[i] = +scale or -scale of element i's chunk. */
void oracle_unpack(const uint32_t* words, const float* scales, int64_t n, int64_t C, float* out) {
    for (int64_t i = 0; i < n; ++i) {
        int bit = (int)((words[i / 32] >> (i % 32)) & 1u);
        float s = scales[i / C];
        out[i] = bit ? s : -s;
    }
}

/*
 * Full-precision Adam warm-up step ("1-bit Adam" index page, Abstract; LIT-278 note, "What the
 * evidence does not cover": the warm-up phase is plain Adam). The W workers' gradients are
 * averaged (the uncompressed allreduce) in fp64 in worker order, rounded once to fp32. R6: no
 * bias correction.
 */
void oracle_warmup_step(int64_t d, int32_t W, float beta1, float beta2, float eps, float lr,
                        float* x, float* m, float* v, const void* g, int gtype) {
    const float omb1 = 1.0f - beta1, omb2 = 1.0f - beta2;
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int32_t w = 0; w < W; ++w) acc += (double)grad_at(g, gtype, (int64_t)w * d + i);
        float gbar = (float)(acc / (double)W);
        float b1m = beta1 * m[i];
        float tg = omb1 * gbar;
        m[i] = b1m + tg;
        float g2 = gbar * gbar;
        float b2v = beta2 * v[i];
        float tv = omb2 * g2;
        v[i] = b2v + tv;
        float den = sqrtf(v[i]) + eps;
        float q = m[i] / den;
        float upd = lr * q;
        x[i] = x[i] - upd;
    }
}

/*
 * Worker side of one compressed step, for all W workers (LIT-278 note, Key takeaways and the
 * Theorem 1 conditions: momentum SGD, error-compensated 1-bit compression, per-chunk scaling).
 *   m_w   = beta1*m + (1-beta1)*g_w           (each worker's local momentum, not stored)
 *   x_w   = m_w + e_w                         (error feedback: add the worker's residual)
 *   s_w,k = ||x_w[chunk k]||_2 / sqrt(C_k)    (R1)
 *   bit   = x_w >= 0                          (R3), packed LSB-first (R4)
 *   e_w   = x_w - (bit ? s : -s)              (new residual: what the message lost)
 * e_w is [W][d], explicit. s_out is [W][nch], bits_w is [W][ceil(d/32)].
 */
void oracle_worker(int64_t d, int32_t W, int64_t C, float beta1, const float* m, const void* g,
                   int gtype, float* e_w, float* s_out, uint32_t* bits_w) {
    const float omb1 = 1.0f - beta1;
    const int64_t nch = chunk_count(d, C), nw = (d + 31) / 32;
    for (int32_t w = 0; w < W; ++w) {
        float* e = e_w + (int64_t)w * d;
        /* pass 1: x_w, kept in the residual buffer until the scales are known */
        for (int64_t i = 0; i < d; ++i) {
            float gf = grad_at(g, gtype, (int64_t)w * d + i);
            float b1m = beta1 * m[i];
            float tg = omb1 * gf;
            float mw = b1m + tg;
            e[i] = mw + e[i];
        }
        oracle_pack(e, d, bits_w + (int64_t)w * nw);
        for (int64_t k = 0; k < nch; ++k) {
            int64_t lo = k * C, len = chunk_len(d, C, k);
            float s = chunk_scale(e + lo, len);
            s_out[(int64_t)w * nch + k] = s;
            /* pass 2: residual */
            for (int64_t i = lo; i < lo + len; ++i) e[i] = e[i] - (sign_bit(e[i]) ? s : -s);
        }
    }
}

/*
 * Bound for R5: every +-s_w of chunk k is an integer multiple of the smallest ulp among the
 * nonzero scales, and every partial sum is bounded by sum |s_w|; if that bound is below 2^53
 * such multiples, each fp64 partial sum is exact and the order of the sum cannot matter.
 */
static int server_sum_is_exact(const float* s, int32_t W, int64_t nch, int64_t k) {
    double umin = 0.0, tot = 0.0;
    for (int32_t w = 0; w < W; ++w) {
        float sv = s[(int64_t)w * nch + k];
        if (sv == 0.0f) continue;
        int ex;
        (void)frexpf(sv, &ex);
        double ulp = ldexp(1.0, ex - 24);
        if (ulp < ldexp(1.0, -149)) ulp = ldexp(1.0, -149);
        if (umin == 0.0 || ulp < umin) umin = ulp;
        tot += fabs((double)sv);
    }
    if (tot == 0.0) return 1;
    return tot / umin <= 9007199254740992.0; /* 2^53 */
}

/*
 * Server side of the compressed allreduce for every chunk (LIT-278 note, Key takeaways;
 * "What the evidence does not cover": the compressed allreduce). For element i of chunk k:
 *   y   = (1/W) * sum_w (bit_w,i ? s_w,k : -s_w,k)   (R5: fp64 sum, one rounding)
 *   z   = y + e_s                                      (server error feedback)
 *   S_k = ||z[chunk k]||_2 / sqrt(C_k)                 (R1)
 *   bs  = z >= 0, packed into bits_s;  e_s = z - (bs ? S : -S)
 * z_tmp is caller scratch of length d (z is needed whole before S_k is known).
 * Returns the number of chunks where R5's exactness bound does not hold.
 */
int64_t oracle_server(int64_t d, int32_t W, int64_t C, const float* s, const uint32_t* bits_w,
                      float* e_s, float* z_tmp, float* S_out, uint32_t* bits_s) {
    const int64_t nch = chunk_count(d, C), nw = (d + 31) / 32;
    int64_t inexact = 0;
    for (int64_t k = 0; k < nch; ++k) {
        if (!server_sum_is_exact(s, W, nch, k)) ++inexact;
        int64_t lo = k * C, len = chunk_len(d, C, k);
        for (int64_t i = lo; i < lo + len; ++i) {
            double acc = 0.0;
            for (int32_t w = 0; w < W; ++w) {
                double sw = (double)s[(int64_t)w * nch + k];
                int bit = (int)((bits_w[(int64_t)w * nw + i / 32] >> (i % 32)) & 1u);
                acc += bit ? sw : -sw;
            }
            float y = (float)(acc / (double)W);
            z_tmp[i] = y + e_s[i];
        }
        float S = chunk_scale(z_tmp + lo, len);
        S_out[k] = S;
        for (int64_t i = lo; i < lo + len; ++i)
            e_s[i] = z_tmp[i] - (sign_bit(z_tmp[i]) ? S : -S);
    }
    oracle_pack(z_tmp, d, bits_s);
    return inexact;
}

/*
 * Every worker decompresses the server's message and writes it back as the shared momentum,
 * then takes the preconditioned step with the frozen variance (LIT-278 note, Key takeaways:
 * fixed preconditioner; R9, R10).
 *   m = bs ? S_k : -S_k ;  x = x - lr * (m / (sqrt(v) + eps))
 */
void oracle_apply(int64_t d, int64_t C, float eps, float lr, const uint32_t* bits_s,
                  const float* S, const float* v, float* m, float* x) {
    for (int64_t i = 0; i < d; ++i) {
        int bit = (int)((bits_s[i / 32] >> (i % 32)) & 1u);
        float Sk = S[i / C];
        m[i] = bit ? Sk : -Sk;
        float den = sqrtf(v[i]) + eps;
        float q = m[i] / den;
        float upd = lr * q;
        x[i] = x[i] - upd;
    }
}

/*
 * One whole compressed step: worker compression, the compressed allreduce (server), then the
 * frozen-variance apply. v is read-only ("1-bit Adam" index page, Abstract: the variance is
 * a fixed preconditioner after the warm-up). z_tmp is caller scratch of length d.
 * Returns the number of chunks where the server sum could not be proven exact (R5).
 */
int64_t oracle_compressed_step(int64_t d, int32_t W, int64_t C, float beta1, float eps, float lr,
                               float* x, float* m, const float* v, float* e_w, float* e_s,
                               const void* g, int gtype, float* s_out, float* S_out,
                               uint32_t* bits_w, uint32_t* bits_s, float* z_tmp) {
    oracle_worker(d, W, C, beta1, m, g, gtype, e_w, s_out, bits_w);
    int64_t inexact = oracle_server(d, W, C, s_out, bits_w, e_s, z_tmp, S_out, bits_s);
    oracle_apply(d, C, eps, lr, bits_s, S_out, v, m, x);
    return inexact;
}
