/*
 * bias_corrected_oracle.c -- the optional bias-corrected warm-up of the 1-bit Adam oracle.
 *
 * TEST INFRASTRUCTURE ONLY, like onebit_oracle.c (same library; no code shared with the CUDA
 * path).
 *
 * The pages do not mention Adam's bias correction ("1-bit Adam" index page, Abstract, and the
 * LIT-278 note cite plain Adam; the method's step x - lr * m / (sqrt(v) + eps) has none), so it
 * is off by default (R6 of onebit_oracle.c). Reading B1, for the flag that turns it on:
 *   - warm-up step t (1-based) keeps m and v uncorrected and steps with the corrected moments
 *         mh = m / c1_t ,  vh = v / c2_t ,  x = x - lr * (mh / (sqrt(vh) + eps))
 *     where c_t = fl32(1 - beta^t), beta^t the fp64 product of t factors beta (the fp32
 *     value) in order and 1 - beta^t taken in fp64 (in fp32 the subtraction would cancel most
 *     digits of 1 - beta2^t); the caller passes c1_t and c2_t;
 *   - the freeze continues from what the last warm-up step used: m = m / c1_T, v = v / c2_T
 *     (the frozen preconditioner is the corrected variance, so the first compressed step does
 *     not jump in size).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float grad_bc_at(const void* g, int gtype, int64_t idx) {
    if (gtype == 1) {
        uint32_t bits = ((uint32_t)((const uint16_t*)g)[idx]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return f;
    }
    return ((const float*)g)[idx];
}

/* One bias-corrected warm-up step (B1); m and v stay uncorrected. */
void oracle_warmup_step_bc(int64_t d, int32_t W, float beta1, float beta2, float eps, float lr,
                           float c1, float c2, float* x, float* m, float* v, const void* g,
                           int gtype) {
    const float omb1 = 1.0f - beta1, omb2 = 1.0f - beta2;
    for (int64_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int32_t w = 0; w < W; ++w) acc += (double)grad_bc_at(g, gtype, (int64_t)w * d + i);
        float gbar = (float)(acc / (double)W);
        float b1m = beta1 * m[i];
        float tg = omb1 * gbar;
        m[i] = b1m + tg;
        float g2 = gbar * gbar;
        float b2v = beta2 * v[i];
        float tv = omb2 * g2;
        v[i] = b2v + tv;
        float mh = m[i] / c1;
        float vh = v[i] / c2;
        float den = sqrtf(vh) + eps;
        float q = mh / den;
        float upd = lr * q;
        x[i] = x[i] - upd;
    }
}

/* The freeze after a bias-corrected warm-up of T steps (B1): m = m / c1_T, v = v / c2_T. */
void oracle_freeze_bc(int64_t d, float c1, float c2, float* m, float* v) {
    for (int64_t i = 0; i < d; ++i) {
        m[i] = m[i] / c1;
        v[i] = v[i] / c2;
    }
}
