/*
 * zero_one_oracle.c -- plain, slow, single-threaded CPU oracle for the compression phase of the
 * 0/1 Adam variant (Lu, Li, Zhang, De Sa, He, "Maximizing Communication Efficiency for
 * Large-scale Training via 0/1 Adam"), built on the 1-bit Adam oracle's compressed allreduce
 * (oracle_pack and oracle_server in onebit_oracle.c, linked into the same library).
 *
 * TEST INFRASTRUCTURE ONLY, like onebit_oracle.c: the product path never calls it and it shares
 * no code, header, table or constant with the CUDA library.
 *
 * What the page fixes (codewithpapers.app "0/1 Adam" page, abstract):
 *   - 1-bit compression and local steps are used together (each alone converges slowly under
 *     Adam's non-linearity);
 *   - each Adam step is linearised by approximating the optimizer states with their stale
 *     estimates and their linear correlation;
 *   - the step stays Adam-like (adaptive), and its linearity is what allows 1-bit compression
 *     and local steps at the same time.
 * The page gives no formulas, so everything below the level of those statements is a reading.
 * Readings (restated in the design notes; R3, R4, R7 and R8 of onebit_oracle.c hold here too):
 *   Z1  the warm-up (full-precision Adam) and the freeze are those of 1-bit Adam; the variant
 *       changes the compression phase only.
 *   Z2  state: every worker w keeps its own momentum m_w and its accumulated update u_w (the
 *       sum of lr_t * m_w over the steps since the last synchronisation) next to its residual
 *       e_w; shared are the synchronised parameters x, the stale variance v and the server
 *       residual e_s. At the freeze m_w = m (the warm-up momentum), u_w = 0, e_w = e_s = 0.
 *   Z3  local step, every step t of the compression phase, each worker:
 *           m_w = beta1*m_w + (1-beta1)*g_w ;  u_w = u_w + lr_t*m_w
 *       (no communication; the Adam-like step with the stale v is implied by u_w, Z7).
 *   Z4  every H-th step (H >= 1) ends with a synchronisation: the accumulated updates go
 *       through 1-bit Adam's compressed allreduce -- x_w = u_w + e_w, per-chunk scale, sign,
 *       e_w = x_w - s*sign; the server's average, residual and recompression -- which yields the
 *       decompressed server message ubar.
 *   Z5  synchronised step: x = x - ubar / (sqrt(v) + eps) (ubar carries the learning rates);
 *       linear correlation: u = sum_t lr_t*m_t, so the momentum estimate is
 *       mbar = ubar / Gamma with Gamma the fp32 sum of lr_t over the interval; every worker
 *       restarts from m_w = mbar, u_w = 0.
 *   Z6  stale variance: at every K-th synchronisation (K >= 1; K = 0: never, v stays frozen as
 *       in 1-bit Adam) v = beta2*v + (1-beta2)*mbar^2, after the parameter step (the step uses
 *       the old v); mbar stands in for the gradient, which the compression phase never
 *       exchanges in full precision.
 *   Z7  worker w's local model between synchronisations is x - u_w / (sqrt(v) + eps), which
 *       equals its stepwise local Adam-like updates in exact arithmetic because v does not
 *       change between synchronisations; it is computed on request (nothing in a step reads
 *       it).
 * With H = 1, K = 0 and a power-of-two learning rate every quantity of the variant is exactly
 * lr times its 1-bit Adam counterpart, so the two produce the same parameters bit for bit.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* from onebit_oracle.c (same library) */
void oracle_pack(const float* x, int64_t n, uint32_t* words);
int64_t oracle_server(int64_t d, int32_t W, int64_t C, const float* s, const uint32_t* bits_w,
                      float* e_s, float* z_tmp, float* S_out, uint32_t* bits_s);

static float grad01_at(const void* g, int gtype, int64_t idx) {
    if (gtype == 1) {
        uint32_t bits = ((uint32_t)((const uint16_t*)g)[idx]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return f;
    }
    return ((const float*)g)[idx];
}

/* Z3: the local step of every worker. m_w and u_w are [W][d]. */
void oracle01_local(int64_t d, int32_t W, float beta1, float lr, float* m_w, float* u_w,
                    const void* g, int gtype) {
    const float omb1 = 1.0f - beta1;
    for (int32_t w = 0; w < W; ++w) {
        for (int64_t i = 0; i < d; ++i) {
            const int64_t j = (int64_t)w * d + i;
            float b1m = beta1 * m_w[j];
            float tg = omb1 * grad01_at(g, gtype, j);
            m_w[j] = b1m + tg;
            float step = lr * m_w[j];
            u_w[j] = u_w[j] + step;
        }
    }
}

/*
 * Z4, worker side: the 1-bit message of every worker's accumulated update with error feedback.
 *   x_w = u_w + e_w ;  s_w,k = ||x_w[chunk k]||_2 / sqrt(C_k) ;  bit = x_w >= 0 ;
 *   e_w = x_w - (bit ? s : -s)
 * e_w ([W][d], explicit) is updated in place; s_out is [W][nch], bits_w [W][ceil(d/32)].
 */
void oracle01_compress(int64_t d, int32_t W, int64_t C, const float* u_w, float* e_w,
                       float* s_out, uint32_t* bits_w) {
    const int64_t nch = (d + C - 1) / C, nw = (d + 31) / 32;
    for (int32_t w = 0; w < W; ++w) {
        float* e = e_w + (int64_t)w * d;
        const float* u = u_w + (int64_t)w * d;
        for (int64_t i = 0; i < d; ++i) e[i] = u[i] + e[i];
        oracle_pack(e, d, bits_w + (int64_t)w * nw);
        for (int64_t k = 0; k < nch; ++k) {
            const int64_t lo = k * C, len = (lo + C > d ? d : lo + C) - lo;
            double ss = 0.0;
            for (int64_t i = lo; i < lo + len; ++i) ss += (double)e[i] * (double)e[i];
            const float s = (float)sqrt(ss / (double)len);
            s_out[(int64_t)w * nch + k] = s;
            for (int64_t i = lo; i < lo + len; ++i) e[i] = e[i] - (e[i] >= 0.0f ? s : -s);
        }
    }
}

/*
 * Z5 and Z6: the synchronised step from the server message (bits_s, S) of the accumulated
 * updates. mbar[d] receives the momentum estimate; v is refreshed when `refresh` is nonzero.
 *   ubar = bs ? S_k : -S_k ;  x = x - ubar / (sqrt(v) + eps) ;  mbar = ubar / gamma ;
 *   (refresh)  v = beta2*v + (1-beta2)*mbar^2
 */
void oracle01_apply(int64_t d, int64_t C, float eps, float gamma, float beta2, int refresh,
                    const uint32_t* bits_s, const float* S, float* v, float* x, float* mbar) {
    const float omb2 = 1.0f - beta2;
    for (int64_t i = 0; i < d; ++i) {
        const int bit = (int)((bits_s[i / 32] >> (i % 32)) & 1u);
        const float Sk = S[i / C];
        const float ubar = bit ? Sk : -Sk;
        float den = sqrtf(v[i]) + eps;
        float q = ubar / den;
        x[i] = x[i] - q;
        mbar[i] = ubar / gamma;
        if (refresh) {
            float b2v = beta2 * v[i];
            float sq = mbar[i] * mbar[i];
            float tv = omb2 * sq;
            v[i] = b2v + tv;
        }
    }
}

/*
 * One step of the compression phase: the local step (Z3) and, when `sync` is nonzero, the
 * synchronisation (Z4-Z6), after which every worker restarts from mbar with u_w = 0.
 * gamma is the fp32 sum of the learning rates since the last synchronisation, this step's
 * included. Outputs of a synchronisation: s_out [W][nch], S_out [nch], bits_w, bits_s,
 * mbar [d]; z_tmp is caller scratch of length d. Returns the number of chunks where the server
 * sum could not be proven exact (R5 of onebit_oracle.c), 0 without a synchronisation.
 */
int64_t oracle01_step(int64_t d, int32_t W, int64_t C, float beta1, float beta2, float eps,
                      float lr, float gamma, int sync, int refresh, float* x, float* m_w,
                      float* u_w, float* v, float* e_w, float* e_s, const void* g, int gtype,
                      float* s_out, float* S_out, uint32_t* bits_w, uint32_t* bits_s,
                      float* mbar, float* z_tmp) {
    oracle01_local(d, W, beta1, lr, m_w, u_w, g, gtype);
    if (!sync) return 0;
    oracle01_compress(d, W, C, u_w, e_w, s_out, bits_w);
    const int64_t inexact = oracle_server(d, W, C, s_out, bits_w, e_s, z_tmp, S_out, bits_s);
    oracle01_apply(d, C, eps, gamma, beta2, refresh, bits_s, S_out, v, x, mbar);
    for (int32_t w = 0; w < W; ++w) {
        for (int64_t i = 0; i < d; ++i) {
            m_w[(int64_t)w * d + i] = mbar[i];
            u_w[(int64_t)w * d + i] = 0.0f;
        }
    }
    return inexact;
}

/* Z7: worker w's local model, out = x - u_w / (sqrt(v) + eps). */
void oracle01_local_model(int64_t d, float eps, const float* x, const float* u, const float* v,
                          float* out) {
    for (int64_t i = 0; i < d; ++i) {
        float den = sqrtf(v[i]) + eps;
        float q = u[i] / den;
        out[i] = x[i] - q;
    }
}
