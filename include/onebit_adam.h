/*
 * onebit_adam.h -- C ABI of the B200 (sm_100a) library for the data-parallel hot path of the
 * compression phase of 1-bit Adam (Tang et al., arXiv 2102.02888).
 *
 * The method (as the pages describe it):
 *   - "1-bit Adam" index page (mlsanity.com/paper/2102.02888), Abstract: Adam's variance becomes
 *     stable after a warm-up phase and is then used as a fixed preconditioner for the rest of
 *     training (the compression phase), where communication uses error-compensated 1-bit
 *     compression.
 *   - LIT-278 note (dmarx.github.io anthology), Key takeaways: the compression phase is 1-bit
 *     compressed momentum SGD with that fixed preconditioner; Theorem 1 assumes
 *     error-compensated 1-bit compression with per-chunk scaling.
 *   - LIT-278 note, "What the evidence does not cover": the warm-up is full-precision Adam; the
 *     compressed allreduce is a custom collective.
 *
 * In this library the W data-parallel workers are a batch dimension in one GPU's memory: the
 * compressed allreduce is a gather over the W workers' packed sign planes in device memory.
 *
 * Entry points, by family:
 *   - onebit_adam_*: one handle with all W workers on one GPU (init, workspace, bind, warm-up,
 *     freeze, compressed step, host-buffer step, state export and import, status, timing);
 *   - onebit_dp_*: a data-parallel rank holding W / R of the workers, one per GPU, with the
 *     compressed allreduce between the GPUs done by the kernels' own stores to peer memory;
 *   - onebit01_*: the 0/1 Adam variant (codewithpapers.app "0/1 Adam" page, abstract): local
 *     steps and a synchronisation through the same compressed allreduce every H steps, on one
 *     GPU or as data-parallel ranks, with checkpoint/resume;
 *   - onebit_pack, onebit_unpack, onebit_compress_static: one vector's 1-bit message;
 *   - host-only queries: onebit_dp_chunk_range, onebit_server_layout, onebit_strerror,
 *     onebit_last_error.
 *
 * Conventions (all calls):
 *   - Every pointer named *_dev or documented as device memory is a CUDA device pointer owned
 *     by the caller, 16-byte aligned, and must stay valid until the work queued on the stream
 *     has finished. The library allocates no device memory, with one exception: the exchange
 *     region of a data-parallel rank (onebit_dp_*), which other ranks map through CUDA IPC and
 *     which therefore must be an allocation of its own.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Device work
 *     is queued on it asynchronously; argument errors are detected on the host and returned
 *     before anything is queued.
 *   - Return values: ONEBIT_OK (0) or a negative onebit_status. ONEBIT_ERR_CUDA means a CUDA
 *     runtime call or kernel launch failed (the CUDA error string is kept, see onebit_last_error).
 *   - Floating point: every fp32 operation of the method is one IEEE round-to-nearest-even
 *     operation (no fused multiply-add, no flush-to-zero); norms and the server average are
 *     accumulated in fp64.
 *   - Sign convention: bit = (x >= 0) (so +0 and -0 give 1, NaN gives 0). Packed planes are
 *     LSB-first uint32 words: element i is bit i%32 of word i/32; bits past the end are 0.
 *   - Chunks: contiguous runs of C elements of the flat d-vector, the last one possibly shorter;
 *     each chunk has its own fp32 scale = sqrt(sum of squares / chunk length).
 */
#ifndef ONEBIT_ADAM_H
#define ONEBIT_ADAM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct onebit_adam_s* onebit_adam_t; /* opaque, host-owned handle */

typedef enum {
    ONEBIT_OK = 0,
    ONEBIT_ERR_ARG = -1,     /* bad size, null pointer, unknown enum value */
    ONEBIT_ERR_ALIGN = -2,   /* C not a multiple of 32, pointer not 16-byte aligned */
    ONEBIT_ERR_PHASE = -3,   /* warm-up after the freeze, compressed step before it, unbound */
    ONEBIT_ERR_CUDA = -4,    /* a CUDA call failed */
    ONEBIT_ERR_SPACE = -5    /* workspace smaller than onebit_adam_workspace_bytes */
} onebit_status;

typedef enum { ONEBIT_F32 = 0, ONEBIT_BF16 = 1 } onebit_dtype;

/* State selectors for onebit_adam_get_state / onebit_adam_set_state. */
typedef enum {
    ONEBIT_STATE_M = 0,     /* momentum m, fp32[d]                                   (get/set) */
    ONEBIT_STATE_V = 1,     /* variance v (frozen after the freeze), fp32[d]         (get/set) */
    ONEBIT_STATE_EW = 2,    /* worker residuals e_w, fp32[W][d]                      (get/set) */
    ONEBIT_STATE_ES = 3,    /* server residual e_s, fp32[d]                          (get/set) */
    ONEBIT_STATE_SW = 4,    /* last step's worker scales s, fp32[W][nch]             (get) */
    ONEBIT_STATE_SS = 5,    /* last step's server scales S, fp32[nch]                (get) */
    ONEBIT_STATE_BITSW = 6, /* last step's worker sign planes, uint32[W][ceil(d/32)] (get;
                               rebuilt from the stored x_w: on one GPU the workers' signs are
                               kept grouped by 8 workers, one byte per element) */
    ONEBIT_STATE_BITSS = 7  /* last step's server sign plane, uint32[ceil(d/32)]     (get) */
} onebit_state;

/* Device status flags (onebit_adam_status). */
#define ONEBIT_FLAG_NAN_WORKER 1u /* some worker's x_w was NaN (its bit is 0) */
#define ONEBIT_FLAG_NAN_SERVER 2u /* some server z was NaN */
#define ONEBIT_FLAG_TIMEOUT 4u    /* a bounded wait gave up: a copy that did not land in the
                                     server kernel, or a data-parallel barrier whose ranks did
                                     not all arrive before the timeout; the step's results are
                                     not valid */

/*
 * Create a handle for d parameters, W workers, chunk length C ("1-bit Adam" index page,
 * Abstract; LIT-278 note, Key takeaways: per-chunk scaling). Host only, no device work.
 *   d >= 0 (d = 0 makes every step a no-op), 1 <= W <= 256, C >= 32 and C % 32 == 0
 *   (ONEBIT_ERR_ALIGN otherwise; C need not divide d), 0 <= beta1, beta2 < 1, eps >= 0, all
 *   finite. *out receives the handle; release it with onebit_adam_destroy.
 */
int onebit_adam_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1,
                     float beta2, float eps);

/* Bytes of device workspace the handle needs for gradients of type grad_dtype. */
int onebit_adam_workspace_bytes(onebit_adam_t h, int32_t grad_dtype, uint64_t* bytes);

/*
 * Give the handle its device workspace (caller-owned, 256-byte aligned, at least
 * onebit_adam_workspace_bytes long) and fix the gradient type. Zeroes m and v on `stream`
 * (Adam's initial state) and puts the handle in the warm-up phase. The workspace holds m, v,
 * the residuals, the sign planes, the scales and the fp64 norm partials.
 */
int onebit_adam_bind(onebit_adam_t h, void* workspace, uint64_t bytes, int32_t grad_dtype,
                     void* stream);

/*
 * One full-precision Adam warm-up step (LIT-278 note, "What the evidence does not cover": the
 * warm-up runs uncompressed Adam). grads: [W][d] of the bound type, device; x: fp32[d], device,
 * updated in place. gbar = fp64 average over workers rounded once; m = b1 m + (1-b1) gbar;
 * v = b2 v + (1-b2) gbar^2; x -= lr * (m / (sqrt(v) + eps)); no bias correction unless
 * onebit_adam_set_bias_correction turned it on. ONEBIT_ERR_PHASE after
 * onebit_adam_freeze_variance.
 */
int onebit_adam_warmup_step(onebit_adam_t h, float* x, const void* grads, float lr,
                            void* stream);

/*
 * Optional bias-corrected warm-up (off by default: the pages' step x - lr * m / (sqrt(v) + eps)
 * has no bias correction, and neither page mentions one). With on = 1, warm-up step t uses
 * Adam's corrected moments m / c1_t and v / c2_t in its step (m and v are stored uncorrected),
 * c_t = fl32(1 - beta^t) with beta^t the fp64 product of t factors beta (the fp32 value) in
 * order; onebit_adam_freeze_variance then continues from the corrected moments, m / c1_T and
 * v / c2_T, so that the first compressed step does not jump in size. Allowed before the first
 * warm-up step only (ONEBIT_ERR_PHASE afterwards); ONEBIT_ERR_ARG for on not in {0, 1} or a
 * data-parallel rank's handle. Host only.
 */
int onebit_adam_set_bias_correction(onebit_adam_t h, int32_t on);

/*
 * End the warm-up: v becomes the fixed preconditioner ("1-bit Adam" index page, Abstract;
 * LIT-278 note, tag list: freeze the variance before compressing). Worker and server residuals
 * and all scales start at zero. Allowed once; ONEBIT_ERR_PHASE afterwards.
 */
int onebit_adam_freeze_variance(onebit_adam_t h, void* stream);

/*
 * One compressed step (LIT-278 note, Key takeaways: 1-bit compressed momentum SGD with error
 * feedback, per-chunk scaling, frozen-variance preconditioner). grads: [W][d], device; x:
 * fp32[d], device, updated in place. For each worker w and element i:
 *   x_w = (b1 m + (1-b1) g_w) + e_w;  s_w,k = ||x_w[chunk k]||_2 / sqrt(C_k);
 *   e_w = x_w - (x_w >= 0 ? s_w,k : -s_w,k)
 * then the compressed allreduce over the W packed planes, per element of chunk k:
 *   z = fl32(fp64 sum_w (+-s_w,k) / W) + e_s;  S_k = ||z[chunk k]||_2 / sqrt(C_k);
 *   e_s = z - (z >= 0 ? S_k : -S_k)
 * and every worker's apply: m = (z >= 0 ? S_k : -S_k); x -= lr * (m / (sqrt(v) + eps)).
 * ONEBIT_ERR_PHASE before onebit_adam_freeze_variance.
 */
int onebit_adam_compressed_step(onebit_adam_t h, float* x, const void* grads, float lr,
                                void* stream);

/*
 * The same compressed step fed from host memory: copies grads_host ([W][d] of the bound type,
 * pinned host memory for an asynchronous copy) into grads_dev, runs the step on x_dev, and
 * copies the updated x_dev back into x_host (fp32[d]). The upload and the step are queued on
 * `stream`; the read-back of x runs on a stream of the handle (created on the first call), so
 * that it overlaps the next call's upload, and the next call's step waits for it. x_host holds
 * this step's result once onebit_adam_host_wait(h, s) has been called and `s` has finished (or
 * the device is synchronized); grads_host may be reused once `stream` has finished.
 */
int onebit_adam_compressed_step_host(onebit_adam_t h, float* x_dev, void* grads_dev,
                                     const void* grads_host, float* x_host, float lr,
                                     void* stream);

/* Make `stream` wait for the last host-buffer step's read-back of x (no-op if there is none). */
int onebit_adam_host_wait(onebit_adam_t h, void* stream);

/*
 * Copy one piece of state into dst (device memory, contiguous, the size listed in
 * onebit_state; onebit_adam_state_bytes gives it). Residuals come back explicit.
 */
int onebit_adam_get_state(onebit_adam_t h, int32_t which, void* dst, void* stream);

/*
 * Copy the part of one piece of state that belongs to chunk k (0 <= k < number of chunks) into
 * dst (device memory, contiguous): M, V, ES: fp32[C_k]; EW: fp32[W][C_k]; SW: fp32[W];
 * SS: fp32[1]; BITSW: uint32[W][ceil(C_k/32)]; BITSS: uint32[ceil(C_k/32)]. Chunks are
 * independent, so a sample of chunks checks every output that depends on them without
 * copying whole W x d buffers. Residuals come back explicit.
 */
int onebit_adam_get_chunk_state(onebit_adam_t h, int32_t which, int64_t k, void* dst,
                                void* stream);

/*
 * Overwrite one piece of state (M, V, EW or ES) from src (device memory, contiguous). Used to
 * resume from a checkpoint: a fresh handle that is bound, frozen and given M, V, EW and ES of
 * another handle continues bit-identically. Setting EW or ES clears the reported scales of the
 * last step. ONEBIT_ERR_ARG for the read-only selectors.
 */
int onebit_adam_set_state(onebit_adam_t h, int32_t which, const void* src, void* stream);

/* Size in bytes of one piece of state. */
int onebit_adam_state_bytes(onebit_adam_t h, int32_t which, uint64_t* bytes);

/*
 * Wait for `stream`, then return the device status flags (ONEBIT_FLAG_*) gathered since the
 * last call in *flags and clear them.
 */
int onebit_adam_status(onebit_adam_t h, void* stream, uint32_t* flags);

/*
 * Shape and progress: out[0..7] = d, W, C, number of chunks, phase (0 unbound, 1 warm-up,
 * 2 compressed), compressed steps taken, gradient dtype (-1 unbound), kernel launches per
 * compressed step (5; 3 or 4 for small buckets, whose chunk-scale reductions fold into the
 * server and apply kernels; 7 for a data-parallel rank).
 */
int onebit_adam_info(onebit_adam_t h, int64_t out[8]);

/*
 * Per-kernel timing with CUDA events recorded on the launching stream. max_steps > 0 starts
 * recording the next max_steps compressed steps (later steps are not recorded); 0 stops and
 * frees the events. onebit_adam_timing_read waits for the last recorded event and returns, in
 * ms_out[0..4], the summed device time of the worker kernel, the worker-scale reduction, the
 * server kernel, the server-scale reduction and the apply kernel (a reduction folded into the
 * next kernel reads 0), and the number of recorded steps in *steps; it then starts a new
 * recording window of the same length.
 */
int onebit_adam_timing(onebit_adam_t h, int32_t max_steps);
int onebit_adam_timing_read(onebit_adam_t h, double ms_out[5], int32_t* steps);

/*
 * The device time of each step of the current recording window, from its first event to its
 * last (step_ms[s] for the first min(cap, steps) steps, in order), and the number of recorded
 * steps in *steps. Waits for the last recorded event; does not end the window (call it before
 * onebit_adam_timing_read). ONEBIT_ERR_ARG for cap < 0, a NULL steps, or a NULL step_ms with
 * cap > 0.
 */
int onebit_adam_timing_steps(onebit_adam_t h, double* step_ms, int32_t cap, int32_t* steps);

/* Release the handle (not the workspace, which the caller owns). NULL is ignored. */
void onebit_adam_destroy(onebit_adam_t h);

/*
 * Sign-pack n fp32 values (device) into ceil(n/32) LSB-first words (device): bit = x >= 0;
 * padding bits are 0. The 1-bit message of the method without its scale. n >= 0.
 */
int onebit_pack(const float* x, int64_t n, uint32_t* words, void* stream);

/*
 * Decompress: out[i] = bit_i ? scales[i / C] : -scales[i / C] for i < n (all device). C >= 1.
 */
int onebit_unpack(const uint32_t* words, const float* scales, int64_t n, int64_t C, float* out,
                  void* stream);

/*
 * Compress one fp32 vector x[n] (device) into its 1-bit message: LSB-first sign words
 * words[ceil(n/32)] (bit = x >= 0) and one scale per chunk of C elements,
 * scales[ceil(n/C)] = sqrt(sum of squares / chunk length) -- the worker compression of the
 * compressed step applied to x itself. The paper has no counterpart of this entry point: it is
 * the library's variant of that kernel for callers that must not allocate device memory, for
 * example code running inside a host application or plugin that hands it only its input and
 * output buffers and owns the whole device memory pool, or latency-critical paths where the
 * implicit synchronisation of cudaMalloc/cudaFree is not acceptable. It allocates nothing: its
 * scratch (the fp64 norm partials) is a fixed 512 KiB array inside the library, which every GPU
 * that loads the library keeps until the process exits.
 *   Limit: ceil(n/C) * ceil(min(C, n)/2048) <= 65536 (for example n <= 134,217,728 when C is a
 *   multiple of 2048); larger inputs return ONEBIT_ERR_SPACE with the reason in
 *   onebit_last_error(), before any device work.
 *   C >= 32, C % 32 == 0 (ONEBIT_ERR_ALIGN otherwise); x 16-byte aligned; n = 0 is a no-op.
 *   The first call on each device looks up the array's device address (with that device
 *   current) and caches it by device ordinal for the life of the process; make that first
 *   call before any stream capture. A device reset (cudaDeviceReset, or a reset of the primary
 *   context) invalidates the cached address: do not call this entry point after one.
 *   All calls share the one array and it keeps the last call's contents; each call writes every
 *   slot it reads before reading it. Calls whose work overlaps on the GPU (for example on two
 *   streams at once) race on the array and must be ordered by the caller.
 */
int onebit_compress_static(const float* x, int64_t n, int64_t C, uint32_t* words, float* scales,
                           void* stream);

/*
 * Self-test of failure detection without a GPU fault: one block arms an mbarrier for bytes
 * that never arrive and waits on it with the same bounded wait the server kernel uses, giving
 * up after `polls` polls (1 <= polls <= 2^22). Writes 1 to *timed_out (device, 4-byte aligned)
 * when the wait gave up -- the expected outcome -- and 0 if it did not. The kernel returns
 * normally and the context stays usable. No counterpart in the paper; this is library
 * plumbing for the bounded waits.
 */
int onebit_selftest_bounded_wait(int32_t polls, uint32_t* timed_out, void* stream);

/*
 * ------------------------------------------------------------------------------------------
 * Data-parallel ranks: the compressed allreduce across GPUs.
 *
 * The pages' compressed allreduce is a collective between machines ("1-bit Adam" index page,
 * Abstract: communication over TCP is the bottleneck; LIT-278 note, "What the evidence does not
 * cover": a custom collective). Here it runs between R GPUs of one NVLink/NVSwitch domain, one
 * process (or, for emulation, one handle) per rank. Rank q holds W / R of the W workers
 * (global workers q*W/R .. (q+1)*W/R - 1) and serves the chunks
 * [q * nch / R, (q+1) * nch / R) (onebit_dp_chunk_range). A compressed step is:
 *   phase 0  worker compression of the rank's workers; each plane word and scale is stored
 *            directly into the receive buffers of the rank that serves its chunk; signal.
 *   phase 1  wait for every rank; server average, residual and recompression of the rank's
 *            chunks; each server plane word and scale is stored into every rank's copy; signal.
 *   phase 2  wait for every rank; apply x -= lr * (m / (sqrt(v) + eps)) on all d elements.
 * The warm-up likewise: phase 0 fp64 sums of the rank's gradients; phase 1 the rank's chunks
 * read every rank's sums in rank order and write the Adam moments into every rank's m and v;
 * phase 2 the x update. The results equal those of one single-GPU handle with all W workers
 * (bit for bit in the compressed phase; in the warm-up whenever the fp64 sums of the gradients
 * are exact, which their grouping by rank can otherwise change in the last bit).
 *
 * A rank's handle is used like a single-GPU one (workspace, bind, warm-up steps, freeze,
 * compressed steps, state), with these additions and differences:
 *   - onebit_dp_init instead of onebit_adam_init; W counts the workers of all ranks.
 *   - onebit_adam_bind also allocates the exchange region (cudaMalloc; freed by
 *     onebit_adam_destroy) and clears it. Every rank must then set its peers (onebit_dp_open_peer
 *     from the peers' onebit_dp_ipc_handle, or onebit_dp_set_peer with addresses valid in this
 *     process) and call onebit_dp_connect; all ranks must have finished connecting (and their
 *     streams that work) before any rank takes a step -- a host barrier between connect and the
 *     first step. Likewise before destroying a handle: every rank's work must have finished
 *     first, and once any rank's handle is destroyed (its exchange region freed) the others
 *     must take no further step or phase.
 *   - Steps and freezes must be taken by all ranks in the same order. Each step contains two
 *     barriers between the ranks (device-side flags, see ONEBIT_FLAG_TIMEOUT): a rank that never
 *     arrives makes the others' waits give up after the timeout (onebit_dp_set_timeout, default
 *     10 s), with ONEBIT_FLAG_TIMEOUT set in their status.
 *   - State: ES is the server residual of the rank's own chunks (fp32[elements of those
 *     chunks]); get_chunk_state(ES, k) needs a chunk k of the rank. EW, SW and BITSW cover the
 *     rank's own workers (BITSW is rebuilt from the stored x_w, so after set_state(EW) it
 *     reflects the residuals that were set). M, V, SS and BITSS cover all d elements and are the
 *     same on every rank; set_state(M) and set_state(V) must be given the same values on every
 *     rank, and set_state(ES) must be called by every rank (each with its own chunks).
 *   - onebit_adam_info reports the rank's own worker count; kernel launches per compressed step
 *     are 7 (two barrier launches).
 * No rank's kernel ever waits on another rank's kernel unboundedly; a step that lost a rank
 * still ends, with ONEBIT_FLAG_TIMEOUT set. The barriers count in device memory, so a step (or
 * a sequence of phases) can be captured in a CUDA graph and replayed like the single-GPU step.
 */

#define ONEBIT_MAX_RANKS 8
#define ONEBIT_IPC_HANDLE_BYTES 64

/*
 * The server kernel's layout for (d, W, C), as a handle of that shape would use it. Host only.
 * out[0] = 1 when its lookup tables are bank-private, out[1] = segments per block, out[2] =
 * dynamic shared memory per block (bytes) on one GPU, out[3] = the same for a data-parallel
 * rank's server, out[4] = server blocks per step on one GPU. The arguments and errors are those
 * of onebit_adam_init.
 */
int onebit_server_layout(int64_t d, int32_t W, int64_t C, int64_t out[5]);

/*
 * Rank q's chunks [*k0, *k1) of nch chunks over R ranks (1 <= R <= 8): contiguous, in rank
 * order, sizes differing by at most one. Host only. ONEBIT_ERR_ARG for nch < 0, R or q out of
 * range, or a NULL output.
 */
int onebit_dp_chunk_range(int64_t nch, int32_t R, int32_t q, int64_t* k0, int64_t* k1);

/*
 * Create the handle of rank `rank` of R (1 <= R <= 8) for d parameters, W workers over all
 * ranks (W % R == 0, W <= 256) and chunk length C; the other arguments and checks are those of
 * onebit_adam_init. Host only. ONEBIT_ERR_ARG for R, rank or W out of range or W % R != 0
 * (*out is then NULL).
 */
int onebit_dp_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1,
                   float beta2, float eps, int32_t R, int32_t rank);

/*
 * out[0..7] = R, rank, W over all ranks, first and end chunk of the rank's chunks, their first
 * element, their element count, exchange region bytes. ONEBIT_ERR_ARG for a single-GPU handle.
 */
int onebit_dp_info(onebit_adam_t h, int64_t out[8]);

/*
 * Base address (device) and size of this rank's exchange region, which the handle owns.
 * ONEBIT_ERR_PHASE before onebit_adam_bind.
 */
int onebit_dp_exchange(onebit_adam_t h, void** base, uint64_t* bytes);

/*
 * CUDA IPC handle (ONEBIT_IPC_HANDLE_BYTES bytes into out, host memory) of the exchange region,
 * for the other ranks' onebit_dp_open_peer. ONEBIT_ERR_PHASE before onebit_adam_bind,
 * ONEBIT_ERR_CUDA if the runtime refuses.
 */
int onebit_dp_ipc_handle(onebit_adam_t h, void* out);

/*
 * Map rank q's exchange region from its IPC handle (a different process on a peer GPU of the
 * same node; peer access is enabled on demand; call with this rank's device current). The
 * handle owns the mapping and releases it in onebit_adam_destroy or when the peer is set
 * again. ONEBIT_ERR_ARG for q out of range or q == rank, ONEBIT_ERR_CUDA if the mapping fails.
 * Invalidates the route until the next onebit_dp_connect.
 */
int onebit_dp_open_peer(onebit_adam_t h, int32_t q, const void* handle);

/*
 * Use `base` (device, 256-byte aligned, valid in this process: another handle's exchange
 * region when several ranks are emulated in one process) as rank q's exchange region; the
 * caller keeps it alive. ONEBIT_ERR_ARG for q out of range, q == rank or NULL,
 * ONEBIT_ERR_ALIGN for a misaligned base. Invalidates the route until onebit_dp_connect.
 */
int onebit_dp_set_peer(onebit_adam_t h, int32_t q, void* base);

/*
 * Build the rank's route (every rank's buffer addresses) from its peers and copy it to the
 * device on `stream`. ONEBIT_ERR_PHASE before onebit_adam_bind or while a peer is not set.
 */
int onebit_dp_connect(onebit_adam_t h, void* stream);

/*
 * Barrier timeout in microseconds (1 .. 3.6e9; ONEBIT_ERR_ARG otherwise). Default 10 s. A wait
 * also ends after 2^28 polls (each followed by a nanosleep of about 256 ns), whichever comes
 * first.
 */
int onebit_dp_set_timeout(onebit_adam_t h, uint64_t timeout_us);

/*
 * One phase (0, 1, 2 in order; see above) of a warm-up or compressed step of this rank, for
 * driving several emulated ranks from one thread: run phase p of every rank before phase p+1
 * of any. Phase 0 reads grads ([W/R][d], device), phase 2 updates x (fp32[d], device); the
 * other pointers may be NULL. ONEBIT_ERR_PHASE for a phase out of order, an unconnected rank,
 * or the wrong phase of the method (warm-up after the freeze, compressed before it);
 * ONEBIT_ERR_ARG for phase > 2, a single-GPU handle, a non-finite lr or a NULL pointer that the
 * phase reads; ONEBIT_ERR_ALIGN for a pointer that is not 16-byte aligned. While a step is
 * driven phase by phase, the freeze and the whole-step entry points return ONEBIT_ERR_PHASE.
 * The whole-step entry points (onebit_adam_warmup_step, onebit_adam_compressed_step) run the
 * three phases with one barrier launch between them and are what separate processes use.
 */
int onebit_dp_warmup_phase(onebit_adam_t h, int32_t phase, float* x, const void* grads,
                           float lr, void* stream);
int onebit_dp_compressed_phase(onebit_adam_t h, int32_t phase, float* x, const void* grads,
                               float lr, void* stream);

/*
 * ------------------------------------------------------------------------------------------
 * The 0/1 Adam variant (codewithpapers.app "0/1 Adam" page, abstract: each Adam step is
 * linearised by approximating the optimizer states with their stale estimates and their linear
 * correlation, which lets 1-bit compression and local steps be used together).
 *
 * The page gives no formulas; the library follows these readings (the oracle's Z1-Z7):
 *   - the warm-up (onebit_adam_warmup_step) and the freeze (onebit_adam_freeze_variance) are
 *     1-bit Adam's;
 *   - every step, each worker w takes a local step on its own momentum and accumulated update:
 *         m_w = beta1*m_w + (1-beta1)*g_w ;  u_w = u_w + lr*m_w
 *   - every H-th step ends with a synchronisation: 1-bit Adam's compressed allreduce of
 *     u_w + e_w (per-chunk scale, signs, worker and server error feedback) gives ubar; then
 *         x = x - ubar / (sqrt(v) + eps) ;  mbar = ubar / Gamma
 *     with Gamma the fp32 sum of the interval's learning rates (the momentum estimate: u is
 *     linear in the momenta); every worker restarts from m_w = mbar, u_w = 0;
 *   - at every K-th synchronisation (K = 0: never) the stale variance is refreshed after the
 *     step: v = beta2*v + (1-beta2)*mbar^2;
 *   - worker w's local model between synchronisations is x - u_w / (sqrt(v) + eps).
 * With H = 1, K = 0 and a power-of-two lr the variant gives 1-bit Adam's parameters bit for bit.
 * A 0/1 handle is a single-GPU handle: the data-parallel entry points do not apply to it, and
 * onebit_adam_compressed_step(_host) returns ONEBIT_ERR_PHASE on it.
 */

/*
 * Create a 0/1 Adam handle: the arguments and checks of onebit_adam_init, plus the
 * synchronisation interval H (1 <= H <= 2^20) and the variance refresh period K in
 * synchronisations (0 <= K <= 2^20; 0 = never). Its workspace (onebit_adam_workspace_bytes)
 * also holds every worker's momentum and accumulated update, fp32[W][d] each. Host only;
 * ONEBIT_ERR_ARG for H or K out of range (*out is then NULL).
 */
int onebit01_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1,
                  float beta2, float eps, int32_t H, int32_t K);

/*
 * One step of the variant's compression phase on `stream`: the local step of every worker
 * (one launch), and on every H-th step the synchronisation as well (four more launches: the
 * worker scales, 1-bit Adam's server stage, the server scales, the synchronised step), which
 * updates x (fp32[d], device, in/out). grads is [W][d] (device), fp32 or bf16 as bound.
 * ONEBIT_ERR_PHASE before the freeze or on a 1-bit Adam handle; ONEBIT_ERR_ARG for a NULL
 * pointer, a non-finite lr, or a synchronisation whose Gamma is 0 or not finite;
 * ONEBIT_ERR_ALIGN for pointers that are not 16-byte aligned. The sign planes, scales and
 * residuals of the last synchronisation are read with onebit_adam_get_state /
 * onebit_adam_get_chunk_state (not ONEBIT_STATE_M, which a 0/1 handle does not hold).
 */
int onebit01_step(onebit_adam_t h, float* x, const void* grads, float lr, void* stream);

/*
 * out[0..5] = H, K, steps since the last synchronisation, synchronisations so far, where the
 * next step's momentum comes from (0: the warm-up momentum, 1: the last synchronisation's
 * mbar, 2: each worker's own, 3: each worker's own, with the accumulated update of the
 * interval's first step rebuilt from it rather than stored), launches of the next step (5 when
 * it synchronises, else 1).
 * Host only; ONEBIT_ERR_ARG for a 1-bit Adam handle.
 */
int onebit01_info(onebit_adam_t h, int64_t out[6]);

/*
 * Every worker's momentum (which = 0) or accumulated update (which = 1) into dst (device):
 * fp32[W][d] for k = -1, fp32[W][C_k] for chunk k. Queued on `stream`. ONEBIT_ERR_ARG for a
 * 1-bit Adam handle, which not in {0, 1}, k out of range or a NULL dst; ONEBIT_ERR_PHASE
 * before the freeze.
 */
int onebit01_get_worker_state(onebit_adam_t h, int32_t which, int64_t k, void* dst,
                              void* stream);

/*
 * Worker w's local model x - u_w / (sqrt(v) + eps) into out (fp32[d], device), with x the
 * synchronised parameters (fp32[d], device). ONEBIT_ERR_ARG for a 1-bit Adam handle, w out of
 * range or a NULL pointer; ONEBIT_ERR_PHASE before the freeze.
 */
int onebit01_local_model(onebit_adam_t h, int32_t w, const float* x, float* out, void* stream);

/*
 * Checkpoint/resume of a 0/1 handle. onebit01_set_worker_state writes every worker's momentum
 * (which = 0) or accumulated update (which = 1) from src (device, fp32[W][d]) and makes the next
 * step start from them, whatever form the state had (the warm-up momentum, the last
 * synchronisation's estimate, or an update not stored): set both. onebit01_get_schedule /
 * onebit01_set_schedule read and write the schedule: ints = {steps since the last
 * synchronisation (0 <= t < H), synchronisations so far}, floats = {Gamma of the steps since the
 * last synchronisation, Gamma of the last synchronisation}. With onebit_adam_get_state /
 * onebit_adam_set_state of v, the worker residuals and the server residual (ONEBIT_STATE_V, _EW,
 * _ES; a 0/1 handle keeps its server plane and scales on _ES), a handle restored after its freeze
 * continues bit for bit like the one saved. ONEBIT_ERR_ARG for a 1-bit Adam handle, which not in
 * {0, 1}, a NULL pointer or a schedule out of range; ONEBIT_ERR_PHASE before the freeze (and, for
 * a data-parallel rank, in the middle of a phase sequence).
 */
int onebit01_set_worker_state(onebit_adam_t h, int32_t which, const void* src, void* stream);
int onebit01_get_schedule(onebit_adam_t h, int64_t ints[2], float floats[2]);
int onebit01_set_schedule(onebit_adam_t h, const int64_t ints[2], const float floats[2]);

/*
 * A data-parallel rank of the 0/1 Adam variant: rank `rank` of R, holding W / R of the W workers
 * (W % R == 0), with onebit_dp_init's chunk ownership, workspace binding, peer connection and
 * barriers, and onebit01_init's schedule (H, K). The warm-up runs as a 1-bit Adam rank's
 * (onebit_dp_warmup_phase or onebit_adam_warmup_step), then onebit_adam_freeze_variance. After
 * the freeze a local step exchanges nothing; a synchronising step sends the sign words of this
 * rank's workers' u_w + e_w to the serving ranks and their scales, runs the server stage of the
 * chunks this rank serves and broadcasts the server words and scales to every rank, as 1-bit
 * Adam's data-parallel step does, then takes the synchronised step on this rank's copy of x.
 * The per-worker state of this rank's workers is read with onebit01_get_worker_state and
 * onebit01_local_model (rows are this rank's workers). The arguments and errors are those of
 * onebit_dp_init and onebit01_init.
 */
int onebit01_dp_init(onebit_adam_t* out, int64_t d, int32_t W, int64_t C, float beta1,
                     float beta2, float eps, int32_t H, int32_t K, int32_t R, int32_t rank);

/*
 * One phase (0, 1, 2 in order) of a 0/1 step of a data-parallel rank, for driving emulated ranks
 * from one thread (phase p of every rank before phase p+1 of any); the whole-step entry point
 * onebit01_step runs the three phases and is what separate processes use. Phase 0: every worker's
 * step, and in a synchronising step the compression and the sends; phase 1: the server stage;
 * phase 2: the synchronised step (x, fp32[d], device). Barriers surround only the exchange of a
 * synchronising step. Phase 0 reads grads ([W/R][d], device). ONEBIT_ERR_PHASE for a phase out
 * of order, an unconnected rank, a 1-bit Adam rank, or before the freeze; ONEBIT_ERR_ARG for
 * phase > 2, a single-GPU handle, a non-finite lr, a synchronisation whose Gamma is 0 or not
 * finite, or a NULL pointer that the phase reads; ONEBIT_ERR_ALIGN for a pointer that is not
 * 16-byte aligned. onebit_dp_compressed_phase returns ONEBIT_ERR_PHASE for a 0/1 rank.
 */
int onebit01_dp_phase(onebit_adam_t h, int32_t phase, float* x, const void* grads, float lr,
                      void* stream);

/* Static description of a status code. */
const char* onebit_strerror(int32_t code);

/* Text of the last CUDA error this thread saw in the library ("" if none). */
const char* onebit_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ONEBIT_ADAM_H */
