/*
 * cf.h -- C ABI of the B200 residual-compression activation codec (libcf).
 *
 * What the codec computes (page titles and sections):
 *  - "Accelerating Parallel Diffusion Model Serving with Residual Compression"
 *    (arXiv 2507.17511), abstract: between parallel devices, send only the
 *    compressed step-wise residual of each activation, and carry the
 *    compression error forward (error feedback) so that it does not
 *    accumulate across denoising steps.
 *  - Same paper, reproducibility table, "Dataset Splits" row (Appendix D,
 *    Figure 8): at least one uncompressed warmup step initialises the base
 *    tensor that later residuals are taken against.
 *  - Same paper, reproducibility table, "Pseudocode" row, Algorithm 3
 *    (Subspace Iteration, rank r): the low-rank compressor.
 *  - xDiT issue 573 ("Proposal: Integrating a compression-based acceleration
 *    method into xDiT"): residuals plus error feedback, 8-16x less traffic.
 *
 * Per communicated tensor ("slot": one layer's activation shard, or its K or
 * its V) and per denoising step t:
 *   sender    A   = (X_t - base) + E          residual plus carried error
 *             payload = Q(A)                   k-bit group codes + fp32 scales,
 *                                              or rank-r factors (U, R, V)
 *             E   = A - deq(payload)           new carried error
 *             base = X_t
 *   receiver  C   = C + deq(payload)           reconstruction cache
 * Step 0 is the uncompressed warmup: base = X_0, E = 0 and C = X_0.  Then
 * C_t + E_t = X_t holds at every step, up to fp32 rounding.
 *
 * Quantiser (the pages give no formula; these are the readings this library
 * takes): groups of G contiguous channels of one token row;
 *   k = 2, 4: s = max|A| over the group, L = 2^(k-1)-1, inv = L/s,
 *             code = clamp(rne(A*inv), -L, L) + L, deq = ((code-L)/L)*s;
 *   k = 1   : code = (A >= 0), deq = code ? s : -s, with
 *             s = (binary-tree sum of |A|)/G (sign_scale 0, the default) or
 *             s = max|A| (sign_scale 1).
 * A group whose scale is below 2^-120, or not finite, is sent as an all-zero
 * group (scale 0, every code the zero level); a non-finite scale also raises
 * CF_E_NONFINITE at the next cf_check.  Every floating-point step is one
 * IEEE-754 binary32 operation with round-to-nearest-even and no fused
 * multiply-add, so results are bit-reproducible.
 *
 * Layouts (all row-major, token rows of `cols` channels, flat index
 * i = row*cols + col):
 *   x, base  bf16 [rows*cols]          err, cache  fp32 [rows*cols]
 *   codes    u8 [rows*cols*k/8]: one LSB-first bit stream; the code of
 *            element i occupies bits [i*k, i*k+k).  Group g = i/G starts at
 *            byte g*G*k/8.
 *   scales   fp32 [rows*cols/G], scales[g] for group g.
 *   low-rank payload: U fp32 [rows x r], R fp32 [r x r] (upper triangular),
 *            V fp32 [cols x r]; the reconstruction is U R V^T.
 *
 * Ownership: the library owns only the context, its device status word and
 * host-side bookkeeping.  Activations, state (base, err, cache), payloads and
 * the workspace are caller memory (device pointers).  The library performs
 * no transmission between devices.
 *
 * Concurrency and errors: every call except cf_create, cf_destroy, cf_check
 * and cf_trace_read is stream-ordered and asynchronous.  Argument, shape, alignment
 * and state errors return before anything is launched and leave all buffers
 * untouched.  Device-side conditions (non-finite scale, a bounded wait that
 * gave up) set bits in the context's status word and are reported by the
 * next cf_check.  The stream-ordered calls allocate no device memory and
 * do not synchronise, so they can be captured into a CUDA graph and replayed
 * (the kernels read the slot pointers given at capture; a quantised step
 * >= 1 is the same launch for every later step).  A context belongs to the
 * device that was current at cf_create; each call makes that device current
 * for its duration and restores the caller's.  A context is not
 * thread-safe; separate contexts are independent.  There is no CPU fallback:
 * without a usable sm_100 device cf_create returns CF_E_CUDA.
 */
#ifndef CF_H
#define CF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct cf_ctx cf_ctx;

typedef enum cf_status {
    CF_OK = 0,
    CF_E_ARG = 1,        /* bad argument value (null pointer, unsupported k/G/r, ...) */
    CF_E_SHAPE = 2,      /* shape not allowed (cols % G, cols % 8, rows < r, ...) */
    CF_E_ALIGN = 3,      /* pointer not 16-byte aligned */
    CF_E_STATE = 4,      /* step > 0 before the warmup step on this context */
    CF_E_NOMEM = 5,      /* host or device allocation failed, or workspace too small */
    CF_E_CUDA = 6,       /* CUDA runtime error (launch, no device, wrong arch) */
    CF_E_NONFINITE = 7,  /* a group scale or a Gram matrix was not finite / not SPD */
    CF_E_TIMEOUT = 8     /* a bounded device-side wait gave up */
} cf_status;

enum { CF_MODE_QUANT = 0, CF_MODE_LOWRANK = 1 };

/* Arithmetic of the low-rank products with A (A Q and A^T P). */
enum {
    CF_PRECISION_AUTO = 0,   /* split products where r > min(m, n) / 8, TF32 elsewhere */
    CF_PRECISION_TF32 = 1,   /* operands rounded to TF32 (nearest): relative error about 2^-12 per product */
    CF_PRECISION_SPLIT = 2   /* "3xTF32": each operand as a TF32 hi + lo pair, three MMAs per step; close to
                                fp32 accuracy, for iterations that follow every rounding (few iterations with a
                                rank that is a large fraction of the matrix), at about twice the shared-memory
                                traffic of the TF32 form */
};

typedef struct cf_config {
    int mode;        /* CF_MODE_QUANT or CF_MODE_LOWRANK */
    int bits;        /* quant: k = 1, 2 or 4 */
    int group;       /* quant: G = 8, 16, 32, 64, 128 or 256; must divide cols */
    int sign_scale;  /* k = 1: 0 = mean |A| scale (default), 1 = absmax scale */
    int rank;        /* low-rank: r, 1..32 */
    int iters;       /* low-rank: T >= 0 subspace iterations */
    int state_bf16;  /* quant: 0 = E and C in fp32 (default); 1 = lean state, E and C in bf16
                        (each new E and C rounded to nearest even when stored; 14.3 instead of
                        22.6 bytes per element for compress + decompress at k = 2, G = 128) */
    int warm_start;  /* low-rank cf_compress: 0 = start Algorithm 3 from the slot's q0 every step
                        (default); 1 = from the second compressed step on, start from the slot's V
                        of the previous step (q0 may then be NULL), so that a small `iters`
                        (e.g. 1) tracks a slowly moving subspace with fewer passes over A */
    int precision;   /* low-rank: CF_PRECISION_AUTO (default), _TF32 or _SPLIT */
} cf_config;

typedef struct cf_shape {
    int64_t rows;    /* tokens of this slot's shard (>= 0) */
    int64_t cols;    /* channels (> 0, multiple of 8) */
} cf_shape;

/* Per-slot device pointers for one call; all 16-byte aligned, all caller
 * owned.  Fields a call does not use may be NULL (see each call), and so may
 * every field of a slot with rows == 0. */
typedef struct cf_slot {
    const void *x;   /* bf16 [rows*cols]  activation X_t (read only) */
    void *base;      /* bf16 [rows*cols]  sender's base tensor X_{t-1} */
    void *err;       /* fp32 [rows*cols]  sender's error-feedback buffer E (bf16 with state_bf16) */
    void *cache;     /* fp32 [rows*cols]  receiver's reconstruction C (bf16 with state_bf16) */
    uint8_t *codes;  /* quant payload codes, rows*cols*k/8 bytes */
    float *scales;   /* quant payload scales, rows*cols/G */
    const float *q0; /* low-rank: Gaussian start block [cols x r] for this call */
    float *U;        /* low-rank payload [rows x r] */
    float *R;        /* low-rank payload [r x r] */
    float *V;        /* low-rank payload [cols x r] */
    void *recon;     /* bf16 [rows*cols] or NULL: receiver output, bf16(cache) after the call
                        (see cf_decompress) */
} cf_slot;

/* Create a context for `nslots` slots of the given shapes (host array).
 * Validates the configuration and the shapes, checks that the current CUDA
 * device has compute capability 10.0 (the only target of sm_100a code), and
 * allocates the device status word on it.
 * nslots may be 0 for a context used only with cf_lowrank.
 * Errors: CF_E_ARG, CF_E_SHAPE, CF_E_NOMEM (a host or device allocation
 * failed), CF_E_CUDA; *out is NULL then.
 * Source: library plumbing with no counterpart in the paper; the
 * configuration selects the compressor -- the k-bit group quantiser of the
 * residual (abstract) or rank-r subspace iteration (Algorithm 3). */
cf_status cf_create(const cf_config *config, int nslots, const cf_shape *shapes, cf_ctx **out);

/* Device workspace cf_compress needs for this context, in bytes (0 in
 * quantised mode; in low-rank mode the fp32 residuals of every slot plus the
 * small per-slot buffers of Algorithm 3).
 * Source: library plumbing; the buffers are those of Algorithm 3
 * (reproducibility table, "Pseudocode" row). */
size_t cf_workspace_bytes(const cf_ctx *ctx);

/* Register caller-owned device workspace (16-byte aligned) used by
 * cf_compress / cf_lowrank until replaced.  Errors: CF_E_ALIGN, CF_E_NOMEM
 * (smaller than cf_workspace_bytes).
 * Source: library plumbing, no counterpart in the paper. */
cf_status cf_set_workspace(cf_ctx *ctx, void *dev_ptr, size_t bytes);

/* Sender side of step `step` for every slot, in one grouped launch.
 *   step 0: warmup -- base = x, err = 0.  Uses x, base, err.
 *   step >= 1, quantised: A = (x - base) + err; codes, scales = Q(A);
 *           err = A - deq; base = x.  Uses x, base, err, codes, scales.
 *   step >= 1, low-rank: A as above into the workspace; Algorithm 3 with
 *           start block q0 (or, with warm_start, the V of the previous
 *           compressed step) gives U, R, V; err = A - U R V^T; base = x.
 *           Uses x, base, err, q0, U, R, V.
 * `slots` is a host array of nslots entries; `cuda_stream` a cudaStream_t
 * (NULL = legacy default stream).  Errors before launch: CF_E_ARG,
 * CF_E_ALIGN, CF_E_STATE (step >= 1 before a warmup), CF_E_NOMEM (workspace
 * missing in low-rank mode); CF_E_CUDA if a launch fails.
 * Source: abstract (send only the compressed step-wise residual, and feed the
 * compression error back into the next step); reproducibility table,
 * "Dataset Splits" row (the uncompressed warmup step sets the base tensor);
 * "Pseudocode" row, Algorithm 3 (the low-rank mode). */
cf_status cf_compress(cf_ctx *ctx, const cf_slot *slots, int step, void *cuda_stream);

/* Receiver side of step `step` for every slot, in one grouped launch.
 *   step 0: warmup -- cache = float(x).  Uses x, cache.
 *   step >= 1, quantised: cache += deq(codes, scales).  Uses codes, scales,
 *           cache.
 *   step >= 1, low-rank: cache += U R V^T.  Uses U, R, V, cache.
 * A slot whose recon is non-NULL also gets recon = bf16(cache) after the
 * update, rounded to nearest even (at step 0 that is x itself), from the same
 * pass: 2 more bytes per element, where a separate cast would read the fp32
 * cache back (4) and write bf16 (2).  It is meant for the consumer of a
 * received K or V, which reads bf16.  The same holds for cf_loopback.
 * Errors as cf_compress (CF_E_STATE: step >= 1 before a receiver warmup;
 * CF_E_ALIGN: recon not 16-byte aligned).
 * Source: abstract (the receiver adds each decompressed residual to the
 * activation it reconstructed at the previous step); reproducibility table,
 * "Dataset Splits" row (the warmup step delivers X_0 uncompressed). */
cf_status cf_decompress(cf_ctx *ctx, const cf_slot *slots, int step, void *cuda_stream);

/* Sender and receiver of step `step` in one pass, for when both sides of a
 * slot live on this device (e.g. the local shard of an all-gather).  The
 * results are bit-identical to cf_compress followed by cf_decompress: the
 * receiver's C += deq reuses the values the sender dequantised, and the
 * payload is still written (for transmission) but not read back.  In
 * quantised mode a step >= 1 is one fused grouped launch moving k/8 + 4/G
 * bytes per element less than the pair; step 0, and every step in low-rank
 * mode, run the two sides one after the other.  Uses x, base, err, cache,
 * codes, scales (and q0, U, R, V in low-rank mode).  Errors as cf_compress
 * (CF_E_STATE: step >= 1 before the warmup).
 * Source: as cf_compress and cf_decompress (abstract; "Dataset Splits" row),
 * with both sides on one device. */
cf_status cf_loopback(cf_ctx *ctx, const cf_slot *slots, int step, void *cuda_stream);

/* Workspace cf_lowrank needs for nmat matrices of m x n at this context's
 * rank: the r-column blocks of Algorithm 3 (Q^T, P^T, P, Z, padded to 16 or
 * 32 columns), the fp64 Gram matrices of their 256-row chunks and R^{-1},
 * about 4*rp*(2m + 2n) + 4*r*(r+1)*ceil(max(m, n)/256) + 8 KB bytes per
 * matrix.  Returns 0 for a quantised-mode context or bad sizes.
 * Source: library plumbing; the blocks are those of Algorithm 3
 * (reproducibility table, "Pseudocode" row). */
size_t cf_lowrank_workspace_bytes(const cf_ctx *ctx, int nmat, int64_t m, int64_t n);

/* Algorithm 3 (subspace iteration, rank r = config.rank, T = config.iters
 * iterations, CholeskyQR orthogonalisation) on nmat given fp32 matrices.
 * All pointer arguments are HOST arrays of nmat DEVICE pointers:
 *   A[i]  fp32 [m x n] row-major (read only; n % 4 == 0)
 *   Q0[i] fp32 [n x r] Gaussian start block (read only)
 *   U[i]  fp32 [m x r]  R[i] fp32 [r x r]  V[i] fp32 [n x r]  (written)
 *   E_opt NULL or E[i] fp32 [m x n]: E = A - U R V^T       (written)
 *   C_opt NULL or C[i] fp32 [m x n]: C += U R V^T          (updated)
 * Uses the registered workspace (>= cf_lowrank_workspace_bytes).  The two
 * products with A (A Q and A^T P) run on the tensor cores, in TF32 with
 * operands rounded to nearest or split into TF32 hi + lo pairs, as
 * config.precision selects; Gram matrices and Cholesky run in fp64.
 * Errors before launch: CF_E_ARG, CF_E_SHAPE (m < r, n < r, n % 4),
 * CF_E_ALIGN, CF_E_NOMEM; device-side: CF_E_NONFINITE (Gram matrix not
 * positive definite), CF_E_TIMEOUT, at the next cf_check.
 * Source: reproducibility table, "Pseudocode" row, Algorithm 3 (Subspace
 * Iteration, rank r); E and C are the error feedback and the receiver's
 * accumulation of the abstract, applied to the rank-r reconstruction. */
cf_status cf_lowrank(cf_ctx *ctx, int nmat, int64_t m, int64_t n, const float *const *A,
                     const float *const *Q0, float *const *U, float *const *R, float *const *V,
                     float *const *E_opt, float *const *C_opt, void *cuda_stream);

/* K or V of a received shard for cf_attention, in one of two forms:
 *   bf16 != NULL : the tensor in bf16, e.g. a slot's recon (bf16 of the
 *                  receiver's cache, written by cf_decompress in its pass);
 *   bf16 == NULL : dequantise-on-load -- the receiver's cache C_{t-1} and
 *                  this step's payload; the attention forms
 *                  C_t = C_{t-1} + deq(codes, scales) exactly as cf_decompress
 *                  does, uses bf16(C_t) and writes C_t to cache_out (if not
 *                  NULL), so the receiver needs no separate decompress. */
typedef struct cf_kv {
    const void *bf16;         /* bf16 [rows*cols], or NULL for dequantise-on-load */
    const float *cache_in;    /* fp32 [rows*cols]: C_{t-1} (read only) */
    float *cache_out;         /* fp32 [rows*cols]: C_t, or NULL; must not overlap any cache_in */
    const uint8_t *codes;     /* this step's codes (the context's k), rows*cols*k/8 bytes */
    const float *scales;      /* this step's scales (the context's G), rows*cols/G */
} cf_kv;

/* Attention of a shard's queries over a received K/V shard, per head of 64
 * channels: for head h (channels [64 h, 64 h + 64) of the token-major
 * layout), out_h = softmax(q_h k_h^T / 8) v_h.
 *   q, out  bf16 [lq x cols] (16-byte aligned); k, v of [lk x cols], both in
 *   the same cf_kv form; cols a multiple of 64 (and of G when dequantising).
 *   lse     fp32 [lq x cols/64] (query-major, 4-byte aligned) or NULL: the
 *   natural log of sum_j exp(q_h . k_j / 8) of every row and head.  A ring
 *   step that attends over one received block at a time merges the partial
 *   outputs with it: over the union of blocks b, out = sum_b exp(lse_b -
 *   lse) out_b with lse = log sum_b exp(lse_b).
 * The products run on the tensor cores in bf16 with fp32 accumulation, the
 * softmax in fp32 (base 2, online over blocks of 128 keys, P rounded to bf16).
 * Dequantise-on-load needs a quantised-mode context with fp32 state (its k
 * and G describe the payload); the bf16 form only uses the context's status
 * word.  The two forms give bit-identical outputs for the same C_t.
 * Stream-ordered; allocates nothing.  Every wait in the kernel is bounded
 * (failure-detection test hook: CF_TEST_STARVE_ATTENTION=1 in the environment
 * when the context is created makes its first cf_attention call time out).
 * Errors before launch: CF_E_ARG (NULL
 * pointer, mixed forms, overlapping caches, out overlapping k or v, wrong
 * context), CF_E_SHAPE (lk <
 * 1, cols not a multiple of 64 or of G), CF_E_ALIGN (q, out, k, v or lse
 * misaligned); device-side:
 * CF_E_TIMEOUT at the next cf_check.
 * Source: reproducibility table, "Pseudocode" row, Algorithms 1 and 2 (each
 * device attends over the key/value blocks it receives from the others);
 * abstract (the receiver adds each decompressed residual to its
 * reconstruction). */
cf_status cf_attention(cf_ctx *ctx, int64_t lq, int64_t lk, int64_t cols, const void *q, const cf_kv *k,
                       const cf_kv *v, void *out, float *lse, void *cuda_stream);

/* Bytes of device scratch that the library keeps on every GPU it is loaded
 * on, for cf_lowrank_noalloc (status word plus the Algorithm 3 buffers). */
#define CF_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* cf_lowrank for callers that cannot allocate device memory.  (The paper has
 * no counterpart: this is an integration aid of this library.)
 *
 * Who needs it: code that must not call cudaMalloc or any allocating library
 * routine at the point where it compresses -- work running inside a caller's
 * pre-reserved memory pool, a plug-in that is handed only the tensors it may
 * touch, or a step that must not change the device's allocation state while
 * other work is in flight.  cf_lowrank needs a context (cf_create allocates
 * its status word) and a caller-allocated workspace; this entry point needs
 * neither.  Its scratch is a fixed CF_NOALLOC_SCRATCH_BYTES (8 MiB) device
 * array inside the library, which every GPU that loads the library holds
 * until the process exits.  It calls no device allocator.
 *
 * Arguments and results are those of cf_lowrank, with the rank r and the
 * iteration count T taken from `config` (mode must be CF_MODE_LOWRANK);
 * A, Q0, U, R, V, E_opt, C_opt are host arrays of nmat device pointers.
 * Limits: the Algorithm 3 buffers of the call -- cf_lowrank_workspace_bytes
 * for the same nmat, m, n and r, about 4*rp*(2m + 2n) + 4*r*(r+1)*ceil(max(m,
 * n)/256) + 8 KB per matrix with rp = 16 (r <= 16) or 32 -- must fit in
 * CF_NOALLOC_SCRATCH_BYTES - 256
 * bytes, and nmat <= 512; otherwise the call returns CF_E_NOMEM and launches
 * nothing.  Eight 4608 x 3072 matrices at r = 16 fit in one call.
 *
 * The call runs on the current device; every pointer must be device memory
 * of that device (else CF_E_ARG).  It is synchronous: it enqueues the work
 * on `cuda_stream` (a stream of the current device), waits for it and
 * returns the device status (CF_OK, CF_E_NONFINITE, CF_E_TIMEOUT or
 * CF_E_CUDA).
 *
 * First call on a device: it looks up the scratch's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  CUDA loads a library's device code lazily by
 * default, when it is first used on a device, and the 8 MiB array comes
 * into existence with it; so the first call into libcf on a device -- this
 * one or any other -- may itself reserve device memory.  A caller whose
 * allocation state must not change should make one call (e.g. on a small
 * matrix) on each device before that region; later calls with the same
 * rank reserve nothing more.
 *
 * Every call shares the one scratch array, which keeps the previous call's
 * contents (the call clears what must start at zero), so calls that overlap
 * on the GPU -- on two streams or from two host threads -- race and must be
 * serialised by the caller.  Errors before launch: CF_E_ARG, CF_E_SHAPE,
 * CF_E_ALIGN, CF_E_NOMEM.
 * Source: none in the paper (an integration aid of this library); it
 * computes what cf_lowrank computes (Algorithm 3, "Pseudocode" row). */
cf_status cf_lowrank_noalloc(const cf_config *config, int nmat, int64_t m, int64_t n, const float *const *A,
                             const float *const *Q0, float *const *U, float *const *R, float *const *V,
                             float *const *E_opt, float *const *C_opt, void *cuda_stream);

/* Per-launch device timing.  While tracing is on (cf_trace_enable(ctx, 1)),
 * every kernel this context launches (in cf_compress, cf_decompress,
 * cf_loopback and cf_lowrank) is bracketed by a pair of CUDA events recorded
 * on its stream; the events come from a pool the context keeps.  Not for use
 * while a stream is being captured into a CUDA graph.  Errors: CF_E_ARG.
 * Source: library plumbing (measurement), no counterpart in the paper. */
cf_status cf_trace_enable(cf_ctx *ctx, int on);

typedef struct cf_trace_entry {
    char kernel[80];   /* kernel name and template arguments, NUL-terminated */
    int launches;      /* traced launches of it since the last cf_trace_read */
    double total_ms;   /* summed event-timed duration of those launches */
} cf_trace_entry;

/* Waits for the traced launches, writes per-kernel totals (in order of first
 * launch) to out[0 .. min(count, max_entries)), clears them and returns the
 * number of distinct kernels (which may exceed max_entries), or -CF_E_ARG /
 * -CF_E_CUDA (an event could not be created, recorded or read), or
 * -CF_E_NOMEM.
 * Source: library plumbing (measurement), no counterpart in the paper. */
int cf_trace_read(cf_ctx *ctx, cf_trace_entry *out, int max_entries);

/* Synchronise `cuda_stream`, read and clear the device status word.
 * Returns CF_OK, CF_E_NONFINITE, CF_E_TIMEOUT or CF_E_CUDA (an asynchronous
 * CUDA error, e.g. from an earlier launch).
 * Source: library plumbing (error reporting), no counterpart in the paper. */
cf_status cf_check(cf_ctx *ctx, void *cuda_stream);

/* Payload bytes of slot `slot` per compressed step: rows*cols*k/8 +
 * 4*rows*cols/G (quantised) or 4*r*(rows + r + cols) (low-rank); 0 for a bad
 * slot index.
 * Source: abstract (only the compressed residual crosses the link); xDiT
 * issue 573 (residuals plus error feedback cut the traffic 8-16x: 16/k of
 * the bf16 activations for k = 2 and k = 1, before the scales' 32/G bits
 * per element). */
size_t cf_payload_bytes(const cf_ctx *ctx, int slot);

/* Human-readable message of the last error on this context ("" if none).
 * The string is owned by the context.
 * Source: library plumbing, no counterpart in the paper. */
const char *cf_last_error(const cf_ctx *ctx);

/* Resume a run from caller-saved state (checkpoint / restart).  All codec
 * state lives in caller memory -- base, err and cache of every slot, and V
 * for the low-rank warm start -- so a checkpoint is a copy of those buffers
 * plus the index of the last step done.  After restoring them, call this on
 * a fresh context with the same configuration and shapes: it records that
 * steps 0..steps_done (the warmup included) have run on both the sender and
 * the receiver side, so the next call may be step steps_done + 1, and a
 * warm-start low-rank context starts Algorithm 3 from the restored V.
 * Enqueues nothing.  Errors: CF_E_ARG (NULL context, steps_done < 0).
 * Source: library plumbing (checkpoint / restart); the state it resumes is
 * the base tensor ("Dataset Splits" row), the error-feedback buffer and the
 * receiver's reconstruction (abstract). */
cf_status cf_resume(cf_ctx *ctx, int64_t steps_done);

/* Free the context (waits for nothing; the caller must not destroy a
 * context while its launches are still running on a stream).
 * Source: library plumbing, no counterpart in the paper. */
cf_status cf_destroy(cf_ctx *ctx);

#ifdef __cplusplus
}
#endif

#endif /* CF_H */
