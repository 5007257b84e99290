// cf_internal.h -- declarations shared by the libcf translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "cf.h"

namespace cf {

// Device status word bits (read and cleared by cf_check).
constexpr uint32_t kStatusNonfinite = 0x1u;
constexpr uint32_t kStatusTimeout = 0x2u;
constexpr uint32_t kStatusNotSpd = 0x4u;

// Slots per grouped launch of the quantised kernels; the descriptor table
// travels as a __grid_constant__ kernel parameter (CUDA 12.1+ allows up to
// 32 KB of parameters), so no per-call device allocation or copy is needed.
constexpr int kMaxSlotsPerLaunch = 128;

struct QuantSlotDesc {
    const void *x;     // bf16
    void *base;        // bf16
    void *err;         // fp32, or bf16 with the lean state
    void *cache;       // fp32, or bf16 with the lean state
    uint8_t *codes;    // packed codes
    float *scales;     // fp32 group scales
    void *recon;       // bf16 copy of the receiver's cache after the call, or null
    int64_t nvec;      // elements / 8
    int64_t tile0;     // first tile index of this slot in the launch (set by launch_quant)
};

struct QuantLaunch {
    int nslots;
    int pad_;
    int64_t ntiles;
    uint32_t *status;
    QuantSlotDesc slot[kMaxSlotsPerLaunch];
};
static_assert(sizeof(QuantLaunch) <= 32764, "a kernel takes at most 32764 bytes of parameters");

enum class QuantOp { WarmupSender, WarmupReceiver, Compress, Decompress, Loopback };

// Launch one grouped quantised kernel over `lp` (host-built slot table;
// tile0/ntiles are filled in here for the chosen kernel's tile size).
// bits/group/sign_scale select the template instance.  Returns cudaSuccess or
// the launch error.
cudaError_t launch_quant(QuantOp op, int bits, int group, int sign_scale, bool lean, QuantLaunch &lp,
                         cudaStream_t stream);

// ---------------------------------------------------------------- low rank

struct LowrankMat {
    const float *A;    // [m x n] row-major
    const float *Q0;   // [n x r]
    float *U;          // [m x r]
    float *R;          // [r x r]
    float *V;          // [n x r]
    float *E;          // [m x n] or null
    float *C;          // [m x n] or null
    void *recon;       // bf16 [m x n] or null: bf16(C) after C += D
};

struct LowrankPlan {
    int nmat;
    int64_t m, n;
    int r, T;
    bool split;        // split (3xTF32) products, see lowrank_split
    bool starve;       // failure-detection test only: the products' loads are withheld (bounded waits time out)
    void *ws;          // device workspace
    size_t ws_bytes;
    uint32_t *status;
};

// Whether the products with A run split (3xTF32) for a config precision
// (CF_PRECISION_*) and an m x n problem of rank r.
bool lowrank_split(int precision, int64_t m, int64_t n, int r);

size_t lowrank_workspace_bytes(int nmat, int64_t m, int64_t n, int r, bool split);

// Runs Algorithm 3 (and the apply step) for plan.nmat matrices.  `mats` is a
// host array.  Returns a cudaError_t from the launches.
cudaError_t run_lowrank(const LowrankPlan &plan, const LowrankMat *mats, cudaStream_t stream);

// Low-rank decompress: C += U R V^T for each matrix (E, A unused).
cudaError_t run_lowrank_decompress(const LowrankPlan &plan, const LowrankMat *mats, cudaStream_t stream);

// Residual materialisation for low-rank mode: A = (x - base) + err (fp32) into
// `a_out`, base <- x.  One launch per slot list.
cudaError_t launch_residual_f32(const void *const *x, void *const *base, const float *const *err,
                                float *const *a_out, const int64_t *n, int nslots, cudaStream_t stream);

// Attention over a received K/V shard (cf_attention): heads of 64 channels,
// K and V as bf16 (kv) or dequantised on load from cache_in + codes/scales
// (dequantise = true), the new cache written to cache_out when non-null;
// the log-sum-exp of every row and head to lse when non-null.
struct AttnArgs {
    const void *q;
    const void *kv[2];
    const float *cache_in[2];
    float *cache_out[2];
    const uint8_t *codes[2];
    const float *scales[2];
    void *out;
    float *lse;          // [lq x cols/64] or null
    int64_t lq, lk, cols;
    int bits, group;
    bool dequantise;
    bool starve;         // failure-detection test only: no loads, 20 ms waits (they time out)
    uint32_t *status;
};
cudaError_t launch_attention(const AttnArgs &a, cudaStream_t stream);

int num_sms();

// Host-side launch log: with CF_LOG=1 in the environment (read once), every
// kernel launch prints one line to stderr with its name, grid, block and
// dynamic shared memory.
void log_launch(const char *kernel, dim3 grid, dim3 block, size_t smem);
bool log_enabled();

// Per-launch device timing (cf_trace_enable / cf_trace_read): while an API
// call of a tracing context runs, trace_on() is true on the calling thread and
// each launch site brackets its kernel with trace_begin / trace_end, which
// record a pair of CUDA events on the launch stream.
bool trace_on();
void trace_begin(const char *kernel, cudaStream_t stream);
void trace_end(cudaStream_t stream);

}  // namespace cf
