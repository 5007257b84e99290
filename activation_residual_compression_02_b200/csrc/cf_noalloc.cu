// cf_noalloc.cu -- cf_lowrank_noalloc: the low-rank call for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they compress: code
// that runs inside a custom or pre-reserved memory pool, plug-ins handed only
// the tensors they must touch, or steps that must not change the device's
// allocation state while other work is in flight.  cf_lowrank needs a
// workspace for the r-column blocks of Algorithm 3 (Q^T, P^T, P, Z and fp64
// Gram matrices), and cf_create allocates a status word.  This entry point
// takes neither a context nor a workspace: its scratch is the file-scope
// device array below, a fixed 8 MiB that every GPU which loads the library
// keeps for the life of the process.  The caller still owns A, Q0 and the
// outputs.
#include <mutex>
#include <new>

#include "cf_internal.h"

namespace cf {
namespace {

constexpr size_t kStatusBytes = 256;
constexpr int kMaxNoallocMats = 512;

// Device scratch of cf_lowrank_noalloc: the status word in the first 256
// bytes, then the Algorithm 3 workspace.  Shared by every call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CF_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch, looked up once per device with that
// device current.  In host code the symbol's name only stands for the
// variable; launching a kernel with it would read the wrong memory, so every
// use goes through the address cudaGetSymbolAddress returns.
cudaError_t scratch_address(void **out)
{
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// True when p is device (or managed) memory of device `dev`.  The kernels run
// on the current device, so a pointer into another GPU's memory, or a host
// pointer, is refused before anything is launched.
bool on_device(const void *p, int dev)
{
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();   // the query's error is the answer, not a sticky state
        return false;
    }
    return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev;
}

}  // namespace
}  // namespace cf

extern "C" cf_status cf_lowrank_noalloc(const cf_config *config, int nmat, int64_t m, int64_t n,
                                        const float *const *A, const float *const *Q0, float *const *U,
                                        float *const *R, float *const *V, float *const *E_opt,
                                        float *const *C_opt, void *cuda_stream)
try {
    using namespace cf;
    if (!config || config->mode != CF_MODE_LOWRANK) return CF_E_ARG;
    const int r = config->rank, T = config->iters;
    if (r < 1 || r > 32 || T < 0 || T > 1000 || nmat < 0) return CF_E_ARG;
    if (config->precision < CF_PRECISION_AUTO || config->precision > CF_PRECISION_SPLIT) return CF_E_ARG;
    if (nmat == 0) return CF_OK;
    if (nmat > kMaxNoallocMats) return CF_E_NOMEM;
    if (!A || !Q0 || !U || !R || !V) return CF_E_ARG;
    if (m < r || n < r || m > INT32_MAX || n > INT32_MAX) return CF_E_SHAPE;
    if (n % 4 != 0) return CF_E_SHAPE;
    // Reject calls whose Algorithm 3 buffers do not fit the fixed scratch.
    const bool split = lowrank_split(config->precision, m, n, r);
    const size_t need = lowrank_workspace_bytes(nmat, m, n, r, split);
    if (need > CF_NOALLOC_SCRATCH_BYTES - kStatusBytes) return CF_E_NOMEM;
    LowrankMat mats[kMaxNoallocMats];
    for (int i = 0; i < nmat; ++i) {
        if (!A[i] || !Q0[i] || !U[i] || !R[i] || !V[i]) return CF_E_ARG;
        float *E = E_opt ? E_opt[i] : nullptr;
        float *C = C_opt ? C_opt[i] : nullptr;
        if (!aligned16(A[i]) || !aligned16(Q0[i]) || !aligned16(U[i]) || !aligned16(R[i]) || !aligned16(V[i]) ||
            !aligned16(E) || !aligned16(C))
            return CF_E_ALIGN;
        mats[i] = LowrankMat{A[i], Q0[i], U[i], R[i], V[i], E, C};
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CF_E_CUDA;
    for (int i = 0; i < nmat; ++i) {
        const LowrankMat &t = mats[i];
        if (!on_device(t.A, dev) || !on_device(t.Q0, dev) || !on_device(t.U, dev) || !on_device(t.R, dev) ||
            !on_device(t.V, dev) || (t.E && !on_device(t.E, dev)) || (t.C && !on_device(t.C, dev)))
            return CF_E_ARG;
    }
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return CF_E_CUDA;
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    uint32_t *status = (uint32_t *)scratch;
    // The array keeps the previous call's contents: the status word must
    // start at zero (run_lowrank zeroes the blocks of Algorithm 3 it needs).
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), stream) != cudaSuccess) return CF_E_CUDA;
    LowrankPlan plan{};
    plan.nmat = nmat;
    plan.m = m;
    plan.n = n;
    plan.r = r;
    plan.T = T;
    plan.split = split;
    plan.ws = (char *)scratch + kStatusBytes;
    plan.ws_bytes = CF_NOALLOC_SCRATCH_BYTES - kStatusBytes;
    plan.status = status;
    if (run_lowrank(plan, mats, stream) != cudaSuccess) return CF_E_CUDA;
    // Without a context there is no cf_check: wait here and report the status.
    if (cudaStreamSynchronize(stream) != cudaSuccess) return CF_E_CUDA;
    uint32_t word = 0;
    if (cudaMemcpy(&word, status, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) return CF_E_CUDA;
    if (word & kStatusTimeout) return CF_E_TIMEOUT;
    if (word & (kStatusNonfinite | kStatusNotSpd)) return CF_E_NONFINITE;
    return CF_OK;
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;   // a host allocation failed: no C++ exception crosses the C ABI
} catch (...) {
    return CF_E_ARG;
}

