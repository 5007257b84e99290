// cf_lowrank.cu -- low-rank mode of the codec (Algorithm 3, subspace iteration).
//
// "Accelerating Parallel Diffusion Model Serving with Residual Compression"
// (arXiv 2507.17511), reproducibility table, "Pseudocode" row, Algorithm 3.
#include "cf_internal.h"

namespace cf {
namespace {

constexpr int kResThreads = 256;

struct ResidualSlots {
    int n;
    int pad_;
    const uint4 *x[kMaxSlotsPerLaunch];
    uint4 *base[kMaxSlotsPerLaunch];
    const float4 *err[kMaxSlotsPerLaunch];
    float4 *a[kMaxSlotsPerLaunch];
    int64_t nvec[kMaxSlotsPerLaunch];
};

// A = (x - base) + err in fp32 (same operation order as the quantised path),
// base <- x.  grid.y = slot.
__global__ void __launch_bounds__(kResThreads) k_residual_f32(const __grid_constant__ ResidualSlots p)
{
    const int s = blockIdx.y;
    const int64_t nvec = p.nvec[s];
    const uint4 *X = p.x[s];
    uint4 *B = p.base[s];
    const float4 *E = p.err[s];
    float4 *A = p.a[s];
    for (int64_t v = (int64_t)blockIdx.x * kResThreads + threadIdx.x; v < nvec; v += (int64_t)gridDim.x * kResThreads) {
        const uint4 xv = __ldcs(X + v);
        const uint4 bv = __ldcs(B + v);
        const float4 e0 = __ldcs(E + 2 * v);
        const float4 e1 = __ldcs(E + 2 * v + 1);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
        const float e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
        float a[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float xl = __uint_as_float(xw[j] << 16), xh = __uint_as_float(xw[j] & 0xffff0000u);
            const float bl = __uint_as_float(bw[j] << 16), bh = __uint_as_float(bw[j] & 0xffff0000u);
            a[2 * j] = __fadd_rn(__fsub_rn(xl, bl), e[2 * j]);
            a[2 * j + 1] = __fadd_rn(__fsub_rn(xh, bh), e[2 * j + 1]);
        }
        __stcs(B + v, xv);
        A[2 * v] = make_float4(a[0], a[1], a[2], a[3]);
        A[2 * v + 1] = make_float4(a[4], a[5], a[6], a[7]);
    }
}

}  // namespace

cudaError_t launch_residual_f32(const void *const *x, void *const *base, const float *const *err, float *const *a_out,
                                const int64_t *n, int nslots, cudaStream_t stream)
{
    for (int first = 0; first < nslots; first += kMaxSlotsPerLaunch) {
        const int cnt = (nslots - first < kMaxSlotsPerLaunch) ? nslots - first : kMaxSlotsPerLaunch;
        ResidualSlots *p = new ResidualSlots;
        p->n = cnt;
        int64_t maxv = 0;
        for (int k = 0; k < cnt; ++k) {
            p->x[k] = (const uint4 *)x[first + k];
            p->base[k] = (uint4 *)base[first + k];
            p->err[k] = (const float4 *)err[first + k];
            p->a[k] = (float4 *)a_out[first + k];
            p->nvec[k] = n[first + k] / 8;
            if (p->nvec[k] > maxv) maxv = p->nvec[k];
        }
        if (maxv > 0) {
            int64_t bx = (maxv + kResThreads - 1) / kResThreads;
            const int64_t cap = (int64_t)num_sms() * 8 / (cnt > 0 ? cnt : 1) + 1;
            if (bx > cap) bx = cap;
            dim3 grid((unsigned)bx, (unsigned)cnt);
            log_launch("k_residual_f32", grid, dim3(kResThreads), 0);
            k_residual_f32<<<grid, kResThreads, 0, stream>>>(*p);
        }
        delete p;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace cf
