// cf_lowrank.cu -- low-rank mode of the codec (Algorithm 3, subspace iteration).
//
// "Accelerating Parallel Diffusion Model Serving with Residual Compression"
// (arXiv 2507.17511), reproducibility table, "Pseudocode" row, Algorithm 3.
#include <string.h>

#include "cf_internal.h"

namespace cf {
namespace {

// Launch shape: persistent CTAs (one per SM) walk a flat tile index over all
// slots; a thread issues the loads of kResUnroll vectors (8 elements each)
// before it computes, as the quantised sender does (the residual moves the
// same streams minus the payload: 14 bytes per element).
constexpr int kResThreads = 256;
constexpr int kResUnroll = 8;
constexpr int64_t kResTileVec = (int64_t)kResThreads * kResUnroll;

struct ResidualSlots {
    int n;
    int pad_;
    int64_t ntiles;
    const uint4 *x[kMaxSlotsPerLaunch];
    uint4 *base[kMaxSlotsPerLaunch];
    const float4 *err[kMaxSlotsPerLaunch];
    float4 *a[kMaxSlotsPerLaunch];
    int64_t nvec[kMaxSlotsPerLaunch];
    int64_t tile0[kMaxSlotsPerLaunch];
};
static_assert(sizeof(ResidualSlots) <= 32764, "a kernel takes at most 32764 bytes of parameters");

// A = (x - base) + err in fp32 (same operation order as the quantised path),
// base <- x.
__global__ void __launch_bounds__(kResThreads, 1) k_residual_f32(const __grid_constant__ ResidualSlots p)
{
    for (int64_t tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        int lo = 0, hi = p.n - 1;   // slot of this tile: last slot whose first tile <= tile
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.tile0[mid] <= tile)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int s = lo;
        const int64_t nvec = p.nvec[s];
        const uint4 *X = p.x[s];
        uint4 *B = p.base[s];
        const float4 *E = p.err[s];
        float4 *A = p.a[s];
        const int64_t v0 = (tile - p.tile0[s]) * kResTileVec + threadIdx.x;
        uint4 xv[kResUnroll], bv[kResUnroll];
        float4 e0[kResUnroll], e1[kResUnroll];
#pragma unroll
        for (int u = 0; u < kResUnroll; ++u) {
            const int64_t v = v0 + (int64_t)u * kResThreads;
            if (v < nvec) {
                xv[u] = __ldcs(X + v);
                bv[u] = __ldcs(B + v);
                e0[u] = __ldcs(E + 2 * v);
                e1[u] = __ldcs(E + 2 * v + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kResUnroll; ++u) {
            const int64_t v = v0 + (int64_t)u * kResThreads;
            if (v >= nvec) continue;
            const uint32_t xw[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
            const uint32_t bw[4] = {bv[u].x, bv[u].y, bv[u].z, bv[u].w};
            const float e[8] = {e0[u].x, e0[u].y, e0[u].z, e0[u].w, e1[u].x, e1[u].y, e1[u].z, e1[u].w};
            float a[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float xl = __uint_as_float(xw[j] << 16), xh = __uint_as_float(xw[j] & 0xffff0000u);
                const float bl = __uint_as_float(bw[j] << 16), bh = __uint_as_float(bw[j] & 0xffff0000u);
                a[2 * j] = __fadd_rn(__fsub_rn(xl, bl), e[2 * j]);
                a[2 * j + 1] = __fadd_rn(__fsub_rn(xh, bh), e[2 * j + 1]);
            }
            __stcs(B + v, xv[u]);
            A[2 * v] = make_float4(a[0], a[1], a[2], a[3]);
            A[2 * v + 1] = make_float4(a[4], a[5], a[6], a[7]);
        }
    }
}

}  // namespace

cudaError_t launch_residual_f32(const void *const *x, void *const *base, const float *const *err, float *const *a_out,
                                const int64_t *n, int nslots, cudaStream_t stream)
{
    ResidualSlots *p = new ResidualSlots;
    cudaError_t e = cudaSuccess;
    for (int first = 0; first < nslots && e == cudaSuccess; first += kMaxSlotsPerLaunch) {
        const int cnt = (nslots - first < kMaxSlotsPerLaunch) ? nslots - first : kMaxSlotsPerLaunch;
        memset(p, 0, sizeof *p);
        p->n = cnt;
        int64_t tiles = 0;
        for (int k = 0; k < cnt; ++k) {
            p->x[k] = (const uint4 *)x[first + k];
            p->base[k] = (uint4 *)base[first + k];
            p->err[k] = (const float4 *)err[first + k];
            p->a[k] = (float4 *)a_out[first + k];
            p->nvec[k] = n[first + k] / 8;
            p->tile0[k] = tiles;
            tiles += (p->nvec[k] + kResTileVec - 1) / kResTileVec;
        }
        p->ntiles = tiles;
        if (tiles > 0) {
            const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
            log_launch("k_residual_f32", dim3(grid), dim3(kResThreads), 0);
            trace_begin("k_residual_f32", stream);
            k_residual_f32<<<grid, kResThreads, 0, stream>>>(*p);
            trace_end(stream);
            e = cudaGetLastError();
        }
    }
    delete p;
    return e;
}

}  // namespace cf
