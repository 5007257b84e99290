// cf_quant.cu -- grouped quantised codec kernels for sm_100a.
//
// "Accelerating Parallel Diffusion Model Serving with Residual Compression"
// (arXiv 2507.17511), abstract: each step sends the compressed residual
// (step-wise activation difference) and carries the compression error
// forward; reproducibility table, "Dataset Splits" row: the warmup step sends
// the activation uncompressed and initialises the base tensor.
//
// One slot is a flat array of n = rows*cols elements; since G divides cols,
// groups never straddle token rows, so every kernel here is 1-D over the
// slot.  A thread owns vectors of 8 consecutive elements (16 bytes of bf16,
// 32 bytes of fp32), G/8 consecutive lanes own one group, and the group
// statistic is a register reduction over 8 elements plus log2(G/8)
// butterfly shuffles.  One launch covers every slot of a step: the slot table
// is a __grid_constant__ parameter and persistent CTAs walk a flat tile
// index.  The work is a pure stream (no reuse), so the design goal is bytes
// in flight: each thread issues all loads of its kUnroll vectors before it
// computes.
//
// Bit-exactness: every floating-point step is an explicit round-to-nearest
// intrinsic (__fadd_rn, __fsub_rn, __fmul_rn, __fdiv_rn), so no FMA
// contraction can change a code; the absmax is an integer max over the
// magnitude bits (exact, and a NaN or infinity is seen as non-finite).
#include <cuda_bf16.h>

#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <unordered_map>

#include "cf_internal.h"
#include "cf_ptx.cuh"

namespace cf {
namespace {

// Launch shape per operation: threads per CTA, vectors (of 8 elements) each
// thread keeps in flight (a tile is threads * unroll vectors), and a cap on
// resident CTAs per SM (0: as many as fit).  Chosen by sweeps on the B200
// over 128..1024 threads, 1..8 vectors and 1..4 CTAs per SM on the 57-slot
// FLUX-shaped step: compress wants many warps to hide its ~150 instructions
// per vector (1024 x 1: 93.5% of the measured copy bandwidth, against 88% for
// 256 x 4 at 2 CTAs/SM); decompress wants about 512 resident threads per SM
// with 4 vectors each (94.5%, against 84% at 4 CTAs/SM).
template <QuantOp OP>
struct QShape {
    static constexpr int kThreads = 256;
    static constexpr int kUnroll = 4;
    static constexpr int kMaxPerSm = 0;
};
template <>
struct QShape<QuantOp::Compress> {
    static constexpr int kThreads = 1024;
    static constexpr int kUnroll = 1;
    static constexpr int kMaxPerSm = 0;
};
template <>
struct QShape<QuantOp::Loopback> {
    // fused sender + receiver: 9 streams per tile; best of the sweep (90.6%
    // of the copy peak), still below the separate pair (94.3%)
    static constexpr int kThreads = 256;
    static constexpr int kUnroll = 8;
    static constexpr int kMaxPerSm = 1;
};
template <>
struct QShape<QuantOp::Decompress> {
    static constexpr int kThreads = 512;
    static constexpr int kUnroll = 4;
    static constexpr int kMaxPerSm = 1;
};
template <QuantOp OP>
constexpr int64_t qtile_vec()
{
    return (int64_t)QShape<OP>::kThreads * QShape<OP>::kUnroll;
}
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kAbsMask = 0x7fffffffu;
constexpr uint32_t kInfBits = 0x7f800000u;
// Scales below 2^-120 denote an all-zero group (keeps L/s finite for k <= 4).
constexpr float kScaleMin = 7.52316384526264e-37f;

__device__ __forceinline__ int find_slot(const QuantLaunch &p, int64_t tile)
{
    int lo = 0, hi = p.nslots - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.slot[mid].tile0 <= tile)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8])
{
    f[0] = bf_lo(v.x); f[1] = bf_hi(v.x);
    f[2] = bf_lo(v.y); f[3] = bf_hi(v.y);
    f[4] = bf_lo(v.z); f[5] = bf_hi(v.z);
    f[6] = bf_lo(v.w); f[7] = bf_hi(v.w);
}

template <int K>
struct CodeWord;
template <> struct CodeWord<1> { using T = uint8_t; };
template <> struct CodeWord<2> { using T = uint16_t; };
template <> struct CodeWord<4> { using T = uint32_t; };

// Per-group scale: absmax (k >= 2, or k = 1 with sign_scale 1) as an integer
// max of the magnitude bits, or for k = 1 the mean of |a| by a perfect
// binary-tree sum (three levels in the lane, then butterfly levels across the
// G/8 lanes; addition is commutative, so both partners of a butterfly hold
// the same node value).
template <int K, int G, int SS>
__device__ __forceinline__ float group_scale(const float (&a)[8], bool &nonfinite)
{
    constexpr int LPG = G / 8;
    if constexpr (K >= 2 || SS == 1) {
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) m = max(m, __float_as_uint(a[j]) & kAbsMask);
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
        nonfinite = m >= kInfBits;
        return __uint_as_float(m);
    } else {
        const float s01 = __fadd_rn(fabsf(a[0]), fabsf(a[1]));
        const float s23 = __fadd_rn(fabsf(a[2]), fabsf(a[3]));
        const float s45 = __fadd_rn(fabsf(a[4]), fabsf(a[5]));
        const float s67 = __fadd_rn(fabsf(a[6]), fabsf(a[7]));
        float t = __fadd_rn(__fadd_rn(s01, s23), __fadd_rn(s45, s67));
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) t = __fadd_rn(t, __shfl_xor_sync(kFull, t, o));
        const float s = __fdiv_rn(t, (float)G);
        nonfinite = !isfinite(s);
        return s;
    }
}

template <QuantOp OP, int K, int G, int SS>
__global__ void __launch_bounds__(QShape<OP>::kThreads) k_quant(const __grid_constant__ QuantLaunch p)
{
    constexpr int kThreads = QShape<OP>::kThreads;
    constexpr int kUnroll = QShape<OP>::kUnroll;
    constexpr int kTileVec = kThreads * kUnroll;
    constexpr int LPG = G / 8;
    constexpr int L = (K >= 2) ? (1 << (K - 1)) - 1 : 1;
    using Word = typename CodeWord<K>::T;

    // Dequantised levels t_c = (c - L) / L, one correctly rounded division each.
    __shared__ float lut[16];
    if (threadIdx.x < 16)
        lut[threadIdx.x] = (K >= 2) ? __fdiv_rn((float)((int)threadIdx.x - L), (float)L) : 0.0f;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    for (int64_t tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x) {
        const int si = find_slot(p, tile);
        const QuantSlotDesc &S = p.slot[si];
        const int64_t nvec = S.nvec;
        const int64_t v0 = (tile - S.tile0) * kTileVec + threadIdx.x;

        if constexpr (OP == QuantOp::WarmupSender) {
            const uint4 *X = static_cast<const uint4 *>(S.x);
            uint4 *B = static_cast<uint4 *>(S.base);
            float4 *E = reinterpret_cast<float4 *>(S.err);
            uint4 xv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) xv[u] = __ldcs(X + v);
            }
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    __stcs(B + v, xv[u]);
                    __stcs(E + 2 * v, z);
                    __stcs(E + 2 * v + 1, z);
                }
            }
        } else if constexpr (OP == QuantOp::WarmupReceiver) {
            const uint4 *X = static_cast<const uint4 *>(S.x);
            float4 *C = reinterpret_cast<float4 *>(S.cache);
            uint4 xv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) xv[u] = __ldcs(X + v);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    float f[8];
                    unpack8(xv[u], f);
                    __stcs(C + 2 * v, make_float4(f[0], f[1], f[2], f[3]));
                    __stcs(C + 2 * v + 1, make_float4(f[4], f[5], f[6], f[7]));
                }
            }
        } else if constexpr (OP == QuantOp::Compress || OP == QuantOp::Loopback) {
            // Loopback = sender and receiver on the same device: the receiver's
            // C += d reuses the d the sender just formed (bit-identical to a
            // separate decompress) and the payload is not read back.
            constexpr bool LB = OP == QuantOp::Loopback;
            const uint4 *X = static_cast<const uint4 *>(S.x);
            uint4 *B = static_cast<uint4 *>(S.base);
            float4 *E = reinterpret_cast<float4 *>(S.err);
            float4 *C = reinterpret_cast<float4 *>(S.cache);
            Word *codes = reinterpret_cast<Word *>(S.codes);
            float *scales = S.scales;

            uint4 xv[kUnroll], bv[kUnroll];
            float4 ea[kUnroll], eb[kUnroll];
            float4 ca[LB ? kUnroll : 1], cb[LB ? kUnroll : 1];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    xv[u] = __ldcs(X + v);
                    bv[u] = __ldcs(B + v);
                    ea[u] = __ldcs(E + 2 * v);
                    eb[u] = __ldcs(E + 2 * v + 1);
                    if constexpr (LB) {
                        ca[u] = __ldcs(C + 2 * v);
                        cb[u] = __ldcs(C + 2 * v + 1);
                    }
                } else {
                    xv[u] = bv[u] = make_uint4(0, 0, 0, 0);
                    ea[u] = eb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if constexpr (LB) ca[u] = cb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                const bool valid = v < nvec;
                // residual against the base tensor plus the carried error
                float xf[8], bf[8], a[8];
                unpack8(xv[u], xf);
                unpack8(bv[u], bf);
                const float e[8] = {ea[u].x, ea[u].y, ea[u].z, ea[u].w, eb[u].x, eb[u].y, eb[u].z, eb[u].w};
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = __fadd_rn(__fsub_rn(xf[j], bf[j]), e[j]);

                bool nonfinite;
                float s = group_scale<K, G, SS>(a, nonfinite);
                const bool zero = nonfinite || !(s >= kScaleMin);
                if (zero) s = 0.0f;
                if (nonfinite && valid) atomicOr(p.status, kStatusNonfinite);

                uint32_t word = 0;
                float d[8];
                if constexpr (K >= 2) {
                    const float inv = __fdiv_rn((float)L, zero ? 1.0f : s);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        int q = __float2int_rn(__fmul_rn(a[j], inv));
                        q = min(max(q, -L), L);
                        const int c = zero ? L : q + L;
                        word |= (uint32_t)c << (K * j);
                        d[j] = __fmul_rn(lut[c], s);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const bool pos = zero || (a[j] >= 0.0f);
                        word |= (uint32_t)pos << j;
                        d[j] = pos ? s : -s;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = __fsub_rn(a[j], d[j]);  // new carried error
                if (valid) {
                    __stcs(B + v, xv[u]);
                    __stcs(E + 2 * v, make_float4(a[0], a[1], a[2], a[3]));
                    __stcs(E + 2 * v + 1, make_float4(a[4], a[5], a[6], a[7]));
                    codes[v] = (Word)word;
                    if ((lane & (LPG - 1)) == 0) scales[v / LPG] = s;
                    if constexpr (LB) {
                        const float4 c0 = ca[u], c1 = cb[u];
                        __stcs(C + 2 * v, make_float4(__fadd_rn(c0.x, d[0]), __fadd_rn(c0.y, d[1]),
                                                      __fadd_rn(c0.z, d[2]), __fadd_rn(c0.w, d[3])));
                        __stcs(C + 2 * v + 1, make_float4(__fadd_rn(c1.x, d[4]), __fadd_rn(c1.y, d[5]),
                                                          __fadd_rn(c1.z, d[6]), __fadd_rn(c1.w, d[7])));
                    }
                }
            }
        } else {  // Decompress
            const Word *codes = reinterpret_cast<const Word *>(S.codes);
            const float *scales = S.scales;
            float4 *C = reinterpret_cast<float4 *>(S.cache);
            Word cw[kUnroll];
            float sv[kUnroll];
            float4 ca[kUnroll], cb[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    cw[u] = __ldcs(codes + v);
                    sv[u] = __ldcs(scales + v / LPG);
                    ca[u] = __ldcs(C + 2 * v);
                    cb[u] = __ldcs(C + 2 * v + 1);
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    const uint32_t w = cw[u];
                    const float s = sv[u];
                    float d[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t c = (w >> (K * j)) & ((1u << K) - 1u);
                        if constexpr (K >= 2)
                            d[j] = __fmul_rn(lut[c], s);
                        else
                            d[j] = c ? s : -s;
                    }
                    const float4 a = ca[u], b = cb[u];
                    __stcs(C + 2 * v, make_float4(__fadd_rn(a.x, d[0]), __fadd_rn(a.y, d[1]),
                                                  __fadd_rn(a.z, d[2]), __fadd_rn(a.w, d[3])));
                    __stcs(C + 2 * v + 1, make_float4(__fadd_rn(b.x, d[4]), __fadd_rn(b.y, d[5]),
                                                      __fadd_rn(b.z, d[6]), __fadd_rn(b.w, d[7])));
                }
            }
        }
    }
}

// ------------------------------------------------ TMA-staged variant ----
// The same arithmetic as k_quant, but the input streams are staged through
// shared memory by one producer thread with bulk-async copies (TMA,
// cp.async.bulk, no tensor map), so that a CTA always has kTmaStages - 1
// tiles in flight without spending registers on them.  Compress stages x,
// base and err (64 B per vector); decompress stages the cache (32 B per
// vector) and loads the small codes/scales directly before it waits.
constexpr int kTmaConsumers = 256;               // 8 consumer warps
constexpr int kTmaThreads = kTmaConsumers + 32;  // + 1 producer warp
constexpr int kTmaVec = 512;                     // vectors per tile (= one stage)
constexpr int kTmaStages = 3;
constexpr unsigned long long kQuantWaitNs = 2000000000ull;

template <QuantOp OP>
__host__ __device__ constexpr int tma_bytes_per_vec()
{
    return OP == QuantOp::Compress ? 64 : 32;
}

struct TmaBarriers {
    uint64_t full[kTmaStages];
    uint64_t empty[kTmaStages];
    int abort_flag;
};

template <QuantOp OP>
constexpr size_t tma_smem_bytes()
{
    return (size_t)kTmaStages * kTmaVec * tma_bytes_per_vec<OP>() + sizeof(TmaBarriers);
}

template <QuantOp OP, int K, int G, int SS>
__global__ void __launch_bounds__(kTmaThreads) k_quant_tma(const __grid_constant__ QuantLaunch p)
{
    using namespace ptx;
    constexpr int LPG = G / 8;
    constexpr int L = (K >= 2) ? (1 << (K - 1)) - 1 : 1;
    constexpr int BPV = tma_bytes_per_vec<OP>();
    constexpr int kStageBytes = kTmaVec * BPV;
    using Word = typename CodeWord<K>::T;

    extern __shared__ __align__(128) uint8_t tma_smem[];
    TmaBarriers *bar = reinterpret_cast<TmaBarriers *>(tma_smem + kTmaStages * kStageBytes);
    __shared__ float lut[16];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid < 16) lut[tid] = (K >= 2) ? __fdiv_rn((float)(tid - L), (float)L) : 0.0f;
    if (tid == 0) {
        for (int s = 0; s < kTmaStages; ++s) {
            mbar_init(&bar->full[s], 1);
            mbar_init(&bar->empty[s], kTmaConsumers / 32);
        }
        bar->abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    volatile int *abort_flag = &bar->abort_flag;

    if (warp == kTmaConsumers / 32) {
        // ---------------------------------------------------- producer --
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            uint32_t it = 0;
            for (int64_t tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++it) {
                const int s = it % kTmaStages;
                const uint32_t ph = (it / kTmaStages) & 1u;
                if (!wait_bounded(&bar->empty[s], ph ^ 1u, abort_flag, p.status, kQuantWaitNs)) break;
                const QuantSlotDesc &S = p.slot[find_slot(p, tile)];
                const int64_t v0 = (tile - S.tile0) * kTmaVec;
                const int64_t left = S.nvec - v0;
                const uint32_t nv = (uint32_t)(left < kTmaVec ? left : kTmaVec);
                uint8_t *st = tma_smem + s * kStageBytes;
                mbar_expect_tx(&bar->full[s], nv * BPV);
                if constexpr (OP == QuantOp::Compress) {
                    bulk_g2s(st, static_cast<const uint4 *>(S.x) + v0, nv * 16, &bar->full[s], pol);
                    bulk_g2s(st + kTmaVec * 16, static_cast<const uint4 *>(S.base) + v0, nv * 16, &bar->full[s], pol);
                    bulk_g2s(st + kTmaVec * 32, S.err + v0 * 8, nv * 32, &bar->full[s], pol);
                } else {
                    bulk_g2s(st, S.cache + v0 * 8, nv * 32, &bar->full[s], pol);
                }
            }
            // every copy this thread issued has landed before the CTA exits
            const uint32_t out = it < (uint32_t)kTmaStages ? it : (uint32_t)kTmaStages;
            for (uint32_t j = it - out; j < it; ++j) {
                volatile int no_abort = 0;
                wait_bounded(&bar->full[j % kTmaStages], (j / kTmaStages) & 1u, &no_abort, p.status, kQuantWaitNs);
            }
        }
        return;
    }

    // ------------------------------------------------------- consumers --
    uint32_t it = 0;
    for (int64_t tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++it) {
        const int s = it % kTmaStages;
        const uint32_t ph = (it / kTmaStages) & 1u;
        const QuantSlotDesc &S = p.slot[find_slot(p, tile)];
        const int64_t v0 = (tile - S.tile0) * kTmaVec;
        const int64_t left = S.nvec - v0;
        const int nv = (int)(left < kTmaVec ? left : kTmaVec);
        const uint8_t *st = tma_smem + s * kStageBytes;

        if constexpr (OP == QuantOp::Compress) {
            bool ok = wait_bounded(&bar->full[s], ph, abort_flag, p.status, kQuantWaitNs);
            if (!__all_sync(kFull, ok)) break;
            uint4 xv[2], bv[2];
            float4 ea[2], eb[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int vl = tid + u * kTmaConsumers;
                if (vl < nv) {
                    xv[u] = reinterpret_cast<const uint4 *>(st)[vl];
                    bv[u] = reinterpret_cast<const uint4 *>(st + kTmaVec * 16)[vl];
                    const float4 *e = reinterpret_cast<const float4 *>(st + kTmaVec * 32);
                    ea[u] = e[2 * vl];
                    eb[u] = e[2 * vl + 1];
                } else {
                    xv[u] = bv[u] = make_uint4(0, 0, 0, 0);
                    ea[u] = eb[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->empty[s]);

            uint4 *B = static_cast<uint4 *>(S.base);
            float4 *E = reinterpret_cast<float4 *>(S.err);
            Word *codes = reinterpret_cast<Word *>(S.codes);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int vl = tid + u * kTmaConsumers;
                const bool valid = vl < nv;
                const int64_t v = v0 + vl;
                float xf[8], bf[8], a[8];
                unpack8(xv[u], xf);
                unpack8(bv[u], bf);
                const float e[8] = {ea[u].x, ea[u].y, ea[u].z, ea[u].w, eb[u].x, eb[u].y, eb[u].z, eb[u].w};
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = __fadd_rn(__fsub_rn(xf[j], bf[j]), e[j]);
                bool nonfinite;
                float sc = group_scale<K, G, SS>(a, nonfinite);
                const bool zero = nonfinite || !(sc >= kScaleMin);
                if (zero) sc = 0.0f;
                if (nonfinite && valid) atomicOr(p.status, kStatusNonfinite);
                uint32_t word = 0;
                if constexpr (K >= 2) {
                    const float inv = __fdiv_rn((float)L, zero ? 1.0f : sc);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        int q = __float2int_rn(__fmul_rn(a[j], inv));
                        q = min(max(q, -L), L);
                        const int c = zero ? L : q + L;
                        word |= (uint32_t)c << (K * j);
                        a[j] = __fsub_rn(a[j], __fmul_rn(lut[c], sc));
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const bool pos = zero || (a[j] >= 0.0f);
                        word |= (uint32_t)pos << j;
                        a[j] = __fsub_rn(a[j], pos ? sc : -sc);
                    }
                }
                if (valid) {
                    __stcs(B + v, xv[u]);
                    __stcs(E + 2 * v, make_float4(a[0], a[1], a[2], a[3]));
                    __stcs(E + 2 * v + 1, make_float4(a[4], a[5], a[6], a[7]));
                    codes[v] = (Word)word;
                    if ((lane & (LPG - 1)) == 0) S.scales[v / LPG] = sc;
                }
            }
        } else {
            // codes and scales do not go through the stage: load them first
            const Word *codes = reinterpret_cast<const Word *>(S.codes);
            Word cw[2];
            float sv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int vl = tid + u * kTmaConsumers;
                if (vl < nv) {
                    cw[u] = __ldcs(codes + v0 + vl);
                    sv[u] = __ldcs(S.scales + (v0 + vl) / LPG);
                } else {
                    cw[u] = 0;
                    sv[u] = 0.0f;
                }
            }
            bool ok = wait_bounded(&bar->full[s], ph, abort_flag, p.status, kQuantWaitNs);
            if (!__all_sync(kFull, ok)) break;
            float4 ca[2], cb[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int vl = tid + u * kTmaConsumers;
                if (vl < nv) {
                    const float4 *c = reinterpret_cast<const float4 *>(st);
                    ca[u] = c[2 * vl];
                    cb[u] = c[2 * vl + 1];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->empty[s]);
            float4 *C = reinterpret_cast<float4 *>(S.cache);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int vl = tid + u * kTmaConsumers;
                if (vl < nv) {
                    const int64_t v = v0 + vl;
                    const uint32_t w = cw[u];
                    const float sc = sv[u];
                    float d[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t c = (w >> (K * j)) & ((1u << K) - 1u);
                        if constexpr (K >= 2)
                            d[j] = __fmul_rn(lut[c], sc);
                        else
                            d[j] = c ? sc : -sc;
                    }
                    const float4 a = ca[u], b = cb[u];
                    __stcs(C + 2 * v, make_float4(__fadd_rn(a.x, d[0]), __fadd_rn(a.y, d[1]), __fadd_rn(a.z, d[2]),
                                                  __fadd_rn(a.w, d[3])));
                    __stcs(C + 2 * v + 1, make_float4(__fadd_rn(b.x, d[4]), __fadd_rn(b.y, d[5]),
                                                      __fadd_rn(b.z, d[6]), __fadd_rn(b.w, d[7])));
                }
            }
        }
    }
}

using KernelFn = void (*)(QuantLaunch);

template <QuantOp OP, int K, int SS, bool TMA>
KernelFn pick_group(int group)
{
    if constexpr (TMA) {
        static_assert(OP == QuantOp::Compress || OP == QuantOp::Decompress, "TMA staging covers compress/decompress");
        switch (group) {
        case 8: return k_quant_tma<OP, K, 8, SS>;
        case 16: return k_quant_tma<OP, K, 16, SS>;
        case 32: return k_quant_tma<OP, K, 32, SS>;
        case 64: return k_quant_tma<OP, K, 64, SS>;
        case 128: return k_quant_tma<OP, K, 128, SS>;
        case 256: return k_quant_tma<OP, K, 256, SS>;
        default: return nullptr;
        }
    } else {
        switch (group) {
        case 8: return k_quant<OP, K, 8, SS>;
        case 16: return k_quant<OP, K, 16, SS>;
        case 32: return k_quant<OP, K, 32, SS>;
        case 64: return k_quant<OP, K, 64, SS>;
        case 128: return k_quant<OP, K, 128, SS>;
        case 256: return k_quant<OP, K, 256, SS>;
        default: return nullptr;
        }
    }
}

template <bool TMA>
KernelFn pick(QuantOp op, int bits, int group, int ss)
{
    switch (op) {
    case QuantOp::WarmupSender: return k_quant<QuantOp::WarmupSender, 2, 8, 0>;
    case QuantOp::WarmupReceiver: return k_quant<QuantOp::WarmupReceiver, 2, 8, 0>;
    case QuantOp::Compress:
        if (bits == 1)
            return ss ? pick_group<QuantOp::Compress, 1, 1, TMA>(group) : pick_group<QuantOp::Compress, 1, 0, TMA>(group);
        if (bits == 2) return pick_group<QuantOp::Compress, 2, 0, TMA>(group);
        if (bits == 4) return pick_group<QuantOp::Compress, 4, 0, TMA>(group);
        return nullptr;
    case QuantOp::Loopback:
        if (bits == 1)
            return ss ? pick_group<QuantOp::Loopback, 1, 1, false>(group) : pick_group<QuantOp::Loopback, 1, 0, false>(group);
        if (bits == 2) return pick_group<QuantOp::Loopback, 2, 0, false>(group);
        if (bits == 4) return pick_group<QuantOp::Loopback, 4, 0, false>(group);
        return nullptr;
    case QuantOp::Decompress:
        if (bits == 1) return pick_group<QuantOp::Decompress, 1, 0, TMA>(group);
        if (bits == 2) return pick_group<QuantOp::Decompress, 2, 0, TMA>(group);
        if (bits == 4) return pick_group<QuantOp::Decompress, 4, 0, TMA>(group);
        return nullptr;
    }
    return nullptr;
}

// Launch shape of one kernel instance: threads, dynamic shared memory and
// resident CTAs per SM (cached; the attribute call raises the dynamic shared
// memory limit of the TMA-staged instances once).
struct Shape {
    int threads;
    size_t smem;
    int per_sm;
};

Shape launch_shape(KernelFn fn, bool tma, QuantOp op)
{
    static std::mutex mu;
    static std::unordered_map<const void *, Shape> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find((const void *)fn);
    if (it != cache.end()) return it->second;
    Shape sh{0, 0, 1};
    int cap = 0;
    switch (op) {
    case QuantOp::WarmupSender:
        sh.threads = QShape<QuantOp::WarmupSender>::kThreads;
        cap = QShape<QuantOp::WarmupSender>::kMaxPerSm;
        break;
    case QuantOp::WarmupReceiver:
        sh.threads = QShape<QuantOp::WarmupReceiver>::kThreads;
        cap = QShape<QuantOp::WarmupReceiver>::kMaxPerSm;
        break;
    case QuantOp::Compress:
        sh.threads = QShape<QuantOp::Compress>::kThreads;
        cap = QShape<QuantOp::Compress>::kMaxPerSm;
        break;
    case QuantOp::Decompress:
        sh.threads = QShape<QuantOp::Decompress>::kThreads;
        cap = QShape<QuantOp::Decompress>::kMaxPerSm;
        break;
    case QuantOp::Loopback:
        sh.threads = QShape<QuantOp::Loopback>::kThreads;
        cap = QShape<QuantOp::Loopback>::kMaxPerSm;
        break;
    }
    if (tma) {
        sh.threads = kTmaThreads;
        sh.smem = op == QuantOp::Compress ? tma_smem_bytes<QuantOp::Compress>() : tma_smem_bytes<QuantOp::Decompress>();
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh.smem);
    }
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, sh.threads, sh.smem) != cudaSuccess || nb < 1) nb = 1;
    sh.per_sm = (!tma && cap > 0 && nb > cap) ? cap : nb;
    cache[(const void *)fn] = sh;
    return sh;
}

// Staging of the compress / decompress streams: "tma" (bulk-async copies
// through shared memory) or "reg" (vector loads straight into registers).
bool use_tma_staging()
{
    static int v = -1;
    if (v < 0) {
        const char *e = getenv("CF_QUANT_STAGING");
        v = (e && strcmp(e, "tma") == 0) ? 1 : 0;
    }
    return v == 1;
}

}  // namespace

int num_sms()
{
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 1;
    }
    return sms;
}

cudaError_t launch_quant(QuantOp op, int bits, int group, int sign_scale, QuantLaunch &lp, cudaStream_t stream)
{
    const bool tma = use_tma_staging() && (op == QuantOp::Compress || op == QuantOp::Decompress);
    KernelFn fn = tma ? pick<true>(op, bits, group, sign_scale) : pick<false>(op, bits, group, sign_scale);
    if (!fn) return cudaErrorInvalidValue;
    // tile prefix of every slot, in this kernel's tile size
    int64_t tile_vec = kTmaVec;
    if (!tma) {
        switch (op) {
        case QuantOp::WarmupSender: tile_vec = qtile_vec<QuantOp::WarmupSender>(); break;
        case QuantOp::WarmupReceiver: tile_vec = qtile_vec<QuantOp::WarmupReceiver>(); break;
        case QuantOp::Compress: tile_vec = qtile_vec<QuantOp::Compress>(); break;
        case QuantOp::Decompress: tile_vec = qtile_vec<QuantOp::Decompress>(); break;
        case QuantOp::Loopback: tile_vec = qtile_vec<QuantOp::Loopback>(); break;
        }
    }
    int64_t tiles = 0;
    for (int k = 0; k < lp.nslots; ++k) {
        lp.slot[k].tile0 = tiles;
        tiles += (lp.slot[k].nvec + tile_vec - 1) / tile_vec;
    }
    lp.ntiles = tiles;
    if (tiles <= 0) return cudaSuccess;
    const Shape sh = launch_shape(fn, tma, op);
    const int64_t cap = (int64_t)num_sms() * sh.per_sm;
    const int grid = (int)(tiles < cap ? tiles : cap);
    fn<<<grid, sh.threads, sh.smem, stream>>>(lp);
    return cudaGetLastError();
}

}  // namespace cf
