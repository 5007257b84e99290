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
#include <stdio.h>

#include <mutex>
#include <unordered_map>

#include "cf_internal.h"

namespace cf {
namespace {

// Launch shape per operation (and, for the fp32-state sender and receiver,
// per code width k): threads per CTA, vectors (of 8 elements) each thread
// keeps in flight (a tile is threads * unroll vectors), and a cap on resident
// CTAs per SM (0: as many as fit).  Chosen by sweeps on the B200 over
// 128..1024 threads (in steps of one or two warps near the optimum), 1..16
// vectors and 1..4 CTAs per SM on the 57-slot FLUX-shaped (k = 2), 30-slot
// CogVideoX-shaped (k = 4) and 60-slot stress (k = 1) steps, as a fraction
// of the measured copy bandwidth:
//   compress   k = 2: 256 x 8 at 1 CTA/SM, 95.2% (1024 x 1: 93.4%; 224 x 8: 90.1%;
//                     288 x 8: 86.6%; 256 x 7: 94.3%)
//              k = 4: 512 x 2, 94.0% (1024 x 1: 89.5%; 256 x 8: 91.4%; 256 x 6: 94.1%)
//              k = 1: 512 x 2, 93.3% (1024 x 1: 89.3%; 256 x 7: 91.3%)
//   decompress k = 2, 4: 448 x 4 at 1 CTA/SM, 98.9% / 97.5% (512 x 4: 94.9% / 93.5%;
//                     416 x 4: 97.2% / 97.2%; 480 x 4: 98.4% / 95.2%; 448 x 5: 94.1% / 92.4%)
//              k = 1: 256 x 8, 98.9% (512 x 4: 89.1%; 448 x 4: 95.6%)
// More resident CTAs per SM, i.e. more concurrent streams into HBM, were
// slower in every case.
template <QuantOp OP, bool LEAN = false>
struct QShapeBase {
    static constexpr int kThreads = 256;
    static constexpr int kUnroll = 4;
    static constexpr int kMaxPerSm = 0;
};
// Warmup step (fp32 state), once per run: sender 384 x 4 (94.2% / 94.5% of the
// copy bandwidth on the FLUX- / CogVideoX-shaped steps; 256 x 4 uncapped:
// 82.3% / 82.6%), receiver 512 x 4 (90.9% / 92.8%; 256 x 4: 72.9% / 73.1%).
template <>
struct QShapeBase<QuantOp::WarmupSender, false> {
    static constexpr int kThreads = 384;
    static constexpr int kUnroll = 4;
    static constexpr int kMaxPerSm = 1;
};
template <>
struct QShapeBase<QuantOp::WarmupReceiver, false> {
    static constexpr int kThreads = 512;
    static constexpr int kUnroll = 4;
    static constexpr int kMaxPerSm = 1;
};
template <>
struct QShapeBase<QuantOp::Compress, false> {
    static constexpr int kThreads = 1024;
    static constexpr int kUnroll = 1;
    static constexpr int kMaxPerSm = 1;   // 2 CTAs of 1024 fit at 32 registers, and are slower
};
template <>
struct QShapeBase<QuantOp::Loopback, false> {
    // fused sender + receiver (9 streams per tile); per-width shapes below
    static constexpr int kThreads = 384;
    static constexpr int kUnroll = 3;
    static constexpr int kMaxPerSm = 1;
};
template <>
struct QShapeBase<QuantOp::Decompress, false> {
    static constexpr int kThreads = 448;
    static constexpr int kUnroll = 4;
    static constexpr int kMaxPerSm = 1;
};
// Lean state (bf16 E and C): half the state bytes per vector, so each thread
// wants more vectors in flight (sweep on the same workload).
template <>
struct QShapeBase<QuantOp::Compress, true> {
    static constexpr int kThreads = 1024;
    static constexpr int kUnroll = 2;
    static constexpr int kMaxPerSm = 1;
};
template <>
struct QShapeBase<QuantOp::Loopback, true> {
    static constexpr int kThreads = 256;
    static constexpr int kUnroll = 8;
    static constexpr int kMaxPerSm = 1;
};
// (896 x 4: 95.1% / 95.1% / 97.3% on the k = 2 / 4 / 1 steps; 1024 x 4: 95.1% /
// 90.7% / 91.4%; 640 x 6: 91.5% / 94.8% / 96.7%)
template <>
struct QShapeBase<QuantOp::Decompress, true> {
    static constexpr int kThreads = 896;
    static constexpr int kUnroll = 4;
    static constexpr int kMaxPerSm = 1;
};
template <QuantOp OP, bool LEAN, int K>
struct QShape : QShapeBase<OP, LEAN> {};
template <int T, int U>
struct QShapeOne {
    static constexpr int kThreads = T;
    static constexpr int kUnroll = U;
    static constexpr int kMaxPerSm = 1;
};
template <>
struct QShape<QuantOp::Compress, false, 2> : QShapeOne<256, 8> {};
template <>
struct QShape<QuantOp::Compress, false, 4> : QShapeOne<512, 2> {};
template <>
struct QShape<QuantOp::Compress, false, 1> : QShapeOne<512, 2> {};
template <>
struct QShape<QuantOp::Decompress, false, 1> : QShapeOne<256, 8> {};
// Loopback (sender and receiver of a step in one kernel): 384 x 3 for k = 2
// and k = 4 (95.4% / 93.4%; 256 x 4: 94.9% / 89.8%; 320 x 4: 93.7% / 91.1%;
// 448 x 3: 91.1% / 88.7%), 256 x 6 for k = 1 (92.7%; 384 x 3: 92.1%); the
// shape is sensitive (256 x 3: 79.7% for k = 2).
template <>
struct QShape<QuantOp::Loopback, false, 1> : QShapeOne<256, 6> {};
// Lean-state sender (bf16 E), steps of the FLUX-, CogVideoX-shaped and stress
// workloads: k = 2 640 x 3 (94.0%; 1024 x 2: 88.3%; 896 x 2: 93.0%; 768 x 3:
// 88.3%; 512 x 3: 89.9%); k = 4 384 x 6 (1024 x 2: 86.6%; 512 x 4: 90.4%;
// 384 x 6: 91.6%); k = 1 256 x 16 (1024 x 2: 86.2%; 256 x 16: 91.2%;
// 256 x 12: 90.6%; 384 x 6: 90.8%).
template <>
struct QShape<QuantOp::Compress, true, 2> : QShapeOne<640, 3> {};
template <>
struct QShape<QuantOp::Compress, true, 4> : QShapeOne<384, 6> {};
template <>
struct QShape<QuantOp::Compress, true, 1> : QShapeOne<256, 16> {};
// Receivers that also write the bf16 reconstruction (RC): one more output
// stream per vector.  The fp32-state receiver with recon runs 384 x 4 (sweep
// on the FLUX- and CogVideoX-shaped steps: 99.0% / 97.8% of the copy
// bandwidth for its 10.28 / 10.56 bytes per element; 512 x 4: 85.1% / 84.2%,
// 256 x 8: 98.6% / 96.5%).
template <QuantOp OP, bool LEAN, int K, bool RC>
struct QShapeR : QShape<OP, LEAN, K> {};
template <int K>
struct QShapeR<QuantOp::Decompress, false, K, true> : QShapeOne<384, 4> {};
template <QuantOp OP, bool LEAN, int K, bool RC>
constexpr int64_t qtile_vec()
{
    return (int64_t)QShapeR<OP, LEAN, K, RC>::kThreads * QShapeR<OP, LEAN, K, RC>::kUnroll;
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

// State vectors (E or C) of 8 elements: fp32 (32 bytes) or, with the lean
// state, bf16 (16 bytes, rounded to nearest even on store).
struct F8 {
    float4 a, b;
};
template <bool LEAN>
struct StateVec {
    using T = F8;
    static __device__ __forceinline__ T load(const void *base, int64_t v)
    {
        const float4 *p = static_cast<const float4 *>(base) + 2 * v;
        return F8{__ldcs(p), __ldcs(p + 1)};
    }
    static __device__ __forceinline__ void unpack(const T &s, float (&f)[8])
    {
        f[0] = s.a.x; f[1] = s.a.y; f[2] = s.a.z; f[3] = s.a.w;
        f[4] = s.b.x; f[5] = s.b.y; f[6] = s.b.z; f[7] = s.b.w;
    }
    static __device__ __forceinline__ T zero() { return F8{make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)}; }
    static __device__ __forceinline__ void store(void *base, int64_t v, const float (&f)[8])
    {
        float4 *p = static_cast<float4 *>(base) + 2 * v;
        __stcs(p, make_float4(f[0], f[1], f[2], f[3]));
        __stcs(p + 1, make_float4(f[4], f[5], f[6], f[7]));
    }
};
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
template <>
struct StateVec<true> {
    using T = uint4;
    static __device__ __forceinline__ T load(const void *base, int64_t v)
    {
        return __ldcs(static_cast<const uint4 *>(base) + v);
    }
    static __device__ __forceinline__ void unpack(const T &s, float (&f)[8]) { unpack8(s, f); }
    static __device__ __forceinline__ T zero() { return make_uint4(0, 0, 0, 0); }
    static __device__ __forceinline__ void store(void *base, int64_t v, const float (&f)[8])
    {
        __stcs(static_cast<uint4 *>(base) + v, make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                          pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
    }
};

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

// RC: the receiver part also writes recon = bf16(C) for every slot whose
// recon pointer is set (instances without RC never touch recon, apart from
// the warmup receiver, which checks the pointer).
template <QuantOp OP, int K, int G, int SS, bool LEAN, bool RC>
__global__ void __launch_bounds__(QShapeR<OP, LEAN, K, RC>::kThreads) k_quant(const __grid_constant__ QuantLaunch p)
{
    using SV = StateVec<LEAN>;
    constexpr int kThreads = QShapeR<OP, LEAN, K, RC>::kThreads;
    constexpr int kUnroll = QShapeR<OP, LEAN, K, RC>::kUnroll;
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
            uint4 xv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) xv[u] = __ldcs(X + v);
            }
            const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    __stcs(B + v, xv[u]);
                    SV::store(S.err, v, z);
                }
            }
        } else if constexpr (OP == QuantOp::WarmupReceiver) {
            const uint4 *X = static_cast<const uint4 *>(S.x);
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
                    SV::store(S.cache, v, f);   // bf16 -> fp32 is exact; fp32 -> bf16 of a bf16 value too
                    if (S.recon) __stcs(static_cast<uint4 *>(S.recon) + v, xv[u]);
                }
            }
        } else if constexpr (OP == QuantOp::Compress || OP == QuantOp::Loopback) {
            // Loopback = sender and receiver on the same device: the receiver's
            // C += d reuses the d the sender just formed (bit-identical to a
            // separate decompress) and the payload is not read back.
            constexpr bool LB = OP == QuantOp::Loopback;
            const uint4 *X = static_cast<const uint4 *>(S.x);
            uint4 *B = static_cast<uint4 *>(S.base);
            Word *codes = reinterpret_cast<Word *>(S.codes);
            float *scales = S.scales;

            uint4 xv[kUnroll], bv[kUnroll];
            typename SV::T ev[kUnroll];
            typename SV::T cv[LB ? kUnroll : 1];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    xv[u] = __ldcs(X + v);
                    bv[u] = __ldcs(B + v);
                    ev[u] = SV::load(S.err, v);
                    if constexpr (LB) cv[u] = SV::load(S.cache, v);
                } else {
                    xv[u] = bv[u] = make_uint4(0, 0, 0, 0);
                    ev[u] = SV::zero();
                    if constexpr (LB) cv[u] = SV::zero();
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                const bool valid = v < nvec;
                // residual against the base tensor plus the carried error
                float xf[8], bf[8], a[8], e[8];
                unpack8(xv[u], xf);
                unpack8(bv[u], bf);
                SV::unpack(ev[u], e);
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
                    SV::store(S.err, v, a);
                    codes[v] = (Word)word;
                    if ((lane & (LPG - 1)) == 0) scales[v / LPG] = s;
                    if constexpr (LB) {
                        float c[8];
                        SV::unpack(cv[u], c);
#pragma unroll
                        for (int j = 0; j < 8; ++j) c[j] = __fadd_rn(c[j], d[j]);
                        SV::store(S.cache, v, c);
                        if (RC && S.recon) StateVec<true>::store(S.recon, v, c);
                    }
                }
            }
        } else if constexpr (!LEAN) {  // Decompress, fp32 cache
            const Word *codes = reinterpret_cast<const Word *>(S.codes);
            const float *scales = S.scales;
            float4 *C = static_cast<float4 *>(S.cache);
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
                    const float c[8] = {__fadd_rn(a.x, d[0]), __fadd_rn(a.y, d[1]), __fadd_rn(a.z, d[2]),
                                        __fadd_rn(a.w, d[3]), __fadd_rn(b.x, d[4]), __fadd_rn(b.y, d[5]),
                                        __fadd_rn(b.z, d[6]), __fadd_rn(b.w, d[7])};
                    __stcs(C + 2 * v, make_float4(c[0], c[1], c[2], c[3]));
                    __stcs(C + 2 * v + 1, make_float4(c[4], c[5], c[6], c[7]));
                    if (RC && S.recon) StateVec<true>::store(S.recon, v, c);
                }
            }
        } else {  // Decompress, bf16 cache (lean state)
            const Word *codes = reinterpret_cast<const Word *>(S.codes);
            const float *scales = S.scales;
            Word cw[kUnroll];
            float sv[kUnroll];
            typename SV::T cv[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + (int64_t)u * kThreads;
                if (v < nvec) {
                    cw[u] = __ldcs(codes + v);
                    sv[u] = __ldcs(scales + v / LPG);
                    cv[u] = SV::load(S.cache, v);
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
                    float c[8];
                    SV::unpack(cv[u], c);
#pragma unroll
                    for (int j = 0; j < 8; ++j) c[j] = __fadd_rn(c[j], d[j]);
                    SV::store(S.cache, v, c);
                    if (RC && S.recon) SV::store(S.recon, v, c);
                }
            }
        }
    }
}

using KernelFn = void (*)(QuantLaunch);

template <QuantOp OP, int K, int SS, bool LEAN, bool RC>
KernelFn pick_group(int group)
{
    switch (group) {
    case 8: return k_quant<OP, K, 8, SS, LEAN, RC>;
    case 16: return k_quant<OP, K, 16, SS, LEAN, RC>;
    case 32: return k_quant<OP, K, 32, SS, LEAN, RC>;
    case 64: return k_quant<OP, K, 64, SS, LEAN, RC>;
    case 128: return k_quant<OP, K, 128, SS, LEAN, RC>;
    case 256: return k_quant<OP, K, 256, SS, LEAN, RC>;
    default: return nullptr;
    }
}

template <QuantOp OP, bool LEAN, bool RC>
KernelFn pick_bits(int bits, int group, int ss)
{
    if (bits == 1) {
        if constexpr (OP == QuantOp::Compress || OP == QuantOp::Loopback)
            if (ss) return pick_group<OP, 1, 1, LEAN, RC>(group);
        return pick_group<OP, 1, 0, LEAN, RC>(group);
    }
    if (bits == 2) return pick_group<OP, 2, 0, LEAN, RC>(group);
    if (bits == 4) return pick_group<OP, 4, 0, LEAN, RC>(group);
    return nullptr;
}

template <bool LEAN>
KernelFn pick(QuantOp op, int bits, int group, int ss, bool rc)
{
    switch (op) {
    case QuantOp::WarmupSender: return k_quant<QuantOp::WarmupSender, 2, 8, 0, LEAN, false>;
    case QuantOp::WarmupReceiver: return k_quant<QuantOp::WarmupReceiver, 2, 8, 0, LEAN, false>;
    case QuantOp::Compress: return pick_bits<QuantOp::Compress, LEAN, false>(bits, group, ss);
    case QuantOp::Decompress:
        return rc ? pick_bits<QuantOp::Decompress, LEAN, true>(bits, group, ss)
                  : pick_bits<QuantOp::Decompress, LEAN, false>(bits, group, ss);
    case QuantOp::Loopback:
        return rc ? pick_bits<QuantOp::Loopback, LEAN, true>(bits, group, ss)
                  : pick_bits<QuantOp::Loopback, LEAN, false>(bits, group, ss);
    }
    return nullptr;
}

// Launch shape of one kernel instance: threads, dynamic shared memory and
// resident CTAs per SM (cached per instance).
struct Shape {
    int threads;
    size_t smem;
    int per_sm;
};

template <QuantOp OP, bool LEAN, int K, bool RC>
void shape_is(int &threads, int &cap, int64_t &tile_vec)
{
    threads = QShapeR<OP, LEAN, K, RC>::kThreads;
    cap = QShapeR<OP, LEAN, K, RC>::kMaxPerSm;
    tile_vec = qtile_vec<OP, LEAN, K, RC>();
}

template <QuantOp OP, bool LEAN, bool RC>
void shape_bits(int bits, int &threads, int &cap, int64_t &tile_vec)
{
    if (bits == 1)
        shape_is<OP, LEAN, 1, RC>(threads, cap, tile_vec);
    else if (bits == 4)
        shape_is<OP, LEAN, 4, RC>(threads, cap, tile_vec);
    else
        shape_is<OP, LEAN, 2, RC>(threads, cap, tile_vec);
}

// The shape of the instance pick() returns: the warmup kernels are the k = 2
// instances.
template <bool LEAN>
void shape_of(QuantOp op, int bits, bool rc, int &threads, int &cap, int64_t &tile_vec)
{
    switch (op) {
    case QuantOp::WarmupSender: shape_is<QuantOp::WarmupSender, LEAN, 2, false>(threads, cap, tile_vec); break;
    case QuantOp::WarmupReceiver: shape_is<QuantOp::WarmupReceiver, LEAN, 2, false>(threads, cap, tile_vec); break;
    case QuantOp::Compress: shape_bits<QuantOp::Compress, LEAN, false>(bits, threads, cap, tile_vec); break;
    case QuantOp::Decompress:
        if (rc)
            shape_bits<QuantOp::Decompress, LEAN, true>(bits, threads, cap, tile_vec);
        else
            shape_bits<QuantOp::Decompress, LEAN, false>(bits, threads, cap, tile_vec);
        break;
    case QuantOp::Loopback:
        if (rc)
            shape_bits<QuantOp::Loopback, LEAN, true>(bits, threads, cap, tile_vec);
        else
            shape_bits<QuantOp::Loopback, LEAN, false>(bits, threads, cap, tile_vec);
        break;
    }
}

Shape launch_shape(KernelFn fn, bool lean, QuantOp op, int bits, bool rc)
{
    static std::mutex mu;
    static std::unordered_map<const void *, Shape> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find((const void *)fn);
    if (it != cache.end()) return it->second;
    Shape sh{0, 0, 1};
    int cap = 0;
    int64_t tile_vec = 0;
    if (lean)
        shape_of<true>(op, bits, rc, sh.threads, cap, tile_vec);
    else
        shape_of<false>(op, bits, rc, sh.threads, cap, tile_vec);
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, sh.threads, sh.smem) != cudaSuccess || nb < 1) nb = 1;
    sh.per_sm = (cap > 0 && nb > cap) ? cap : nb;
    cache[(const void *)fn] = sh;
    return sh;
}

}  // namespace

int num_sms()
{
    // per device (a process may drive several GPUs)
    static std::mutex mu;
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (sms[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        sms[dev] = v > 0 ? v : 1;
    }
    return sms[dev];
}

cudaError_t launch_quant(QuantOp op, int bits, int group, int sign_scale, bool lean, QuantLaunch &lp,
                         cudaStream_t stream)
{
    // the receiver instances that write recon are used when a slot asks for it
    bool rc = false;
    if (op == QuantOp::Decompress || op == QuantOp::Loopback)
        for (int k = 0; k < lp.nslots; ++k) rc = rc || lp.slot[k].recon != nullptr;
    KernelFn fn = lean ? pick<true>(op, bits, group, sign_scale, rc) : pick<false>(op, bits, group, sign_scale, rc);
    if (!fn) return cudaErrorInvalidValue;
    // tile prefix of every slot, in this kernel's tile size
    int threads = 0, cap = 0;
    int64_t tile_vec = 0;
    if (lean)
        shape_of<true>(op, bits, rc, threads, cap, tile_vec);
    else
        shape_of<false>(op, bits, rc, threads, cap, tile_vec);
    int64_t tiles = 0;
    for (int k = 0; k < lp.nslots; ++k) {
        lp.slot[k].tile0 = tiles;
        tiles += (lp.slot[k].nvec + tile_vec - 1) / tile_vec;
    }
    lp.ntiles = tiles;
    if (tiles <= 0) return cudaSuccess;
    const Shape sh = launch_shape(fn, lean, op, bits, rc);
    const int64_t cap_blocks = (int64_t)num_sms() * sh.per_sm;
    const int grid = (int)(tiles < cap_blocks ? tiles : cap_blocks);
    const bool traced = trace_on();
    if (log_enabled() || traced) {
        char name[80];
        snprintf(name, sizeof name, "k_quant<op %d, k %d, G %d, ss %d, %s%s>", (int)op, bits, group, sign_scale,
                 lean ? "bf16 state" : "fp32 state", rc ? ", recon" : "");
        log_launch(name, dim3(grid), dim3(sh.threads), sh.smem);
        if (traced) trace_begin(name, stream);
    }
    fn<<<grid, sh.threads, sh.smem, stream>>>(lp);
    if (traced) trace_end(stream);
    return cudaGetLastError();
}

}  // namespace cf
