// cf_attention.cu -- attention over a received K/V shard, with K and V read
// either as bf16 or straight from the receiver's codec state.
//
// "Accelerating Parallel Diffusion Model Serving with Residual Compression"
// (arXiv 2507.17511), reproducibility table, "Pseudocode" row, Algorithms 1
// and 2: every device attends with its own queries over the key/value blocks
// of the other devices, which reach it compressed (all-gathered for patch
// parallelism, passed round a ring for ring attention).  The receiver of such
// a block keeps the reconstruction C of each K or V slot and adds the
// decompressed residual of every step to it (abstract: residual compression
// with error feedback).
//
// Per head h (channels [64 h, 64 h + 64) of the token-major [rows x cols]
// layout of the codec):  O_h = softmax(Q_h K_h^T / 8) V_h.  K and V come in one
// of two forms:
//   * bf16 -- e.g. the receiver's recon, bf16(C_t), written by cf_decompress
//     in the same pass as C_t;
//   * dequantise-on-load -- the receiver's fp32 cache C_{t-1} plus this step's
//     codes and scales: the loader forms C_t = C_{t-1} + deq(code, scale) with
//     the decompress arithmetic (one binary32 multiply and one add, round to
//     nearest even), rounds it to bf16 for the tensor cores, and the CTAs of
//     the first query block write C_t to cache_out, so no separate decompress
//     runs.  The two forms give bit-identical outputs.
//
// One CTA per (128-query block, head), 8 warps (two per SM sub-partition, so
// that a thread may hold up to 255 registers):
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t); online
//              softmax in base 2 over 128-key blocks, P written to shared
//              memory in bf16, O rescaled in TMEM;
//   warp 4     allocates TMEM (S: 128 columns, O: 64) and issues
//              tcgen05.mma.kind::f16 (bf16 operands, fp32 accumulators):
//              S = Q K^T, then O += P V;
//   warps 5-7  load Q once, then K and V blocks into a two-deep ring
//              (K-major, 128-byte swizzle; V transposed in registers so that
//              every operand is K-major).
// Every mbarrier wait is bounded; on expiry the CTA raises an abort flag and
// the status word's timeout bit, drains its MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include <mutex>

#include "cf_internal.h"
#include "cf_ptx.cuh"
#include "cf_tc.cuh"

namespace cf {
namespace {

using namespace ptx;
using namespace tc;

constexpr int kHeadDim = 64;
constexpr int kBlockQ = 128;           // queries per CTA (MMA M)
constexpr int kBlockK = 128;           // keys per block (S's N, PV's K)
constexpr int kAttnThreads = 256;      // 8 warps
constexpr int kLoaders = 96;           // warps 5-7
constexpr int kRing = 2;               // K/V blocks in flight
constexpr int kTileBytes = 128 * kHeadDim * 2;   // a 128 x 64 bf16 tile: 16 KB
constexpr uint64_t kAttnWaitNs = 2000000000ull;

struct AttnSmem {
    uint64_t q_full;
    uint64_t ld_full[kRing];
    uint64_t ld_free[kRing];
    uint64_t s_full;
    uint64_t s_free;
    uint64_t p_full;
    uint64_t pv_done;
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    float lut[16];
};

struct AttnParams {
    const uint16_t *q;            // bf16 [lq x cols]
    const uint16_t *kv[2];        // bf16 [lk x cols] (form 0)
    const float *cache_in[2];     // fp32 [lk x cols] (form 1)
    float *cache_out[2];          // fp32 [lk x cols] or null (form 1)
    const uint8_t *codes[2];      // k-bit stream (form 1)
    const float *scales[2];       // fp32 per group (form 1)
    uint16_t *out;                // bf16 [lq x cols]
    int lq, lk, cols;
    int group;
    float scale_log2;             // log2(e) / sqrt(64)
    uint32_t *status;
    unsigned long long wait_ns;
};

// Byte offset of 16-byte piece `chunk` (0..7) of row `row` in a [rows x 64]
// bf16 tile stored K-major with the 128-byte swizzle (8-row groups of 1 KB).
__device__ __forceinline__ uint32_t sw128(int row, int chunk)
{
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M = 128.
__device__ __forceinline__ uint32_t instr_desc_bf16(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBlockQ >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, kLayoutSw128); }

// A bounded wait whose outcome is the same for every lane of the warp, so that
// the warp never splits across the .sync.aligned tcgen05 instructions after it.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *status,
                                          unsigned long long ns)
{
    const bool ok = wait_bounded(bar, parity, abort_flag, status, ns);
    return __all_sync(0xffffffffu, ok);
}

// Eight consecutive channels of K or V at flat element index i0 (a multiple
// of 8), as four bf16 pairs.  FORM 0 reads bf16; FORM 1 forms C + deq as the
// receiver's decompress does and, when `wb` is set, writes it to cache_out.
template <int FORM, int K>
__device__ __forceinline__ void load8(const AttnParams &p, int which, int64_t i0, bool wb, const float *lut,
                                      uint32_t (&w)[4])
{
    if constexpr (FORM == 0) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.kv[which] + i0));
        w[0] = v.x;
        w[1] = v.y;
        w[2] = v.z;
        w[3] = v.w;
    } else {
        const int64_t v8 = i0 >> 3;
        uint32_t code;
        if constexpr (K == 4)
            code = __ldg(reinterpret_cast<const uint32_t *>(p.codes[which]) + v8);
        else if constexpr (K == 2)
            code = __ldg(reinterpret_cast<const uint16_t *>(p.codes[which]) + v8);
        else
            code = __ldg(p.codes[which] + v8);
        const float s = __ldg(p.scales[which] + i0 / p.group);
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p.cache_in[which] + i0));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(p.cache_in[which] + i0) + 1);
        const float cin[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float c[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t cj = (code >> (K * j)) & ((1u << K) - 1u);
            const float d = (K >= 2) ? __fmul_rn(lut[cj], s) : (cj ? s : -s);
            c[j] = __fadd_rn(cin[j], d);
        }
        if (wb) {
            float4 *o = reinterpret_cast<float4 *>(p.cache_out[which] + i0);
            o[0] = make_float4(c[0], c[1], c[2], c[3]);
            o[1] = make_float4(c[4], c[5], c[6], c[7]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = bf16x2(c[2 * j], c[2 * j + 1]);
    }
}

template <int FORM, int K>
__global__ void __launch_bounds__(kAttnThreads, 1) k_attention(const __grid_constant__ AttnParams p)
{
    extern __shared__ __align__(1024) uint8_t attn_smem[];
    uint8_t *base = (uint8_t *)(((uintptr_t)attn_smem + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = base;                                    // [128 x 64] bf16
    uint8_t *sK = sQ + kTileBytes;                         // kRing x [128 keys x 64]
    uint8_t *sV = sK + kRing * kTileBytes;                 // kRing x 2 x [64 dims x 64 keys] (V transposed)
    uint8_t *sP = sV + kRing * kTileBytes;                 // 2 x [128 queries x 64 keys]
    AttnSmem *S = reinterpret_cast<AttnSmem *>(sP + 2 * kTileBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = blockIdx.x, head = blockIdx.y;
    const int q0 = qb * kBlockQ;
    const int nkb = (p.lk + kBlockK - 1) / kBlockK;
    const int col0 = head * kHeadDim;

    if (threadIdx.x == 0) {
        mbar_init(&S->q_full, kLoaders);
        for (int b = 0; b < kRing; ++b) {
            mbar_init(&S->ld_full[b], kLoaders);
            mbar_init(&S->ld_free[b], 1);
        }
        mbar_init(&S->s_full, 1);
        mbar_init(&S->s_free, 128);
        mbar_init(&S->p_full, 128);
        mbar_init(&S->pv_done, 1);
        mbar_init(&S->drain, 1);
        S->abort_flag = 0;
        mbar_init_fence();
    }
    if (threadIdx.x < 16) {
        const int L = (1 << (K - 1)) - 1;
        S->lut[threadIdx.x] = (K >= 2) ? __fdiv_rn((float)((int)threadIdx.x - L), (float)L) : 0.0f;
    }
    if (warp == 4) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S->tmem_base)),
                     "r"(256)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    const uint32_t tS = tmem, tO = tmem + 128;   // S: columns 0..127, O: 128..191
    volatile int *abort_flag = &S->abort_flag;
    const unsigned long long wait_ns = p.wait_ns;

    if (warp >= 5) {
        // ------------------------------------------------------- loaders --
        const int lt = threadIdx.x - 160;   // 0..kLoaders-1
        // Q: 128 rows x 8 pieces; rows past lq are zero
        for (int u = lt; u < kBlockQ * 8; u += kLoaders) {
            const int row = u >> 3, ch = u & 7;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (q0 + row < p.lq) v = __ldg(reinterpret_cast<const uint4 *>(p.q + (int64_t)(q0 + row) * p.cols + col0 + 8 * ch));
            *reinterpret_cast<uint4 *>(sQ + sw128(row, ch)) = v;
        }
        fence_proxy_async();
        mbar_arrive(&S->q_full);
        const bool wb = FORM == 1 && qb == 0;
        for (int j = 0; j < nkb; ++j) {
            const int b = j % kRing;
            if (j >= kRing && !warp_wait(&S->ld_free[b], (uint32_t)((j / kRing) - 1) & 1u, abort_flag, p.status, wait_ns))
                break;
            const int k0 = j * kBlockK;
            uint8_t *tk = sK + b * kTileBytes;
            uint8_t *tv = sV + b * kTileBytes;
            // K: 128 keys x 8 pieces of 8 channels, K-major as loaded
            for (int u = lt; u < kBlockK * 8; u += kLoaders) {
                const int row = u >> 3, ch = u & 7;
                uint32_t w[4] = {0u, 0u, 0u, 0u};
                if (k0 + row < p.lk) load8<FORM, K>(p, 0, (int64_t)(k0 + row) * p.cols + col0 + 8 * ch, wb, S->lut, w);
                *reinterpret_cast<uint4 *>(tk + sw128(row, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            // V: 8-key x 8-channel blocks, transposed in registers so that V^T
            // (channels x keys) is K-major like the other operands
            for (int bi = lt; bi < (kBlockK / 8) * 8; bi += kLoaders) {
                const int kg = bi >> 3, dg = bi & 7;    // keys 8 kg .. 8 kg + 7, channels 8 dg .. 8 dg + 7
                uint32_t in[8][4];
#pragma unroll
                for (int r = 0; r < 8; ++r) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) in[r][c] = 0u;
                    const int key = k0 + 8 * kg + r;
                    if (key < p.lk) load8<FORM, K>(p, 1, (int64_t)key * p.cols + col0 + 8 * dg, wb, S->lut, in[r]);
                }
                uint8_t *blk = tv + (kg >> 3) * (kTileBytes / 2);   // keys 0-63 or 64-127 of the block
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t sel = (c & 1) ? 0x7632u : 0x5410u;
                    uint4 o;
                    o.x = __byte_perm(in[0][c >> 1], in[1][c >> 1], sel);
                    o.y = __byte_perm(in[2][c >> 1], in[3][c >> 1], sel);
                    o.z = __byte_perm(in[4][c >> 1], in[5][c >> 1], sel);
                    o.w = __byte_perm(in[6][c >> 1], in[7][c >> 1], sel);
                    *reinterpret_cast<uint4 *>(blk + sw128(8 * dg + c, kg & 7)) = o;
                }
            }
            fence_proxy_async();
            mbar_arrive(&S->ld_full[b]);
        }
    } else if (warp == 4) {
        // ---------------------------------------------------- MMA issuer --
        const uint32_t idS = instr_desc_bf16(kBlockK), idO = instr_desc_bf16(kHeadDim);
        const uint32_t aQ = smem_u32(sQ);
        bool ok = warp_wait(&S->q_full, 0u, abort_flag, p.status, wait_ns) &&
                  warp_wait(&S->ld_full[0], 0u, abort_flag, p.status, wait_ns);
        if (ok) {
            tc_fence_after();
            if (lane == 0) {
                const uint32_t bK = smem_u32(sK);
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) mma_bf16(tS, kdesc(aQ + 32 * kk), kdesc(bK + 32 * kk), idS, kk > 0);
                tc_commit(&S->s_full);
            }
            __syncwarp();
        }
        for (int j = 0; j < nkb && ok; ++j) {
            if (j + 1 < nkb) {
                const int b1 = (j + 1) % kRing;
                ok = warp_wait(&S->ld_full[b1], (uint32_t)((j + 1) / kRing) & 1u, abort_flag, p.status, wait_ns) &&
                     warp_wait(&S->s_free, (uint32_t)j & 1u, abort_flag, p.status, wait_ns);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t bK = smem_u32(sK + b1 * kTileBytes);
#pragma unroll
                    for (int kk = 0; kk < kHeadDim / 16; ++kk)
                        mma_bf16(tS, kdesc(aQ + 32 * kk), kdesc(bK + 32 * kk), idS, kk > 0);
                    tc_commit(&S->s_full);
                }
                __syncwarp();
            }
            ok = warp_wait(&S->p_full, (uint32_t)j & 1u, abort_flag, p.status, wait_ns);
            if (!ok) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t aP = smem_u32(sP), bV = smem_u32(sV + (j % kRing) * kTileBytes);
#pragma unroll
                for (int kk = 0; kk < kBlockK / 16; ++kk) {
                    const uint32_t half = (uint32_t)(kk >> 2), off = 32u * (uint32_t)(kk & 3);
                    mma_bf16(tO, kdesc(aP + half * kTileBytes + off), kdesc(bV + half * (kTileBytes / 2) + off), idO,
                             (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&S->pv_done);
                tc_commit(&S->ld_free[j % kRing]);
            }
            __syncwarp();
        }
        // Drain: every MMA this thread issued has completed before TMEM is freed.
        if (lane == 0) {
            tc_commit(&S->drain);
            volatile int no_abort = 0;
            wait_bounded(&S->drain, 0u, &no_abort, p.status, kAttnWaitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- softmax --
        const int row = threadIdx.x;                        // query row of this thread = TMEM lane
        const uint32_t lanebase = (uint32_t)(32 * warp) << 16;
        float m = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            if (!warp_wait(&S->s_full, (uint32_t)j & 1u, abort_flag, p.status, wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kBlockK];
#pragma unroll
            for (int c = 0; c < kBlockK; c += 16) {
                uint32_t v[16];
                tc_ld16(tS + lanebase + (uint32_t)c, v);
                tc_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) s[c + e] = __uint_as_float(v[e]);
            }
            tc_fence_before();
            mbar_arrive(&S->s_free);
            // scores in base 2; keys past lk do not count
            const int kvalid = p.lk - j * kBlockK;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kBlockK; ++c) {
                s[c] = c < kvalid ? s[c] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[c]);
            }
            const float m_new = fmaxf(m, mx);
            const float alpha = exp2f(m - m_new);     // 0 on the first block (m = -inf)
            float sum = 0.0f;
#pragma unroll
            for (int c = 0; c < kBlockK; ++c) {
                s[c] = exp2f(s[c] - m_new);
                sum += s[c];
            }
            l = l * alpha + sum;
            m = m_new;
            uint32_t pw[kBlockK / 2];   // P in bf16 pairs: half the registers across the wait below
#pragma unroll
            for (int c = 0; c < kBlockK; c += 2) pw[c >> 1] = bf16x2(s[c], s[c + 1]);
            if (j > 0) {
                // P and O are free once the previous block's P V has completed
                if (!warp_wait(&S->pv_done, (uint32_t)(j - 1) & 1u, abort_flag, p.status, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
#pragma unroll
            for (int c = 0; c < kBlockK; c += 8) {
                const uint4 w = make_uint4(pw[c >> 1], pw[(c >> 1) + 1], pw[(c >> 1) + 2], pw[(c >> 1) + 3]);
                *reinterpret_cast<uint4 *>(sP + (c >> 6) * kTileBytes + sw128(row, (c & 63) >> 3)) = w;
            }
            if (j > 0) {
#pragma unroll
                for (int c = 0; c < kHeadDim; c += 16) {
                    uint32_t v[16];
                    tc_ld16(tO + lanebase + (uint32_t)c, v);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                    tmem_st16(tO + lanebase + (uint32_t)c, v);
                }
                tmem_wait_st();
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&S->p_full);
        }
        if (ok && warp_wait(&S->pv_done, (uint32_t)(nkb - 1) & 1u, abort_flag, p.status, wait_ns)) {
            tc_fence_after();
            const float inv = 1.0f / l;
            uint32_t o[kHeadDim / 2];
#pragma unroll
            for (int c = 0; c < kHeadDim; c += 16) {
                uint32_t v[16];
                tc_ld16(tO + lanebase + (uint32_t)c, v);
                tc_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; e += 2)
                    o[(c + e) >> 1] = bf16x2(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv);
            }
            if (q0 + row < p.lq) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (int64_t)(q0 + row) * p.cols + col0);
#pragma unroll
                for (int c = 0; c < kHeadDim / 8; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 4) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256) : "memory");
    }
}

constexpr size_t kAttnSmemBytes = 1024 + (size_t)(1 + 2 * kRing + 2) * kTileBytes + sizeof(AttnSmem);
static_assert(kAttnSmemBytes <= 227 * 1024, "attention shared memory exceeds 227 KB");

template <int FORM, int K>
cudaError_t attn_launch_k(const AttnParams &p, cudaStream_t stream)
{
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64 || !done[dev]) {
            e = cudaFuncSetAttribute(k_attention<FORM, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kAttnSmemBytes);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) done[dev] = true;
        }
    }
    const dim3 grid((unsigned)((p.lq + kBlockQ - 1) / kBlockQ), (unsigned)(p.cols / kHeadDim));
    const char *name = FORM == 0 ? "k_attention<bf16>" : "k_attention<dequantise>";
    log_launch(name, grid, dim3(kAttnThreads), kAttnSmemBytes);
    trace_begin(name, stream);
    k_attention<FORM, K><<<grid, kAttnThreads, kAttnSmemBytes, stream>>>(p);
    trace_end(stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs &a, cudaStream_t stream)
{
    AttnParams p{};
    p.q = static_cast<const uint16_t *>(a.q);
    for (int i = 0; i < 2; ++i) {
        p.kv[i] = static_cast<const uint16_t *>(a.kv[i]);
        p.cache_in[i] = a.cache_in[i];
        p.cache_out[i] = a.cache_out[i];
        p.codes[i] = a.codes[i];
        p.scales[i] = a.scales[i];
    }
    p.out = static_cast<uint16_t *>(a.out);
    p.lq = (int)a.lq;
    p.lk = (int)a.lk;
    p.cols = (int)a.cols;
    p.group = a.group;
    p.scale_log2 = 1.4426950408889634f / 8.0f;   // log2(e) / sqrt(64)
    p.status = a.status;
    p.wait_ns = kAttnWaitNs;
    if (!a.dequantise) return attn_launch_k<0, 2>(p, stream);
    switch (a.bits) {
    case 1: return attn_launch_k<1, 1>(p, stream);
    case 2: return attn_launch_k<1, 2>(p, stream);
    default: return attn_launch_k<1, 4>(p, stream);
    }
}

}  // namespace cf
