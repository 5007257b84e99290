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
// One CTA per (256-query block, head): two 128-query tiles, t = 0 and 1, whose
// softmax work alternates with the other tile's products on the tensor cores.
//   warps 0-3, 4-7  softmax of tile 0, tile 1: thread r of a tile owns query
//              row r (TMEM lane r); online softmax in base 2 over 128-key
//              blocks, P written to tensor memory in bf16; O rescaled in
//              TMEM only when a row's running maximum grows by more than 2^8
//              (otherwise the stale maximum is kept: the normalisation at the
//              end divides by a sum taken against the same maximum).  The two
//              warps of a sub-partition (one per tile) take turns at the
//              exponentials, passing the turn halfway through a block, so one
//              tile's loads and maximum overlap the other's use of the unit.
//              On request each row's log-sum-exp goes to lse (the weight that
//              merges partial results over several received blocks);
//   warp 8(-9) allocates TMEM (S_t: 128 columns each, O_t: 64, P_t: 64) and
//              issues tcgen05.mma.kind::f16 (bf16 operands, fp32
//              accumulators): S_t = Q_t K^T from shared memory, then
//              O_t += P_t V with P_t read from tensor memory.  In the bf16
//              form warps 8 and 9 each issue one tile's products (a single
//              issuing thread, at a few hundred cycles per group of MMAs and
//              commit, would bound the kernel); in the other, warp 8 issues
//              both;
//   the rest   load Q once (TMA), then K and V blocks into a ring shared by
//              both tiles: in the bf16 form by TMA (a [128 x 64] box with the
//              128-byte swizzle lands in the layout the MMA reads); in the
//              other, the fp32 cache rows of 32-key sub-chunks by TMA and
//              their codes and scales by cp.async into a ring of staging
//              slots, three sub-chunks ahead of the one being dequantised
//              and stored swizzled.  Q and K are K-major operands; V is read
//              MN-major (the channels of a key are contiguous), so no operand
//              is transposed.
// Every mbarrier wait is bounded; on expiry the CTA raises an abort flag and
// the status word's timeout bit, drains its MMAs, frees TMEM and returns (a
// test hook, AttnParams::starve, withholds every load to make that happen).
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
constexpr int kBlockQ = 128;           // queries per tile (MMA M)
constexpr int kTiles = 2;              // query tiles per CTA
constexpr int kBlockK = 128;           // keys per block (S's N, PV's K)
constexpr int kMmaWarp = 8;
constexpr int kTileBytes = 128 * kHeadDim * 2;   // a 128 x 64 bf16 tile: 16 KB
constexpr int kMaxRing = 3;
constexpr uint64_t kAttnWaitNs = 2000000000ull;
// Tensor memory columns: S_t at 128 t, O_t at 256 + 64 t, P_t at 384 + 64 t.
constexpr uint32_t kTmemCols = 512;
// Rescale O only when the running maximum grows by more than 2^8 (base 2).
constexpr float kRescaleLog2 = 8.0f;
// Dequantise-on-load staging: sub-chunks of 32 keys (K and V: fp32 cache,
// codes, scales) stream through a ring of kSlots shared-memory slots.
constexpr int kSub = 32;
constexpr int kSlots = 4;
constexpr int kSlotC = 2 * kSub * kHeadDim * 4;     // 16 KB of cache
constexpr int kSlotCodes = 2 * kSub * 32;           // up to 32 code bytes per key row (k = 4)
constexpr int kSlotScales = 2 * kSub * 8 * 4;       // up to 8 scales per key row (G = 8)
constexpr int kSlotBytes = kSlotC + kSlotCodes + kSlotScales;

// Per form: MMA issuer warps (one per tile in the bf16 form, whose issue
// rate would otherwise bound it), loader warps, threads and K/V ring depth.
template <int FORM>
struct AttnCfg {
    static constexpr int kIssuers = FORM == 0 ? 2 : 1;
    static constexpr int kLoader0 = 32 * (kMmaWarp + kIssuers);   // first loader thread
    static constexpr int kLoaders = FORM == 0 ? 32 : 96;
    static constexpr int kThreads = kLoader0 + kLoaders;
    static constexpr int kRing = FORM == 0 ? 3 : 2;
};

struct AttnSmem {
    uint64_t st_full[kSlots];     // staging slot landed (TMA bytes + every loader's cp.async)
    uint64_t st_free[kSlots];     // staging slot read by the three loader warps
    uint64_t q_full;
    uint64_t ld_full[kMaxRing];   // K and V of a block in the ring
    uint64_t ld_free[kMaxRing];   // both tiles' products with that block done
    uint64_t s_full[kTiles];      // S_t computed
    uint64_t s_free[kTiles];      // S_t read by the tile's four softmax warps
    uint64_t p_full[kTiles];      // P_t (and any O_t rescale) in tensor memory
    uint64_t pv_done[kTiles];     // O_t += P_t V complete
    uint64_t turn[kTiles][4];     // per sub-partition: tile t may run its exponentials
    uint64_t drain[kTiles];
    uint32_t tmem_base;
    int abort_flag;
    float lut[16];
};

struct __align__(64) AttnParams {
    CUtensorMap tq;               // Q, bf16 [lq x cols], box 64 x 128
    CUtensorMap tk, tv;           // K, V (bf16 form), same boxes
    CUtensorMap tc[2];            // cache_in of K and V (dequantise form), fp32, box 64 x 32
    const uint16_t *q;            // bf16 [lq x cols]
    const uint16_t *kv[2];        // bf16 [lk x cols] (form 0)
    const float *cache_in[2];     // fp32 [lk x cols] (form 1)
    float *cache_out[2];          // fp32 [lk x cols] or null (form 1)
    const uint8_t *codes[2];      // k-bit stream (form 1)
    const float *scales[2];       // fp32 per group (form 1)
    uint16_t *out;                // bf16 [lq x cols]
    float *lse;                   // fp32 [lq x cols/64] or null
    int lq, lk, cols;
    int group;
    int group_lg;                 // log2(group)
    float scale_log2;             // log2(e) / sqrt(64)
    uint32_t *status;
    unsigned long long wait_ns;
    int starve;                   // failure-detection test: the loaders issue nothing
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

// Instruction descriptor, kind::f16: D fp32, A and B bf16, A K-major, B K-major
// or MN-major (b_mn), M = 128.
__device__ __forceinline__ uint32_t instr_desc_bf16(int n, int b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kBlockQ >> 4) << 24);
}

// 2^x on the special-function unit (ex2.approx: a relative error near 2^-22,
// below the bf16 rounding P gets next).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
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

// The same with the A operand in tensor memory: lane i holds row i of A, and
// each 32-bit column two consecutive K elements (the lower one in the low
// half), so one K = 16 step reads 8 columns.
__device__ __forceinline__ void mma_bf16_ta(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
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

// K-major [rows x 64] bf16 tile, 128-byte swizzle: 8-row groups 1 KB apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t saddr) { return smem_desc(saddr, 16, 1024, kLayoutSw128); }
// MN-major [keys x 64] bf16 tile (V: 64 channels of a key contiguous), 128-byte
// swizzle: one 64-wide atom along N, 8-key groups 1 KB apart along K.  Both
// offsets are 1 KB, so the single N atom reads the same either way.
__device__ __forceinline__ uint64_t vdesc(uint32_t saddr) { return smem_desc(saddr, 1024, 1024, kLayoutSw128); }

// A bounded wait whose outcome is the same for every lane of the warp, so that
// the warp never splits across the .sync.aligned tcgen05 instructions after it.
// The first test is inline (a barrier already past costs one try_wait); only a
// wait that has to spin calls the bounded loop.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *status,
                                          unsigned long long ns)
{
    bool ok = mbar_try_wait(smem_u32(bar), parity);
    if (!ok) ok = wait_bounded(bar, parity, abort_flag, status, ns);
    return __all_sync(0xffffffffu, ok);
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ void cp_async(void *dst, const void *src, int bytes)
{
    if (bytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
    else if (bytes == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Loads from shared memory by 32-bit shared-window address (the staging and
// tile pointers are derived by arithmetic, which would otherwise make them
// generic accesses).
__device__ __forceinline__ float4 lds128(uint32_t a)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a)
{
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t a)
{
    unsigned short v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(a));
    return v & 0xffu;
}
// The mbarrier gets one arrival once this thread's earlier cp.async copies
// have landed (the arrival counts towards the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void sts128(uint32_t a, uint4 v)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int FORM, int K>
__global__ void __launch_bounds__(AttnCfg<FORM>::kThreads, 1) k_attention(const __grid_constant__ AttnParams p)
{
    constexpr int kRing = AttnCfg<FORM>::kRing;
    constexpr int kLoaders = AttnCfg<FORM>::kLoaders;
    extern __shared__ __align__(1024) uint8_t attn_smem[];
    uint8_t *base = (uint8_t *)(((uintptr_t)attn_smem + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = base;                                    // kTiles x [128 queries x 64] K-major
    uint8_t *sK = sQ + kTiles * kTileBytes;                // kRing x [128 keys x 64] K-major
    uint8_t *sV = sK + kRing * kTileBytes;                 // kRing x [128 keys x 64] (read MN-major)
    uint8_t *sStage = sV + kRing * kTileBytes;             // dequantise-on-load: kSlots staging slots
    AttnSmem *S = reinterpret_cast<AttnSmem *>(sStage + (FORM == 1 ? kSlots * kSlotBytes : 0));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = blockIdx.x, head = blockIdx.y;
    const int q0 = qb * (kTiles * kBlockQ);
    const int nkb = (p.lk + kBlockK - 1) / kBlockK;
    const int col0 = head * kHeadDim;
    constexpr uint32_t kLdArrivals = FORM == 0 ? 1u : (uint32_t)kLoaders;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&S->st_full[i], kLoaders + 1);   // every loader's cp.async arrival + the TMA thread's
            mbar_init(&S->st_free[i], kLoaders / 32);  // one arrival per loader warp
        }
        mbar_init(&S->q_full, 1);
        for (int b = 0; b < kRing; ++b) {
            mbar_init(&S->ld_full[b], kLdArrivals);
            mbar_init(&S->ld_free[b], AttnCfg<FORM>::kIssuers);   // one commit per issuer
        }
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(&S->s_full[t], 1);
            mbar_init(&S->s_free[t], 4);               // one arrival per softmax warp of the tile
            mbar_init(&S->p_full[t], 4);
            mbar_init(&S->pv_done[t], 1);
            for (int w = 0; w < 4; ++w) mbar_init(&S->turn[t][w], 1);
        }
        for (int t = 0; t < kTiles; ++t) mbar_init(&S->drain[t], 1);
        S->abort_flag = 0;
        mbar_init_fence();
    }
    if (threadIdx.x < 16) {
        const int L = (1 << (K - 1)) - 1;
        S->lut[threadIdx.x] = (K >= 2) ? __fdiv_rn((float)((int)threadIdx.x - L), (float)L) : 0.0f;
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S->tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    volatile int *abort_flag = &S->abort_flag;
    const unsigned long long wait_ns = p.wait_ns;

    constexpr int kLoader0 = AttnCfg<FORM>::kLoader0;
    if (threadIdx.x >= kLoader0) {
        // ------------------------------------------------------- loaders --
        const int lt = threadIdx.x - kLoader0;   // 0..kLoaders-1
        // Fault injection for the failure-detection test: with nothing loaded,
        // the MMA issuers' bounded wait on Q runs out, they raise the abort
        // flag and every other wait of the CTA gives up.
        if (p.starve) goto loaders_done;
        if (lt == 0) {
            // Q of both tiles by TMA; rows past lq read as zero
            mbar_expect_tx(&S->q_full, (uint32_t)(kTiles * kTileBytes));
            for (int t = 0; t < kTiles; ++t) tma_load_2d(sQ + t * kTileBytes, &p.tq, col0, q0 + t * kBlockQ, &S->q_full);
        }
        if constexpr (FORM == 0) {
            // K and V boxes by TMA (keys past lk read as zero), one thread
            if (lt == 0) {
                for (int j = 0; j < nkb; ++j) {
                    const int b = j % kRing;
                    if (j >= kRing &&
                        !wait_bounded(&S->ld_free[b], (uint32_t)((j / kRing) - 1) & 1u, abort_flag, p.status, wait_ns))
                        break;
                    mbar_expect_tx(&S->ld_full[b], 2u * kTileBytes);
                    tma_load_2d(sK + b * kTileBytes, &p.tk, col0, j * kBlockK, &S->ld_full[b]);
                    tma_load_2d(sV + b * kTileBytes, &p.tv, col0, j * kBlockK, &S->ld_full[b]);
                }
            }
        } else {
            // Dequantise-on-load.  Sub-chunk g (keys 32 g .. 32 g + 31 of K and
            // V) is staged in slot g % kSlots: the fp32 cache rows by TMA (one
            // 64 x 32 box per tensor, keys past lk zero-filled), the code bytes
            // and scales by cp.async; the slot's mbarrier completes when all
            // have landed.  Staging runs three sub-chunks ahead of the one being
            // dequantised into the bf16 tiles of its key block.
            const bool wb = qb == 0;                      // the first query block writes the new cache
            const int ngs = nkb * (kBlockK / kSub);
            constexpr int kCodeRow = 8 * K;                // code bytes per key row of a head (64 channels)
            constexpr int kCodePiece = kCodeRow >= 16 ? 16 : kCodeRow;
            constexpr int kCodePieces = kCodeRow / kCodePiece;
            const int ns = p.group >= kHeadDim ? 1 : kHeadDim / p.group;   // scales per key row of a head
            const int sc_piece = ns >= 4 ? 16 : 4 * ns;
            const int sc_lg = ns == 8 ? 1 : 0;             // two 16-byte pieces at G = 8
            const int cpg = p.cols / p.group, c0g = col0 / p.group;      // scale index = key * cpg + c0g
            const uint32_t stage0 = smem_u32(sStage);
            auto issue = [&](int g) {                     // every loader thread; the slot is free
                const int k0 = g * kSub, slot = g & (kSlots - 1);
                uint8_t *st = sStage + slot * kSlotBytes;
                if (lt == 0) {
                    mbar_expect_tx(&S->st_full[slot], 2u * kSub * kHeadDim * 4);
                    tma_load_2d(st, &p.tc[0], col0, k0, &S->st_full[slot]);
                    tma_load_2d(st + kSub * 256, &p.tc[1], col0, k0, &S->st_full[slot]);
                }
                for (int u = lt; u < 2 * kSub * kCodePieces; u += kLoaders) {
                    const int w = u / (kSub * kCodePieces), rem = u - w * (kSub * kCodePieces);
                    const int r = rem / kCodePieces, q = rem - r * kCodePieces;
                    if (k0 + r < p.lk)
                        cp_async(st + kSlotC + w * (kSub * 32) + r * 32 + q * kCodePiece,
                                 p.codes[w] + ((int64_t)(k0 + r) * p.cols + col0) * K / 8 + q * kCodePiece, kCodePiece);
                }
                for (int u = lt; u < (2 * kSub) << sc_lg; u += kLoaders) {
                    const int wr = u >> sc_lg, q = u & ((1 << sc_lg) - 1);
                    const int w = wr >> 5, r = wr & (kSub - 1);
                    if (k0 + r < p.lk)
                        cp_async(st + kSlotC + kSlotCodes + w * (kSub * 32) + r * 32 + q * sc_piece,
                                 p.scales[w] + (int64_t)(k0 + r) * cpg + c0g + q * (sc_piece / 4), sc_piece);
                }
                cp_async_arrive(&S->st_full[slot]);
            };
            for (int g = 0; g < kSlots - 1 && g < ngs; ++g) issue(g);
            const uint32_t lut = smem_u32(S->lut);
            for (int g = 0; g < ngs; ++g) {
                const int j = g / (kBlockK / kSub), sub = g % (kBlockK / kSub), b = j % kRing;
                const int slot = g & (kSlots - 1);
                // stage sub-chunk g + 3 into the slot of sub-chunk g - 1 once every loader warp has read it
                const int gn = g + kSlots - 1;
                if (gn < ngs) {
                    if (gn >= kSlots && !warp_wait(&S->st_free[gn & (kSlots - 1)], (uint32_t)((gn / kSlots) - 1) & 1u,
                                                   abort_flag, p.status, wait_ns))
                        break;
                    issue(gn);
                }
                if (!warp_wait(&S->st_full[slot], (uint32_t)(g / kSlots) & 1u, abort_flag, p.status, wait_ns)) break;
                if (sub == 0 && j >= kRing &&
                    !warp_wait(&S->ld_free[b], (uint32_t)((j / kRing) - 1) & 1u, abort_flag, p.status, wait_ns))
                    break;
                const uint32_t st = stage0 + (uint32_t)(slot * kSlotBytes);
                const uint32_t tk = smem_u32(sK + b * kTileBytes), tv = smem_u32(sV + b * kTileBytes);
                for (int u = lt; u < 2 * kSub * 8; u += kLoaders) {
                    const int w = u >> 8, r = (u >> 3) & (kSub - 1), pc = u & 7;
                    const int key = g * kSub + r;
                    uint4 o = make_uint4(0u, 0u, 0u, 0u);
                    if (key < p.lk) {
                        const uint32_t cs = st + (uint32_t)(w * (kSub * 256) + r * 256 + 32 * pc);
                        const float4 a = lds128(cs), bb = lds128(cs + 16);
                        const uint32_t cb = st + (uint32_t)(kSlotC + w * (kSub * 32) + r * 32 + K * pc);
                        const uint32_t code = K == 4 ? lds32(cb) : (K == 2 ? lds16(cb) : lds8(cb));
                        const float sc = __uint_as_float(lds32(st + (uint32_t)(kSlotC + kSlotCodes + w * (kSub * 32) +
                                                                               r * 32 + 4 * ((8 * pc) >> p.group_lg))));
                        const float cin[8] = {a.x, a.y, a.z, a.w, bb.x, bb.y, bb.z, bb.w};
                        float c[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            // the decompress arithmetic: one binary32 multiply and one add, never fused
                            const uint32_t ce = (code >> (K * e)) & ((1u << K) - 1u);
                            const float d = (K >= 2) ? __fmul_rn(__uint_as_float(lds32(lut + 4 * ce)), sc) : (ce ? sc : -sc);
                            c[e] = __fadd_rn(cin[e], d);
                        }
                        if (wb) {
                            float4 *dst = reinterpret_cast<float4 *>(p.cache_out[w] + (int64_t)key * p.cols + col0 + 8 * pc);
                            dst[0] = make_float4(c[0], c[1], c[2], c[3]);
                            dst[1] = make_float4(c[4], c[5], c[6], c[7]);
                        }
                        o = make_uint4(bf16x2(c[0], c[1]), bf16x2(c[2], c[3]), bf16x2(c[4], c[5]), bf16x2(c[6], c[7]));
                    }
                    sts128((w ? tv : tk) + sw128(sub * kSub + r, pc), o);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->st_free[slot]);
                if (sub == kBlockK / kSub - 1) {
                    fence_proxy_async();
                    mbar_arrive(&S->ld_full[b]);
                }
            }
            cp_wait_all();
        }
    loaders_done:;
    } else if (warp >= kMmaWarp) {
        // ---------------------------------------------------- MMA issuer --
        // Per key block j: S_0(j + 1) as soon as tile 0's softmax has read
        // S_0(j), O_0 += P_0(j) V(j) once P_0(j) is in tensor memory, then the
        // same for tile 1; so the tensor cores work on one tile while the
        // other tile's softmax runs.
        const uint32_t idS = instr_desc_bf16(kBlockK, 0), idO = instr_desc_bf16(kHeadDim, 1);
        auto issue_s = [&](int t, int b) {       // S_t = Q_t K_b^T (lane 0)
            const uint32_t aQ = smem_u32(sQ + t * kTileBytes), bK = smem_u32(sK + b * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < kHeadDim / 16; ++kk)
                mma_bf16(tmem + 128u * (uint32_t)t, kdesc(aQ + 32 * kk), kdesc(bK + 32 * kk), idS, kk > 0);
            tc_commit(&S->s_full[t]);
        };
        auto issue_pv = [&](int t, int b, bool first) {   // O_t += P_t V_b (lane 0)
            const uint32_t bV = smem_u32(sV + b * kTileBytes);
            const uint32_t tO = tmem + 256u + 64u * (uint32_t)t, tP = tmem + 384u + 64u * (uint32_t)t;
#pragma unroll
            for (int kk = 0; kk < kBlockK / 16; ++kk)
                // keys 16 kk .. 16 kk + 15: P's columns 8 kk .., V's 8-key groups 2 kk and 2 kk + 1
                mma_bf16_ta(tO, tP + 8u * (uint32_t)kk, vdesc(bV + 2048u * (uint32_t)kk), idO,
                            (!first || kk > 0) ? 1u : 0u);
            tc_commit(&S->pv_done[t]);
        };
        bool ok = warp_wait(&S->q_full, 0u, abort_flag, p.status, wait_ns) &&
                  warp_wait(&S->ld_full[0], 0u, abort_flag, p.status, wait_ns);
        if constexpr (AttnCfg<FORM>::kIssuers == 2) {
            // one issuer per tile: S_t(j + 1) once the tile's softmax has read
            // S_t(j), O_t += P_t(j) V(j) once P_t(j) is in tensor memory
            const int t = warp - kMmaWarp;
            if (ok) {
                tc_fence_after();
                if (lane == 0) issue_s(t, 0);
                __syncwarp();
            }
            for (int j = 0; j < nkb && ok; ++j) {
                const int b = j % kRing, b1 = (j + 1) % kRing;
                const uint32_t par = (uint32_t)j & 1u;
                if (j + 1 < nkb) {
                    ok = warp_wait(&S->ld_full[b1], (uint32_t)((j + 1) / kRing) & 1u, abort_flag, p.status, wait_ns) &&
                         warp_wait(&S->s_free[t], par, abort_flag, p.status, wait_ns);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) issue_s(t, b1);
                    __syncwarp();
                }
                ok = warp_wait(&S->p_full[t], par, abort_flag, p.status, wait_ns);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    issue_pv(t, b, j == 0);
                    tc_commit(&S->ld_free[b]);
                }
                __syncwarp();
            }
        } else {
            // one issuer for both tiles: S_0(j + 1), O_0 += P_0(j) V(j), then
            // the same for tile 1
            if (ok) {
                tc_fence_after();
                if (lane == 0) {
                    issue_s(0, 0);
                    issue_s(1, 0);
                }
                __syncwarp();
            }
            for (int j = 0; j < nkb && ok; ++j) {
                const int b = j % kRing, b1 = (j + 1) % kRing;
                const uint32_t par = (uint32_t)j & 1u;
                if (j + 1 < nkb) {
                    ok = warp_wait(&S->ld_full[b1], (uint32_t)((j + 1) / kRing) & 1u, abort_flag, p.status, wait_ns) &&
                         warp_wait(&S->s_free[0], par, abort_flag, p.status, wait_ns);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) issue_s(0, b1);
                    __syncwarp();
                }
                ok = warp_wait(&S->p_full[0], par, abort_flag, p.status, wait_ns);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) issue_pv(0, b, j == 0);
                __syncwarp();
                if (j + 1 < nkb) {
                    ok = warp_wait(&S->s_free[1], par, abort_flag, p.status, wait_ns);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) issue_s(1, b1);
                    __syncwarp();
                }
                ok = warp_wait(&S->p_full[1], par, abort_flag, p.status, wait_ns);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    issue_pv(1, b, j == 0);
                    tc_commit(&S->ld_free[b]);
                }
                __syncwarp();
            }
        }
        // Drain: every MMA this thread issued has completed before TMEM is freed.
        if (lane == 0) {
            uint64_t *dr = &S->drain[warp - kMmaWarp];
            tc_commit(dr);
            volatile int no_abort = 0;
            wait_bounded(dr, 0u, &no_abort, p.status, kAttnWaitNs);
        }
        __syncwarp();
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------- softmax --
        const int t = warp >> 2;                            // query tile
        const int row = 32 * (warp & 3) + lane;             // query row of the tile = TMEM lane
        const uint32_t lanebase = (uint32_t)(32 * (warp & 3)) << 16;
        const uint32_t tS = tmem + 128u * (uint32_t)t + lanebase;
        const uint32_t tO = tmem + 256u + 64u * (uint32_t)t + lanebase;
        const uint32_t tP = tmem + 384u + 64u * (uint32_t)t + lanebase;
        const float c2 = p.scale_log2;
        float m = -INFINITY, l = 0.0f;                      // reference maximum (raw score) and sum against it
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            if (!warp_wait(&S->s_full[t], (uint32_t)j & 1u, abort_flag, p.status, wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kBlockK];
#pragma unroll
            for (int c = 0; c < kBlockK; c += 16) {
                uint32_t v[16];
                tc_ld16(tS + (uint32_t)c, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) s[c + e] = __uint_as_float(v[e]);
            }
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->s_free[t]);
            // keys past lk do not count (the last block only; uniform across the CTA)
            const int kvalid = p.lk - j * kBlockK;
            if (kvalid < kBlockK) {
#pragma unroll
                for (int c = 0; c < kBlockK; ++c) s[c] = c < kvalid ? s[c] : -INFINITY;
            }
            float mx[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) mx[e] = fmaxf(s[2 * e], s[2 * e + 1]);
#pragma unroll
            for (int c = 8; c < kBlockK; c += 8) {
#pragma unroll
                for (int e = 0; e < 4; ++e) mx[e] = fmax3(mx[e], s[c + 2 * e], s[c + 2 * e + 1]);
            }
            const float m_blk = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
            // move the reference maximum only when it grows by more than 2^8 in base 2
            const bool grow = (m_blk - m) * c2 > kRescaleLog2;   // true on the first block (m = -inf)
            const bool rescale = __any_sync(0xffffffffu, grow) && j > 0;
            float alpha = 1.0f;
            if (grow) {
                alpha = ex2((m - m_blk) * c2);                    // 0 on the first block
                m = m_blk;
            }
            const float mc = m * c2;
            if (j > 0) {
                // P_t and O_t are free once the previous block's P V has completed
                if (!warp_wait(&S->pv_done[t], (uint32_t)(j - 1) & 1u, abort_flag, p.status, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            // The two tiles' warps on this sub-partition take turns at the
            // exponentials (tile 0 first in every block; the turn passes when
            // half of a block's are done), so that one tile's loads, maximum
            // and waits overlap the other's use of the unit.
            if ((t == 1 || j > 0) &&
                !warp_wait(&S->turn[t][warp & 3], (uint32_t)(t == 1 ? j : j - 1) & 1u, abort_flag, p.status, wait_ns)) {
                ok = false;
                break;
            }
            // P = 2^(s c2 - m c2) in 32-key chunks, each packed to bf16 pairs and
            // stored to tensor memory as soon as it is formed
            float sm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < kBlockK; q += 32) {
                uint32_t v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float x0 = ex2(fmaf(s[q + 2 * e], c2, -mc)), x1 = ex2(fmaf(s[q + 2 * e + 1], c2, -mc));
                    sm[(2 * e) & 7] += x0;
                    sm[(2 * e + 1) & 7] += x1;
                    v[e] = bf16x2(x0, x1);
                }
                tmem_st16(tP + (uint32_t)(q >> 1), v);
                if (q == 32 * 2) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S->turn[t ^ 1][warp & 3]);
                }
            }
            l = l * alpha + (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));
            if (rescale) {
#pragma unroll
                for (int c = 0; c < kHeadDim; c += 32) {
                    uint32_t v0[16], v1[16];
                    tc_ld16(tO + (uint32_t)c, v0);
                    tc_ld16(tO + (uint32_t)c + 16u, v1);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        v0[e] = __float_as_uint(__uint_as_float(v0[e]) * alpha);
                        v1[e] = __float_as_uint(__uint_as_float(v1[e]) * alpha);
                    }
                    tmem_st16(tO + (uint32_t)c, v0);
                    tmem_st16(tO + (uint32_t)c + 16u, v1);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->p_full[t]);
        }
        if (ok && warp_wait(&S->pv_done[t], (uint32_t)(nkb - 1) & 1u, abort_flag, p.status, wait_ns)) {
            tc_fence_after();
            const float inv = 1.0f / l;
            uint32_t ov[kHeadDim];
#pragma unroll
            for (int c = 0; c < kHeadDim; c += 16) {
                uint32_t v[16];
                tc_ld16(tO + (uint32_t)c, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) ov[c + e] = v[e];
            }
            tc_wait_ld();
            uint32_t o[kHeadDim / 2];
#pragma unroll
            for (int c = 0; c < kHeadDim; c += 2)
                o[c >> 1] = bf16x2(__uint_as_float(ov[c]) * inv, __uint_as_float(ov[c + 1]) * inv);
            const int qrow = q0 + t * kBlockQ + row;
            if (qrow < p.lq) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (int64_t)qrow * p.cols + col0);
#pragma unroll
                for (int c = 0; c < kHeadDim / 8; ++c) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                // log sum_j e^(s_j / 8) = ln 2 * (m log2(e) / 8 + log2 l): l was summed against the reference m
                if (p.lse) p.lse[(int64_t)qrow * (p.cols / kHeadDim) + head] = (m * c2 + log2f(l)) * 0.69314718055994531f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

template <int FORM>
constexpr size_t attn_smem_bytes()
{
    return 1024 + (size_t)(kTiles + 2 * AttnCfg<FORM>::kRing) * kTileBytes +
           (FORM == 1 ? (size_t)kSlots * kSlotBytes : 0) + sizeof(AttnSmem);
}
static_assert(attn_smem_bytes<0>() <= 227 * 1024, "attention shared memory exceeds 227 KB");
static_assert(attn_smem_bytes<1>() <= 227 * 1024, "attention shared memory exceeds 227 KB");
// One CTA per SM: the 512 tensor-memory columns it allocates are the SM's all.
static_assert(attn_smem_bytes<0>() > 114 * 1024 && attn_smem_bytes<1>() > 114 * 1024,
              "a second resident CTA would wait for tensor memory");

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
                                     (int)attn_smem_bytes<FORM>());
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) done[dev] = true;
        }
    }
    constexpr int kQ = kTiles * kBlockQ;
    const dim3 grid((unsigned)((p.lq + kQ - 1) / kQ), (unsigned)(p.cols / kHeadDim));
    const char *name = FORM == 0 ? "k_attention<bf16>" : "k_attention<dequantise>";
    log_launch(name, grid, dim3(AttnCfg<FORM>::kThreads), attn_smem_bytes<FORM>());
    trace_begin(name, stream);
    k_attention<FORM, K><<<grid, AttnCfg<FORM>::kThreads, attn_smem_bytes<FORM>(), stream>>>(p);
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
    p.lse = a.lse;
    p.lq = (int)a.lq;
    p.lk = (int)a.lk;
    p.cols = (int)a.cols;
    p.group = a.group;
    p.group_lg = 0;
    while (p.group > 0 && (1 << (p.group_lg + 1)) <= p.group) ++p.group_lg;
    p.scale_log2 = 1.4426950408889634f / 8.0f;   // log2(e) / sqrt(64)
    p.status = a.status;
    p.wait_ns = kAttnWaitNs;
    if (a.starve) {
        p.starve = 1;
        p.wait_ns = 20000000ull;
    }
    // Q (both forms) and bf16 K, V by TMA: [rows x cols] bf16, a 64-channel x 128-row box
    if (!make_map_bf16(&p.tq, a.q, (uint64_t)a.cols, (uint64_t)a.lq, (uint64_t)a.cols, kHeadDim, kBlockQ))
        return cudaErrorInvalidValue;
    if (!a.dequantise &&
        (!make_map_bf16(&p.tk, a.kv[0], (uint64_t)a.cols, (uint64_t)a.lk, (uint64_t)a.cols, kHeadDim, kBlockK) ||
         !make_map_bf16(&p.tv, a.kv[1], (uint64_t)a.cols, (uint64_t)a.lk, (uint64_t)a.cols, kHeadDim, kBlockK)))
        return cudaErrorInvalidValue;
    // the caches (dequantise form): fp32 [lk x cols], a 64-channel x 32-key box, no swizzle
    if (a.dequantise &&
        (!make_map(&p.tc[0], a.cache_in[0], (uint64_t)a.cols, (uint64_t)a.lk, (uint64_t)a.cols, kHeadDim, kSub,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
         !make_map(&p.tc[1], a.cache_in[1], (uint64_t)a.cols, (uint64_t)a.lk, (uint64_t)a.cols, kHeadDim, kSub,
                   CU_TENSOR_MAP_SWIZZLE_NONE)))
        return cudaErrorInvalidValue;
    if (!a.dequantise) return attn_launch_k<0, 2>(p, stream);
    switch (a.bits) {
    case 1: return attn_launch_k<1, 1>(p, stream);
    case 2: return attn_launch_k<1, 2>(p, stream);
    default: return attn_launch_k<1, 4>(p, stream);
    }
}

}  // namespace cf
