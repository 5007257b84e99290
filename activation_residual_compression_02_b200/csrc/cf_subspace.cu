// cf_subspace.cu -- Algorithm 3 (rank-r subspace iteration) for sm_100a.
//
// "Accelerating Parallel Diffusion Model Serving with Residual Compression"
// (arXiv 2507.17511), reproducibility table, "Pseudocode" row, Algorithm 3:
//   Q = orth(random Q0); repeat T: Z = A^T (A Q), Q = orth(Z);
//   U = orth(A Q); V = Q.
// orth() is CholeskyQR (G = Y^T Y, R = chol(G), Y R^{-1}); keeping the R of
// the last step gives the payload (U, R, V) whose reconstruction is U R V^T.
//
// Kernels (one grouped launch each, over every matrix of the call):
//  * k_gemm_tf32: the two products with A.  P = A Q (A K-major) and
//    Z = A^T P (A read as an MN-major operand straight from its row-major
//    storage, staged with the 128-byte/32-byte-atom swizzle that MN-major
//    32-bit operands require).  A warp-specialised persistent tcgen05 kernel: one TMA warp
//    streams stages of two or three 128x32 fp32 boxes of A (128-byte swizzle)
//    plus the matching r-column slices of Q^T / P^T; four warps round each A tile to TF32 in
//    shared memory (round to nearest: the tensor core would otherwise drop the
//    low mantissa bits, a bias of about 2^-11 that alone costs ~7e-4 of the
//    reconstruction); one thread issues tcgen05.mma (M=128, N=16/32, K=8)
//    into a double-buffered TMEM accumulator; four warps drain TMEM with
//    tcgen05.ld and write the r-column result.  The work is HBM-bound (8 flop
//    per byte of A), so the tensor cores only have to keep up with the stream.
//  * k_cholqr_factor / k_cholqr_apply: CholeskyQR in fp64 -- Gram matrices
//    of 256-row chunks, summed in chunk order by the last CTA of each
//    matrix, which factors G = R^T R and inverts R; then Y R^{-1} row by row.
//  * k_apply: D = U (R V^T) on CUDA cores (K = r is far too thin for the
//    tensor cores; the step is an HBM stream), fused with E = A - D and
//    C += D.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the
// CTA raises an abort flag and a status bit, drains its own TMA loads and
// MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <stdlib.h>

#include <algorithm>
#include <mutex>

#include "cf_internal.h"
#include "cf_ptx.cuh"
#include "cf_tc.cuh"

namespace cf {
namespace {

// ------------------------------------------------------------ constants --
constexpr int kBM = 128;            // MMA M: rows of an output tile
constexpr int kBoxK = 32;           // K of one TMA box: 32 fp32 = 128 bytes, the swizzle span
constexpr int kBoxBytes = kBM * kBoxK * 4;   // one 128 x 32 box of A: 16 KB
constexpr int kGemmThreads = 320;   // 10 warps: TMA, MMA, 4 convert, 4 epilogue
constexpr int kMaxGemmMats = 160;   // 128-byte tensor maps in the kernel parameters

// Pipeline shape per padded rank RP (the MMA's N).  A stage holds NB boxes of
// A side by side in K, so each row of A is read NB x 128 contiguous bytes at
// a time and the per-stage handshakes (barrier, TF32 rounding, fence, MMA
// batch) are paid once per NB boxes.  Measured on the 57 x 4608 x 3072 pass
// with one CTA per SM: one box per stage with 8 stages ran at 5.2-5.6 TB/s;
// three boxes with four stages at 6.6 TB/s, bit-identical.  RP = 32 needs
// twice the B space and keeps two boxes with five stages (one CTA per SM).
//
// Accumulation in chunks of K.  The tensor core's fp32 accumulator loses a
// fraction of an ulp towards zero at each accumulating MMA, so one long
// accumulation chain shrinks the product by a factor that grows with K
// (measured on exactly rank-16 matrices: P = A Q was 2.8e-5 small at
// K = 4096 and 1.6e-4 at K = 32768, and E = A - U R V^T inherits it).  The
// MMA therefore restarts its accumulator every CH stages (about 1000 of K),
// and the epilogue adds the chunk sums on the CUDA cores with round to
// nearest, in chunk order, so the loss stays at its K = 1000 level.
//
// At RP = 16 and with at least two tiles per SM, two CTAs share an SM (two
// boxes x three stages each): more independent TMA streams per SM than one
// CTA with three boxes x four stages, 0.475 against 0.482 ms per pass over the
// 57 x 4608 x 3072 batch.  With fewer tiles (a few matrices) the one-CTA form
// is faster (4 matrices: 43.5 / 51.0 against 48.8 / 67.0 us for A Q / A^T P),
// so the host picks the form by tile count.
//
// Split products (SPLIT, "3xTF32"): each operand is carried as two TF32
// parts, x = hi + lo with hi = tf32(x) and lo = tf32(x - hi), and each
// product is hi_A hi_B + (lo_A hi_B + hi_A lo_B), dropping lo_A lo_B (about
// 2^-22 of the product): close to fp32 accuracy, for iterations that are
// ill-conditioned with respect to operand rounding.  The converter warps
// write lo_A beside hi_A; the producer loads hi_B and lo_B blocks.  The two
// correction products accumulate into their own TMEM accumulator, so the
// main accumulation chain is as long as in the plain form; the epilogue adds
// the two.  The stages are smaller (A takes twice the shared memory).
template <int RP, int CPS, bool SPLIT = false>
struct GemmCfg {
    static constexpr int NB = SPLIT ? (RP == 16 ? 2 : 1) : ((RP == 16 && CPS == 1) ? 3 : 2);   // boxes of A per stage
    static constexpr int ST = SPLIT ? (RP == 16 ? 3 : 5) : (RP == 16 ? (CPS == 2 ? 3 : 4) : 5); // pipeline stages
    static constexpr int BK = NB * kBoxK;               // K per stage
    static constexpr int CH = 1024 / BK;                // stages per accumulation chunk (960 or 1024 of K)
    static constexpr int NP = SPLIT ? 2 : 1;            // TF32 parts per operand
    static constexpr int ATile = NB * kBoxBytes;        // A bytes per stage and part
    static constexpr int BBox = RP * kBoxK * 4;         // one RP x 32 box of Q^T / P^T
    static constexpr int BTile = NB * BBox;             // B bytes per stage and part
    static constexpr int TmemCols = SPLIT ? 128 : 64;   // two accumulators of up to 32 columns (+ two for corrections)
};
constexpr uint64_t kWaitNs = 2000000000ull;

struct __align__(64) GemmMat {
    CUtensorMap ta;    // A (fp32, row-major m x n) of this matrix
};

struct GemmParams {
    GemmMat mat[kMaxGemmMats];
    CUtensorMap tb;    // B^T blocks of every matrix, 3-D {K, rp, matrix}: Q^T or P^T (K-major)
    CUtensorMap tb_lo; // split products: the lo parts of the same blocks
    float *out;        // output of matrix 0; matrix i at out + i * out_stride
    float *out_lo;     // split products, out_mode 0: lo parts of the transposed output (same strides)
    int64_t out_stride;
    int nmat;
    int tiles_per_mat;
    int ktiles;
    int out_rows;      // valid output rows (m for A Q, n for A^T P)
    int rp;            // N of the MMA (16 or 32)
    int mn_major;      // 0: out = A Q (A K-major); 1: out = A^T P (A MN-major)
    int out_mode;      // 0: transposed + TF32-rounded [rp][out_ld]; 1: exact row-major [rows][rp]
    int out_ld;        // leading dimension of the transposed output
    uint32_t *status;
    unsigned long long wait_ns;
    int starve;        // fault-injection hook for tests: the producer issues no loads
};

using namespace ptx;
using namespace tc;


template <int ST>
struct GemmSmem {
    uint64_t full[ST];
    uint64_t conv[ST];
    uint64_t empty[ST];
    uint64_t accf[2];
    uint64_t acce[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
};

// ------------------------------------------------------------ the GEMM ----
template <int RP, int CPS, bool SPLIT>
__global__ void __launch_bounds__(kGemmThreads, CPS) k_gemm_tf32(const __grid_constant__ GemmParams p)
{
    using C = GemmCfg<RP, CPS, SPLIT>;
    constexpr int kStages = C::ST;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = base;                                   // kStages x NB boxes of A (hi part)
    uint8_t *sAlo = sA + kStages * C::ATile;              // SPLIT: the lo parts, same layout
    uint8_t *sB = sA + C::NP * kStages * C::ATile;        // kStages x NP x NB boxes of Q^T / P^T
    GemmSmem<kStages> *S = (GemmSmem<kStages> *)(sB + C::NP * kStages * C::BTile);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int total_tiles = p.nmat * p.tiles_per_mat;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->conv[s], 128);
            mbar_init(&S->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S->accf[b], 1);
            mbar_init(&S->acce[b], 128);
        }
        mbar_init(&S->drain, 1);
        S->abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S->tmem_base)),
                     "r"(C::TmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    volatile int *abort_flag = &S->abort_flag;
    const unsigned long long wait_ns = p.wait_ns;
    const uint32_t stage_bytes = (uint32_t)(C::ATile + C::NP * C::BTile);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = !p.starve;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const int mi = tile / p.tiles_per_mat;
                const int mt = tile - mi * p.tiles_per_mat;
                const GemmMat &M = p.mat[mi];
                for (int kt = 0; kt < p.ktiles; ++kt, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!wait_bounded(&S->empty[s], ph ^ 1u, abort_flag, p.status, wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(&S->full[s], stage_bytes);
                    // NB boxes side by side in K; boxes past the end of K
                    // are zero-filled by the TMA unit and still count their
                    // full bytes.
#pragma unroll
                    for (int h = 0; h < C::NB; ++h) {
                        uint8_t *a = sA + s * C::ATile + h * kBoxBytes;
                        const int k0 = kt * C::BK + h * kBoxK;
                        if (!p.mn_major) {
                            tma_load_2d(a, &M.ta, k0, mt * kBM, &S->full[s]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                tma_load_2d(a + j * 4096, &M.ta, mt * kBM + 32 * j, k0, &S->full[s]);
                        }
                        uint8_t *b = sB + s * C::NP * C::BTile + h * C::BBox;
                        tma_load_3d(b, &p.tb, k0, 0, mi, &S->full[s]);
                        if (SPLIT) tma_load_3d(b + C::BTile, &p.tb_lo, k0, 0, mi, &S->full[s]);
                    }
                }
            }
            // Drain: every load this thread issued has landed before exit.
            const uint32_t outstanding = it < (uint32_t)kStages ? it : (uint32_t)kStages;
            for (uint32_t j = it - outstanding; j < it; ++j) {
                volatile int no_abort = 0;
                wait_bounded(&S->full[j % kStages], (j / kStages) & 1u, &no_abort, p.status, kWaitNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        const uint32_t idesc = instr_desc_tf32(RP, p.mn_major);
        uint32_t it = 0, lc = 0;   // stage counter; accumulation-chunk counter (selects the TMEM buffer)
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            for (int k0 = 0; k0 < p.ktiles && ok; k0 += C::CH, ++lc) {
                const int k1 = min(p.ktiles, k0 + C::CH);
                const int b = lc & 1;
                const uint32_t aph = (lc >> 1) & 1u;
                if (!wait_bounded(&S->acce[b], aph ^ 1u, abort_flag, p.status, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dtm = tmem + (uint32_t)(b * 32);
                const uint32_t dcor = dtm + 64;   // SPLIT: accumulator of the correction products
                for (int kt = k0; kt < k1; ++kt, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!wait_bounded(&S->conv[s], ph, abort_flag, p.status, wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a0 = smem_u32(sA + s * C::ATile);
                        const uint32_t b0 = smem_u32(sB + s * C::NP * C::BTile);
#pragma unroll
                        for (int k = 0; k < C::BK / 8; ++k) {
                            // K step k: box k / 4, 8-element slice k % 4 of it
                            const uint32_t ah = a0 + (k / 4) * kBoxBytes, bh = b0 + (k / 4) * C::BBox;
                            const uint32_t kk = (uint32_t)(k % 4);
                            const uint64_t ad = p.mn_major ? smem_desc(ah + kk * 1024, 4096, 512, kLayoutSw128Atom32)
                                                           : smem_desc(ah + kk * 32, 16, 1024, kLayoutSw128);
                            const uint64_t bd = smem_desc(bh + kk * 32, 16, 1024, kLayoutSw128);
                            const uint32_t acc = (kt > k0 || k > 0) ? 1u : 0u;
                            if (SPLIT) {
                                // the lo parts sit kStages * ATile (A) and BTile (B) bytes further on
                                const uint32_t alo = ah + (uint32_t)(kStages * C::ATile);
                                const uint64_t adl = p.mn_major ? smem_desc(alo + kk * 1024, 4096, 512, kLayoutSw128Atom32)
                                                                : smem_desc(alo + kk * 32, 16, 1024, kLayoutSw128);
                                const uint64_t bdl = smem_desc(bh + (uint32_t)C::BTile + kk * 32, 16, 1024, kLayoutSw128);
                                tc_mma_tf32(dcor, adl, bd, idesc, acc);
                                tc_mma_tf32(dcor, ad, bdl, idesc, 1u);
                            }
                            tc_mma_tf32(dtm, ad, bd, idesc, acc);
                        }
                        tc_commit(&S->empty[s]);
                    }
                    __syncwarp();
                }
                if (ok && lane == 0) tc_commit(&S->accf[b]);
                __syncwarp();
            }
        }
        // Drain: all MMAs this thread issued have completed before TMEM is freed.
        if (lane == 0) {
            tc_commit(&S->drain);
            volatile int no_abort = 0;
            wait_bounded(&S->drain, 0, &no_abort, p.status, kWaitNs);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------ TF32 rounding of A tiles --
        const int ct = threadIdx.x - 64;
        uint32_t it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            for (int kt = 0; kt < p.ktiles; ++kt, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1u;
                if (!wait_bounded(&S->full[s], ph, abort_flag, p.status, wait_ns)) {
                    ok = false;
                    break;
                }
                float4 *a = (float4 *)(sA + s * C::ATile);
                float4 *alo = (float4 *)(sAlo + s * C::ATile);
#pragma unroll
                for (int i = 0; i < C::ATile / 16 / 128; ++i) {
                    const float4 v = a[ct + 128 * i];
                    const float4 h = make_float4(round_tf32(v.x), round_tf32(v.y), round_tf32(v.z), round_tf32(v.w));
                    a[ct + 128 * i] = h;
                    if (SPLIT)
                        alo[ct + 128 * i] = make_float4(round_tf32(v.x - h.x), round_tf32(v.y - h.y),
                                                        round_tf32(v.z - h.z), round_tf32(v.w - h.w));
                }
                fence_proxy_async();
                mbar_arrive(&S->conv[s]);
            }
        }
    } else {
        // ----------------------------------------------------- epilogue --
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        uint32_t lc = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
            // sum of the tile's accumulation chunks, in chunk order, rounded to nearest
            float acc[RP];
            for (int k0 = 0; k0 < p.ktiles; k0 += C::CH, ++lc) {
                const int b = lc & 1;
                const uint32_t aph = (lc >> 1) & 1u;
                if (!wait_bounded(&S->accf[b], aph, abort_flag, p.status, wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[32];
                const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * 32);
                {
                    uint32_t lo[16];
                    tc_ld16(taddr, lo);
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = lo[c];
                }
                if (RP > 16) {
                    uint32_t hi[16];
                    tc_ld16(taddr + 16, hi);
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[16 + c] = hi[c];
                }
                if (SPLIT) {
                    // chunk = main + corrections, one rounding
                    uint32_t w[32];
                    uint32_t t16[16];
                    tc_ld16(taddr + 64, t16);
#pragma unroll
                    for (int c = 0; c < 16; ++c) w[c] = t16[c];
                    if (RP > 16) {
                        tc_ld16(taddr + 80, t16);
#pragma unroll
                        for (int c = 0; c < 16; ++c) w[16 + c] = t16[c];
                    }
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < RP; ++c) v[c] = __float_as_uint(__fadd_rn(__uint_as_float(v[c]), __uint_as_float(w[c])));
                }
                tc_wait_ld();
                tc_fence_before();
                mbar_arrive(&S->acce[b]);
#pragma unroll
                for (int c = 0; c < RP; ++c)
                    acc[c] = k0 == 0 ? __uint_as_float(v[c]) : __fadd_rn(acc[c], __uint_as_float(v[c]));
            }
            if (!ok) break;

            const int mi = tile / p.tiles_per_mat;
            const int mt = tile - mi * p.tiles_per_mat;
            const int row = mt * kBM + 32 * q + lane;
            float *out = p.out + (int64_t)mi * p.out_stride;
            if (row < p.out_rows) {
                if (p.out_mode == 0) {
#pragma unroll
                    for (int c = 0; c < RP; ++c) {
                        const float hi = round_tf32(acc[c]);
                        out[(int64_t)c * p.out_ld + row] = hi;
                        if (SPLIT) p.out_lo[(int64_t)mi * p.out_stride + (int64_t)c * p.out_ld + row] = round_tf32(acc[c] - hi);
                    }
                } else {
                    float4 *o = (float4 *)(out + (int64_t)row * RP);
#pragma unroll
                    for (int c = 0; c < RP; c += 4)
                        o[c / 4] = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TmemCols) : "memory");
    }
}

template <int RP, int CPS, bool SPLIT>
constexpr size_t gemm_smem_bytes()
{
    using C = GemmCfg<RP, CPS, SPLIT>;
    return 1024 + (size_t)C::NP * C::ST * (C::ATile + C::BTile) + sizeof(GemmSmem<C::ST>);
}
static_assert(gemm_smem_bytes<16, 1, false>() <= 227 * 1024, "GEMM shared memory (RP = 16) exceeds 227 KB");
static_assert(2 * (gemm_smem_bytes<16, 2, false>() + 1024) <= 228 * 1024,
              "two GEMM CTAs (RP = 16) do not fit in one SM's shared memory");
static_assert(gemm_smem_bytes<32, 1, false>() <= 227 * 1024, "GEMM shared memory (RP = 32) exceeds 227 KB");
static_assert(gemm_smem_bytes<16, 1, true>() <= 227 * 1024, "split GEMM shared memory (RP = 16) exceeds 227 KB");
static_assert(gemm_smem_bytes<32, 1, true>() <= 227 * 1024, "split GEMM shared memory (RP = 32) exceeds 227 KB");

// ------------------------------------------------------ CholeskyQR -------
// Two launches per orthonormalisation.  k_cholqr_factor: CTA (chunk, matrix)
// forms the Gram matrix of its kCqrRows rows in fp64 and stores it; the CTA
// that finishes last for a matrix (a counter per matrix) sums the stored Gram
// matrices in chunk order -- so the result does not depend on timing --,
// factors G = R^T R with one warp and inverts R with one warp.
// k_cholqr_apply: every row times R^{-1} in fp64 (the columns of a row are
// independent, so each thread keeps many multiply-adds in flight).
constexpr int kCqrThreads = 256;
constexpr int kCqrRows = 256;   // rows per Gram CTA

struct CholMat {
    const float *Y;       // input block [rows x ld]
    double *Gpart;        // Gram matrix of every chunk, packed upper triangles [chunks][r (r + 1) / 2]
    unsigned int *count;  // chunks done (zero before the launch; the last CTA resets it)
    double *Rinv;         // R^{-1} [32 x 32], upper triangular
    float *Qt;            // mode Q: rounded transposed output [rp x qt_ld] (rows >= r stay zero)
    float *Qt_lo;         // mode Q, split products: the lo parts of Qt (or null)
    float *Qexact;        // mode Q: optional exact output [rows x r] (V)
    float *U;             // mode U: [rows x r]
    float *R;             // mode U: [r x r]
};

constexpr int kMaxCholMats = 192;

struct CholParams {
    CholMat mat[kMaxCholMats];
    int nmat;
    int rows;
    int ld;             // row stride of Y (r or rp)
    int r;
    int qt_ld;
    uint32_t *status;
};

// Upper Cholesky factor of G (G = R^T R) by one warp: lane j owns column j.
// Step p: lane p forms the diagonal, then every lane q > p forms R[p][q].
// A pivot that is not positive (G not positive definite) is reported and
// replaced by 1 so that the solve stays finite.
__device__ void cholesky_upper_warp(const double *G, double *R, double *inv_diag, int r, uint32_t *status,
                                    bool report)
{
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < 32 * 32; i += 32) R[i] = 0.0;
    __syncwarp();
    for (int pp = 0; pp < r; ++pp) {
        if (lane == pp) {
            double diag = G[pp * 32 + pp];
            for (int k = 0; k < pp; ++k) diag -= R[k * 32 + pp] * R[k * 32 + pp];
            if (!(diag > 0.0) || !isfinite(diag)) {
                if (report) atomicOr(status, kStatusNotSpd);
                diag = 1.0;
            }
            const double d = sqrt(diag);
            R[pp * 32 + pp] = d;
            inv_diag[pp] = 1.0 / d;
        }
        __syncwarp();
        if (lane > pp && lane < r) {
            double v = G[pp * 32 + lane];
            for (int k = 0; k < pp; ++k) v -= R[k * 32 + pp] * R[k * 32 + lane];
            R[pp * 32 + lane] = v * inv_diag[pp];
        }
        __syncwarp();
    }
}

// R^{-1} of the upper triangular R by one warp: lane j forms column j by back
// substitution, Ri[i][j] = -(sum_{i < k <= j} R[i][k] Ri[k][j]) / R[i][i].
__device__ void inverse_upper_warp(const double *R, const double *inv_diag, double *Ri, int r)
{
    const int j = threadIdx.x & 31;
    for (int i = 0; i < 32; ++i) Ri[i * 32 + j] = 0.0;
    if (j < r) {
        Ri[j * 32 + j] = inv_diag[j];
        for (int i = j - 1; i >= 0; --i) {
            double acc = 0.0;
            for (int k = i + 1; k <= j; ++k) acc += R[i * 32 + k] * Ri[k * 32 + j];
            Ri[i * 32 + j] = -acc * inv_diag[i];
        }
    }
    __syncwarp();
}

// Copy n floats between global memory and a row-padded shared tile (row
// stride 33, `ld` floats per row), 16 bytes at a time where the block allows:
// a CTA's rows are one contiguous, 16-byte aligned block of n = rows * ld
// floats.
template <bool TO_SHARED>
__device__ __forceinline__ void block_copy(float *gptr, float *tile, int n, int ld)
{
    const int n4 = n >> 2;
    for (int i4 = threadIdx.x; i4 < n4; i4 += kCqrThreads) {
        const int i = i4 << 2;
        if (TO_SHARED) {
            const float4 v = reinterpret_cast<const float4 *>(gptr)[i4];
            const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) tile[((i + u) / ld) * 33 + (i + u) % ld] = e[u];
        } else {
            float e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) e[u] = tile[((i + u) / ld) * 33 + (i + u) % ld];
            reinterpret_cast<float4 *>(gptr)[i4] = make_float4(e[0], e[1], e[2], e[3]);
        }
    }
    for (int i = (n4 << 2) + threadIdx.x; i < n; i += kCqrThreads) {
        if (TO_SHARED)
            tile[(i / ld) * 33 + i % ld] = gptr[i];
        else
            gptr[i] = tile[(i / ld) * 33 + i % ld];
    }
}

// Gram matrix, Cholesky factor and its inverse for every matrix of the
// launch (MODE 1 also stores R, the payload of the final step).
template <int MODE>
__global__ void __launch_bounds__(kCqrThreads, 3) k_cholqr_factor(const __grid_constant__ CholParams p)
{
    const CholMat &M = p.mat[blockIdx.y];
    const int r = p.r;
    const int npairs = r * (r + 1) / 2;
    const int row0 = blockIdx.x * kCqrRows;
    const int nrows = min(kCqrRows, p.rows - row0);
    // The staged rows (phase 1) and the r x r matrices of the last CTA
    // (phase 2) share one buffer: 33.8 KB, of which phase 2 uses 24 KB.
    __shared__ __align__(16) unsigned char sbuf[kCqrRows * 33 * 4];
    static_assert(3 * 32 * 32 * sizeof(double) <= sizeof(sbuf), "phase-2 matrices exceed the staging buffer");
    float *ys = reinterpret_cast<float *>(sbuf);
    double *Gs = reinterpret_cast<double *>(sbuf);
    double *Rs = Gs + 32 * 32;
    double *Ri = Rs + 32 * 32;
    __shared__ double inv_diag[32];
    __shared__ int is_last;
    if (p.ld == r) {
        block_copy<true>(const_cast<float *>(M.Y) + (int64_t)row0 * p.ld, ys, nrows * r, r);
    } else {
        for (int i = threadIdx.x; i < nrows * r; i += kCqrThreads) {
            const int rr = i / r, c = i - rr * r;
            ys[rr * 33 + c] = M.Y[(int64_t)(row0 + rr) * p.ld + c];
        }
    }
    __syncthreads();
    for (int pidx = threadIdx.x; pidx < npairs; pidx += kCqrThreads) {
        // pair index -> (i, j), i <= j
        int i = 0, rem = pidx;
        while (rem >= r - i) {
            rem -= r - i;
            ++i;
        }
        const int j = i + rem;
        // four interleaved partial sums (rows k = 4q + u), added in a fixed
        // order at the end: a quarter of the dependent fp64 chain
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        int k = 0;
        for (; k + 4 <= nrows; k += 4) {
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] += (double)ys[(k + u) * 33 + i] * (double)ys[(k + u) * 33 + j];
        }
        for (; k < nrows; ++k) acc[0] += (double)ys[k * 33 + i] * (double)ys[k * 33 + j];
        M.Gpart[(int64_t)blockIdx.x * npairs + pidx] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    // The last CTA of this matrix to get here finishes the factorisation.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = atomicAdd(M.count, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    for (int pidx = threadIdx.x; pidx < npairs; pidx += kCqrThreads) {
        int i = 0, rem = pidx;
        while (rem >= r - i) {
            rem -= r - i;
            ++i;
        }
        const int j = i + rem;
        // loads of eight chunks in flight at a time, added in chunk order
        double g = 0.0;
        for (unsigned c0 = 0; c0 < gridDim.x; c0 += 8) {
            double v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = c0 + u < gridDim.x ? __ldcg(M.Gpart + (int64_t)(c0 + u) * npairs + pidx) : 0.0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (c0 + u < gridDim.x) g += v[u];
        }
        Gs[i * 32 + j] = g;
    }
    if (threadIdx.x == 0) *M.count = 0u;   // ready for the next orthonormalisation
    __syncthreads();
    if (threadIdx.x < 32) {
        cholesky_upper_warp(Gs, Rs, inv_diag, r, p.status, true);
        inverse_upper_warp(Rs, inv_diag, Ri, r);
    }
    __syncthreads();
    if (MODE == 1) {
        for (int i = threadIdx.x; i < r * r; i += kCqrThreads) {
            const int a = i / r, b = i - a * r;
            M.R[i] = (float)Rs[a * 32 + b];
        }
    }
    for (int i = threadIdx.x; i < 32 * 32; i += kCqrThreads) M.Rinv[i] = Ri[i];
}

// Q = Y R^{-1} row by row.  MODE 0: Q into Qt (TF32-rounded, transposed)
// [+ Qexact]; MODE 1: U.  The CTA's rows come in, and its row-major outputs
// go out, through a shared tile with 16-byte accesses; a thread keeps its
// row (RMAX doubles) in registers and forms one output column at a time, so
// that several CTAs fit on an SM.
template <int MODE, int RMAX>
__global__ void __launch_bounds__(kCqrThreads) k_cholqr_apply(const __grid_constant__ CholParams p)
{
    const CholMat &M = p.mat[blockIdx.y];
    const int r = p.r;
    __shared__ double Ri[32 * 32];
    __shared__ float tile[kCqrThreads * 33];
    const int row0 = blockIdx.x * kCqrThreads;
    const int nrows = min(kCqrThreads, p.rows - row0);
    for (int i = threadIdx.x; i < 32 * 32; i += kCqrThreads) Ri[i] = M.Rinv[i];
    block_copy<true>(const_cast<float *>(M.Y) + (int64_t)row0 * p.ld, tile, nrows * p.ld, p.ld);
    __syncthreads();
    const int t = threadIdx.x;
    const int row = row0 + t;
    double yv[RMAX];
#pragma unroll
    for (int k = 0; k < RMAX; ++k) yv[k] = (k < r && t < nrows) ? (double)tile[t * 33 + k] : 0.0;
    __syncthreads();   // every row is in registers: the tile now collects outputs
    float *out = MODE == 0 ? M.Qexact : M.U;
#pragma unroll
    for (int c = 0; c < RMAX; ++c) {
        if (c < r) {
            double acc = 0.0;
#pragma unroll
            for (int k = 0; k <= c; ++k) acc += yv[k] * Ri[k * 32 + c];
            if (MODE == 0 && t < nrows) {
                const float f = (float)acc, hi = round_tf32(f);
                M.Qt[(int64_t)c * p.qt_ld + row] = hi;
                if (M.Qt_lo) M.Qt_lo[(int64_t)c * p.qt_ld + row] = round_tf32(f - hi);
            }
            tile[t * 33 + c] = (float)acc;
        }
    }
    if (out) {
        __syncthreads();
        block_copy<false>(out + (int64_t)row0 * r, tile, nrows * r, r);
    }
}

// -------------------------------------------------------------- apply ----
// D = U (R V^T) with E = A - D and/or C += D.  W = R V^T is held in
// registers: a thread owns CPT adjacent columns (4 for r <= 16, 2 for
// r <= 32) for all RMAX rows of W and walks a long strip of rows; warp w
// takes rows w, w + 8, ... of the strip, RF rows at a time, so that every
// thread keeps RF rows of A (and C) in flight.  The U row of each step is
// the same for all lanes of a warp (a broadcast load through L1).
constexpr int kApplyThreads = 256;
constexpr int kApplyRows = 1024;    // rows per CTA strip

struct ApplyMat {
    const float *A;   // [m x n] or null
    const float *U;   // [m x r]
    const float *R;   // [r x r]
    const float *V;   // [n x r]
    float *E;         // [m x n] or null: E = A - D
    float *C;         // [m x n] or null: C += D
    void *recon;      // bf16 [m x n] or null: bf16(C) after C += D (only with C)
};

constexpr int kMaxApplyMats = 192;

struct ApplyParams {
    ApplyMat mat[kMaxApplyMats];
    int nmat;
    int m, n, r;
    int row_tiles, col_tiles;
};
static_assert(sizeof(ApplyParams) <= 32764, "a kernel takes at most 32764 bytes of parameters");

template <int CPT>
struct Vec;
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}
template <> struct Vec<4> {
    using T = float4;
    static __device__ __forceinline__ void load(const float *p, float (&v)[4])
    {
        const float4 x = __ldcs((const float4 *)p);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[4])
    {
        __stcs((float4 *)p, make_float4(v[0], v[1], v[2], v[3]));
    }
    // bf16, rounded to nearest even, at element offset off of a bf16 array
    static __device__ __forceinline__ void store_bf16(void *base, int64_t off, const float (&v)[4])
    {
        __stcs(reinterpret_cast<uint2 *>(static_cast<uint16_t *>(base) + off),
               make_uint2(bf16x2_rn(v[0], v[1]), bf16x2_rn(v[2], v[3])));
    }
};
template <> struct Vec<2> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[2])
    {
        const float2 x = __ldcs((const float2 *)p);
        v[0] = x.x; v[1] = x.y;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[2])
    {
        __stcs((float2 *)p, make_float2(v[0], v[1]));
    }
    static __device__ __forceinline__ void store_bf16(void *base, int64_t off, const float (&v)[2])
    {
        __stcs(reinterpret_cast<unsigned int *>(static_cast<uint16_t *>(base) + off), bf16x2_rn(v[0], v[1]));
    }
};

template <int RMAX, bool HAS_E, bool HAS_C>
__global__ void __launch_bounds__(kApplyThreads, 2) k_apply(const __grid_constant__ ApplyParams p)
{
    constexpr int CPT = 64 / RMAX;                     // columns per thread
    constexpr int COLS = 32 * CPT;                     // columns per CTA
    constexpr int RF = (HAS_E && HAS_C) ? 3 : 6;       // rows in flight per thread
    const int per_mat = p.row_tiles * p.col_tiles;
    const int mi = blockIdx.x / per_mat;
    const int t = blockIdx.x - mi * per_mat;
    const int ct = t % p.col_tiles, rt = t / p.col_tiles;
    const ApplyMat &M = p.mat[mi];
    const int r = p.r, n = p.n, m = p.m;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int row0 = rt * kApplyRows;
    const int row_end = min(m, row0 + kApplyRows);
    const int col = ct * COLS + lane * CPT;

    __shared__ float Rs[32 * 33];
    __shared__ float Vs[COLS * (RMAX + 1)];
    for (int i = threadIdx.x; i < 32 * 33; i += kApplyThreads) {
        const int a = i / 33, b = i - a * 33;
        Rs[i] = (a < r && b < r) ? M.R[a * r + b] : 0.0f;
    }
    for (int i = threadIdx.x; i < COLS * RMAX; i += kApplyThreads) {
        const int j = i / RMAX, c = i - j * RMAX;
        const int gc = ct * COLS + j;
        Vs[j * (RMAX + 1) + c] = (gc < n && c < r) ? M.V[(int64_t)gc * r + c] : 0.0f;
    }
    __syncthreads();
    // W[k][col + c] = sum_{q >= k} R[k][q] V[col + c][q]
    float w[RMAX][CPT];
#pragma unroll
    for (int k = 0; k < RMAX; ++k)
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            float acc = 0.0f;
            const int j = lane * CPT + c;
#pragma unroll
            for (int q = 0; q < RMAX; ++q) acc = fmaf(Rs[k * 33 + q], Vs[j * (RMAX + 1) + q], acc);
            w[k][c] = acc;
        }
    if (col >= n) return;   // n % 4 == 0: a thread's columns are all in or all out

    for (int base = row0 + warp; base < row_end; base += 8 * RF) {
        float av[RF][CPT], cv[RF][CPT];
#pragma unroll
        for (int u = 0; u < RF; ++u) {
            const int row = base + 8 * u;
            if (row < row_end) {
                const int64_t off = (int64_t)row * n + col;
                if (HAS_E && M.E) Vec<CPT>::load(M.A + off, av[u]);
                if (HAS_C && M.C) Vec<CPT>::load(M.C + off, cv[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < RF; ++u) {
            const int row = base + 8 * u;
            if (row >= row_end) break;
            float ur[RMAX];
            const float *urow = M.U + (int64_t)row * r;
#pragma unroll
            for (int k = 0; k < RMAX; ++k) ur[k] = (k < r) ? __ldg(urow + k) : 0.0f;
            float d[CPT];
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < RMAX; ++k) acc = fmaf(ur[k], w[k][c], acc);
                d[c] = acc;
            }
            const int64_t off = (int64_t)row * n + col;
            if (HAS_E && M.E) {
                float e[CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c) e[c] = av[u][c] - d[c];
                Vec<CPT>::store(M.E + off, e);
            }
            if (HAS_C && M.C) {
                float o[CPT];
#pragma unroll
                for (int c = 0; c < CPT; ++c) o[c] = cv[u][c] + d[c];
                Vec<CPT>::store(M.C + off, o);
                if (M.recon) Vec<CPT>::store_bf16(M.recon, off, o);
            }
        }
    }
}

// Apply for r <= 16 with r % 4 == 0: the same arithmetic as k_apply<16>, but
// the rows of A (and C) and U travel through a per-thread ring of cp.async
// copies in shared memory, kAsyncStages deep, so that each thread keeps
// (kAsyncStages - 1) * kAsyncRF rows in flight without holding them in
// registers.  A thread only reads its own A/C copies; the U row of a warp is
// copied by lanes 0..r/4-1 and shared after __syncwarp.
constexpr int kAsyncRF = 4;

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool HAS_E, bool HAS_C>
__host__ __device__ constexpr int async_stages()
{
    // E and C: 3 stages (smem); C only: 5 (85.4% of measured on the receiver of
    // the 57 x 4608 x 3072 step, 4 stages: 84.6%); E only: 4
    return (HAS_E && HAS_C) ? 3 : (HAS_C ? 5 : 4);
}

template <bool HAS_E, bool HAS_C>
constexpr size_t async_smem_bytes()
{
    return (size_t)async_stages<HAS_E, HAS_C>() * kAsyncRF *
           ((HAS_E ? kApplyThreads * 16 : 0) + (HAS_C ? kApplyThreads * 16 : 0) + 8 * 64);
}

// Paired fp32 arithmetic of sm_100 (PTX .f32x2): two independent
// round-to-nearest FMAs in one instruction, on 64-bit register pairs whose
// low half is the first element.
__device__ __forceinline__ unsigned long long f32x2_pack(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ unsigned long long f32x2_fma(unsigned long long a, unsigned long long b,
                                                        unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ float f32x2_sum(unsigned long long a)
{
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a));
    return lo + hi;
}

template <bool HAS_E, bool HAS_C>
__global__ void __launch_bounds__(kApplyThreads, 2) k_apply_async(const __grid_constant__ ApplyParams p)
{
    constexpr int S = async_stages<HAS_E, HAS_C>();
    constexpr int RF = kAsyncRF;
    constexpr int CPT = 4, COLS = 128, RMAX = 16;
    const int per_mat = p.row_tiles * p.col_tiles;
    const int mi = blockIdx.x / per_mat;
    const int t = blockIdx.x - mi * per_mat;
    const int ct = t % p.col_tiles, rt = t / p.col_tiles;
    const ApplyMat &M = p.mat[mi];
    const int r = p.r, n = p.n, m = p.m;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row0 = rt * kApplyRows;
    const int row_end = min(m, row0 + kApplyRows);
    const int col = ct * COLS + lane * CPT;
    const bool col_ok = col < n;    // n % 4 == 0: a thread's 4 columns are all in or all out

    extern __shared__ __align__(16) uint8_t apply_smem[];
    float4 *ringA = reinterpret_cast<float4 *>(apply_smem);
    float4 *ringC = ringA + (HAS_E ? S * RF * kApplyThreads : 0);
    float *ringU = reinterpret_cast<float *>(ringC + (HAS_C ? S * RF * kApplyThreads : 0));
    __shared__ float Rs[32 * 33];
    __shared__ float Vs[COLS * (RMAX + 1)];
    for (int i = tid; i < 32 * 33; i += kApplyThreads) {
        const int a = i / 33, b = i - a * 33;
        Rs[i] = (a < r && b < r) ? M.R[a * r + b] : 0.0f;
    }
    for (int i = tid; i < COLS * RMAX; i += kApplyThreads) {
        const int j = i / RMAX, c = i - j * RMAX;
        const int gc = ct * COLS + j;
        Vs[j * (RMAX + 1) + c] = (gc < n && c < r) ? M.V[(int64_t)gc * r + c] : 0.0f;
    }
    // U slots past column r are never copied: they must read as zero
    for (int i = tid; i < S * RF * 8 * 16; i += kApplyThreads) ringU[i] = 0.0f;
    __syncthreads();
    // W[k][c] for k = 2h (low half) and 2h + 1 (high half) of wp[h][c]: the
    // row products below accumulate even and odd k in the two halves of a pair
    // (half the FMA instructions; the kernel is otherwise issue-bound).
    unsigned long long wp[RMAX / 2][CPT];
#pragma unroll
    for (int h = 0; h < RMAX / 2; ++h)
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            float acc[2] = {0.0f, 0.0f};
            const int j = lane * CPT + c;
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int q = 0; q < RMAX; ++q) acc[e] = fmaf(Rs[(2 * h + e) * 33 + q], Vs[j * (RMAX + 1) + q], acc[e]);
            wp[h][c] = f32x2_pack(acc[0], acc[1]);
        }

    const int nrows = row_end - row0;
    const int ngroups = nrows > 0 ? (nrows + 8 * RF - 1) / (8 * RF) : 0;
    const int uchunks = r / 4;
    auto issue = [&](int g, int slot) {
#pragma unroll
        for (int u = 0; u < RF; ++u) {
            const int row = row0 + g * 8 * RF + warp + 8 * u;
            const bool valid = row < row_end;
            const int safe_row = valid ? row : row0;
            const int64_t off = (int64_t)safe_row * n + (col_ok ? col : 0);
            // a matrix without E (or C) reads nothing: zero bytes from a valid address
            if (HAS_E)
                cp_async16(&ringA[(slot * RF + u) * kApplyThreads + tid], M.E ? M.A + off : M.U,
                           valid && col_ok && M.E != nullptr);
            if (HAS_C)
                cp_async16(&ringC[(slot * RF + u) * kApplyThreads + tid], M.C ? M.C + off : M.U,
                           valid && col_ok && M.C != nullptr);
            if (lane < uchunks)
                cp_async16(&ringU[((slot * RF + u) * 8 + warp) * 16 + lane * 4], M.U + (int64_t)safe_row * r + lane * 4,
                           valid);
        }
    };
#pragma unroll
    for (int s = 0; s < S - 1; ++s) {
        if (s < ngroups) issue(s, s);
        cp_async_commit();
    }
    for (int g = 0; g < ngroups; ++g) {
        const int gi = g + S - 1;
        if (gi < ngroups) issue(gi, gi % S);
        cp_async_commit();
        cp_async_wait<S - 1>();
        __syncwarp();
        const int slot = g % S;
#pragma unroll
        for (int u = 0; u < RF; ++u) {
            const int row = row0 + g * 8 * RF + warp + 8 * u;
            if (row >= row_end || !col_ok) continue;
            // U row as (u_2h, u_2h+1) pairs, straight from shared memory
            const ulonglong2 *urow = reinterpret_cast<const ulonglong2 *>(&ringU[((slot * RF + u) * 8 + warp) * 16]);
            unsigned long long dp[CPT] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int k4 = 0; k4 < RMAX / 4; ++k4) {
                const ulonglong2 uk = urow[k4];
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    dp[c] = f32x2_fma(uk.x, wp[2 * k4][c], dp[c]);
                    dp[c] = f32x2_fma(uk.y, wp[2 * k4 + 1][c], dp[c]);
                }
            }
            float d[CPT];
#pragma unroll
            for (int c = 0; c < CPT; ++c) d[c] = f32x2_sum(dp[c]);
            const int64_t off = (int64_t)row * n + col;
            if (HAS_E && M.E) {
                const float4 a = ringA[(slot * RF + u) * kApplyThreads + tid];
                __stcs((float4 *)(M.E + off), make_float4(a.x - d[0], a.y - d[1], a.z - d[2], a.w - d[3]));
            }
            if (HAS_C && M.C) {
                const float4 c = ringC[(slot * RF + u) * kApplyThreads + tid];
                const float o[CPT] = {c.x + d[0], c.y + d[1], c.z + d[2], c.w + d[3]};
                Vec<CPT>::store(M.C + off, o);
                if (M.recon) Vec<CPT>::store_bf16(M.recon, off, o);
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
}

// ----------------------------------------------------------- host side ---

int64_t rup(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
    int rp;
    bool split;                           // split (3xTF32) products: lo parts of Q^T and P^T too
    int64_t mp, np;                       // padded leading dims (multiples of 32)
    size_t qt, pt, qt_lo, pt_lo, pe, z, cnt, gp, ri, total;   // byte offsets inside the workspace
    int chunks;                           // Gram chunks of the tallest block
};

WsLayout layout(int nmat, int64_t m, int64_t n, int r, bool split)
{
    WsLayout L{};
    L.rp = r <= 16 ? 16 : 32;
    L.split = split;
    L.mp = rup(m, 32);
    L.np = rup(n, 32);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (size_t)rup((int64_t)bytes, 256);
        return o;
    };
    L.qt = take((size_t)nmat * L.rp * L.np * 4);
    L.pt = take((size_t)nmat * L.rp * L.mp * 4);
    L.qt_lo = split ? take((size_t)nmat * L.rp * L.np * 4) : 0;
    L.pt_lo = split ? take((size_t)nmat * L.rp * L.mp * 4) : 0;
    L.pe = take((size_t)nmat * m * L.rp * 4);
    L.z = take((size_t)nmat * n * L.rp * 4);
    L.cnt = take((size_t)nmat * sizeof(unsigned int));
    L.chunks = (int)((std::max(m, n) + kCqrRows - 1) / kCqrRows);
    L.gp = take((size_t)nmat * L.chunks * (r * (r + 1) / 2) * 8);
    L.ri = take((size_t)nmat * 32 * 32 * 8);
    L.total = off;
    return L;
}

template <int RP, int CPS, bool SPLIT>
cudaError_t gemm_launch_rp(GemmParams &gp, int grid, cudaStream_t stream)
{
    // the shared-memory opt-in is a per-device function attribute: set it once per device
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64 || !done[dev]) {
            e = cudaFuncSetAttribute(k_gemm_tf32<RP, CPS, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)gemm_smem_bytes<RP, CPS, SPLIT>());
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) done[dev] = true;
        }
    }
    const char *name = SPLIT ? (RP == 16 ? "k_gemm_tf32<16,split>" : "k_gemm_tf32<32,split>")
                             : (RP == 16 ? "k_gemm_tf32<16>" : "k_gemm_tf32<32>");
    log_launch(name, dim3(grid), dim3(kGemmThreads), gemm_smem_bytes<RP, CPS, SPLIT>());
    trace_begin(name, stream);
    k_gemm_tf32<RP, CPS, SPLIT><<<grid, kGemmThreads, gemm_smem_bytes<RP, CPS, SPLIT>(), stream>>>(gp);
    trace_end(stream);
    return cudaGetLastError();
}

// Resident CTAs per SM for a launch of `total_tiles` tiles (see GemmCfg).
int gemm_cps(int rp, bool split, int64_t total_tiles)
{
    return !split && rp == 16 && total_tiles >= 2 * (int64_t)num_sms() ? 2 : 1;
}

cudaError_t gemm_launch(GemmParams &gp, int total_tiles, int cps, bool split, cudaStream_t stream)
{
    const int grid = total_tiles < cps * num_sms() ? total_tiles : cps * num_sms();
    if (grid <= 0) return cudaSuccess;
    if (split) return gp.rp != 16 ? gemm_launch_rp<32, 1, true>(gp, grid, stream) : gemm_launch_rp<16, 1, true>(gp, grid, stream);
    if (gp.rp != 16) return gemm_launch_rp<32, 1, false>(gp, grid, stream);
    return cps == 2 ? gemm_launch_rp<16, 2, false>(gp, grid, stream) : gemm_launch_rp<16, 1, false>(gp, grid, stream);
}

int gemm_bk(int rp, int cps, bool split)
{
    if (split) return rp != 16 ? GemmCfg<32, 1, true>::BK : GemmCfg<16, 1, true>::BK;
    return rp != 16 ? GemmCfg<32, 1>::BK : (cps == 2 ? GemmCfg<16, 2>::BK : GemmCfg<16, 1>::BK);
}

// out_i = A_i Q_i (mn_major = 0) or A_i^T P_i (mn_major = 1) for every matrix.
cudaError_t gemm_pass(const LowrankPlan &pl, const LowrankMat *mats, const WsLayout &L, int mn_major, int out_mode,
                      cudaStream_t stream)
{
    char *ws = (char *)pl.ws;
    const int64_t m = pl.m, n = pl.n;
    GemmParams *gp = new GemmParams;
    cudaError_t err = cudaSuccess;
    for (int first = 0; first < pl.nmat && err == cudaSuccess; first += kMaxGemmMats) {
        const int cnt = pl.nmat - first < kMaxGemmMats ? pl.nmat - first : kMaxGemmMats;
        memset(gp, 0, sizeof *gp);
        gp->nmat = cnt;
        gp->rp = L.rp;
        gp->mn_major = mn_major;
        gp->out_mode = out_mode;
        gp->status = pl.status;
        gp->wait_ns = kWaitNs;
        // Fault injection for the failure-detection test (see LowrankPlan::starve):
        // the producer loads nothing, so the consumers' bounded waits on the
        // "tile landed" barriers run out (after 20 ms) and the kernel returns
        // with the timeout bit set in the status word.
        if (pl.starve) {
            gp->starve = 1;
            gp->wait_ns = 20000000ull;
        }
        bool ok;
        const int cps = gemm_cps(L.rp, L.split, (int64_t)cnt * (((!mn_major ? m : n) + kBM - 1) / kBM));
        const int bk = gemm_bk(L.rp, cps, L.split);
        if (!mn_major) {
            gp->tiles_per_mat = (int)((m + kBM - 1) / kBM);
            gp->ktiles = (int)((n + bk - 1) / bk);
            gp->out_rows = (int)m;
            gp->out_ld = (int)L.mp;
            ok = make_map3(&gp->tb, ws + L.qt + (size_t)first * L.rp * L.np * 4, n, L.rp, cnt, L.np, L.rp * L.np,
                           kBoxK, L.rp);
            if (ok && L.split)
                ok = make_map3(&gp->tb_lo, ws + L.qt_lo + (size_t)first * L.rp * L.np * 4, n, L.rp, cnt, L.np,
                               L.rp * L.np, kBoxK, L.rp);
            if (out_mode == 0) {
                gp->out = (float *)(ws + L.pt) + (size_t)first * L.rp * L.mp;
                gp->out_lo = L.split ? (float *)(ws + L.pt_lo) + (size_t)first * L.rp * L.mp : nullptr;
                gp->out_stride = L.rp * L.mp;
            } else {
                gp->out = (float *)(ws + L.pe) + (size_t)first * m * L.rp;
                gp->out_stride = m * L.rp;
            }
        } else {
            gp->tiles_per_mat = (int)((n + kBM - 1) / kBM);
            gp->ktiles = (int)((m + bk - 1) / bk);
            gp->out_rows = (int)n;
            gp->out_ld = 0;
            ok = make_map3(&gp->tb, ws + L.pt + (size_t)first * L.rp * L.mp * 4, m, L.rp, cnt, L.mp, L.rp * L.mp,
                           kBoxK, L.rp);
            if (ok && L.split)
                ok = make_map3(&gp->tb_lo, ws + L.pt_lo + (size_t)first * L.rp * L.mp * 4, m, L.rp, cnt, L.mp,
                               L.rp * L.mp, kBoxK, L.rp);
            gp->out = (float *)(ws + L.z) + (size_t)first * n * L.rp;
            gp->out_stride = n * L.rp;
        }
        for (int k = 0; k < cnt && ok; ++k) {
            const LowrankMat &s = mats[first + k];
            ok = !mn_major ? make_map(&gp->mat[k].ta, s.A, n, m, n, kBoxK, kBM)
                           : make_map(&gp->mat[k].ta, s.A, n, m, n, 32, kBoxK, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
        }
        if (!ok) {
            err = cudaErrorInvalidValue;
            break;
        }
        err = gemm_launch(*gp, cnt * gp->tiles_per_mat, cps, L.split, stream);
    }
    delete gp;
    return err;
}

// CholeskyQR of a tall block for every matrix: mode 0 writes Qt (+ V when
// `final_v`), mode 1 writes U and R.  Two launches (per 192 matrices).
cudaError_t cholqr_pass(const LowrankPlan &pl, const LowrankMat *mats, const WsLayout &L, int src, int mode,
                        bool final_v, cudaStream_t stream)
{
    char *ws = (char *)pl.ws;
    const int64_t m = pl.m, n = pl.n;
    const int r = pl.r;
    const int npairs = r * (r + 1) / 2;
    // src: 0 = Q0 (n x r), 1 = Z (n x rp), 2 = P exact (m x rp)
    const int rows = (int)(src == 2 ? m : n);
    const int ld = src == 0 ? r : L.rp;
    CholParams *cp = new CholParams;
    cudaError_t err = cudaSuccess;
    for (int first = 0; first < pl.nmat && err == cudaSuccess; first += kMaxCholMats) {
        const int cnt = pl.nmat - first < kMaxCholMats ? pl.nmat - first : kMaxCholMats;
        memset(cp, 0, sizeof *cp);
        cp->nmat = cnt;
        cp->rows = rows;
        cp->ld = ld;
        cp->r = r;
        cp->qt_ld = (int)L.np;
        cp->status = pl.status;
        for (int k = 0; k < cnt; ++k) {
            const int i = first + k;
            CholMat &c = cp->mat[k];
            c.Y = src == 0 ? mats[i].Q0
                           : (src == 1 ? (const float *)(ws + L.z + (size_t)i * n * L.rp * 4)
                                       : (const float *)(ws + L.pe + (size_t)i * m * L.rp * 4));
            c.Gpart = (double *)(ws + L.gp + (size_t)i * L.chunks * npairs * 8);
            c.count = (unsigned int *)(ws + L.cnt) + i;
            c.Rinv = (double *)(ws + L.ri + (size_t)i * 32 * 32 * 8);
            c.Qt = (float *)(ws + L.qt + (size_t)i * L.rp * L.np * 4);
            c.Qt_lo = L.split ? (float *)(ws + L.qt_lo + (size_t)i * L.rp * L.np * 4) : nullptr;
            c.Qexact = final_v ? mats[i].V : nullptr;
            c.U = mats[i].U;
            c.R = mats[i].R;
        }
        dim3 fgrid((unsigned)((rows + kCqrRows - 1) / kCqrRows), (unsigned)cnt);
        dim3 agrid((unsigned)((rows + kCqrThreads - 1) / kCqrThreads), (unsigned)cnt);
        const bool r16 = r <= 16;
        const char *fname = mode == 0 ? "k_cholqr_factor<Q>" : "k_cholqr_factor<U>";
        const char *aname = mode == 0 ? "k_cholqr_apply<Q>" : "k_cholqr_apply<U>";
        log_launch(fname, fgrid, dim3(kCqrThreads), 0);
        log_launch(aname, agrid, dim3(kCqrThreads), 0);
        trace_begin(fname, stream);
        if (mode == 0)
            k_cholqr_factor<0><<<fgrid, kCqrThreads, 0, stream>>>(*cp);
        else
            k_cholqr_factor<1><<<fgrid, kCqrThreads, 0, stream>>>(*cp);
        trace_end(stream);
        trace_begin(aname, stream);
        if (mode == 0) {
            if (r16)
                k_cholqr_apply<0, 16><<<agrid, kCqrThreads, 0, stream>>>(*cp);
            else
                k_cholqr_apply<0, 32><<<agrid, kCqrThreads, 0, stream>>>(*cp);
        } else {
            if (r16)
                k_cholqr_apply<1, 16><<<agrid, kCqrThreads, 0, stream>>>(*cp);
            else
                k_cholqr_apply<1, 32><<<agrid, kCqrThreads, 0, stream>>>(*cp);
        }
        trace_end(stream);
        err = cudaGetLastError();
    }
    delete cp;
    return err;
}

cudaError_t apply_pass(const LowrankPlan &pl, const LowrankMat *mats, bool sender, cudaStream_t stream)
{
    ApplyParams *ap = new ApplyParams;
    cudaError_t err = cudaSuccess;
    const int rmax = pl.r <= 16 ? 16 : 32;
    const int cols = 32 * (64 / rmax);
    for (int first = 0; first < pl.nmat && err == cudaSuccess; first += kMaxApplyMats) {
        const int cnt = pl.nmat - first < kMaxApplyMats ? pl.nmat - first : kMaxApplyMats;
        memset(ap, 0, sizeof *ap);
        ap->nmat = cnt;
        ap->m = (int)pl.m;
        ap->n = (int)pl.n;
        ap->r = pl.r;
        ap->row_tiles = (int)((pl.m + kApplyRows - 1) / kApplyRows);
        ap->col_tiles = (int)((pl.n + cols - 1) / cols);
        bool has_e = false, has_c = false;
        for (int k = 0; k < cnt; ++k) {
            const LowrankMat &s = mats[first + k];
            ApplyMat &a = ap->mat[k];
            a.A = s.A;
            a.U = s.U;
            a.R = s.R;
            a.V = s.V;
            a.E = sender ? s.E : nullptr;
            a.C = s.C;
            a.recon = s.C ? s.recon : nullptr;
            has_e = has_e || a.E;
            has_c = has_c || a.C;
        }
        if (!has_e && !has_c) continue;
        const unsigned blocks = (unsigned)((int64_t)cnt * ap->row_tiles * ap->col_tiles);
        using Fn = void (*)(ApplyParams);
        Fn fn;
        if (rmax == 16 && pl.r % 4 == 0) {
            // copies through a cp.async ring (U rows are 16-byte chunks when r % 4 == 0)
            size_t smem;
            if (has_e && has_c) {
                fn = k_apply_async<true, true>;
                smem = async_smem_bytes<true, true>();
            } else if (has_e) {
                fn = k_apply_async<true, false>;
                smem = async_smem_bytes<true, false>();
            } else {
                fn = k_apply_async<false, true>;
                smem = async_smem_bytes<false, true>();
            }
            cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            log_launch("k_apply_async", dim3(blocks), dim3(kApplyThreads), smem);
            trace_begin("k_apply_async", stream);
            fn<<<blocks, kApplyThreads, smem, stream>>>(*ap);
            trace_end(stream);
            err = cudaGetLastError();
            continue;
        }
        if (rmax == 16)
            fn = has_e ? (has_c ? k_apply<16, true, true> : k_apply<16, true, false>) : k_apply<16, false, true>;
        else
            fn = has_e ? (has_c ? k_apply<32, true, true> : k_apply<32, true, false>) : k_apply<32, false, true>;
        log_launch("k_apply", dim3(blocks), dim3(kApplyThreads), 0);
        trace_begin("k_apply", stream);
        fn<<<blocks, kApplyThreads, 0, stream>>>(*ap);
        trace_end(stream);
        err = cudaGetLastError();
    }
    delete ap;
    return err;
}

}  // namespace

bool lowrank_split(int precision, int64_t m, int64_t n, int r)
{
    if (precision == CF_PRECISION_SPLIT) return true;
    if (precision == CF_PRECISION_TF32) return false;
    // automatic: split products where the rank is a large fraction of the
    // smaller dimension, i.e. where a few iterations leave the subspace far
    // from converged and the result follows every rounding of the products
    return (int64_t)8 * r > std::min(m, n);
}

size_t lowrank_workspace_bytes(int nmat, int64_t m, int64_t n, int r, bool split)
{
    return layout(nmat, m, n, r, split).total;
}

cudaError_t run_lowrank(const LowrankPlan &pl, const LowrankMat *mats, cudaStream_t stream)
{
    if (pl.nmat <= 0) return cudaSuccess;
    if (pl.m > INT32_MAX || pl.n > INT32_MAX) return cudaErrorInvalidValue;
    const WsLayout L = layout(pl.nmat, pl.m, pl.n, pl.r, pl.split);
    if (pl.ws_bytes < L.total) return cudaErrorInvalidValue;
    char *ws = (char *)pl.ws;
    // Padded rows of Q^T (rows r..rp-1) must be zero: they feed zero columns.
    cudaError_t err = cudaMemsetAsync(ws + L.qt, 0, (size_t)pl.nmat * L.rp * L.np * 4, stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(ws + L.pt, 0, (size_t)pl.nmat * L.rp * L.mp * 4, stream);
    if (err == cudaSuccess && L.split) err = cudaMemsetAsync(ws + L.qt_lo, 0, (size_t)pl.nmat * L.rp * L.np * 4, stream);
    if (err == cudaSuccess && L.split) err = cudaMemsetAsync(ws + L.pt_lo, 0, (size_t)pl.nmat * L.rp * L.mp * 4, stream);
    // CholeskyQR chunk counters start at zero (each launch leaves them at zero)
    if (err == cudaSuccess) err = cudaMemsetAsync(ws + L.cnt, 0, (size_t)pl.nmat * sizeof(unsigned int), stream);
    // Line 1: Q = orth(Q0).
    if (err == cudaSuccess) err = cholqr_pass(pl, mats, L, 0, 0, pl.T == 0, stream);
    // Lines 2-5: T times Z = A^T (A Q), Q = orth(Z).
    for (int t = 0; t < pl.T && err == cudaSuccess; ++t) {
        err = gemm_pass(pl, mats, L, 0, 0, stream);                      // P^T = (A Q)^T, TF32-rounded
        if (err == cudaSuccess) err = gemm_pass(pl, mats, L, 1, 1, stream);   // Z = A^T P
        if (err == cudaSuccess) err = cholqr_pass(pl, mats, L, 1, 0, t == pl.T - 1, stream);
    }
    // Lines 6-8: P = A Q; (U, R) = orth(P); V = Q.
    if (err == cudaSuccess) err = gemm_pass(pl, mats, L, 0, 1, stream);
    if (err == cudaSuccess) err = cholqr_pass(pl, mats, L, 2, 1, false, stream);
    // Apply: E = A - U R V^T and/or C += U R V^T.
    if (err == cudaSuccess) err = apply_pass(pl, mats, true, stream);
    return err;
}

cudaError_t run_lowrank_decompress(const LowrankPlan &pl, const LowrankMat *mats, cudaStream_t stream)
{
    if (pl.m > INT32_MAX || pl.n > INT32_MAX) return cudaErrorInvalidValue;
    return apply_pass(pl, mats, false, stream);
}

}  // namespace cf
