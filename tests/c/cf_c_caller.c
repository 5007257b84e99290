/* A plain C caller of libcf: the C ABI used without Python or torch.
 *
 * One quantised slot (k = 2, G = 128) of 300 x 768 bf16 activations whose
 * step-to-step change is the same constant c in every element.  With the
 * pages' residual + error-feedback scheme (abstract of "Accelerating Parallel
 * Diffusion Model Serving with Residual Compression"), each residual group is
 * constant, so absmax quantisation represents it exactly: after every step the
 * receiver cache equals X_t and the error buffer is zero.  The program checks
 * that, plus the argument errors, and prints "ok".  Build:
 *   gcc -std=c11 -I include -I <cuda>/include cf_c_caller.c -L <pkg> -lcf -L <cuda>/lib64 -lcudart
 */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "cf.h"

#define ROWS 300
#define COLS 768
#define N (ROWS * COLS)

static int fail(const char *what, int code)
{
    fprintf(stderr, "FAIL %s (%d)\n", what, code);
    return 1;
}

static unsigned short to_bf16(float f)   /* exact for the values used here */
{
    unsigned int u;
    memcpy(&u, &f, 4);
    return (unsigned short)(u >> 16);
}

int main(void)
{
    cf_config cfg;
    memset(&cfg, 0, sizeof cfg);
    cfg.mode = CF_MODE_QUANT;
    cfg.bits = 2;
    cfg.group = 128;
    cf_shape shape = {ROWS, COLS};
    cf_ctx *ctx = NULL;
    int st = cf_create(&cfg, 1, &shape, &ctx);
    if (st != CF_OK) return fail("cf_create", st);

    cf_shape bad = {ROWS, 100};
    cf_ctx *ctx2 = NULL;
    if (cf_create(&cfg, 1, &bad, &ctx2) != CF_E_SHAPE || ctx2) return fail("cols % 8 must be refused", 0);

    void *x, *base, *err, *cache, *codes, *scales;
    if (cudaMalloc(&x, N * 2) || cudaMalloc(&base, N * 2) || cudaMalloc(&err, N * 4) || cudaMalloc(&cache, N * 4) ||
        cudaMalloc(&codes, N * 2 / 8) || cudaMalloc(&scales, N / 128 * 4))
        return fail("cudaMalloc", 0);
    unsigned short *hx = malloc(N * 2);
    float *hc = malloc(N * 4), *he = malloc(N * 4);

    cf_slot slot;
    memset(&slot, 0, sizeof slot);
    slot.x = x;
    slot.base = base;
    slot.err = err;
    slot.cache = cache;
    slot.codes = codes;
    slot.scales = scales;

    if (cf_compress(ctx, &slot, 1, NULL) != CF_E_STATE) return fail("step 1 before the warmup must be refused", 0);

    for (int t = 0; t < 4; ++t) {
        /* X_t = (i % 7 - 3) / 4 + t / 2: every step adds the constant 1/2 (exact in bf16) */
        for (int i = 0; i < N; ++i) hx[i] = to_bf16((float)(i % 7 - 3) * 0.25f + 0.5f * (float)t);
        if (cudaMemcpy(x, hx, N * 2, cudaMemcpyHostToDevice)) return fail("copy in", t);
        if ((st = cf_compress(ctx, &slot, t, NULL)) != CF_OK) return fail(cf_last_error(ctx), st);
        if ((st = cf_decompress(ctx, &slot, t, NULL)) != CF_OK) return fail(cf_last_error(ctx), st);
        if ((st = cf_check(ctx, NULL)) != CF_OK) return fail("cf_check", st);
        if (cudaMemcpy(hc, cache, N * 4, cudaMemcpyDeviceToHost) || cudaMemcpy(he, err, N * 4, cudaMemcpyDeviceToHost))
            return fail("copy out", t);
        for (int i = 0; i < N; ++i) {
            const float want = (float)(i % 7 - 3) * 0.25f + 0.5f * (float)t;
            if (hc[i] != want || he[i] != 0.0f) {
                fprintf(stderr, "step %d element %d: cache %g err %g, want %g and 0\n", t, i, hc[i], he[i], want);
                return 1;
            }
        }
    }
    if (cf_payload_bytes(ctx, 0) != (size_t)(N * 2 / 8 + N / 128 * 4)) return fail("cf_payload_bytes", 0);
    cf_destroy(ctx);
    printf("ok\n");
    return 0;
}
