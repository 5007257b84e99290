// Host allocation failures injected into libcf's cf_create, on the host.
//
// This test program replaces the global C++ allocation functions with a fake
// that can be told to fail the N-th allocation after it is armed (the
// throwing forms throw std::bad_alloc, the nothrow forms return NULL).  The
// executable's definitions take precedence over libstdc++'s for every shared
// library in the process, libcf included.  For every N up to the number of
// allocations cf_create makes, the call must return an error -- CF_E_NOMEM
// where libcf's own allocation failed -- with *out left NULL, and must not
// let an exception escape the C ABI (the process would abort).  Afterwards,
// disarmed, cf_create works again.  No GPU fault is involved: the GPU is only
// needed because cf_create checks for an sm_100 device before it allocates.
// Prints "ok".
#include <cstdio>
#include <cstdlib>
#include <new>

#include <cuda_runtime_api.h>

#include "cf.h"

namespace {
long g_fail_at = 0;   // 0: disarmed; N > 0: the N-th allocation after arming fails
long g_count = 0;     // allocations since arming

bool fail_now()
{
    if (g_fail_at <= 0) return false;
    return ++g_count == g_fail_at;
}

void arm(long n)
{
    g_fail_at = n;
    g_count = 0;
}
}  // namespace

void *operator new(std::size_t n)
{
    if (fail_now()) throw std::bad_alloc();
    void *p = std::malloc(n ? n : 1);
    if (!p) throw std::bad_alloc();
    return p;
}
void *operator new[](std::size_t n)
{
    if (fail_now()) throw std::bad_alloc();
    void *p = std::malloc(n ? n : 1);
    if (!p) throw std::bad_alloc();
    return p;
}
void *operator new(std::size_t n, const std::nothrow_t &) noexcept { return fail_now() ? nullptr : std::malloc(n ? n : 1); }
void *operator new[](std::size_t n, const std::nothrow_t &) noexcept { return fail_now() ? nullptr : std::malloc(n ? n : 1); }
void operator delete(void *p) noexcept { std::free(p); }
void operator delete[](void *p) noexcept { std::free(p); }
void operator delete(void *p, std::size_t) noexcept { std::free(p); }
void operator delete[](void *p, std::size_t) noexcept { std::free(p); }
void operator delete(void *p, const std::nothrow_t &) noexcept { std::free(p); }
void operator delete[](void *p, const std::nothrow_t &) noexcept { std::free(p); }

static int fail(const char *what, long n, int st)
{
    std::fprintf(stderr, "FAIL %s (N = %ld, status %d)\n", what, n, st);
    return 1;
}

int main()
{
    if (cudaFree(nullptr) != cudaSuccess) return fail("CUDA initialisation", 0, -1);   // context first, unarmed
    cf_config cfg{};
    cfg.mode = CF_MODE_QUANT;
    cfg.bits = 2;
    cfg.group = 128;
    const cf_shape shapes[3] = {{64, 256}, {0, 128}, {37, 512}};

    // how many allocations an unarmed cf_create makes
    arm(1L << 40);
    cf_ctx *ctx = nullptr;
    int st = cf_create(&cfg, 3, shapes, &ctx);
    const long made = g_count;
    arm(0);
    if (st != CF_OK || !ctx) return fail("unarmed cf_create", 0, st);
    cf_destroy(ctx);
    if (made < 2) return fail("cf_create should allocate the context and the shape table", made, st);

    int nomem = 0;
    for (long n = 1; n <= made; ++n) {
        ctx = reinterpret_cast<cf_ctx *>(0x1);
        arm(n);
        st = cf_create(&cfg, 3, shapes, &ctx);
        arm(0);
        if (st == CF_OK) return fail("cf_create succeeded with a failed allocation", n, st);
        if (ctx != nullptr) return fail("*out not NULL after a failed cf_create", n, st);
        if (st == CF_E_NOMEM) ++nomem;
        else if (st != CF_E_CUDA) return fail("unexpected status", n, st);
    }
    // the context and the shape table are libcf's own: at least those two fail with CF_E_NOMEM
    if (nomem < 2) return fail("too few CF_E_NOMEM results", nomem, 0);

    // disarmed, the library works again
    st = cf_create(&cfg, 3, shapes, &ctx);
    if (st != CF_OK || !ctx) return fail("cf_create after the injected failures", 0, st);
    if (cf_payload_bytes(ctx, 0) != 64 * 256 * 2 / 8 + 4 * (64 * 256 / 128)) return fail("payload bytes", 0, 0);
    cf_destroy(ctx);
    std::printf("ok\n");
    return 0;
}
