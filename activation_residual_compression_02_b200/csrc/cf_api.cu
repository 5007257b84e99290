// cf_api.cu -- the libcf C ABI: validation, context, grouped launches.
//
// Semantics follow "Accelerating Parallel Diffusion Model Serving with
// Residual Compression" (arXiv 2507.17511): abstract (send the compressed
// step-wise residual, keep an error-feedback buffer), reproducibility table
// "Dataset Splits" row (an uncompressed warmup step initialises the base
// tensor) and "Pseudocode" row, Algorithm 3 (rank-r subspace iteration).
#include <stdarg.h>
#include <stdlib.h>
#include <stdio.h>
#include <string.h>

#include <new>
#include <string>
#include <vector>

#include "cf_internal.h"

namespace cf {

// Event pairs of traced launches, summed per kernel name by cf_trace_read.
struct Tracer {
    struct Rec {
        std::string kernel;
        cudaEvent_t e0, e1;
    };
    std::vector<Rec> recs;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pool;   // events free for reuse
    bool failed = false;                                     // an event could not be created or recorded
    ~Tracer()
    {
        for (auto &r : recs) pool.emplace_back(r.e0, r.e1);
        for (auto &e : pool) {
            cudaEventDestroy(e.first);
            cudaEventDestroy(e.second);
        }
    }
};

}  // namespace cf

struct cf_ctx {
    cf_config cfg{};
    bool tracing = false;
    cf::Tracer tracer;
    std::vector<cf_shape> shapes;
    uint32_t *d_status = nullptr;
    void *ws = nullptr;
    size_t ws_bytes = 0;
    bool warm_sender = false;
    bool warm_receiver = false;
    int64_t lowrank_steps = 0;   // compressed low-rank steps done (for warm_start)
    bool starve_once = false;    // failure-detection test: the next cf_lowrank withholds its loads
    bool starve_attention_once = false;   // the same for the next cf_attention
    int device = 0;
    std::string err;
};

namespace cf {

bool log_enabled()
{
    static const bool on = [] {
        const char *v = getenv("CF_LOG");
        return v && v[0] == '1';
    }();
    return on;
}

void log_launch(const char *kernel, dim3 grid, dim3 block, size_t smem)
{
    if (!log_enabled()) return;
    fprintf(stderr, "cf: launch %s grid (%u, %u, %u) block (%u, %u, %u) smem %zu\n", kernel, grid.x, grid.y, grid.z,
            block.x, block.y, block.z, smem);
}

namespace {
thread_local Tracer *t_tracer = nullptr;   // the tracer of the API call running on this thread
}

bool trace_on() { return t_tracer != nullptr; }

void trace_begin(const char *kernel, cudaStream_t stream)
{
    Tracer *t = t_tracer;
    if (!t) return;
    std::pair<cudaEvent_t, cudaEvent_t> ev;
    if (!t->pool.empty()) {
        ev = t->pool.back();
        t->pool.pop_back();
    } else if (cudaEventCreate(&ev.first) != cudaSuccess) {
        t->failed = true;
        return;
    } else if (cudaEventCreate(&ev.second) != cudaSuccess) {
        cudaEventDestroy(ev.first);
        t->failed = true;
        return;
    }
    if (cudaEventRecord(ev.first, stream) != cudaSuccess) t->failed = true;
    t->recs.push_back(Tracer::Rec{kernel, ev.first, ev.second});
}

void trace_end(cudaStream_t stream)
{
    Tracer *t = t_tracer;
    if (!t || t->recs.empty()) return;
    if (cudaEventRecord(t->recs.back().e1, stream) != cudaSuccess) t->failed = true;
}

}  // namespace cf

namespace {

// Makes the context's device current for the duration of one API call (a
// process may drive several GPUs, each with its own contexts) and restores
// the caller's device afterwards.
struct DeviceGuard {
    int prev = -1;
    explicit DeviceGuard(const cf_ctx *ctx)
    {
        int cur = 0;
        if (ctx && cudaGetDevice(&cur) == cudaSuccess && cur != ctx->device && cudaSetDevice(ctx->device) == cudaSuccess)
            prev = cur;
    }
    ~DeviceGuard()
    {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

// Sets this thread's tracer for the duration of one API call of a tracing context.
struct TraceGuard {
    explicit TraceGuard(cf_ctx *ctx)
    {
        if (ctx && ctx->tracing) cf::t_tracer = &ctx->tracer;
    }
    ~TraceGuard() { cf::t_tracer = nullptr; }
};

cf_status fail(cf_ctx *ctx, cf_status st, const char *fmt, ...)
{
    if (ctx) {
        char buf[512];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        ctx->err = buf;
    }
    return st;
}

cf_status cuda_fail(cf_ctx *ctx, cudaError_t e, const char *what)
{
    return fail(ctx, CF_E_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

cf_status validate_config(const cf_config *c, std::string &why)
{
    if (c->mode == CF_MODE_QUANT) {
        if (c->bits != 1 && c->bits != 2 && c->bits != 4) { why = "bits must be 1, 2 or 4"; return CF_E_ARG; }
        if (!pow2(c->group) || c->group < 8 || c->group > 256) { why = "group must be a power of two in [8, 256]"; return CF_E_ARG; }
        if (c->sign_scale != 0 && c->sign_scale != 1) { why = "sign_scale must be 0 or 1"; return CF_E_ARG; }
        if (c->state_bf16 != 0 && c->state_bf16 != 1) { why = "state_bf16 must be 0 or 1"; return CF_E_ARG; }
        if (c->warm_start != 0) { why = "warm_start is a low-rank-mode option"; return CF_E_ARG; }
        if (c->precision != 0) { why = "precision is a low-rank-mode option"; return CF_E_ARG; }
        return CF_OK;
    }
    if (c->mode == CF_MODE_LOWRANK) {
        if (c->state_bf16 != 0) { why = "the lean bf16 state is a quantised-mode option"; return CF_E_ARG; }
        if (c->warm_start != 0 && c->warm_start != 1) { why = "warm_start must be 0 or 1"; return CF_E_ARG; }
        if (c->rank < 1 || c->rank > 32) { why = "rank must be in [1, 32]"; return CF_E_ARG; }
        if (c->iters < 0 || c->iters > 1000) { why = "iters must be in [0, 1000]"; return CF_E_ARG; }
        if (c->precision < CF_PRECISION_AUTO || c->precision > CF_PRECISION_SPLIT) {
            why = "precision must be CF_PRECISION_AUTO, _TF32 or _SPLIT";
            return CF_E_ARG;
        }
        return CF_OK;
    }
    why = "mode must be CF_MODE_QUANT or CF_MODE_LOWRANK";
    return CF_E_ARG;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Low-rank mode workspace: the fp32 residual of every slot (256-byte
// aligned), then the Algorithm 3 buffers for the largest run of equal shapes.
size_t lowrank_residual_bytes(const cf_ctx *ctx)
{
    size_t b = 0;
    for (const cf_shape &s : ctx->shapes) b += round_up((size_t)(s.rows * s.cols) * 4, 256);
    return b;
}

template <class F>
void for_each_run(const std::vector<cf_shape> &shapes, F f)
{
    size_t i = 0;
    while (i < shapes.size()) {
        size_t j = i + 1;
        while (j < shapes.size() && shapes[j].rows == shapes[i].rows && shapes[j].cols == shapes[i].cols) ++j;
        f(i, j);
        i = j;
    }
}

size_t lowrank_mode_bytes(const cf_ctx *ctx)
{
    size_t algo = 0;
    for_each_run(ctx->shapes, [&](size_t i, size_t j) {
        const cf_shape &sh = ctx->shapes[i];
        const size_t b = cf::lowrank_workspace_bytes((int)(j - i), sh.rows, sh.cols, ctx->cfg.rank,
                                                     cf::lowrank_split(ctx->cfg.precision, sh.rows, sh.cols,
                                                                       ctx->cfg.rank));
        if (b > algo) algo = b;
    });
    return lowrank_residual_bytes(ctx) + algo;
}

cf_status check_quant_slot(cf_ctx *ctx, const cf_slot &s, int i, bool sender, int step)
{
    if (step == 0) {
        if (!s.x) return fail(ctx, CF_E_ARG, "slot %d: x is NULL", i);
        if (!aligned16(s.x)) return fail(ctx, CF_E_ALIGN, "slot %d: x not 16-byte aligned", i);
        if (sender) {
            if (!s.base || !s.err) return fail(ctx, CF_E_ARG, "slot %d: base/err is NULL", i);
            if (!aligned16(s.base) || !aligned16(s.err)) return fail(ctx, CF_E_ALIGN, "slot %d: base/err not 16-byte aligned", i);
        } else {
            if (!s.cache) return fail(ctx, CF_E_ARG, "slot %d: cache is NULL", i);
            if (!aligned16(s.cache) || !aligned16(s.recon))
                return fail(ctx, CF_E_ALIGN, "slot %d: cache/recon not 16-byte aligned", i);
        }
        return CF_OK;
    }
    if (sender) {
        if (!s.x || !s.base || !s.err || !s.codes || !s.scales)
            return fail(ctx, CF_E_ARG, "slot %d: x/base/err/codes/scales must be non-NULL", i);
        if (!aligned16(s.x) || !aligned16(s.base) || !aligned16(s.err) || !aligned16(s.codes) || !aligned16(s.scales))
            return fail(ctx, CF_E_ALIGN, "slot %d: pointers must be 16-byte aligned", i);
    } else {
        if (!s.codes || !s.scales || !s.cache) return fail(ctx, CF_E_ARG, "slot %d: codes/scales/cache must be non-NULL", i);
        if (!aligned16(s.codes) || !aligned16(s.scales) || !aligned16(s.cache) || !aligned16(s.recon))
            return fail(ctx, CF_E_ALIGN, "slot %d: pointers must be 16-byte aligned", i);
    }
    return CF_OK;
}

cf_status run_quant(cf_ctx *ctx, const cf_slot *slots, cf::QuantOp op, cudaStream_t stream)
{
    const int n = (int)ctx->shapes.size();
    cf::QuantLaunch *lp = new (std::nothrow) cf::QuantLaunch;
    if (!lp) return fail(ctx, CF_E_NOMEM, "host allocation failed");
    for (int first = 0; first < n; first += cf::kMaxSlotsPerLaunch) {
        const int cnt = (n - first < cf::kMaxSlotsPerLaunch) ? n - first : cf::kMaxSlotsPerLaunch;
        memset(lp, 0, sizeof *lp);
        lp->nslots = cnt;
        lp->status = ctx->d_status;
        for (int k = 0; k < cnt; ++k) {
            const cf_slot &s = slots[first + k];
            const cf_shape &sh = ctx->shapes[first + k];
            const int64_t elems = sh.rows * sh.cols;
            cf::QuantSlotDesc &d = lp->slot[k];
            d.x = s.x;
            d.base = s.base;
            d.err = s.err;
            d.cache = s.cache;
            d.codes = s.codes;
            d.scales = s.scales;
            d.recon = op == cf::QuantOp::Compress || op == cf::QuantOp::WarmupSender ? nullptr : s.recon;
            d.nvec = elems / 8;
        }
        cudaError_t e = cf::launch_quant(op, ctx->cfg.bits, ctx->cfg.group, ctx->cfg.sign_scale, ctx->cfg.state_bf16 != 0,
                                         *lp, stream);
        if (e != cudaSuccess) {
            delete lp;
            return cuda_fail(ctx, e, "quantised codec launch");
        }
    }
    delete lp;
    return CF_OK;
}

cf_status run_lowrank_mode(cf_ctx *ctx, const cf_slot *slots, bool sender, cudaStream_t stream)
{
    const size_t need = sender ? lowrank_mode_bytes(ctx) : 0;
    if (sender && (!ctx->ws || ctx->ws_bytes < need))
        return fail(ctx, CF_E_NOMEM, "low-rank mode needs %zu bytes of workspace (cf_set_workspace)", need);
    const int n = (int)ctx->shapes.size();
    const int r = ctx->cfg.rank;
    // warm start: from the second compressed step on, Algorithm 3 starts from
    // the V each slot received in the previous step
    const bool warm = sender && ctx->cfg.warm_start && ctx->lowrank_steps > 0;
    for (int i = 0; i < n; ++i) {
        const cf_slot &s = slots[i];
        if (ctx->shapes[i].rows == 0) continue;  // an empty slot is never touched
        if (!s.U || !s.R || !s.V) return fail(ctx, CF_E_ARG, "slot %d: U/R/V must be non-NULL", i);
        if (!aligned16(s.U) || !aligned16(s.R) || !aligned16(s.V))
            return fail(ctx, CF_E_ALIGN, "slot %d: U/R/V must be 16-byte aligned", i);
        if (sender) {
            if (!s.x || !s.base || !s.err || (!s.q0 && !warm))
                return fail(ctx, CF_E_ARG, "slot %d: x/base/err/q0 must be non-NULL", i);
            if (!aligned16(s.x) || !aligned16(s.base) || !aligned16(s.err) || !aligned16(s.q0))
                return fail(ctx, CF_E_ALIGN, "slot %d: x/base/err/q0 must be 16-byte aligned", i);
            if (ctx->shapes[i].rows > 0 && (ctx->shapes[i].rows < r || ctx->shapes[i].cols < r))
                return fail(ctx, CF_E_SHAPE, "slot %d: rows and cols must be >= rank", i);
        } else {
            if (!s.cache) return fail(ctx, CF_E_ARG, "slot %d: cache must be non-NULL", i);
            if (!aligned16(s.cache) || !aligned16(s.recon))
                return fail(ctx, CF_E_ALIGN, "slot %d: cache/recon must be 16-byte aligned", i);
        }
    }
    // fp32 residual of every slot, base <- x
    std::vector<float *> a_ptr(n);
    {
        char *p = (char *)ctx->ws;
        for (int i = 0; i < n; ++i) {
            a_ptr[i] = (float *)p;
            if (sender) p += round_up((size_t)(ctx->shapes[i].rows * ctx->shapes[i].cols) * 4, 256);
        }
    }
    if (sender) {
        std::vector<const void *> xs(n);
        std::vector<void *> bs(n);
        std::vector<const float *> es(n);
        std::vector<int64_t> ns(n);
        for (int i = 0; i < n; ++i) {
            xs[i] = slots[i].x;
            bs[i] = slots[i].base;
            es[i] = static_cast<const float *>(slots[i].err);
            ns[i] = ctx->shapes[i].rows * ctx->shapes[i].cols;
        }
        cudaError_t e = cf::launch_residual_f32(xs.data(), bs.data(), es.data(), a_ptr.data(), ns.data(), n, stream);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "residual launch");
    }
    char *algo_ws = (char *)ctx->ws + (sender ? lowrank_residual_bytes(ctx) : 0);
    cf_status st = CF_OK;
    for_each_run(ctx->shapes, [&](size_t i, size_t j) {
        if (st != CF_OK) return;
        const cf_shape sh = ctx->shapes[i];
        if (sh.rows == 0) return;
        std::vector<cf::LowrankMat> mats(j - i);
        for (size_t k = i; k < j; ++k) {
            cf::LowrankMat &m = mats[k - i];
            m.A = a_ptr[k];
            m.Q0 = warm ? slots[k].V : slots[k].q0;
            m.U = slots[k].U;
            m.R = slots[k].R;
            m.V = slots[k].V;
            m.E = sender ? static_cast<float *>(slots[k].err) : nullptr;
            m.C = sender ? nullptr : static_cast<float *>(slots[k].cache);
            m.recon = sender ? nullptr : slots[k].recon;
        }
        cf::LowrankPlan plan{};
        plan.nmat = (int)(j - i);
        plan.m = sh.rows;
        plan.n = sh.cols;
        plan.r = ctx->cfg.rank;
        plan.T = ctx->cfg.iters;
        plan.split = cf::lowrank_split(ctx->cfg.precision, sh.rows, sh.cols, ctx->cfg.rank);
        plan.ws = algo_ws;
        plan.ws_bytes = ctx->ws_bytes - (size_t)(algo_ws - (char *)ctx->ws);
        plan.status = ctx->d_status;
        cudaError_t e = sender ? cf::run_lowrank(plan, mats.data(), stream)
                               : cf::run_lowrank_decompress(plan, mats.data(), stream);
        if (e != cudaSuccess) st = cuda_fail(ctx, e, sender ? "low-rank compress" : "low-rank decompress");
    });
    if (st == CF_OK && sender) ++ctx->lowrank_steps;
    return st;
}

cf_status codec_call(cf_ctx *ctx, const cf_slot *slots, int step, void *stream_, bool sender)
{
    if (!ctx) return CF_E_ARG;
    DeviceGuard device(ctx);
    TraceGuard trace(ctx);
    if (step < 0) return fail(ctx, CF_E_ARG, "step must be >= 0");
    const int n = (int)ctx->shapes.size();
    if (n > 0 && !slots) return fail(ctx, CF_E_ARG, "slots is NULL");
    cudaStream_t stream = (cudaStream_t)stream_;
    if (step > 0 && !(sender ? ctx->warm_sender : ctx->warm_receiver))
        return fail(ctx, CF_E_STATE, "step %d before the warmup step (step 0) on this context", step);

    if (step == 0 || ctx->cfg.mode == CF_MODE_QUANT) {
        for (int i = 0; i < n; ++i) {
            if (ctx->shapes[i].rows == 0) continue;  // an empty slot is never touched
            cf_status st = check_quant_slot(ctx, slots[i], i, sender, step);
            if (st != CF_OK) return st;
        }
        cf::QuantOp op = step == 0 ? (sender ? cf::QuantOp::WarmupSender : cf::QuantOp::WarmupReceiver)
                                   : (sender ? cf::QuantOp::Compress : cf::QuantOp::Decompress);
        cf_status st = run_quant(ctx, slots, op, stream);
        if (st != CF_OK) return st;
    } else {
        cf_status st = run_lowrank_mode(ctx, slots, sender, stream);
        if (st != CF_OK) return st;
    }
    if (step == 0) (sender ? ctx->warm_sender : ctx->warm_receiver) = true;
    ctx->err.clear();
    return CF_OK;
}

}  // namespace

extern "C" {

cf_status cf_create(const cf_config *config, int nslots, const cf_shape *shapes, cf_ctx **out)
try {
    if (!out) return CF_E_ARG;
    *out = nullptr;
    if (!config || nslots < 0 || (nslots > 0 && !shapes)) return CF_E_ARG;
    std::string why;
    cf_status st = validate_config(config, why);
    if (st != CF_OK) return st;
    for (int i = 0; i < nslots; ++i) {
        const cf_shape &s = shapes[i];
        if (s.rows < 0 || s.cols <= 0 || s.cols % 8 != 0) return CF_E_SHAPE;
        if (s.rows > ((int64_t)1 << 40) / s.cols) return CF_E_SHAPE;
        if (config->mode == CF_MODE_QUANT && s.cols % config->group != 0) return CF_E_SHAPE;
        if (config->mode == CF_MODE_LOWRANK && s.rows > 0 && (s.rows < config->rank || s.cols < config->rank))
            return CF_E_SHAPE;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CF_E_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return CF_E_CUDA;
    if (prop.major != 10 || prop.minor != 0) return CF_E_CUDA;  // sm_100a code runs on compute capability 10.0 only

    cf_ctx *ctx = new (std::nothrow) cf_ctx;
    if (!ctx) return CF_E_NOMEM;
    ctx->cfg = *config;
    ctx->device = dev;
    // Failure-detection test hook, read once here: with CF_TEST_STARVE_GEMM=1
    // in the environment when the context is created, the context's first
    // cf_lowrank call issues no loads in its products, so their bounded waits
    // run out and the next cf_check reports CF_E_TIMEOUT (no GPU fault).
    const char *starve = getenv("CF_TEST_STARVE_GEMM");
    ctx->starve_once = config->mode == CF_MODE_LOWRANK && starve && starve[0] == '1';
    // Likewise CF_TEST_STARVE_ATTENTION=1: the context's first cf_attention call
    // issues no loads and gives up on its waits after 20 ms.
    const char *starve_attn = getenv("CF_TEST_STARVE_ATTENTION");
    ctx->starve_attention_once = starve_attn && starve_attn[0] == '1';
    try {
        ctx->shapes.assign(shapes, shapes + nslots);
    } catch (const std::bad_alloc &) {
        delete ctx;
        return CF_E_NOMEM;
    }
    if (cudaMalloc(&ctx->d_status, 256) != cudaSuccess) {
        delete ctx;
        return CF_E_NOMEM;
    }
    if (cudaMemset(ctx->d_status, 0, 256) != cudaSuccess) {
        cudaFree(ctx->d_status);
        delete ctx;
        return CF_E_CUDA;
    }
    *out = ctx;
    return CF_OK;
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;   // a host allocation failed: no C++ exception crosses the C ABI
} catch (...) {
    return CF_E_ARG;
}

size_t cf_workspace_bytes(const cf_ctx *ctx)
{
    if (!ctx || ctx->cfg.mode != CF_MODE_LOWRANK) return 0;
    return lowrank_mode_bytes(ctx);
}

cf_status cf_set_workspace(cf_ctx *ctx, void *dev_ptr, size_t bytes)
{
    if (!ctx) return CF_E_ARG;
    if (bytes > 0 && !dev_ptr) return fail(ctx, CF_E_ARG, "workspace pointer is NULL");
    if (!aligned16(dev_ptr)) return fail(ctx, CF_E_ALIGN, "workspace must be 16-byte aligned");
    ctx->ws = dev_ptr;
    ctx->ws_bytes = bytes;
    return CF_OK;
}

cf_status cf_compress(cf_ctx *ctx, const cf_slot *slots, int step, void *cuda_stream)
try {
    return codec_call(ctx, slots, step, cuda_stream, true);
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;
} catch (...) {
    return CF_E_ARG;
}

cf_status cf_decompress(cf_ctx *ctx, const cf_slot *slots, int step, void *cuda_stream)
try {
    return codec_call(ctx, slots, step, cuda_stream, false);
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;
} catch (...) {
    return CF_E_ARG;
}

cf_status cf_loopback(cf_ctx *ctx, const cf_slot *slots, int step, void *cuda_stream)
try {
    if (!ctx) return CF_E_ARG;
    if (step == 0 || ctx->cfg.mode != CF_MODE_QUANT) {
        cf_status st = codec_call(ctx, slots, step, cuda_stream, true);
        if (st != CF_OK) return st;
        return codec_call(ctx, slots, step, cuda_stream, false);
    }
    if (!(ctx->warm_sender && ctx->warm_receiver))
        return fail(ctx, CF_E_STATE, "step %d before the warmup step (step 0) on this context", step);
    DeviceGuard device(ctx);
    TraceGuard trace(ctx);
    const int n = (int)ctx->shapes.size();
    if (n > 0 && !slots) return fail(ctx, CF_E_ARG, "slots is NULL");
    for (int i = 0; i < n; ++i) {
        if (ctx->shapes[i].rows == 0) continue;
        cf_status st = check_quant_slot(ctx, slots[i], i, true, step);
        if (st == CF_OK) st = check_quant_slot(ctx, slots[i], i, false, step);
        if (st != CF_OK) return st;
    }
    cf_status st = run_quant(ctx, slots, cf::QuantOp::Loopback, (cudaStream_t)cuda_stream);
    if (st == CF_OK) ctx->err.clear();
    return st;
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;
} catch (...) {
    return CF_E_ARG;
}

size_t cf_lowrank_workspace_bytes(const cf_ctx *ctx, int nmat, int64_t m, int64_t n)
{
    if (!ctx || ctx->cfg.mode != CF_MODE_LOWRANK || nmat < 0 || m < ctx->cfg.rank || n < ctx->cfg.rank) return 0;
    return cf::lowrank_workspace_bytes(nmat, m, n, ctx->cfg.rank,
                                       cf::lowrank_split(ctx->cfg.precision, m, n, ctx->cfg.rank));
}

cf_status cf_lowrank(cf_ctx *ctx, int nmat, int64_t m, int64_t n, const float *const *A, const float *const *Q0,
                     float *const *U, float *const *R, float *const *V, float *const *E_opt, float *const *C_opt,
                     void *cuda_stream)
try {
    if (!ctx) return CF_E_ARG;
    DeviceGuard device(ctx);
    TraceGuard trace(ctx);
    if (ctx->cfg.mode != CF_MODE_LOWRANK) return fail(ctx, CF_E_ARG, "context is not in low-rank mode");
    if (nmat < 0) return fail(ctx, CF_E_ARG, "nmat must be >= 0");
    if (nmat == 0) return CF_OK;
    if (!A || !Q0 || !U || !R || !V) return fail(ctx, CF_E_ARG, "A/Q0/U/R/V arrays must be non-NULL");
    const int r = ctx->cfg.rank;
    if (m < r || n < r) return fail(ctx, CF_E_SHAPE, "m and n must be >= rank");
    if (n % 4 != 0) return fail(ctx, CF_E_SHAPE, "n must be a multiple of 4 (16-byte rows)");
    if (m > ((int64_t)1 << 40) / n) return fail(ctx, CF_E_SHAPE, "matrix too large");
    const bool split = cf::lowrank_split(ctx->cfg.precision, m, n, r);
    const size_t need = cf::lowrank_workspace_bytes(nmat, m, n, r, split);
    if (!ctx->ws || ctx->ws_bytes < need)
        return fail(ctx, CF_E_NOMEM, "cf_lowrank needs %zu bytes of workspace (cf_set_workspace)", need);
    std::vector<cf::LowrankMat> mats(nmat);
    for (int i = 0; i < nmat; ++i) {
        if (!A[i] || !Q0[i] || !U[i] || !R[i] || !V[i]) return fail(ctx, CF_E_ARG, "matrix %d: NULL pointer", i);
        if (!aligned16(A[i]) || !aligned16(Q0[i]) || !aligned16(U[i]) || !aligned16(R[i]) || !aligned16(V[i]))
            return fail(ctx, CF_E_ALIGN, "matrix %d: pointers must be 16-byte aligned", i);
        float *E = E_opt ? E_opt[i] : nullptr;
        float *C = C_opt ? C_opt[i] : nullptr;
        if (!aligned16(E) || !aligned16(C)) return fail(ctx, CF_E_ALIGN, "matrix %d: E/C must be 16-byte aligned", i);
        mats[i] = cf::LowrankMat{A[i], Q0[i], U[i], R[i], V[i], E, C};
    }
    cf::LowrankPlan plan{};
    plan.nmat = nmat;
    plan.m = m;
    plan.n = n;
    plan.r = r;
    plan.T = ctx->cfg.iters;
    plan.split = split;
    plan.starve = ctx->starve_once;
    ctx->starve_once = false;
    plan.ws = ctx->ws;
    plan.ws_bytes = ctx->ws_bytes;
    plan.status = ctx->d_status;
    cudaError_t e = cf::run_lowrank(plan, mats.data(), (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "cf_lowrank");
    ctx->err.clear();
    return CF_OK;
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;
} catch (...) {
    return CF_E_ARG;
}

namespace {
bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return a && b && x < y + nb && y < x + na;
}
}  // namespace

cf_status cf_attention(cf_ctx *ctx, int64_t lq, int64_t lk, int64_t cols, const void *q, const cf_kv *k,
                       const cf_kv *v, void *out, float *lse, void *cuda_stream)
try {
    if (!ctx) return CF_E_ARG;
    DeviceGuard device(ctx);
    TraceGuard trace(ctx);
    if (lq < 0 || lk < 1 || cols < 64 || cols % 64 != 0)
        return fail(ctx, CF_E_SHAPE, "need lq >= 0, lk >= 1 and cols a positive multiple of 64 (heads of 64)");
    if (lq > ((int64_t)1 << 40) / cols || lk > ((int64_t)1 << 40) / cols || cols / 64 > 65535 ||
        lq > INT32_MAX || lk > INT32_MAX)
        return fail(ctx, CF_E_SHAPE, "shard too large");
    if (lq == 0) return CF_OK;
    if (!q || !k || !v || !out) return fail(ctx, CF_E_ARG, "q, k, v and out must be non-NULL");
    if (!aligned16(q) || !aligned16(out)) return fail(ctx, CF_E_ALIGN, "q and out must be 16-byte aligned");
    if (lse && ((uintptr_t)lse & 3u) != 0) return fail(ctx, CF_E_ALIGN, "lse must be 4-byte aligned");
    const bool deq = k->bf16 == nullptr;
    if ((v->bf16 == nullptr) != deq) return fail(ctx, CF_E_ARG, "k and v must come in the same form");
    cf::AttnArgs a{};
    a.q = q;
    a.out = out;
    a.lse = lse;
    a.lq = lq;
    a.lk = lk;
    a.cols = cols;
    a.dequantise = deq;
    a.status = ctx->d_status;
    const cf_kv *kv[2] = {k, v};
    const size_t state_bytes = (size_t)lk * (size_t)cols * 4;
    for (int i = 0; i < 2; ++i) {
        const cf_kv &t = *kv[i];
        if (!deq) {
            if (!aligned16(t.bf16)) return fail(ctx, CF_E_ALIGN, "k/v bf16 must be 16-byte aligned");
            a.kv[i] = t.bf16;
            continue;
        }
        if (ctx->cfg.mode != CF_MODE_QUANT || ctx->cfg.state_bf16)
            return fail(ctx, CF_E_ARG, "dequantise-on-load needs a quantised-mode context with fp32 state");
        if (cols % ctx->cfg.group != 0) return fail(ctx, CF_E_SHAPE, "cols must be a multiple of the group size");
        if (!t.cache_in || !t.codes || !t.scales)
            return fail(ctx, CF_E_ARG, "dequantise-on-load needs cache_in, codes and scales");
        if (!aligned16(t.cache_in) || !aligned16(t.cache_out) || !aligned16(t.codes) || !aligned16(t.scales))
            return fail(ctx, CF_E_ALIGN, "k/v state and payload must be 16-byte aligned");
        a.cache_in[i] = t.cache_in;
        a.cache_out[i] = t.cache_out;
        a.codes[i] = t.codes;
        a.scales[i] = t.scales;
    }
    {
        // out is written while other CTAs still read K and V (or the caches)
        const size_t out_bytes = (size_t)lq * (size_t)cols * 2;
        for (int i = 0; i < 2; ++i) {
            const void *src = deq ? (const void *)a.cache_in[i] : a.kv[i];
            const size_t src_bytes = deq ? state_bytes : (size_t)lk * (size_t)cols * 2;
            if (ranges_overlap(out, out_bytes, src, src_bytes))
                return fail(ctx, CF_E_ARG, "out must not overlap k or v");
        }
    }
    if (deq) {
        // the CTAs of the first query block write C_t while the others still read C_{t-1}
        for (int i = 0; i < 2; ++i)
            for (int j = 0; j < 2; ++j)
                if (ranges_overlap(a.cache_out[i], state_bytes, a.cache_in[j], state_bytes))
                    return fail(ctx, CF_E_ARG, "cache_out must not overlap cache_in");
        if (ranges_overlap(a.cache_out[0], state_bytes, a.cache_out[1], state_bytes))
            return fail(ctx, CF_E_ARG, "the cache_out of k and v overlap");
        a.bits = ctx->cfg.bits;
        a.group = ctx->cfg.group;
    }
    a.starve = ctx->starve_attention_once;
    ctx->starve_attention_once = false;
    cudaError_t e = cf::launch_attention(a, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "cf_attention");
    ctx->err.clear();
    return CF_OK;
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;
} catch (...) {
    return CF_E_ARG;
}

cf_status cf_check(cf_ctx *ctx, void *cuda_stream)
{
    if (!ctx) return CF_E_ARG;
    DeviceGuard device(ctx);
    cudaStream_t stream = (cudaStream_t)cuda_stream;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "stream synchronize");
    uint32_t word = 0;
    e = cudaMemcpy(&word, ctx->d_status, sizeof word, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "status read");
    if (word != 0) {
        e = cudaMemset(ctx->d_status, 0, sizeof word);
        if (e != cudaSuccess) return cuda_fail(ctx, e, "status clear");
    }
    if (word & cf::kStatusTimeout) return fail(ctx, CF_E_TIMEOUT, "a bounded device-side wait gave up");
    if (word & cf::kStatusNonfinite) return fail(ctx, CF_E_NONFINITE, "a group scale was not finite");
    if (word & cf::kStatusNotSpd) return fail(ctx, CF_E_NONFINITE, "a Gram matrix was not positive definite");
    return CF_OK;
}

size_t cf_payload_bytes(const cf_ctx *ctx, int slot)
{
    if (!ctx || slot < 0 || slot >= (int)ctx->shapes.size()) return 0;
    const cf_shape &s = ctx->shapes[slot];
    const size_t n = (size_t)(s.rows * s.cols);
    if (ctx->cfg.mode == CF_MODE_QUANT) return n * ctx->cfg.bits / 8 + 4 * (n / ctx->cfg.group);
    const size_t r = (size_t)ctx->cfg.rank;
    return 4 * r * ((size_t)s.rows + r + (size_t)s.cols);
}

const char *cf_last_error(const cf_ctx *ctx)
{
    if (!ctx) return "null context";
    return ctx->err.c_str();
}

cf_status cf_resume(cf_ctx *ctx, int64_t steps_done)
try {
    if (!ctx) return CF_E_ARG;
    if (steps_done < 0) return fail(ctx, CF_E_ARG, "steps_done must be >= 0");
    ctx->warm_sender = true;
    ctx->warm_receiver = true;
    ctx->lowrank_steps = steps_done;   // compressed steps after the warmup
    ctx->err.clear();
    return CF_OK;
} catch (const std::bad_alloc &) {
    return CF_E_NOMEM;
} catch (...) {
    return CF_E_ARG;
}

cf_status cf_trace_enable(cf_ctx *ctx, int on)
{
    if (!ctx) return CF_E_ARG;
    if (on != 0 && on != 1) return fail(ctx, CF_E_ARG, "on must be 0 or 1");
    ctx->tracing = on != 0;
    return CF_OK;
}

int cf_trace_read(cf_ctx *ctx, cf_trace_entry *out, int max_entries)
try {
    if (!ctx || max_entries < 0 || (max_entries > 0 && !out)) return -CF_E_ARG;
    DeviceGuard device(ctx);
    cf::Tracer &t = ctx->tracer;
    struct Sum {
        std::string kernel;
        int launches;
        double ms;
    };
    std::vector<Sum> sums;   // in order of first launch
    bool bad = t.failed;
    for (auto &r : t.recs) {
        float ms = 0.0f;
        if (cudaEventSynchronize(r.e1) != cudaSuccess || cudaEventElapsedTime(&ms, r.e0, r.e1) != cudaSuccess) {
            bad = true;
            ms = 0.0f;
        }
        size_t k = 0;
        while (k < sums.size() && sums[k].kernel != r.kernel) ++k;
        if (k == sums.size()) sums.push_back(Sum{r.kernel, 0, 0.0});
        sums[k].launches += 1;
        sums[k].ms += ms;
        t.pool.emplace_back(r.e0, r.e1);
    }
    t.recs.clear();
    t.failed = false;
    for (size_t k = 0; k < sums.size() && (int)k < max_entries; ++k) {
        memset(&out[k], 0, sizeof out[k]);
        snprintf(out[k].kernel, sizeof out[k].kernel, "%s", sums[k].kernel.c_str());
        out[k].launches = sums[k].launches;
        out[k].total_ms = sums[k].ms;
    }
    if (bad) {
        fail(ctx, CF_E_CUDA, "a trace event could not be created, recorded or read");
        return -CF_E_CUDA;
    }
    return (int)sums.size();
} catch (const std::bad_alloc &) {
    return -CF_E_NOMEM;
} catch (...) {
    return -CF_E_ARG;
}

cf_status cf_destroy(cf_ctx *ctx)
{
    if (!ctx) return CF_E_ARG;
    DeviceGuard device(ctx);
    if (ctx->d_status) cudaFree(ctx->d_status);
    delete ctx;
    return CF_OK;
}

}  // extern "C"
