// C-ABI entry points of libkda: host-side validation, engine choice, dispatch.
#include <math.h>
#include <stdarg.h>
#include <atomic>
#include <stdio.h>
#include <string.h>

#include "kda_internal.cuh"

namespace kda {

static thread_local char g_err[512];

void clear_error() { g_err[0] = 0; }

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

kda_status_t fail(kda_status_t s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

static std::atomic<uint64_t> g_launches{0};

kda_status_t check_launch(const char *what) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return KDA_OK;
}

static bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

static size_t esize(kda_dtype_t dt) { return dt == KDA_F32 ? 4 : 2; }

static bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

struct Buf {
    const void *p;
    size_t n;
    const char *name;
};

// Checks that `out` overlaps none of `ins` (except an input listed as `allowed_equal`
// that starts at the same address with the same size).
static kda_status_t check_no_overlap(const Buf &out, const Buf *ins, int nin,
                                     const void *allowed_equal = nullptr) {
    for (int i = 0; i < nin; ++i) {
        if (!ins[i].p) continue;
        if (allowed_equal && ins[i].p == allowed_equal && out.p == allowed_equal && ins[i].n == out.n)
            continue;
        if (overlap(out.p, out.n, ins[i].p, ins[i].n))
            return fail(KDA_ERR_INVALID_ARG, "output %s overlaps input %s", out.name, ins[i].name);
    }
    return KDA_OK;
}

static kda_status_t check_dtype(kda_dtype_t dt) {
    if (dt != KDA_F32 && dt != KDA_BF16) return fail(KDA_ERR_UNSUPPORTED, "dtype %d not supported", (int)dt);
    return KDA_OK;
}

static kda_status_t check_gmin(float g_min) {
    if (!(isfinite(g_min) && g_min < 0.0f))
        return fail(KDA_ERR_INVALID_ARG, "g_min must be a finite negative number (got %g)", (double)g_min);
    return KDA_OK;
}

#define KDA_TRY(expr)                      \
    do {                                   \
        kda_status_t s_ = (expr);          \
        if (s_ != KDA_OK) return s_;       \
    } while (0)

// Pointers must be non-NULL (REQ) and aligned to their element size `al`.
#define KDA_REQ_PTR(p, name, al)                                                               \
    do {                                                                                       \
        if (!(p)) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", name);                        \
        if (!aligned_to(p, al)) return fail(KDA_ERR_INVALID_ARG, "%s is not %d-byte aligned", name, (int)(al)); \
    } while (0)

#define KDA_OPT_PTR(p, name, al)                                                               \
    do {                                                                                       \
        if ((p) && !aligned_to(p, al))                                                         \
            return fail(KDA_ERR_INVALID_ARG, "%s is not %d-byte aligned", name, (int)(al));     \
    } while (0)

// gdn: the scalar-decay (Gated DeltaNet) entry points, whose z / log_decay are (B, S, H).
static kda_status_t chunk_validate(const kda_chunk_args *a, int *chunk_out, bool *use_tc, bool gdn) {
    if (!a) return fail(KDA_ERR_INVALID_ARG, "args is NULL");
    KDA_TRY(check_dtype(a->dtype));
    KDA_TRY(check_gmin(a->g_min));
    if (a->B < 0 || a->S < 0 || a->H < 1 || a->D_k < 1 || a->D_v < 1)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%lld S=%lld H=%d D_k=%d D_v=%d",
                    (long long)a->B, (long long)a->S, a->H, a->D_k, a->D_v);
    if (a->D_k > 128 || a->D_v > 128)
        return fail(KDA_ERR_UNSUPPORTED, "D_k and D_v must be <= 128 (got %d, %d)", a->D_k, a->D_v);
    int chunk = a->chunk == 0 ? 64 : a->chunk;
    if (chunk < 1) return fail(KDA_ERR_INVALID_ARG, "chunk must be positive (got %d)", a->chunk);
    if (chunk > 64) return fail(KDA_ERR_UNSUPPORTED, "chunk must be <= 64 (got %d)", chunk);
    if (a->engine != KDA_ENGINE_AUTO && a->engine != KDA_ENGINE_SIMT && a->engine != KDA_ENGINE_TC)
        return fail(KDA_ERR_INVALID_ARG, "unknown engine %d", (int)a->engine);
    *chunk_out = chunk;
    const bool tc_ok = gdn ? gdn_tc_supported(*a, chunk) : chunk_tc_supported(*a, chunk);
    if (a->engine == KDA_ENGINE_TC && !tc_ok)
        return fail(KDA_ERR_UNSUPPORTED, gdn ? "tensor-core engine needs bf16, D_k = D_v = 128 and chunk 64"
                                             : "tensor-core engine needs bf16, D_k = D_v = 128, chunk 64 and g_min >= -5.5");
    *use_tc = (a->engine == KDA_ENGINE_TC) || (a->engine == KDA_ENGINE_AUTO && tc_ok);
    if (a->gate_logits && !(isfinite(a->eps) && a->eps >= 0.0f))
        return fail(KDA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    return KDA_OK;
}

}  // namespace kda

using namespace kda;

extern "C" {

const char *kda_status_string(kda_status_t s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    }
    return "KDA_ERR_UNKNOWN";
}

const char *kda_last_error(void) { return g_err; }

int kda_version(void) { return 100; }

uint64_t kda_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

kda_status_t kda_gate(const void *z, kda_dtype_t dtype, int64_t n, float g_min, float *log_alpha,
                      void *stream) {
    g_err[0] = 0;
    KDA_TRY(check_dtype(dtype));
    if (n < 0) return fail(KDA_ERR_INVALID_ARG, "n must be >= 0");
    KDA_TRY(check_gmin(g_min));
    if (n == 0) return KDA_OK;
    KDA_REQ_PTR(z, "z", esize(dtype));
    KDA_REQ_PTR(log_alpha, "log_alpha", 4);
    Buf in{z, (size_t)n * esize(dtype), "z"};
    KDA_TRY(check_no_overlap(Buf{log_alpha, (size_t)n * 4, "log_alpha"}, &in, 1));
    return launch_gate(z, dtype, n, g_min, log_alpha, (cudaStream_t)stream);
}

static kda_status_t chunk_workspace_impl(const kda_chunk_args *a, size_t *bytes, bool gdn) {
    if (!bytes) return fail(KDA_ERR_INVALID_ARG, "bytes is NULL");
    int chunk = 0;
    bool tc = false;
    KDA_TRY(chunk_validate(a, &chunk, &tc, gdn));
    *bytes = tc ? chunk_tc_workspace(*a) : chunk_simt_workspace(*a, chunk);
    return KDA_OK;
}

static kda_status_t chunk_fwd_impl(const kda_chunk_args *a, bool gdn) {
    int chunk = 0;
    bool tc = false;
    KDA_TRY(chunk_validate(a, &chunk, &tc, gdn));
    if (a->B == 0) return KDA_OK;
    const size_t es = esize(a->dtype);
    const size_t nk = (size_t)a->B * a->S * a->H * a->D_k;
    const size_t nv = (size_t)a->B * a->S * a->H * a->D_v;
    const size_t nb = (size_t)a->B * a->S * a->H;
    const size_t nz = gdn ? nb : nk;  // decay inputs: one per key channel, or one per (token, head)
    const size_t ns = (size_t)a->B * a->H * a->D_k * a->D_v * 4;
    if (a->S > 0) {
        KDA_REQ_PTR(a->q, "q", es);
        KDA_REQ_PTR(a->k, "k", es);
        KDA_REQ_PTR(a->v, "v", es);
        KDA_REQ_PTR(a->beta, "beta", es);
        KDA_REQ_PTR(a->o, "o", es);
        if (!a->log_decay) KDA_REQ_PTR(a->z, "z (or log_decay)", es);
        KDA_OPT_PTR(a->log_decay, "log_decay", 4);
        KDA_OPT_PTR(a->gate_logits, "gate_logits", es);
    }
    KDA_OPT_PTR(a->initial_state, "initial_state", 4);
    KDA_OPT_PTR(a->final_state, "final_state", 4);
    KDA_OPT_PTR(a->workspace, "workspace", 256);
    KDA_OPT_PTR(a->dev_status, "dev_status", 4);
    const bool aligned = gdn ? gdn_tc_aligned(*a) : chunk_tc_aligned(*a);
    if (tc && a->engine == KDA_ENGINE_TC && !aligned)
        return fail(KDA_ERR_INVALID_ARG, "the tensor-core engine needs 16-byte aligned q, k, v, z, beta, o");
    if (tc && !aligned) tc = false;
    const size_t need = tc ? chunk_tc_workspace(*a) : chunk_simt_workspace(*a, chunk);
    if (need > 0 && (!a->workspace || a->workspace_bytes < need))
        return fail(KDA_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need,
                    a->workspace ? a->workspace_bytes : (size_t)0);
    const Buf ins[] = {
        {a->S ? a->q : nullptr, nk * es, "q"},
        {a->S ? a->k : nullptr, nk * es, "k"},
        {a->S ? a->v : nullptr, nv * es, "v"},
        {a->S && !a->log_decay ? a->z : nullptr, nz * es, "z"},
        {a->S ? a->log_decay : nullptr, nz * 4, "log_decay"},
        {a->S ? a->beta : nullptr, nb * es, "beta"},
        {a->S ? a->gate_logits : nullptr, nv * es, "gate_logits"},
        {a->initial_state, ns, "initial_state"},
        {need ? a->workspace : nullptr, need, "workspace"},
    };
    const int nin = (int)(sizeof(ins) / sizeof(ins[0]));
    if (a->S > 0) KDA_TRY(check_no_overlap(Buf{a->o, nv * es, "o"}, ins, nin));
    if (a->final_state) {
        KDA_TRY(check_no_overlap(Buf{a->final_state, ns, "final_state"}, ins, nin, a->initial_state));
        if (a->S > 0 && overlap(a->final_state, ns, a->o, nv * es))
            return fail(KDA_ERR_INVALID_ARG, "final_state overlaps o");
    }
    cudaStream_t st = (cudaStream_t)a->stream;
    if (tc) return gdn ? launch_gdn_tc(*a, st) : launch_chunk_tc(*a, st);
    KDA_TRY(launch_chunk_simt(*a, chunk, st, gdn));
    if (a->gate_logits && a->S > 0)
        return launch_norm_gate(a->o, a->gate_logits, a->B * a->S, a->H, a->D_v, a->eps, a->o,
                                a->dtype, st);
    return KDA_OK;
}

kda_status_t kda_chunk_workspace_size(const kda_chunk_args *a, size_t *bytes) {
    g_err[0] = 0;
    return chunk_workspace_impl(a, bytes, false);
}

kda_status_t kda_chunk_fwd(const kda_chunk_args *a) {
    g_err[0] = 0;
    return chunk_fwd_impl(a, false);
}

kda_status_t kda_gdn_chunk_workspace_size(const kda_chunk_args *a, size_t *bytes) {
    g_err[0] = 0;
    return chunk_workspace_impl(a, bytes, true);
}

kda_status_t kda_gdn_chunk_fwd(const kda_chunk_args *a) {
    g_err[0] = 0;
    return chunk_fwd_impl(a, true);
}

static kda_status_t rec_bwd_validate(const kda_recurrent_bwd_args *a) {
    if (!a) return fail(KDA_ERR_INVALID_ARG, "args is NULL");
    KDA_TRY(check_dtype(a->dtype));
    KDA_TRY(check_gmin(a->g_min));
    if (a->B < 0 || a->S < 0 || a->H < 1 || a->D_k < 1 || a->D_v < 1)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes B=%lld S=%lld H=%d D_k=%d D_v=%d", (long long)a->B,
                    (long long)a->S, a->H, a->D_k, a->D_v);
    if (a->D_k > 128 || a->D_v > 128)
        return fail(KDA_ERR_UNSUPPORTED, "D_k and D_v must be <= 128 (got %d, %d)", a->D_k, a->D_v);
    if ((int64_t)a->B * a->H > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "B*H too large");
    return KDA_OK;
}

kda_status_t kda_recurrent_bwd_workspace_size(const kda_recurrent_bwd_args *a, size_t *bytes) {
    g_err[0] = 0;
    if (!bytes) return fail(KDA_ERR_INVALID_ARG, "bytes is NULL");
    KDA_TRY(rec_bwd_validate(a));
    *bytes = rec_bwd_workspace(a->B, a->S, a->H, a->D_k, a->D_v);
    return KDA_OK;
}

// The SIMT chunk paths launch one CTA per (b, h, chunk): at most 2^31 - 1 of them.
static kda_status_t check_chunk_units(int64_t B, int64_t S, int H, const char *what) {
    const int64_t nc = (S + 63) / 64;
    if (B > 0 && nc > 0 && B * H > 0x7fffffffLL / nc)
        return fail(KDA_ERR_UNSUPPORTED, "%s: B*H*chunks exceeds 2^31 - 1", what);
    return KDA_OK;
}

kda_status_t kda_chunk_bwd_workspace_size(const kda_recurrent_bwd_args *a, size_t *bytes) {
    g_err[0] = 0;
    if (!bytes) return fail(KDA_ERR_INVALID_ARG, "bytes is NULL");
    KDA_TRY(rec_bwd_validate(a));
    KDA_TRY(check_chunk_units(a->B, a->S, a->H, "chunk backward"));
    *bytes = chunk_bwd_workspace(a->B, a->S, a->H, a->D_k, a->D_v);
    return KDA_OK;
}

// The pointer, workspace and overlap checks both backward entry points share (need: the workspace bytes).
static kda_status_t bwd_check_buffers(const kda_recurrent_bwd_args *a, size_t need) {
    const size_t es = esize(a->dtype);
    const size_t nk = (size_t)a->B * a->S * a->H * a->D_k, nv = (size_t)a->B * a->S * a->H * a->D_v;
    const size_t nb = (size_t)a->B * a->S * a->H, ns = (size_t)a->B * a->H * a->D_k * a->D_v * 4;
    if (a->S > 0) {
        KDA_REQ_PTR(a->q, "q", es);
        KDA_REQ_PTR(a->k, "k", es);
        KDA_REQ_PTR(a->v, "v", es);
        KDA_REQ_PTR(a->beta, "beta", es);
        KDA_REQ_PTR(a->d_o, "d_o", es);
        if (!a->log_decay) KDA_REQ_PTR(a->z, "z (or log_decay)", es);
        KDA_OPT_PTR(a->log_decay, "log_decay", 4);
        KDA_REQ_PTR(a->dq, "dq", 4);
        KDA_REQ_PTR(a->dk, "dk", 4);
        KDA_REQ_PTR(a->dv, "dv", 4);
        KDA_REQ_PTR(a->dbeta, "dbeta", 4);
        KDA_REQ_PTR(a->dz, "dz", 4);
    }
    KDA_OPT_PTR(a->initial_state, "initial_state", 4);
    KDA_OPT_PTR(a->d_final_state, "d_final_state", 4);
    KDA_OPT_PTR(a->d_initial_state, "d_initial_state", 4);
    KDA_OPT_PTR(a->workspace, "workspace", 256);
    if (a->S > 0 && need > 0 && (!a->workspace || a->workspace_bytes < need))
        return fail(KDA_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need,
                    a->workspace ? a->workspace_bytes : (size_t)0);
    const Buf ins[] = {
        {a->S ? a->q : nullptr, nk * es, "q"}, {a->S ? a->k : nullptr, nk * es, "k"},
        {a->S ? a->v : nullptr, nv * es, "v"}, {a->S && !a->log_decay ? a->z : nullptr, nk * es, "z"},
        {a->S ? a->log_decay : nullptr, nk * 4, "log_decay"}, {a->S ? a->beta : nullptr, nb * es, "beta"},
        {a->S ? a->d_o : nullptr, nv * es, "d_o"}, {a->initial_state, ns, "initial_state"},
        {a->d_final_state, ns, "d_final_state"}, {a->S && need ? a->workspace : nullptr, need, "workspace"},
    };
    const int nin = (int)(sizeof(ins) / sizeof(ins[0]));
    const Buf outs[] = {{a->S ? a->dq : nullptr, nk * 4, "dq"}, {a->S ? a->dk : nullptr, nk * 4, "dk"},
                        {a->S ? a->dv : nullptr, nv * 4, "dv"}, {a->S ? a->dbeta : nullptr, nb * 4, "dbeta"},
                        {a->S ? a->dz : nullptr, nk * 4, "dz"}, {a->d_initial_state, ns, "d_initial_state"}};
    for (const Buf &o : outs) {
        if (!o.p) continue;
        KDA_TRY(check_no_overlap(o, ins, nin));
        for (const Buf &o2 : outs)
            if (&o2 != &o && o2.p && overlap(o.p, o.n, o2.p, o2.n))
                return fail(KDA_ERR_INVALID_ARG, "outputs %s and %s overlap", o.name, o2.name);
    }
    return KDA_OK;
}

kda_status_t kda_recurrent_bwd(const kda_recurrent_bwd_args *a) {
    g_err[0] = 0;
    KDA_TRY(rec_bwd_validate(a));
    if (a->B == 0) return KDA_OK;
    KDA_TRY(bwd_check_buffers(a, rec_bwd_workspace(a->B, a->S, a->H, a->D_k, a->D_v)));
    return launch_rec_bwd(*a, (cudaStream_t)a->stream);
}

kda_status_t kda_chunk_bwd(const kda_recurrent_bwd_args *a) {
    g_err[0] = 0;
    KDA_TRY(rec_bwd_validate(a));
    if (a->B == 0) return KDA_OK;
    KDA_TRY(check_chunk_units(a->B, a->S, a->H, "chunk backward"));
    KDA_TRY(bwd_check_buffers(a, chunk_bwd_workspace(a->B, a->S, a->H, a->D_k, a->D_v)));
    return launch_chunk_bwd(*a, (cudaStream_t)a->stream);
}

// The checks both DPLR entry points share: sizes, dtype, g_min, pointers and overlaps.
static kda_status_t dplr_validate(const kda_dplr_args *a) {
    if (!a) return fail(KDA_ERR_INVALID_ARG, "args is NULL");
    KDA_TRY(check_dtype(a->dtype));
    KDA_TRY(check_gmin(a->g_min));
    if (a->B < 0 || a->S < 0 || a->H < 1 || a->D_k < 1 || a->D_v < 1)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (a->D_k > 128 || a->D_v > 128) return fail(KDA_ERR_UNSUPPORTED, "D_k and D_v must be <= 128");
    if ((int64_t)a->B * a->H > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "B*H too large");
    if (a->B == 0) return KDA_OK;
    const size_t es = esize(a->dtype);
    const size_t nk = (size_t)a->B * a->S * a->H * a->D_k, nv = (size_t)a->B * a->S * a->H * a->D_v;
    const size_t ns = (size_t)a->B * a->H * a->D_k * a->D_v * 4;
    if (a->S > 0) {
        KDA_REQ_PTR(a->q, "q", es);
        KDA_REQ_PTR(a->k, "k", es);
        KDA_REQ_PTR(a->v, "v", es);
        KDA_REQ_PTR(a->a, "a", es);
        KDA_REQ_PTR(a->b, "b", es);
        KDA_REQ_PTR(a->o, "o", es);
        if (!a->log_decay) KDA_REQ_PTR(a->z, "z (or log_decay)", es);
        KDA_OPT_PTR(a->log_decay, "log_decay", 4);
    }
    KDA_OPT_PTR(a->initial_state, "initial_state", 4);
    KDA_OPT_PTR(a->final_state, "final_state", 4);
    const Buf ins[] = {
        {a->S ? a->q : nullptr, nk * es, "q"}, {a->S ? a->k : nullptr, nk * es, "k"},
        {a->S ? a->v : nullptr, nv * es, "v"}, {a->S ? a->a : nullptr, nk * es, "a"},
        {a->S ? a->b : nullptr, nk * es, "b"}, {a->S && !a->log_decay ? a->z : nullptr, nk * es, "z"},
        {a->S ? a->log_decay : nullptr, nk * 4, "log_decay"}, {a->initial_state, ns, "initial_state"},
    };
    const int nin = (int)(sizeof(ins) / sizeof(ins[0]));
    if (a->S > 0) KDA_TRY(check_no_overlap(Buf{a->o, nv * es, "o"}, ins, nin));
    if (a->final_state) {
        KDA_TRY(check_no_overlap(Buf{a->final_state, ns, "final_state"}, ins, nin));
        if (a->S > 0 && overlap(a->final_state, ns, a->o, nv * es)) return fail(KDA_ERR_INVALID_ARG, "final_state overlaps o");
    }
    return KDA_OK;
}

// An empty sequence: final_state = initial_state (or zero).
static kda_status_t dplr_empty(const kda_dplr_args *a) {
    const size_t ns = (size_t)a->B * a->H * a->D_k * a->D_v * 4;
    if (a->final_state) {
        cudaError_t e = a->initial_state ? cudaMemcpyAsync(a->final_state, a->initial_state, ns,
                                                           cudaMemcpyDeviceToDevice, (cudaStream_t)a->stream)
                                         : cudaMemsetAsync(a->final_state, 0, ns, (cudaStream_t)a->stream);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "empty sequence: %s", cudaGetErrorString(e));
    }
    return KDA_OK;
}

kda_status_t kda_dplr_recurrent_fwd(const kda_dplr_args *a) {
    g_err[0] = 0;
    KDA_TRY(dplr_validate(a));
    if (a->B == 0) return KDA_OK;
    if (a->S == 0) return dplr_empty(a);
    return launch_dplr(*a, (cudaStream_t)a->stream);
}

kda_status_t kda_dplr_chunk_workspace_size(const kda_dplr_args *a, size_t *bytes) {
    g_err[0] = 0;
    if (!bytes) return fail(KDA_ERR_INVALID_ARG, "bytes is NULL");
    if (!a) return fail(KDA_ERR_INVALID_ARG, "args is NULL");
    if (a->B < 0 || a->S < 0 || a->H < 1 || a->D_k < 1 || a->D_v < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (a->D_k > 128 || a->D_v > 128) return fail(KDA_ERR_UNSUPPORTED, "D_k and D_v must be <= 128");
    KDA_TRY(check_chunk_units(a->B, a->S, a->H, "chunked DPLR"));
    *bytes = dplr_chunk_workspace(a->B, a->S, a->H, a->D_k, a->D_v);
    return KDA_OK;
}

kda_status_t kda_dplr_chunk_fwd(const kda_dplr_args *a, void *workspace, size_t workspace_bytes) {
    g_err[0] = 0;
    KDA_TRY(dplr_validate(a));
    if (a->B == 0) return KDA_OK;
    KDA_TRY(check_chunk_units(a->B, a->S, a->H, "chunked DPLR"));
    if (a->S == 0) return dplr_empty(a);
    KDA_OPT_PTR(workspace, "workspace", 256);
    const size_t need = dplr_chunk_workspace(a->B, a->S, a->H, a->D_k, a->D_v);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", need, workspace ? workspace_bytes : (size_t)0);
    const size_t es = esize(a->dtype);
    const size_t nk = (size_t)a->B * a->S * a->H * a->D_k, nv = (size_t)a->B * a->S * a->H * a->D_v;
    const size_t ns = (size_t)a->B * a->H * a->D_k * a->D_v * 4;
    const Buf ins[] = {
        {a->q, nk * es, "q"}, {a->k, nk * es, "k"}, {a->v, nv * es, "v"}, {a->a, nk * es, "a"}, {a->b, nk * es, "b"},
        {!a->log_decay ? a->z : nullptr, nk * es, "z"}, {a->log_decay, nk * 4, "log_decay"},
        {a->initial_state, ns, "initial_state"}, {a->o, nv * es, "o"}, {a->final_state, ns, "final_state"},
    };
    KDA_TRY(check_no_overlap(Buf{workspace, need, "workspace"}, ins, (int)(sizeof(ins) / sizeof(ins[0]))));
    return launch_dplr_chunk(*a, workspace, (cudaStream_t)a->stream);
}

kda_status_t kda_decode_step(const kda_decode_args *a) {
    g_err[0] = 0;
    if (!a) return fail(KDA_ERR_INVALID_ARG, "args is NULL");
    KDA_TRY(check_dtype(a->dtype));
    if (a->B < 0 || a->H < 1 || a->D_k < 1 || a->D_v < 1)
        return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (a->D_k > 128 || a->D_v > 128)
        return fail(KDA_ERR_UNSUPPORTED, "D_k and D_v must be <= 128");
    if (a->B == 0) return KDA_OK;
    const size_t es = esize(a->dtype);
    KDA_REQ_PTR(a->q, "q", es);
    KDA_REQ_PTR(a->k, "k", es);
    KDA_REQ_PTR(a->v, "v", es);
    KDA_REQ_PTR(a->beta, "beta", es);
    KDA_REQ_PTR(a->state, "state", 4);
    KDA_REQ_PTR(a->o, "o", es);
    KDA_TRY(check_gmin(a->g_min));
    if (!a->log_decay) KDA_REQ_PTR(a->z, "z (or log_decay)", es);
    KDA_OPT_PTR(a->log_decay, "log_decay", 4);
    KDA_OPT_PTR(a->gate_logits, "gate_logits", es);
    if (a->gate_logits && !(isfinite(a->eps) && a->eps >= 0.0f))
        return fail(KDA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const size_t nk = (size_t)a->B * a->H * a->D_k, nv = (size_t)a->B * a->H * a->D_v;
    const size_t ns = (size_t)a->B * a->H * a->D_k * a->D_v * 4;
    const Buf ins[] = {
        {a->q, nk * es, "q"}, {a->k, nk * es, "k"}, {a->v, nv * es, "v"},
        {a->log_decay ? nullptr : a->z, nk * es, "z"}, {a->log_decay, nk * 4, "log_decay"},
        {a->beta, (size_t)a->B * a->H * es, "beta"}, {a->gate_logits, nv * es, "gate_logits"},
    };
    const int nin = (int)(sizeof(ins) / sizeof(ins[0]));
    KDA_TRY(check_no_overlap(Buf{a->state, ns, "state"}, ins, nin));
    KDA_TRY(check_no_overlap(Buf{a->o, nv * es, "o"}, ins, nin));
    if (overlap(a->o, nv * es, a->state, ns)) return fail(KDA_ERR_INVALID_ARG, "o overlaps state");
    return launch_decode(*a, (cudaStream_t)a->stream);
}

kda_status_t kda_norm_gate(const void *o, const void *gl, int64_t N, int32_t H, int32_t Dv,
                           float eps, void *x, kda_dtype_t dtype, void *stream) {
    g_err[0] = 0;
    KDA_TRY(check_dtype(dtype));
    if (N < 0 || H < 1 || Dv < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (!(isfinite(eps) && eps >= 0.0f)) return fail(KDA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (N == 0) return KDA_OK;
    KDA_REQ_PTR(o, "o", esize(dtype));
    KDA_REQ_PTR(gl, "gate_logits", esize(dtype));
    KDA_REQ_PTR(x, "x", esize(dtype));
    const size_t n = (size_t)N * H * Dv * esize(dtype);
    const Buf ins[] = {{x == o ? nullptr : o, n, "o"}, {gl, n, "gate_logits"}};
    KDA_TRY(check_no_overlap(Buf{x, n, "x"}, ins, 2));
    if (x != o && overlap(x, n, o, n)) return fail(KDA_ERR_INVALID_ARG, "x partially overlaps o");
    return launch_norm_gate(o, gl, N, H, Dv, eps, x, dtype, (cudaStream_t)stream);
}

kda_status_t kda_out_proj(const void *x, const void *W, int64_t N, int32_t K, int32_t Dm, void *y,
                          kda_dtype_t dtype, void *stream) {
    g_err[0] = 0;
    KDA_TRY(check_dtype(dtype));
    if (N < 0 || K < 1 || Dm < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (N == 0) return KDA_OK;
    const size_t es = esize(dtype);
    KDA_REQ_PTR(x, "x", es);
    KDA_REQ_PTR(W, "W_o", es);
    KDA_REQ_PTR(y, "y", es);
    const Buf ins[] = {{x, (size_t)N * K * es, "x"}, {W, (size_t)Dm * K * es, "W_o"}};
    KDA_TRY(check_no_overlap(Buf{y, (size_t)N * Dm * es, "y"}, ins, 2));
    if (proj_tc_supported(N, K, Dm, dtype) && aligned_to(x, 16) && aligned_to(W, 16) && aligned_to(y, 16))
        return launch_proj_tc(x, W, N, K, Dm, y, (cudaStream_t)stream);
    return launch_proj_simt(x, W, N, K, Dm, y, dtype, (cudaStream_t)stream);
}

kda_status_t kda_out_norm_gate_proj_workspace_size(int64_t N, int32_t H, int32_t Dv, kda_dtype_t dtype,
                                                   size_t *bytes) {
    g_err[0] = 0;
    KDA_TRY(check_dtype(dtype));
    if (!bytes) return fail(KDA_ERR_INVALID_ARG, "bytes is NULL");
    if (N < 0 || H < 1 || Dv < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    *bytes = (size_t)N * H * Dv * esize(dtype);
    return KDA_OK;
}

kda_status_t kda_out_norm_gate_proj(const void *o, const void *gl, const void *W, int64_t N, int32_t H,
                                    int32_t Dv, int32_t Dm, float eps, void *y, kda_dtype_t dtype,
                                    void *ws, size_t ws_bytes, void *stream) {
    g_err[0] = 0;
    KDA_TRY(check_dtype(dtype));
    if (N < 0 || H < 1 || Dv < 1 || Dm < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (!(isfinite(eps) && eps >= 0.0f)) return fail(KDA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    if (N == 0) return KDA_OK;
    const size_t es = esize(dtype);
    KDA_REQ_PTR(o, "o", es);
    KDA_REQ_PTR(gl, "gate_logits", es);
    KDA_REQ_PTR(W, "W_o", es);
    KDA_REQ_PTR(y, "y", es);
    KDA_REQ_PTR(ws, "workspace", 256);
    const size_t nx = (size_t)N * H * Dv * es;
    if (ws_bytes < nx) return fail(KDA_ERR_WORKSPACE, "workspace needs %zu bytes (got %zu)", nx, ws_bytes);
    const Buf ins[] = {{o, nx, "o"}, {gl, nx, "gate_logits"}, {W, (size_t)Dm * H * Dv * es, "W_o"}};
    KDA_TRY(check_no_overlap(Buf{y, (size_t)N * Dm * es, "y"}, ins, 3));
    KDA_TRY(check_no_overlap(Buf{ws, nx, "workspace"}, ins, 3));
    if (overlap(ws, nx, y, (size_t)N * Dm * es)) return fail(KDA_ERR_INVALID_ARG, "workspace overlaps y");
    cudaStream_t st = (cudaStream_t)stream;
    KDA_TRY(launch_norm_gate(o, gl, N, H, Dv, eps, ws, dtype, st));
    const int K = H * Dv;
    if (proj_tc_supported(N, K, Dm, dtype) && aligned_to(W, 16) && aligned_to(y, 16))
        return launch_proj_tc(ws, W, N, K, Dm, y, st);
    return launch_proj_simt(ws, W, N, K, Dm, y, dtype, st);
}

}  // extern "C"
