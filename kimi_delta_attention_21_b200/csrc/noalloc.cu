// kda_out_norm_gate_proj_noalloc: the norm + gate + projection step for
// callers that cannot allocate device memory.
//
// kda_out_norm_gate_proj needs a caller workspace for the normalised, gated
// activations between its two kernels.  Some callers have no way to provide
// one: an integration point that hands the library only its input and output
// buffers (a plugin interface with no workspace hook), or a serving loop that
// must not call cudaMalloc while it runs because the call can synchronise the
// device and stall every other stream.  This entry point keeps that
// intermediate in a fixed scratch array that lives in the library's own device
// memory instead, so it needs nothing from the caller but inputs and outputs
// and never calls cudaMalloc, cudaFree or any allocating routine.
//
// The scratch array is a file-scope device array of NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits.  All
// calls on a device share it and it keeps the last call's contents; every
// byte a call reads is first written by the same call, so nothing needs
// clearing.  Two calls whose kernels overlap on the GPU (other streams, other
// host threads) race on the array and must be ordered by the caller.
#include <mutex>

#include "kda_internal.cuh"

namespace kda {

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(8) << 20;  // 8 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_setup_mu;
void *g_scratch_addr[MAX_DEVICES];

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side handle, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
kda_status_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= MAX_DEVICES) return fail(KDA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(KDA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return KDA_OK;
}

bool ptr_overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

bool aligned(const void *p, size_t al) { return (reinterpret_cast<uintptr_t>(p) & (al - 1)) == 0; }

}  // namespace

}  // namespace kda

extern "C" kda_status_t kda_out_norm_gate_proj_noalloc(const void *o, const void *gate_logits, const void *W_o,
                                                       int64_t N, int32_t H, int32_t D_v, int32_t D_model,
                                                       float eps, void *y, kda_dtype_t dtype, void *stream) {
    using namespace kda;
    clear_error();
    if (dtype != KDA_F32 && dtype != KDA_BF16) return fail(KDA_ERR_UNSUPPORTED, "dtype %d not supported", (int)dtype);
    if (N < 0 || H < 1 || D_v < 1 || D_model < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (!(isfinite(eps) && eps >= 0.0f)) return fail(KDA_ERR_INVALID_ARG, "eps must be finite and >= 0");
    const size_t es = dtype == KDA_F32 ? 4 : 2;
    // the limit is checked on N before any product that could wrap
    const size_t row_bytes = (size_t)H * (size_t)D_v * es;
    if (row_bytes > NOALLOC_SCRATCH_BYTES || (uint64_t)N > NOALLOC_SCRATCH_BYTES / row_bytes)
        return fail(KDA_ERR_UNSUPPORTED,
                    "N*H*D_v*element_size (N = %lld, %zu bytes per row) exceeds the fixed %zu-byte scratch of the "
                    "no-allocation entry point; use kda_out_norm_gate_proj with a workspace",
                    (long long)N, row_bytes, NOALLOC_SCRATCH_BYTES);
    const size_t nx = (size_t)N * row_bytes;
    if (N == 0) return KDA_OK;
    const void *ptrs[] = {o, gate_logits, W_o, y};
    const char *names[] = {"o", "gate_logits", "W_o", "y"};
    for (int i = 0; i < 4; ++i) {
        if (!ptrs[i]) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
        if (!aligned(ptrs[i], es)) return fail(KDA_ERR_INVALID_ARG, "%s is not %zu-byte aligned", names[i], es);
    }
    const size_t ny = (size_t)N * D_model * es, nw = (size_t)D_model * H * D_v * es;
    if (ptr_overlap(y, ny, o, nx) || ptr_overlap(y, ny, gate_logits, nx) || ptr_overlap(y, ny, W_o, nw))
        return fail(KDA_ERR_INVALID_ARG, "output y overlaps an input");
    void *scratch = nullptr;
    kda_status_t s = scratch_address(&scratch);
    if (s != KDA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    s = launch_norm_gate(o, gate_logits, N, H, D_v, eps, scratch, dtype, st);
    if (s != KDA_OK) return s;
    const int K = H * D_v;
    if (proj_tc_supported(N, K, D_model, dtype) && aligned(W_o, 16) && aligned(y, 16))
        return launch_proj_tc(scratch, W_o, N, K, D_model, y, st);
    return launch_proj_simt(scratch, W_o, N, K, D_model, y, dtype, st);
}
