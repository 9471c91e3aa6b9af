// Internal declarations shared by the CUDA translation units of libkda.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "kda.h"

namespace kda {

// ----------------------------------------------------------------- host-side error state
void clear_error();
void set_error(const char *fmt, ...);
kda_status_t fail(kda_status_t s, const char *fmt, ...);
kda_status_t check_launch(const char *what);

// ----------------------------------------------------------------- element access
__device__ __forceinline__ float load_elem(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float *p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16 *p, int64_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
}

// Accumulator type of the exact-fp32 kernels: fp32 inputs accumulate their
// reductions in fp64 so that results stay within 1e-6 absolute / 1e-5 relative
// of an fp64 evaluation; bf16 inputs accumulate in fp32.
template <typename T> struct AccT { using type = float; };
template <> struct AccT<float> { using type = double; };

// sigmoid in full fp32 precision (expf, not the fast approximation)
__device__ __forceinline__ float sigmoid_precise(float x) { return 1.0f / (1.0f + expf(-x)); }

// A caller-supplied log(alpha), clamped to the documented range [g_min, 0]
// (a NaN becomes g_min).  Values outside it would leave the layer's
// definition and, on the tensor-core path, the range its decay factors cover.
__device__ __forceinline__ float clamp_log_decay(float g, float g_min) { return fminf(0.0f, fmaxf(g, g_min)); }

// log(alpha) from the decay logits: g_min * sigmoid(z)
__device__ __forceinline__ float log_alpha_of(float z, float g_min) {
    return g_min * sigmoid_precise(z);
}

// ----------------------------------------------------------------- checked builds
// A build with -DKDA_CHECKED tests every global write through an offset the library computes itself
// (workspace records, segment maps and entering states, checkpoints and stashes, final states, staged
// outputs) against the buffer it has to land in: a write that would leave its buffer is skipped and
// counted in a device counter (kda_device_bounds_errors), never trapped.  Other builds compile the
// test away.
#ifdef KDA_CHECKED
__device__ __forceinline__ bool in_bounds(const void *p, size_t n, const void *base, size_t size,
                                          unsigned int *errors) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(base);
    const bool ok = base != nullptr && a >= b && n <= size && a - b <= size - n;
    if (!ok && errors) atomicAdd(errors, 1u);
    return ok;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(const void *, size_t, const void *, size_t, unsigned int *) {
    return true;
}
#endif
unsigned int *device_bounds_counter();  // device address of the counter (host)

// ----------------------------------------------------------------- asynchronous global -> shared copies
// One fp32 element by cp.async (4-byte aligned addresses); with fill == false the destination gets
// zero and nothing is read.  A thread's copies have landed after cp_async_wait<n>() leaves at most n of
// its committed groups pending; other threads see them after a block barrier that follows.
__device__ __forceinline__ void cp_async4(float *smem_dst, const float *gsrc, bool fill = true) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
                 "l"(gsrc), "r"(fill ? 4 : 0)
                 : "memory");
}
// Four fp32 elements (16-byte aligned addresses); zero and no read with fill == false.
__device__ __forceinline__ void cp_async16_fill(float *smem_dst, const float *gsrc, bool fill = true) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
                 "l"(gsrc), "r"(fill ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ----------------------------------------------------------------- launchers (one per .cu)
kda_status_t launch_gate(const void *z, kda_dtype_t dt, int64_t n, float g_min, float *out,
                         cudaStream_t st);

kda_status_t launch_decode(const kda_decode_args &a, cudaStream_t st);

// SIMT chunk engine: exact fp32 arithmetic, any D_k, D_v <= 128, chunk <= 64.  scalar_decay: z or
// log_decay hold one value per (token, head) (B, S, H), the decay of every key channel (GDN).
kda_status_t launch_chunk_simt(const kda_chunk_args &a, int chunk, cudaStream_t st, bool scalar_decay = false);
size_t chunk_simt_workspace(const kda_chunk_args &a, int chunk);

// tcgen05 chunk engine: bf16, D_k = D_v = 128, chunk 64.
bool chunk_tc_supported(const kda_chunk_args &a, int chunk);
bool chunk_tc_aligned(const kda_chunk_args &a);
size_t chunk_tc_workspace(const kda_chunk_args &a);
kda_status_t launch_chunk_tc(const kda_chunk_args &a, cudaStream_t st);

// tcgen05 chunk engine for the scalar-decay (GDN) case: bf16, D_k = D_v = 128, chunk 64, any g_min.
// Same workspace as the KDA engine (chunk_tc_workspace).
bool gdn_tc_supported(const kda_chunk_args &a, int chunk);
bool gdn_tc_aligned(const kda_chunk_args &a);
kda_status_t launch_gdn_tc(const kda_chunk_args &a, cudaStream_t st);

// Recurrent backward (exact fp32): checkpoints every 64 tokens, per-block stash.
size_t rec_bwd_workspace(int64_t B, int64_t S, int H, int Dk, int Dv);
kda_status_t launch_rec_bwd(const kda_recurrent_bwd_args &a, cudaStream_t st);

// Chunkwise backward (exact fp32): per-chunk records, forward and backward state chains.
size_t chunk_bwd_workspace(int64_t B, int64_t S, int H, int Dk, int Dv);
kda_status_t launch_chunk_bwd(const kda_recurrent_bwd_args &a, cudaStream_t st);

// General DPLR recurrence, token by token (the comparator), and in chunk form (per-chunk records).
kda_status_t launch_dplr(const kda_dplr_args &a, cudaStream_t st);
size_t dplr_chunk_workspace(int64_t B, int64_t S, int H, int Dk, int Dv);
kda_status_t launch_dplr_chunk(const kda_dplr_args &a, void *workspace, cudaStream_t st);

kda_status_t launch_norm_gate(const void *o, const void *gl, int64_t N, int H, int Dv, float eps,
                              void *x, kda_dtype_t dt, cudaStream_t st);

kda_status_t launch_proj_simt(const void *x, const void *W, int64_t N, int K, int Dm, void *y,
                              kda_dtype_t dt, cudaStream_t st);
bool proj_tc_supported(int64_t N, int K, int Dm, kda_dtype_t dt);
kda_status_t launch_proj_tc(const void *x, const void *W, int64_t N, int K, int Dm, void *y,
                            cudaStream_t st);

// Launch with programmatic stream serialisation (the kernel starts early and waits in device code
// for the previous kernel of the stream before it touches global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace kda
