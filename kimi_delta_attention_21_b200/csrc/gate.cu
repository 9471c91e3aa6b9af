// Decay gate: log(alpha) = g_min * sigmoid(z) ("KDA Recurrence" page, gate formula).
// HBM-bound elementwise pass: 16-byte loads, grid sized to the SM count.
#include "kda_internal.cuh"

namespace kda {

template <typename T>
__global__ void __launch_bounds__(256) gate_kernel(const T *__restrict__ z, int64_t n, float g_min,
                                                   float *__restrict__ out, bool vec) {
    constexpr int V = 16 / sizeof(T);  // elements per 16-byte load
    const int64_t nvec = vec ? n / V : 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
        const uint4 raw = reinterpret_cast<const uint4 *>(z)[i];
        const T *e = reinterpret_cast<const T *>(&raw);
        float r[V];
#pragma unroll
        for (int j = 0; j < V; ++j) r[j] = log_alpha_of(load_elem(e, j), g_min);
        float4 *o = reinterpret_cast<float4 *>(out + i * V);
#pragma unroll
        for (int j = 0; j < V / 4; ++j) o[j] = make_float4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
    }
    for (int64_t i = nvec * V + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = log_alpha_of(load_elem(z, i), g_min);
}

kda_status_t launch_gate(const void *z, kda_dtype_t dt, int64_t n, float g_min, float *out,
                         cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (n / 8 + 255) / 256;
    const int grid = (int)(want < (int64_t)sms * 8 ? (want > 0 ? want : 1) : (int64_t)sms * 8);
    const bool vec = ((reinterpret_cast<uintptr_t>(z) | reinterpret_cast<uintptr_t>(out)) & 15u) == 0;
    if (dt == KDA_F32)
        gate_kernel<float><<<grid, 256, 0, st>>>((const float *)z, n, g_min, out, vec);
    else
        gate_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)z, n, g_min, out, vec);
    return check_launch("gate_kernel");
}

}  // namespace kda
