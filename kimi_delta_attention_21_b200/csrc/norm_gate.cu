// Per-head RMS normalisation over D_v, then the sigmoid output gate
// ("KDA Recurrence" page, problem statement; eps inside the root, no learned
// scale):  x = o / sqrt(mean(o^2) + eps) * sigmoid(gate).
// One warp per (token, head) row; safe in place (x == o).
#include "kda_internal.cuh"

namespace kda {

template <typename T>
__global__ void __launch_bounds__(256) norm_gate_kernel(const T *o, const T *__restrict__ gl, int64_t rows,
                                                        int Dv, float eps, T *x) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;
    using AT = typename AccT<T>::type;
    const T *src = o + row * Dv;
    AT ss = 0;
    for (int j = lane; j < Dv; j += 32) {
        const AT u = load_elem(src, j);
        ss += u * u;
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const AT inv = AT(1) / sqrt(ss / (AT)Dv + (AT)eps);
    for (int j = lane; j < Dv; j += 32) {
        const AT u = load_elem(src, j);
        store_elem(x, row * Dv + j, (float)(u * inv * (AT)sigmoid_precise(load_elem(gl, row * Dv + j))));
    }
}

kda_status_t launch_norm_gate(const void *o, const void *gl, int64_t N, int H, int Dv, float eps, void *x,
                              kda_dtype_t dt, cudaStream_t st) {
    const int64_t rows = N * H;
    const int64_t blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "too many rows");
    if (dt == KDA_F32)
        norm_gate_kernel<float><<<(unsigned)blocks, 256, 0, st>>>((const float *)o, (const float *)gl, rows, Dv,
                                                                  eps, (float *)x);
    else
        norm_gate_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)gl, rows, Dv, eps, (__nv_bfloat16 *)x);
    return check_launch("norm_gate_kernel");
}

}  // namespace kda
