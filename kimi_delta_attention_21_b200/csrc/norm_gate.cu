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

// bf16 rows of exactly 128 values: 16 lanes per row, 8 values (16 bytes) per
// lane, two rows per warp; HBM-bound on 3 * 256 bytes per row.
__global__ void __launch_bounds__(256) norm_gate128_bf16_kernel(const __nv_bfloat16 *o,
                                                               const __nv_bfloat16 *__restrict__ gl,
                                                               int64_t rows, float eps, __nv_bfloat16 *x) {
    const int lane = threadIdx.x & 31, half = lane >> 4, sub = lane & 15;
    const int64_t row = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 2 + half;
    const bool valid = row < rows;
    uint4 ov = make_uint4(0, 0, 0, 0), gv = make_uint4(0, 0, 0, 0);
    if (valid) {
        ov = reinterpret_cast<const uint4 *>(o + row * 128)[sub];
        gv = reinterpret_cast<const uint4 *>(gl + row * 128)[sub];
    }
    const __nv_bfloat162 *oh = reinterpret_cast<const __nv_bfloat162 *>(&ov);
    const __nv_bfloat162 *gh = reinterpret_cast<const __nv_bfloat162 *>(&gv);
    float f[8], g[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 a = __bfloat1622float2(oh[j]), b = __bfloat1622float2(gh[j]);
        f[2 * j] = a.x; f[2 * j + 1] = a.y; g[2 * j] = b.x; g[2 * j + 1] = b.y;
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) ss += f[j] * f[j];
#pragma unroll
    for (int m = 8; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);  // within each 16-lane half
    const float inv = 1.0f / sqrtf(ss * (1.0f / 128.0f) + eps);
    uint4 out;
    __nv_bfloat162 *xh = reinterpret_cast<__nv_bfloat162 *>(&out);
#pragma unroll
    for (int j = 0; j < 4; ++j)
        xh[j] = __floats2bfloat162_rn(f[2 * j] * inv * sigmoid_precise(g[2 * j]),
                                      f[2 * j + 1] * inv * sigmoid_precise(g[2 * j + 1]));
    if (valid) reinterpret_cast<uint4 *>(x + row * 128)[sub] = out;
}

kda_status_t launch_norm_gate(const void *o, const void *gl, int64_t N, int H, int Dv, float eps, void *x,
                              kda_dtype_t dt, cudaStream_t st) {
    const int64_t rows = N * H;
    const bool aligned = ((reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(gl) |
                           reinterpret_cast<uintptr_t>(x)) & 15u) == 0;
    if (dt == KDA_BF16 && Dv == 128 && aligned) {
        const int64_t blocks = (rows + 15) / 16;  // 8 warps x 2 rows
        if (blocks > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "too many rows");
        norm_gate128_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)gl, rows, eps, (__nv_bfloat16 *)x);
        return check_launch("norm_gate128_bf16_kernel");
    }
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
