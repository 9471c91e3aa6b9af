// Building blocks of the exact-fp32 SIMT chunk kernels (the chunkwise backward and the chunked DPLR
// forward): chunk geometry, staging of record blocks and input rows into shared memory, and a
// register-tiled product of two shared-memory blocks.
#pragma once

#include "kda_internal.cuh"

namespace kda {
namespace simt {

constexpr int CB_C = 64;    // tokens per chunk
constexpr int CB_NT = 256;   // threads per CTA of the chain kernels
constexpr int CB_NTC = 512;  // threads per CTA of the per-chunk kernels
constexpr int CB_VS = 16;   // value columns per chain CTA

__host__ __device__ inline int cb_pad8(int x) { return (x + 7) & ~7; }
__host__ __device__ inline int cb_max(int a, int b) { return a > b ? a : b; }

// exp of a decay exponent (a difference <= 0, or a cumulative log-decay <= 0)
__device__ __forceinline__ float cb_exp(float x) { return __expf(x); }

// Staging into shared memory.  Record blocks (fp32) go by cp.async, every element of a tile in flight at
// once; dst[r * ld + c] = src[r * D + c] for r < rows, c < D, and zero for r < rows_p, c < D_p outside
// that (the padding the products read).  16-byte copies where D, D_p, ld and both addresses allow them.
// (r, c) advance by a fixed step per pass: no division per element.
__device__ __forceinline__ void cb_copy(float *dst, int ld, const float *src, int rows, int D, int rows_p,
                                        int D_p) {
    const int nt = blockDim.x;
    const bool wide = ((D | D_p | ld) & 3) == 0 &&
                      ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0;
    const int e = wide ? 4 : 1, W = D_p / e, n = rows_p * W, sr = nt / W, sc = nt - sr * W;
    int r = threadIdx.x / W, c = threadIdx.x - r * W;
    for (int idx = threadIdx.x; idx < n; idx += nt) {
        const bool in = r < rows && e * c < D;
        const float *g = src + (in ? (int64_t)r * D + e * c : 0);
        if (wide) cp_async16_fill(dst + r * ld + e * c, g, in);
        else cp_async4(dst + r * ld + c, g, in);
        c += sc;
        r += sr;
        if (c >= W) {
            c -= W;
            ++r;
        }
    }
}
// columns j0 .. j0 + 15 of a [rows][D] block into [rows][16] (zero past D)
__device__ __forceinline__ void cb_copy_cols(float *dst, const float *src, int rows, int D, int j0) {
    const int nt = blockDim.x;
    const bool wide = ((D | j0) & 3) == 0 &&
                      ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0;
    const int e = wide ? 4 : 1, W = CB_VS / e, n = rows * W;
    for (int idx = threadIdx.x; idx < n; idx += nt) {
        const int r = idx / W, c = idx - r * W;  // (W is 4 or 16: a shift)
        const bool in = j0 + e * c < D;
        const float *g = src + (in ? (int64_t)r * D + j0 + e * c : 0);
        if (wide) cp_async16_fill(dst + r * CB_VS + e * c, g, in);
        else cp_async4(dst + r * CB_VS + c, g, in);
    }
}
// Token rows of an input tensor (rs elements from one row to the next), converted to fp32, times
// e^{gsrc[r * D + c]} when gsrc is given (a record block): rows < valid, columns < D; zero elsewhere up
// to rows x D_p.  Eight loads in flight per thread.
template <typename T>
__device__ __forceinline__ void cb_load_rows(float *dst, int ld, const T *src, int64_t rs, int rows, int valid,
                                             int D, int D_p, const float *gsrc = nullptr) {
    const int nt = blockDim.x, n = rows * D_p, sr = nt / D_p, sc = nt - sr * D_p;
    int r0 = threadIdx.x / D_p, c0 = threadIdx.x - r0 * D_p;
    for (int base = threadIdx.x; base < n; base += 8 * nt) {
        float v[8], g[8];
        int rr[8], cc[8];
        int r = r0, c = c0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            rr[u] = r;
            cc[u] = c;
            const bool in = base + u * nt < n && r < valid && c < D;
            v[u] = in ? load_elem(src, (int64_t)r * rs + c) : 0.f;
            g[u] = (in && gsrc) ? gsrc[(int64_t)r * D + c] : 0.f;
            c += sc;
            r += sr;
            if (c >= D_p) {
                c -= D_p;
                ++r;
            }
        }
        r0 = r;
        c0 = c;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (base + u * nt < n) dst[rr[u] * ld + cc[u]] = gsrc ? v[u] * cb_exp(g[u]) : v[u];
    }
}

// out(r, c) = sum_k X(r, k) Y(c, k) for r < R, c < N (R, N multiples of 4), each thread a 4 x 4 block
// of strided elements (rows rt + a R/4, columns ct + b N/4, so that neighbouring threads read
// neighbouring rows of Y).  X(r, k) = X[r * ldx + k], or X[k * ldx + r] with XT; likewise Y.
template <bool XT, bool YT, typename F>
__device__ __forceinline__ void cb_mm(const float *X, int ldx, const float *Y, int ldy, int R, int N, int K,
                                      F &&emit) {
    const int R4 = R >> 2, N4 = N >> 2;
    for (int tile = threadIdx.x; tile < R4 * N4; tile += blockDim.x) {
        const int rt = tile / N4, ct = tile - rt * N4;
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
        for (int k = 0; k < K; ++k) {
            float x[4], y[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = rt + a * R4, c = ct + a * N4;
                x[a] = XT ? X[(int64_t)k * ldx + r] : X[(int64_t)r * ldx + k];
                y[a] = YT ? Y[(int64_t)k * ldy + c] : Y[(int64_t)c * ldy + k];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(x[a], y[b], acc[a][b]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) emit(rt + a * R4, ct + b * N4, acc[a][b]);
    }
}

}  // namespace simt
}  // namespace kda
