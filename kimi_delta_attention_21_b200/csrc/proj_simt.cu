// Exact-fp32 SIMT GEMM for the output projection y = x W_o^T (head concat is
// the row-major (N, H*D_v) layout of x).  Used for fp32 and for shapes the
// tcgen05 GEMM does not cover.  64x64 output tile per CTA, 4x4 per thread.
#include "kda_internal.cuh"

namespace kda {

namespace {
constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__global__ void __launch_bounds__(256) proj_simt_kernel(const T *__restrict__ x, const T *__restrict__ W,
                                                        int64_t N, int K, int Dm, T *__restrict__ y) {
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    const int64_t n0 = (int64_t)blockIdx.y * BM;
    const int m0 = blockIdx.x * BN;
    using AT = typename AccT<T>::type;
    AT acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += BK) {
        for (int e = tid; e < BM * BK; e += 256) {
            const int r = e / BK, kk = e % BK;
            const int64_t n = n0 + r;
            const int kq = k0 + kk;
            As[kk][r] = (n < N && kq < K) ? load_elem(x, n * K + kq) : 0.f;
            const int m = m0 + r;
            Bs[kk][r] = (m < Dm && kq < K) ? load_elem(W, (int64_t)m * K + kq) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] += (AT)a[i] * (AT)b[j];
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t n = n0 + ty * 4 + i;
        if (n >= N) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = m0 + tx * 4 + j;
            if (m < Dm) store_elem(y, n * Dm + m, (float)acc[i][j]);
        }
    }
}
}  // namespace

kda_status_t launch_proj_simt(const void *x, const void *W, int64_t N, int K, int Dm, void *y, kda_dtype_t dt,
                              cudaStream_t st) {
    const int64_t gy = (N + BM - 1) / BM;
    if (gy > 65535) return fail(KDA_ERR_UNSUPPORTED, "N too large for the SIMT projection");
    const dim3 grid((unsigned)((Dm + BN - 1) / BN), (unsigned)gy);
    if (dt == KDA_F32)
        proj_simt_kernel<float><<<grid, 256, 0, st>>>((const float *)x, (const float *)W, N, K, Dm, (float *)y);
    else
        proj_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)W,
                                                              N, K, Dm, (__nv_bfloat16 *)y);
    return check_launch("proj_simt_kernel");
}

}  // namespace kda
