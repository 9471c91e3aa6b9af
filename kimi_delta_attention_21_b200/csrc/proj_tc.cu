// Output projection on the 5th-generation tensor cores (tcgen05 + TMEM + TMA):
//   y[n, m] = sum_i x[n, i] * W_o[m, i]      (head concat is x's row-major layout)
// bf16 operands, fp32 accumulation in TMEM, bf16 output.
//
// One CTA computes a 128 x BN tile of y (BN = 256, or 64 when there are few
// rows, as in decode, so that the grid still covers the SMs).  Warp 0 (one
// thread) streams 128x64 tiles of x and BNx64 tiles of W_o into a 4-stage
// shared-memory ring with TMA (128-byte swizzle); warp 1 (one thread) issues
// tcgen05.mma (M=128, N=BN, K=16) into a BN-column TMEM accumulator and
// releases each stage with tcgen05.commit; then all four warps read the
// accumulator back (tcgen05.ld 32x32b, one row per thread) and store bf16.
#include "kda_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace kda {

namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64, ST = 4;

template <int BN> struct ProjCfg {
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr size_t SMEM_BYTES = ST * STAGE_BYTES + 1024 /*alignment slack*/ + 256 /*barriers*/;
    static constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
};

template <int BN>
__global__ void __launch_bounds__(128, 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
               int K, __nv_bfloat16 *__restrict__ y, unsigned int *timeouts) {
    using Cfg = ProjCfg<BN>;
    constexpr uint32_t A_BYTES = Cfg::A_BYTES, B_BYTES = Cfg::B_BYTES, STAGE_BYTES = Cfg::STAGE_BYTES;
    constexpr uint32_t TMEM_COLS = Cfg::TMEM_COLS;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = sm;
    uint8_t *sB = sm + ST * A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + ST * STAGE_BYTES);
    uint64_t *empty = full + ST;
    uint64_t *done = empty + ST;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int KB = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fence_barrier_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool timed_out = false;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        int kb = 0;
        for (; kb < KB; ++kb) {
            const int s = kb % ST;
            if (kb >= ST && !mbar_wait(&empty[s], ((kb / ST) - 1) & 1)) {
                timed_out = true;
                break;
            }
            mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
            tma_load_2d(sA + s * A_BYTES, &tmA, &full[s], kb * BK, m0);
            tma_load_2d(sB + s * B_BYTES, &tmB, &full[s], kb * BK, n0);
        }
        if (timed_out) {
            // let the copies already issued land before the CTA can exit
            for (int j = (kb > ST ? kb - ST : 0); j < kb; ++j) mbar_wait(&full[j % ST], (j / ST) & 1);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t idesc = idesc_f16(BM, BN, 0, 0);
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % ST;
            if (!mbar_wait(&full[s], (kb / ST) & 1)) {
                timed_out = true;
                break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(sA + s * A_BYTES), b0 = smem_u32(sB + s * B_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
                const uint64_t ad = smem_desc(a0 + k * 32, 16, 1024, LAYOUT_SW128);
                const uint64_t bd = smem_desc(b0 + k * 32, 16, 1024, LAYOUT_SW128);
                mma_f16_ss(tmem, ad, bd, idesc, (kb | k) != 0);
            }
            mma_commit(&empty[s]);
        }
        mma_commit(done);
    }
    __syncwarp();

    // ---------------- epilogue: TMEM -> registers -> bf16 -> global
    const bool ready = mbar_wait(done, 0);
    tc_fence_after();
    if (ready) {
        const int row = m0 + warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            if (n0 + c >= N) break;  // warp-uniform
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem + lane_base + (uint32_t)c, r);
            tmem_wait_ld();
            if (row < M) {
                __nv_bfloat16 *dst = y + (int64_t)row * N + n0 + c;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    if (n0 + c + 8 * g + 8 > N) break;
                    uint4 v;
                    uint32_t *pv = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[8 * g + 2 * j]),
                                                                 __uint_as_float(r[8 * g + 2 * j + 1]));
                        pv[j] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    *reinterpret_cast<uint4 *>(dst + 8 * g) = v;
                }
            }
        }
    } else {
        timed_out = true;
    }
    if (timed_out && timeouts) atomicAdd(timeouts, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace

bool proj_tc_supported(int64_t N, int K, int Dm, kda_dtype_t dt) {
    return dt == KDA_BF16 && K % 8 == 0 && Dm % 8 == 0 && N <= 0x7fffffff && (N + BM - 1) / BM <= 65535;
}

template <int BN>
static kda_status_t launch_proj_tc_bn(const CUtensorMap &ta, const void *W, int64_t N, int K, int Dm, void *y,
                                      cudaStream_t st) {
    using Cfg = ProjCfg<BN>;
    CUtensorMap tb;
    kda_status_t s = make_tmap_2d(&tb, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)Dm, (uint64_t)K,
                                  (uint64_t)K, BN, BK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != KDA_OK) return s;
    cudaFuncSetAttribute(proj_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
    const dim3 grid((unsigned)((Dm + BN - 1) / BN), (unsigned)((N + BM - 1) / BM));
    proj_tc_kernel<BN><<<grid, 128, Cfg::SMEM_BYTES, st>>>(ta, tb, (int)N, Dm, K, (__nv_bfloat16 *)y,
                                                          device_timeout_counter());
    return check_launch("proj_tc_kernel");
}

kda_status_t launch_proj_tc(const void *x, const void *W, int64_t N, int K, int Dm, void *y, cudaStream_t st) {
    CUtensorMap ta;
    kda_status_t s = make_tmap_2d(&ta, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)N, (uint64_t)K,
                                  (uint64_t)K, BM, BK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != KDA_OK) return s;
    // few rows (decode): narrow tiles so that the grid covers the SMs
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles256 = ((N + BM - 1) / BM) * ((Dm + 255) / 256);
    if (tiles256 < sms) return launch_proj_tc_bn<64>(ta, W, N, K, Dm, y, st);
    return launch_proj_tc_bn<256>(ta, W, N, K, Dm, y, st);
}

}  // namespace kda
