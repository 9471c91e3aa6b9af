// Output projection on the 5th-generation tensor cores (tcgen05 + TMEM + TMA):
//   y[n, m] = sum_i x[n, i] * W_o[m, i]      (head concat is x's row-major layout)
// bf16 operands, fp32 accumulation in TMEM, bf16 output.
//
// Persistent, warp-specialised: one CTA per SM walks 128 x BN output tiles.
//   warp 0       TMA producer: 128x64 tiles of x and BNx64 tiles of W_o into a
//                STAGES-deep shared-memory ring (128-byte swizzle);
//   warp 1       MMA issuer: tcgen05.mma (M=128, N=BN, K=16) into one of two
//                BN-column TMEM accumulators, releasing ring slots with
//                tcgen05.commit;
//   warps 2..5   epilogue: tcgen05.ld (32x32b, one row per thread) -> bf16 ->
//                global, then hand the accumulator back.
// With two accumulators a tile's epilogue overlaps the next tile's main loop.
#include "kda_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace kda {

namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64;

template <int BN> struct ProjCfg {
    static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
    static constexpr uint32_t A_BYTES = BM * BK * 2;
    static constexpr uint32_t B_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr uint32_t TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
    static constexpr size_t SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*alignment slack*/ + 256 /*barriers*/;
};

template <int BN>
__global__ void __launch_bounds__(192, 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
               int K, __nv_bfloat16 *__restrict__ y, unsigned int *timeouts) {
    pdl_trigger();
    pdl_wait();
    using Cfg = ProjCfg<BN>;
    constexpr int ST = Cfg::STAGES;
    extern __shared__ uint8_t smraw[];
    // first 1024-byte boundary, by pointer arithmetic on the shared base (keeps accesses ld/st.shared)
    uint8_t *sm = smraw + ((1024u - (static_cast<uint32_t>(__cvta_generic_to_shared(smraw)) & 1023u)) & 1023u);
    uint8_t *sA = sm;
    uint8_t *sB = sm + ST * Cfg::A_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + ST * Cfg::STAGE_BYTES);
    uint64_t *empty = full + ST;
    uint64_t *acc_full = empty + ST;     // [2] MMA -> epilogue
    uint64_t *acc_empty = acc_full + 2;  // [2] epilogue -> MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int tiles = tiles_m * tiles_n;
    const int KB = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);  // one arrival per epilogue warp
        }
        fence_barrier_init();
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool timed_out = false;

    // tiles walk N fastest inside groups of 8 M-tiles, so CTAs running at the same
    // time share their x rows and W_o rows in L2
    auto tile_mn = [&](int t, int &m0, int &n0) {
        const int group = 8;
        const int gm = t / (group * tiles_n);
        const int rem = t % (group * tiles_n);
        const int rows = min(group, tiles_m - gm * group);
        m0 = (gm * group + rem % rows) * BM;
        n0 = (rem / rows) * BN;
    };

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer
        int it = 0;
        for (int t = blockIdx.x; t < tiles && !timed_out; t += gridDim.x) {
            int m0, n0;
            tile_mn(t, m0, n0);
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % ST;
                if (it >= ST && !mbar_wait(&empty[s], ((it / ST) - 1) & 1)) {
                    timed_out = true;
                    break;
                }
                mbar_arrive_expect_tx(&full[s], Cfg::STAGE_BYTES);
                tma_load_2d(sA + s * Cfg::A_BYTES, &tmA, &full[s], kb * BK, m0);
                tma_load_2d(sB + s * Cfg::B_BYTES, &tmB, &full[s], kb * BK, n0);
            }
        }
        if (timed_out)  // let the copies already issued land before the CTA can exit
            for (int j = (it > ST ? it - ST : 0); j < it; ++j) mbar_wait(&full[j % ST], (j / ST) & 1);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t idesc = idesc_f16(BM, BN, 0, 0);
        int it = 0, lt = 0;
        for (int t = blockIdx.x; t < tiles && !timed_out; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            // the epilogue must have drained this accumulator (used two tiles ago)
            if (lt >= 2 && !mbar_wait(&acc_empty[buf], ((lt >> 1) - 1) & 1)) {
                timed_out = true;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem + buf * BN;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % ST;
                if (!mbar_wait(&full[s], (it / ST) & 1)) {
                    timed_out = true;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = smem_desc(smem_u32(sA + s * Cfg::A_BYTES), 16, 1024, LAYOUT_SW128);
                const uint64_t bd = smem_desc(smem_u32(sB + s * Cfg::B_BYTES), 16, 1024, LAYOUT_SW128);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    mma_f16_ss(d, ad + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc, (kb | k) != 0);
                mma_commit(&empty[s]);
            }
            mma_commit(&acc_full[buf]);
        }
    } else if (warp >= 2) {
        // ---------------- epilogue: TMEM -> registers -> bf16 -> global
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
            const int buf = lt & 1;
            int m0, n0;
            tile_mn(t, m0, n0);
            if (!mbar_wait(&acc_full[buf], (lt >> 1) & 1)) {
                timed_out = true;
                break;
            }
            tc_fence_after();
            const int row = m0 + 32 * q + lane;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + lane_base + buf * BN + (uint32_t)c, r);
                tmem_wait_ld();
                if (row < M && n0 + c < N) {
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
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }
    if (timed_out && timeouts) atomicAdd(timeouts, 1u);
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

template <int BN>
kda_status_t launch_proj_tc_bn(const CUtensorMap &ta, const void *W, int64_t N, int K, int Dm, void *y, int sms,
                               cudaStream_t st) {
    using Cfg = ProjCfg<BN>;
    CUtensorMap tb;
    kda_status_t s = make_tmap_2d(&tb, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)Dm, (uint64_t)K,
                                  (uint64_t)K, BN, BK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != KDA_OK) return s;
    cudaFuncSetAttribute(proj_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM_BYTES);
    const int64_t tiles = ((N + BM - 1) / BM) * ((Dm + BN - 1) / BN);
    const int grid = (int)(tiles < sms ? tiles : sms);
    cudaError_t e = launch_pdl(proj_tc_kernel<BN>, dim3(grid), dim3(192), Cfg::SMEM_BYTES, st, ta, tb, (int)N, Dm, K,
                               (__nv_bfloat16 *)y, device_timeout_counter());
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "proj_tc_kernel: %s", cudaGetErrorString(e));
    return check_launch("proj_tc_kernel");
}

}  // namespace

bool proj_tc_supported(int64_t N, int K, int Dm, kda_dtype_t dt) {
    return dt == KDA_BF16 && K % 8 == 0 && Dm % 8 == 0 && N <= 0x7fffffff;
}

kda_status_t launch_proj_tc(const void *x, const void *W, int64_t N, int K, int Dm, void *y, cudaStream_t st) {
    CUtensorMap ta;
    kda_status_t s = make_tmap_2d(&ta, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)N, (uint64_t)K,
                                  (uint64_t)K, BM, BK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != KDA_OK) return s;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // few rows (decode): narrow tiles so that more SMs take part
    const int64_t tiles256 = ((N + BM - 1) / BM) * ((Dm + 255) / 256);
    if (tiles256 < sms) return launch_proj_tc_bn<64>(ta, W, N, K, Dm, y, sms, st);
    return launch_proj_tc_bn<256>(ta, W, N, K, Dm, y, sms, st);
}

}  // namespace kda
