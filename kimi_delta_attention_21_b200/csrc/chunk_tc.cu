// Tensor-core (tcgen05 / TMEM / TMA) chunk engine for the KDA prefill:
// bf16 inputs, D_k = D_v = 128, chunks of C = 64 tokens, fp32 state.
//
// Algebra (Kimi Linear report, section 3.1 and appendix B, Props. 1-2 with
// beta_r multiplying the whole bracket of Eqs. 17 and 19).  Inside a chunk,
// G_r = sum_{i<=r} log alpha_i per key channel, and with decayed products
// <x, y>_{r,i} = sum_c x_c y_c exp(G_rc - G_ic):
//
//   A[r,i] = beta_r <k_r, k_i>_{r,i}   (i < r)     M[r,i] = <q_r, k_i>_{r,i}   (i <= r)
//   T      = (I + A)^{-1}              (unit lower triangular)
//   W      = T Diag(beta)(K * e^G),    U = T Diag(beta) V          (Eqs. 17, 19 stacked)
//   V'     = U - W S                   (S: state entering the chunk)
//   O      = (Q * e^G) S + M V'        (o_t = S_t^T q_t, read after the update)
//   S     <- Diag(e^{G_C}) S + (K * e^{G_C - G})^T V'
//
// Two kernels:
//  * chunk_prep_kernel, one CTA per (chunk, head, batch), all chunks in
//    parallel: TMA loads of q, k, v, z; the cumulative log-decay; decay-scaled
//    operands; A^T and M^T on tcgen05; the blocked inverse T in fp32 SIMT;
//    [W | U] = T [beta K e^G | beta V] on tcgen05.  It writes one workspace
//    record per chunk holding Q*e^G, K*e^{G_C-G}, W and M^T as ready-made
//    128-byte-swizzled shared-memory images, U split by value-column slice,
//    and e^{G_C}.
//  * chunk_state_kernel, one CTA per (value-column slice, head, batch), walks
//    the chunks in order with the state slice resident in TMEM, streaming the
//    records with bulk copies (two stages), and writes o~ and the final state.
//
// Decay factors as GEMM operands.  exp(G_r - G_i) is split into a row factor
// and a column factor around a reference point.  G spans up to |g_min| * 64
// per chunk, so one reference per chunk would overflow; instead each 16-token
// block R has its own reference m_R = G at token 16R+7.  For rows r in block R
// the row factor is exp(G_r - m_R) (|exponent| <= 8 |g_min|) and the column
// factor of token i <= r is exp(m_R - G_i), which is <= 1 for i in earlier
// blocks and <= exp(8 |g_min|) inside the block.  With g_min >= -5.5 every
// factor and every product (masked ones included) stays inside the fp32/bf16
// range.  The factors are assembled from exp(G - b_{R-1}), exp(b_R - G)
// (b_R = G at the last token of block R) and per-channel block constants, so
// no intermediate underflows unless the true value does.
//
// Precision of M.  Rounding the decay-scaled q and k to bf16 costs ~2^-9 of
// sum_c |q_c k_c| in every product; on the diagonal 16x16 blocks of M (no
// decay to shrink the terms) that error can be a large part of a small
// q_r . k_i, and the per-head RMS normalisation then turns it into a large
// output error for tokens whose o~ is small.  The diagonal blocks of M are
// therefore computed with split operands, x = hi + lo (both bf16): the MMA
// adds hi*lo + lo*hi on top of hi*hi, which leaves ~2^-17 relative error.
#include "kda_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace kda {

namespace {

using namespace sm100;

constexpr int CH = 64;   // chunk length
constexpr int DD = 128;  // D_k = D_v
constexpr float TC_GMIN_LIMIT = -5.5f;

// ---------------------------------------------------------------- workspace record (per b, h, chunk)
constexpr uint32_t REC_QG = 0;        // Q * e^G          K-major SW128 image [2 atoms][64 rows][128 B]
constexpr uint32_t REC_KT = 16384;    // K * e^{G_C - G}  same image (MN-major A operand of K~^T V')
constexpr uint32_t REC_W = 32768;     // W                same image
constexpr uint32_t REC_MT = 49152;    // M^T              [64 rows i][128 B: r] (MN-major A operand of M V')
constexpr uint32_t REC_U = 57344;     // U                [128/NV slices][64 rows][NV] bf16
constexpr uint32_t REC_GAM = 73728;   // e^{G_C}          128 fp32
constexpr uint32_t REC_IMG = 57344;   // bytes of the four images
constexpr uint32_t REC_BYTES = 74240;

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]);
    u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]);
    u.w = pack_bf16x2(f[6], f[7]);
    return u;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 x = __bfloat1622float2(h[j]);
        f[2 * j] = x.x;
        f[2 * j + 1] = x.y;
    }
}

__device__ __forceinline__ void load8f(const float *p, float (&f)[8]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// The tensor-core engine works on bf16 data and every exponent it takes is
// bounded (|x| <= 8 |g_min| + |g_min| * 64), so the hardware exp2 approximation
// (a few ulp of fp32) is far below the bf16 rounding it feeds.
__device__ __forceinline__ float fexp(float x) { return __expf(x); }
__device__ __forceinline__ float log_alpha_fast(float z, float g_min) {
    return g_min * __fdividef(1.0f, 1.0f + __expf(-z));
}

// A descriptor for base + off: the start-address field holds address >> 4 in 14
// bits, which cannot carry for shared-memory addresses below 256 KB.
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t off_bytes) { return d + (off_bytes >> 4); }

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void report_timeout(unsigned int *timeouts, int *dev_status) {
    if (timeouts) atomicAdd(timeouts, 1u);
    if (dev_status) atomicExch(dev_status, (int)KDA_ERR_TIMEOUT);
}

// ================================================================ K2a: chunk_prep_kernel
// Persistent: one CTA per SM walks (chunk, head, batch) units.  The next unit's
// q, k and z tiles are loaded by TMA as soon as this unit's copies of them are
// dead (after the A/M MMAs), v after the W/U MMA, and the workspace bulk
// stores drain while the next unit is computed.
// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t P_QI = 0;         // q image; becomes Q e^G (stored as soon as P2 ends)
constexpr uint32_t P_KI = 16384;     // k image; becomes K e^{G_C - G}
constexpr uint32_t P_VI = 32768;     // v image; becomes beta V (MN-major B operand of the W|U MMA)
constexpr uint32_t P_ZI = 49152;     // z image; becomes lo part of the q row operand
constexpr uint32_t P_KC = 65536;     // column operands, 4 versions packed [2 atoms][160 rows][128 B]; later W, U
constexpr uint32_t P_KR = 106496;    // row operand from k [2 atoms][64 rows][128 B]; later the M^T image
constexpr uint32_t P_QR = 122880;    // row operand from q; later the T image
constexpr uint32_t P_RH = 139264;    // beta K e^G image (MN-major B) + lo part of the diagonal column operand
constexpr uint32_t P_SG = 172032;    // G fp32 [64][132]; later A [64][65] and T [64][68] fp32
constexpr uint32_t P_TAB = 206080;   // per-channel block constants [26][128] fp32
constexpr uint32_t P_XS = 219392;    // scratch for the blocked inverse [3][256] fp32
constexpr uint32_t P_BETA = 222464;  // beta [64] fp32
constexpr uint32_t P_GAM = 222720;   // e^{G_C} [128] fp32
constexpr uint32_t P_BAR = 223232;   // 3 mbarriers + TMEM slot
constexpr uint32_t P_END = 223312;
constexpr size_t PREP_SMEM = P_END + 1024;
constexpr uint32_t P_MT = P_KR, P_TI = P_QR;
constexpr uint32_t P_KLO = P_RH + 16384;
constexpr uint32_t P_SA = P_SG, P_ST = P_SG + 16640;
constexpr uint32_t P_WI = P_KC, P_UI = P_KC + 16384;
constexpr int SG_LD = 132, SA_LD = 65, ST_LD = 68;
constexpr uint32_t KC_ATOM = 160 * 128;  // bytes per atom column of the packed column operand

// table rows: b_R (0-3), F_R = e^{b_{R-1} - m_R} (4-7), E_R = e^{b_{R-1}} (8-11),
// D_R = e^{b_3 - b_R} (12-15), C_{V,R} = e^{m_V - b_R} for R <= V (16 + V(V+1)/2 + R)
__device__ __forceinline__ int tab_c(int V, int R) { return 16 + V * (V + 1) / 2 + R; }
__device__ __forceinline__ int kc_row0(int V) { return 8 * V * (V + 1); }  // 0, 16, 48, 96

struct PrepArgs {
    int S, H, Nc, Nv;
    int64_t units;  // Nc * H * B
    float g_min;
    const __nv_bfloat16 *beta;
    const float *log_decay;
    uint8_t *ws;
    unsigned int *timeouts;
    int *dev_status;
};

__global__ void __launch_bounds__(256, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tz, PrepArgs p) {
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + P_BAR);
    uint64_t *bar_am = bar_in + 1;
    uint64_t *bar_wu = bar_in + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + P_BAR + 24);
    float *sG = reinterpret_cast<float *>(sm + P_SG);
    float *tab = reinterpret_cast<float *>(sm + P_TAB);
    float *sbeta = reinterpret_cast<float *>(sm + P_BETA);
    float *sgam = reinterpret_cast<float *>(sm + P_GAM);
    const uint32_t in_bytes = (p.log_decay ? 6u : 8u) * 8192u;

    auto unit_coords = [&](int64_t u, int &n, int &h, int &b) {
        n = (int)(u % p.Nc);
        const int64_t bh = u / p.Nc;
        h = (int)(bh % p.H);
        b = (int)(bh / p.H);
    };
    auto load_qkz = [&](int64_t u) {  // arms bar_in for the whole unit
        int n, h, b;
        unit_coords(u, n, h, b);
        mbar_arrive_expect_tx(bar_in, in_bytes);
        for (int a = 0; a < 2; ++a) {
            tma_load_4d(sm + P_QI + a * 8192, &tq, bar_in, 64 * a, h, n * CH, b);
            tma_load_4d(sm + P_KI + a * 8192, &tk, bar_in, 64 * a, h, n * CH, b);
            if (!p.log_decay) tma_load_4d(sm + P_ZI + a * 8192, &tz, bar_in, 64 * a, h, n * CH, b);
        }
    };
    auto load_v = [&](int64_t u) {
        int n, h, b;
        unit_coords(u, n, h, b);
        for (int a = 0; a < 2; ++a) tma_load_4d(sm + P_VI + a * 8192, &tv, bar_in, 64 * a, h, n * CH, b);
    };

    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_am, 1);
        mbar_init(bar_wu, 1);
        fence_barrier_init();
        if ((int64_t)blockIdx.x < p.units) {
            load_qkz(blockIdx.x);
            load_v(blockIdx.x);
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    int it = 0;
    for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++it) {
        int n, h, b;
        unit_coords(u, n, h, b);
        const int t0 = n * CH;
        const int len = min(CH, p.S - t0);
        const int64_t u_next = u + gridDim.x;
        const uint32_t par = it & 1;
        // the previous unit's bulk stores must have read their shared sources
        if (tid == 0) bulk_wait_read_all();
        if (tid < CH)
            sbeta[tid] = (tid < len) ? __bfloat162float(p.beta[((int64_t)b * p.S + t0 + tid) * p.H + h]) : 0.f;
        ok = mbar_wait(bar_in, par);
        ok = __syncthreads_and(ok);
        if (!ok) break;

        // ---------------- P1: G = in-chunk cumulative log-decay (rows past the sequence end: no decay)
        {
            const int c = tid & 127, half = tid >> 7;
            float g[32];
            if (p.log_decay) {
#pragma unroll
                for (int rr = 0; rr < 32; ++rr) {
                    const int r = half * 32 + rr;
                    g[rr] = (r < len) ? p.log_decay[(((int64_t)b * p.S + t0 + r) * p.H + h) * DD + c] : 0.f;
                }
            } else {
                const uint8_t *zc = sm + P_ZI + (c >> 6) * 8192 + (c & 7) * 2;
                const uint32_t ch = (c & 63) >> 3;
#pragma unroll
                for (int rr = 0; rr < 32; ++rr) {
                    const int r = half * 32 + rr;
                    const float zv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(zc + sw128(r, ch)));
                    g[rr] = (r < len) ? log_alpha_fast(zv, p.g_min) : 0.f;
                }
            }
            float acc = 0.f;
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) {
                acc += g[rr];
                g[rr] = acc;
            }
            if (half == 0) sG[31 * SG_LD + c] = acc;
            __syncthreads();
            const float base = half ? sG[31 * SG_LD + c] : 0.f;
            __syncthreads();
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) sG[(half * 32 + rr) * SG_LD + c] = g[rr] + base;
        }
        __syncthreads();
        // ---------------- per-channel block constants
        if (tid < 128) {
            const int c = tid;
            float bb[4], mm[4];
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                bb[R] = sG[(16 * R + 15) * SG_LD + c];
                mm[R] = sG[(16 * R + 7) * SG_LD + c];
            }
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                const float bm1 = R ? bb[R - 1] : 0.f;
                tab[R * 128 + c] = bb[R];
                tab[(4 + R) * 128 + c] = fexp(bm1 - mm[R]);
                tab[(8 + R) * 128 + c] = fexp(bm1);
                tab[(12 + R) * 128 + c] = fexp(bb[3] - bb[R]);
            }
#pragma unroll
            for (int V = 0; V < 4; ++V)
#pragma unroll
                for (int R = 0; R <= V; ++R) tab[tab_c(V, R) * 128 + c] = fexp(mm[V] - bb[R]);
            sgam[c] = fexp(bb[3]);
        }
        __syncthreads();
        // ---------------- P2: decay-scaled operands (one thread per row r and 4 chunks of 8 channels)
        {
            const int r = tid & 63, grp = tid >> 6, R = r >> 4;
            const float beta_r = sbeta[r];
#pragma unroll 1
            for (int mi = 0; mi < 4; ++mi) {
                const int j = grp + 4 * mi;
                const int atom = j >> 3, jj = j & 7, c0 = 8 * j;
                const uint32_t img = atom * 8192 + sw128(r, jj);
                float qv[8], kv[8], vv[8], G[8], bR[8], bRm1[8], F[8], E[8], Dd[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + P_QI + img), qv);
                unpack8(*reinterpret_cast<const uint4 *>(sm + P_KI + img), kv);
                unpack8(*reinterpret_cast<const uint4 *>(sm + P_VI + img), vv);
                load8f(sG + r * SG_LD + c0, G);
                load8f(tab + R * 128 + c0, bR);
                if (R > 0) {
                    load8f(tab + (R - 1) * 128 + c0, bRm1);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) bRm1[e] = 0.f;
                }
                load8f(tab + (4 + R) * 128 + c0, F);
                load8f(tab + (8 + R) * 128 + c0, E);
                load8f(tab + (12 + R) * 128 + c0, Dd);
                float e1[8], e3[8], t[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    e1[e] = fexp(G[e] - bRm1[e]);
                    e3[e] = fexp(bR[e] - G[e]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = kv[e] * e1[e] * F[e];
                *reinterpret_cast<uint4 *>(sm + P_KR + img) = pack8(t);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = qv[e] * e1[e] * F[e];
                {
                    const uint4 hi = pack8(t);
                    *reinterpret_cast<uint4 *>(sm + P_QR + img) = hi;
                    float hf[8], lo[8];
                    unpack8(hi, hf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) lo[e] = t[e] - hf[e];
                    *reinterpret_cast<uint4 *>(sm + P_ZI + img) = pack8(lo);  // z image is dead
                }
                for (int V = R; V < 4; ++V) {
                    float Cv[8];
                    load8f(tab + tab_c(V, R) * 128 + c0, Cv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = kv[e] * e3[e] * Cv[e];
                    const uint4 hi = pack8(t);
                    *reinterpret_cast<uint4 *>(sm + P_KC + atom * KC_ATOM + sw128(kc_row0(V) + r, jj)) = hi;
                    if (V == R) {  // diagonal block: keep the rounding residue
                        float hf[8], lo[8];
                        unpack8(hi, hf);
#pragma unroll
                        for (int e = 0; e < 8; ++e) lo[e] = t[e] - hf[e];
                        *reinterpret_cast<uint4 *>(sm + P_KLO + img) = pack8(lo);
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = qv[e] * e1[e] * E[e];
                *reinterpret_cast<uint4 *>(sm + P_QI + img) = pack8(t);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = kv[e] * e3[e] * Dd[e];
                *reinterpret_cast<uint4 *>(sm + P_KI + img) = pack8(t);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = beta_r * kv[e] * e1[e] * E[e];
                *reinterpret_cast<uint4 *>(sm + P_RH + img) = pack8(t);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = beta_r * vv[e];
                *reinterpret_cast<uint4 *>(sm + P_VI + img) = pack8(t);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        uint8_t *rec = p.ws + ((size_t)(b * p.H + h) * p.Nc + n) * REC_BYTES;
        // ---------------- Q e^G and K e^{G_C - G} leave now; tcgen05: A^T (cols 0-63), M^T (64-127),
        // residues of M's diagonal blocks (128-191)
        if (tid == 0) {
            bulk_store(rec + REC_QG, sm + P_QI, 16384);
            bulk_store(rec + REC_KT, sm + P_KI, 16384);
            bulk_commit();
            tc_fence_after();
            constexpr uint32_t id = idesc_f16(64, 16, 0, 0);
            const uint64_t kc = smem_desc(smem_u32(sm + P_KC), 16, 1024, LAYOUT_SW128);
            const uint64_t kr = smem_desc(smem_u32(sm + P_KR), 16, 1024, LAYOUT_SW128);
            const uint64_t qr = smem_desc(smem_u32(sm + P_QR), 16, 1024, LAYOUT_SW128);
            const uint64_t klo = smem_desc(smem_u32(sm + P_KLO), 16, 1024, LAYOUT_SW128);
            const uint64_t qlo = smem_desc(smem_u32(sm + P_ZI), 16, 1024, LAYOUT_SW128);
            // lo(k) * hi(q) for all four diagonal blocks at once: rows i of the residue image
            // carry the scaling of their own block, so the products are right wherever i and
            // r share a block (the only entries read)
            constexpr uint32_t id64 = idesc_f16(64, 64, 0, 0);
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                const uint32_t ko = (s8 >> 2), kb = (s8 & 3) * 32;
                mma_f16_ss(tmem + 128, dadd(klo, ko * 8192 + kb), dadd(qr, ko * 8192 + kb), id64, s8 > 0);
            }
#pragma unroll
            for (int V = 0; V < 4; ++V) {
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8) {
                    const uint32_t ko = (s8 >> 2), kb = (s8 & 3) * 32;
                    const uint64_t a = dadd(kc, ko * KC_ATOM + kc_row0(V) * 128 + kb);
                    const uint64_t bk = dadd(kr, ko * 8192 + V * 2048 + kb);
                    const uint64_t bq = dadd(qr, ko * 8192 + V * 2048 + kb);
                    mma_f16_ss(tmem + 16 * V, a, bk, id, s8 > 0);
                    mma_f16_ss(tmem + 64 + 16 * V, a, bq, id, s8 > 0);
                    // hi(k) * lo(q) on block V's columns, added to the residue above
                    mma_f16_ss(tmem + 128 + 16 * V, a, dadd(qlo, ko * 8192 + V * 2048 + kb), id, 1);
                }
            }
            mma_commit(bar_am);
        }
        ok = mbar_wait(bar_am, par);
        ok = __syncthreads_and(ok);
        tc_fence_after();
        if (!ok) break;
        // q, k, z images are dead (their stores have read them once the group drains): prefetch
        if (tid == 0 && u_next < p.units) {
            bulk_wait_read_all();
            load_qkz(u_next);
        }

        // ---------------- P3: A (masked, beta-weighted, fp32) and the M^T image
        {
            const int q4 = warp & 3, role = warp >> 2;
            const int i = 16 * q4 + lane;
            uint32_t va[32], vb[32], vd[16];
            const uint32_t taddr = tmem + ((uint32_t)(32 * q4) << 16) + 64 * role;
            tmem_ld_32x32b_x32(taddr, va);
            tmem_ld_32x32b_x32(taddr + 32, vb);
            tmem_ld_32x32b_x16(tmem + ((uint32_t)(32 * q4) << 16) + 128 + 16 * q4, vd);
            tmem_wait_ld();
            if (lane < 16) {
                if (role == 0) {
                    float *sA = reinterpret_cast<float *>(sm + P_SA);
#pragma unroll
                    for (int r = 0; r < 64; ++r) {
                        const float v = __uint_as_float(r < 32 ? va[r] : vb[r - 32]);
                        sA[r * SA_LD + i] = (i < r) ? sbeta[r] * v : 0.f;
                    }
                } else {
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        float t[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int r = 8 * cc + e;
                            float v = __uint_as_float(r < 32 ? va[r] : vb[r - 32]);
                            if ((r >> 4) == q4) v += __uint_as_float(vd[r & 15]);
                            t[e] = (i <= r) ? v : 0.f;
                        }
                        *reinterpret_cast<uint4 *>(sm + P_MT + sw128(i, cc)) = pack8(t);
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---------------- P4: T = (I + A)^{-1} by blocks of 16 (fp32)
        {
            const float *sA = reinterpret_cast<const float *>(sm + P_SA);
            float *sT = reinterpret_cast<float *>(sm + P_ST);
            float *xs = reinterpret_cast<float *>(sm + P_XS);
            for (int e = tid; e < 64 * ST_LD / 4; e += 256)
                reinterpret_cast<float4 *>(sT)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            __syncthreads();
            if (tid < 64) {  // diagonal block R, column jc: forward substitution
                const int R = tid >> 4, jc = tid & 15, o = 16 * R;
                float col[16];
#pragma unroll
                for (int a = 0; a < 16; ++a) {
                    float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int m = 0; m < a; ++m) part[m & 3] += sA[(o + a) * SA_LD + o + m] * col[m];
                    const float x = ((a == jc) ? 1.f : 0.f) - ((part[0] + part[1]) + (part[2] + part[3]));
                    col[a] = (a < jc) ? 0.f : x;
                }
#pragma unroll
                for (int a = 0; a < 16; ++a) sT[(o + a) * ST_LD + o + jc] = col[a];
            }
            __syncthreads();
            // blocks below the diagonal, one distance d = R - I at a time, 4 columns per thread:
            //   X = A[16R+a, 16I:16R] T[16I:16R, 16I+bc..+3],  T_RI = -T_RR X
#pragma unroll
            for (int d = 1; d < 4; ++d) {
                const int e = tid;
                const bool act = e < (4 - d) * 64;
                const int blk = e >> 6, R = d + blk, I = R - d, a = (e >> 2) & 15, bc = (e & 3) * 4;
                if (act) {
                    const float *arow = sA + (16 * R + a) * SA_LD + 16 * I;
                    const float *tblk = sT + 16 * I * ST_LD + 16 * I + bc;
                    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int k = 0; k < 16 * d; ++k) {
                        const float av = arow[k];
                        const float4 tv = *reinterpret_cast<const float4 *>(tblk + k * ST_LD);
                        x.x += av * tv.x; x.y += av * tv.y; x.z += av * tv.z; x.w += av * tv.w;
                    }
                    *reinterpret_cast<float4 *>(xs + blk * 256 + a * 16 + bc) = x;
                }
                __syncthreads();
                if (act) {
                    const float *trow = sT + (16 * R + a) * ST_LD + 16 * R;
                    const float *xb = xs + blk * 256 + bc;
                    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float tv = trow[m];  // zero above the diagonal
                        const float4 xv = *reinterpret_cast<const float4 *>(xb + m * 16);
                        y.x += tv * xv.x; y.y += tv * xv.y; y.z += tv * xv.z; y.w += tv * xv.w;
                    }
                    *reinterpret_cast<float4 *>(sT + (16 * R + a) * ST_LD + 16 * I + bc) =
                        make_float4(-y.x, -y.y, -y.z, -y.w);
                }
                __syncthreads();
            }
            {  // T image (K-major, 64 rows x 64 cols)
                const int r = tid >> 2, part = tid & 3;
#pragma unroll
                for (int uu = 0; uu < 2; ++uu) {
                    const int cc = 2 * part + uu;
                    float t[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = sT[r * ST_LD + 8 * cc + e];
                    *reinterpret_cast<uint4 *>(sm + P_TI + sw128(r, cc)) = pack8(t);
                }
            }
            fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncthreads();

        // ---------------- tcgen05: W = T (beta K e^G), U = T (beta V)   (M=64, N=128+128, K=64, B MN-major)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_f16(64, 128, 0, 1);
            const uint64_t ti = smem_desc(smem_u32(sm + P_TI), 16, 1024, LAYOUT_SW128);
            const uint64_t rw = smem_desc(smem_u32(sm + P_RH), 8192, 1024, LAYOUT_SW128);
            const uint64_t ru = smem_desc(smem_u32(sm + P_VI), 8192, 1024, LAYOUT_SW128);
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                mma_f16_ss(tmem, dadd(ti, s4 * 32), dadd(rw, s4 * 2048), id, s4 > 0);
                mma_f16_ss(tmem + 128, dadd(ti, s4 * 32), dadd(ru, s4 * 2048), id, s4 > 0);
            }
            mma_commit(bar_wu);
        }
        ok = mbar_wait(bar_wu, par);
        ok = __syncthreads_and(ok);
        tc_fence_after();
        if (!ok) break;
        if (tid == 0 && u_next < p.units) load_v(u_next);  // beta V has been consumed

        // ---------------- P5: W image and U slices
        {
            const int q4 = warp & 3, half = warp >> 2;
            const int r = 16 * q4 + lane;
#pragma unroll 1
            for (int cb = 0; cb < 4; ++cb) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q4) << 16) + 128 * half + 32 * cb, v);
                tmem_wait_ld();
                if (lane < 16) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float t[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) t[e] = __uint_as_float(v[8 * g + e]);
                        if (half == 0) {
                            const int j = 4 * cb + g;
                            *reinterpret_cast<uint4 *>(sm + P_WI + (j >> 3) * 8192 + sw128(r, j & 7)) = pack8(t);
                        } else {
                            const int jv = 32 * cb + 8 * g;
                            const int slice = jv / p.Nv, within = jv % p.Nv;
                            *reinterpret_cast<uint4 *>(sm + P_UI + slice * (64 * p.Nv * 2) +
                                                       (r * p.Nv + within) * 2) = pack8(t);
                        }
                    }
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            bulk_store(rec + REC_W, sm + P_WI, 16384);
            bulk_store(rec + REC_MT, sm + P_MT, 8192);
            bulk_store(rec + REC_U, sm + P_UI, 16384);
            bulk_store(rec + REC_GAM, sgam, 512);
            bulk_commit();
        }
    }

    if (tid == 0) {
        bulk_wait_all();
        if (!ok) report_timeout(p.timeouts, p.dev_status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ================================================================ K2b: chunk_state_kernel
struct StateArgs {
    int S, H, Nc;
    const uint8_t *ws;
    const float *S0;
    float *Sf;
    __nv_bfloat16 *o;
    unsigned int *timeouts;
    int *dev_status;
};

template <int NV> struct StateCfg {
    static constexpr uint32_t U_BYTES = 64 * NV * 2;
    static constexpr uint32_t STAGE_RAW = REC_IMG + U_BYTES + 512;
    static constexpr uint32_t STAGE = (STAGE_RAW + 1023) & ~1023u;
    static constexpr uint32_t S_U = REC_IMG;
    static constexpr uint32_t S_GAM = REC_IMG + U_BYTES;
    static constexpr uint32_t B_ST = 2 * STAGE;          // S^T image [2 atoms][NV rows][128 B]
    static constexpr uint32_t B_VT = B_ST + NV * 256;    // V'^T image [NV rows][128 B]
    static constexpr uint32_t B_BAR = B_VT + NV * 128;
    static constexpr uint32_t END = B_BAR + 64;
    static constexpr size_t SMEM = END + 1024;
    static constexpr uint32_t TCOLS = 4 * NV <= 32 ? 32 : (4 * NV <= 64 ? 64 : (4 * NV <= 128 ? 128 : 256));
    static constexpr uint32_t EXPECT = REC_IMG + U_BYTES + 512;
};

template <int NV>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[NV]) {
#pragma unroll
    for (int k = 0; k < NV / 16; ++k) {
        uint32_t t[16];
        tmem_ld_32x32b_x16(taddr + 16 * k, t);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[16 * k + e] = t[e];
    }
}

template <int NV>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&v)[NV]) {
#pragma unroll
    for (int k = 0; k < NV / 16; ++k) {
        uint32_t t[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) t[e] = v[16 * k + e];
        tmem_st_32x32b_x16(taddr + 16 * k, t);
    }
}

// S^T image element (row j, column c) for the K-major B operand [2 atoms][NV rows][128 B]
template <int NV>
__device__ __forceinline__ void write_st_row(uint8_t *img, int c, const float *vals) {
#pragma unroll
    for (int j = 0; j < NV; ++j)
        *reinterpret_cast<__nv_bfloat16 *>(img + (c >> 6) * (NV * 128) + sw128(j, (c & 63) >> 3) + (c & 7) * 2) =
            __float2bfloat16_rn(vals[j]);
}

template <int NV>
__global__ void __launch_bounds__(128, 1) chunk_state_kernel(StateArgs p) {
    using Cfg = StateCfg<NV>;
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int j0 = slice * NV;
    const int bh = b * p.H + h;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + Cfg::B_BAR);
    uint64_t *bar_po = full + 2;
    uint64_t *bar_so = full + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Cfg::B_BAR + 32);
    uint8_t *st_img = sm + Cfg::B_ST;
    uint8_t *vt_img = sm + Cfg::B_VT;
    const uint8_t *rec0 = p.ws + (size_t)bh * p.Nc * REC_BYTES;
    __shared__ int s_fail;

    auto issue_chunk = [&](int n, int stg) {
        uint8_t *dst = sm + stg * Cfg::STAGE;
        const uint8_t *src = rec0 + (size_t)n * REC_BYTES;
        mbar_arrive_expect_tx(&full[stg], Cfg::EXPECT);
        bulk_load(dst, src, REC_IMG, &full[stg]);
        bulk_load(dst + Cfg::S_U, src + REC_U + slice * Cfg::U_BYTES, Cfg::U_BYTES, &full[stg]);
        bulk_load(dst + Cfg::S_GAM, src + REC_GAM, 512, &full[stg]);
    };

    if (tid == 0) {
        s_fail = 0;
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(bar_po, 1);
        mbar_init(bar_so, 1);
        fence_barrier_init();
        for (int n = 0; n < 2 && n < p.Nc; ++n) issue_chunk(n, n);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, Cfg::TCOLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const uint32_t S_COL = 0, P_COL = NV, O_COL0 = 2 * NV;
    const int c = tid;  // state row (key channel) owned by this thread

    // ---------------- initial state -> TMEM accumulator
    {
        uint32_t su[NV];
        if (p.S0) {
            const float4 *src = reinterpret_cast<const float4 *>(p.S0 + ((size_t)bh * DD + c) * DD + j0);
#pragma unroll
            for (int k = 0; k < NV / 4; ++k) {
                const float4 x = src[k];
                su[4 * k] = __float_as_uint(x.x); su[4 * k + 1] = __float_as_uint(x.y);
                su[4 * k + 2] = __float_as_uint(x.z); su[4 * k + 3] = __float_as_uint(x.w);
            }
        } else {
#pragma unroll
            for (int j = 0; j < NV; ++j) su[j] = 0u;
        }
        tmem_st_cols<NV>(tmem + lane_base + S_COL, su);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    constexpr uint32_t id_p = idesc_f16(64, NV, 0, 0);
    constexpr uint32_t id_o = idesc_f16(64, NV, 1, 0);
    constexpr uint32_t id_s = idesc_f16(128, NV, 1, 0);
    const uint64_t d_st = smem_desc(smem_u32(st_img), 16, 1024, LAYOUT_SW128);
    const uint64_t d_vt = smem_desc(smem_u32(vt_img), 16, 1024, LAYOUT_SW128);
    const uint64_t d_k16 = smem_desc(smem_u32(sm), 16, 1024, LAYOUT_SW128);     // K-major images
    const uint64_t d_mn = smem_desc(smem_u32(sm), 8192, 1024, LAYOUT_SW128);    // MN-major images

    // O of chunk m (TMEM buffer m & 1) -> o~ rows of the chunk (this thread's token row)
    auto store_o = [&](int m) {
        uint32_t ov[NV];
        tmem_ld_cols<NV>(tmem + lane_base + O_COL0 + (m & 1) * NV, ov);
        tmem_wait_ld();
        const int r = 16 * warp + lane;
        const int t = m * CH + r;
        if (lane < 16 && t < p.S) {
            __nv_bfloat16 *dst = p.o + (((size_t)b * p.S + t) * p.H + h) * DD + j0;
#pragma unroll
            for (int k = 0; k < NV / 8; ++k) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(ov[8 * k + e]);
                reinterpret_cast<uint4 *>(dst)[k] = pack8(f);
            }
        }
    };

    bool ok = true;
    for (int n = 0; n < p.Nc; ++n) {
        const int stg = n & 1;
        uint8_t *sg = sm + stg * Cfg::STAGE;
        const uint32_t sgo = stg * Cfg::STAGE;
        const uint32_t ocol = O_COL0 + (n & 1) * NV;
        // ---------- this chunk's record; S_n -> bf16 operand; S <- Diag(e^{G_C}) S_n in TMEM
        if (!mbar_wait(&full[stg], (n >> 1) & 1)) s_fail = 1;
        {
            uint32_t sv[NV];
            tmem_ld_cols<NV>(tmem + lane_base + S_COL, sv);
            tmem_wait_ld();
            float sf[NV];
#pragma unroll
            for (int j = 0; j < NV; ++j) sf[j] = __uint_as_float(sv[j]);
            write_st_row<NV>(st_img, c, sf);
            const float gam = reinterpret_cast<const float *>(sg + Cfg::S_GAM)[c];
#pragma unroll
            for (int j = 0; j < NV; ++j) sv[j] = __float_as_uint(sf[j] * gam);
            tmem_st_cols<NV>(tmem + lane_base + S_COL, sv);
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_fail) { ok = false; break; }
        // ---------- P = W S and O = (Q e^G) S
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t ko = s >> 2, kb = (s & 3) * 32;
                const uint64_t bd = dadd(d_st, ko * (NV * 128) + kb);
                mma_f16_ss(tmem + P_COL, dadd(d_k16, sgo + REC_W + ko * 8192 + kb), bd, id_p, s > 0);
                mma_f16_ss(tmem + ocol, dadd(d_k16, sgo + REC_QG + ko * 8192 + kb), bd, id_p, s > 0);
            }
            mma_commit(bar_po);
        }
        if (n > 0) store_o(n - 1);  // overlaps the MMAs just issued
        if (!mbar_wait(bar_po, n & 1)) s_fail = 1;
        tc_fence_after();
        // ---------- V' = U - P (token rows of the M=64 accumulator layout)
        {
            uint32_t pv[NV];
            tmem_ld_cols<NV>(tmem + lane_base + P_COL, pv);
            tmem_wait_ld();
            if (lane < 16) {
                const int r = 16 * warp + lane;
                const __nv_bfloat16 *u = reinterpret_cast<const __nv_bfloat16 *>(sg + Cfg::S_U) + r * NV;
#pragma unroll
                for (int j = 0; j < NV; ++j) {
                    const float vp = __bfloat162float(u[j]) - __uint_as_float(pv[j]);
                    *reinterpret_cast<__nv_bfloat16 *>(vt_img + sw128(j, r >> 3) + (r & 7) * 2) =
                        __float2bfloat16_rn(vp);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_fail) { ok = false; break; }
        // ---------- O += M V' and S += (K e^{G_C - G})^T V'
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint64_t bd = dadd(d_vt, s * 32);
                mma_f16_ss(tmem + ocol, dadd(d_mn, sgo + REC_MT + s * 2048), bd, id_o, 1);
                mma_f16_ss(tmem + S_COL, dadd(d_mn, sgo + REC_KT + s * 2048), bd, id_s, 1);
            }
            mma_commit(bar_so);
        }
        if (!mbar_wait(bar_so, n & 1)) s_fail = 1;
        tc_fence_after();
        __syncthreads();
        if (s_fail) { ok = false; break; }
        if (tid == 0 && n + 2 < p.Nc) issue_chunk(n + 2, stg);
    }
    if (ok && p.Nc > 0) store_o(p.Nc - 1);

    if (ok) {
        if (p.Sf) {
            uint32_t sv[NV];
            tmem_ld_cols<NV>(tmem + lane_base + S_COL, sv);
            tmem_wait_ld();
            float4 *dst = reinterpret_cast<float4 *>(p.Sf + ((size_t)bh * DD + c) * DD + j0);
#pragma unroll
            for (int k = 0; k < NV / 4; ++k)
                dst[k] = make_float4(__uint_as_float(sv[4 * k]), __uint_as_float(sv[4 * k + 1]),
                                     __uint_as_float(sv[4 * k + 2]), __uint_as_float(sv[4 * k + 3]));
        }
    } else if (tid == 0) {
        report_timeout(p.timeouts, p.dev_status);
        // let bulk copies already issued land before the CTA exits
        for (int s = 0; s < 2; ++s) mbar_wait(&full[s], 0, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TCOLS);
}

template <int NV>
kda_status_t launch_state(const StateArgs &sa, int B, int H, cudaStream_t st) {
    using Cfg = StateCfg<NV>;
    cudaFuncSetAttribute(chunk_state_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
    chunk_state_kernel<NV><<<dim3(DD / NV, H, B), 128, Cfg::SMEM, st>>>(sa);
    return check_launch("chunk_state_kernel");
}

// (B, S, H, 128) bf16 tensor seen as 4-D (channel, head, token, batch); a box is
// 64 channels x 1 head x 64 tokens x 1 batch row, 128-byte swizzled, and tokens
// past the end of a sequence read as zero.
kda_status_t make_tmap_tokens(CUtensorMap *m, const void *base, int H, int64_t S, int64_t B, uint64_t rs,
                              uint64_t ss, uint64_t bs) {
    const uint64_t dims[4] = {(uint64_t)DD, (uint64_t)H, (uint64_t)S, (uint64_t)B};
    const uint64_t strides[3] = {rs, ss, bs};
    const uint32_t box[4] = {64, 1, CH, 1};
    return make_tmap_nd(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 4, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

int pick_nv(int64_t BH) {
    if (BH >= 148) return 64;
    if (BH >= 74) return 32;
    return 16;
}

}  // namespace

bool chunk_tc_supported(const kda_chunk_args &a, int chunk) {
    return a.dtype == KDA_BF16 && a.D_k == DD && a.D_v == DD && chunk == CH && a.g_min >= TC_GMIN_LIMIT &&
           a.B <= 65535 && a.H <= 65535 && a.S <= 0x7fffffffLL - CH;
}

bool chunk_tc_aligned(const kda_chunk_args &a) {
    auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    bool okp = al(a.q) && al(a.k) && al(a.v) && al(a.o) && al(a.initial_state) && al(a.final_state);
    if (!a.log_decay) okp = okp && al(a.z);
    return okp;
}

size_t chunk_tc_workspace(const kda_chunk_args &a) {
    const int64_t Nc = (a.S + CH - 1) / CH;
    return (size_t)a.B * a.H * Nc * REC_BYTES;
}

kda_status_t launch_chunk_tc(const kda_chunk_args &a, cudaStream_t st) {
    const int64_t Nc = (a.S + CH - 1) / CH;
    const int nv = pick_nv((int64_t)a.B * a.H);
    unsigned int *timeouts = device_timeout_counter();
    if (Nc > 0) {
        CUtensorMap tq, tk, tv, tz;
        const uint64_t rs = (uint64_t)DD, ss = (uint64_t)a.H * DD, bs = (uint64_t)a.S * a.H * DD;
        kda_status_t s;
        s = make_tmap_tokens(&tq, a.q, a.H, a.S, a.B, rs, ss, bs);
        if (s != KDA_OK) return s;
        s = make_tmap_tokens(&tk, a.k, a.H, a.S, a.B, rs, ss, bs);
        if (s != KDA_OK) return s;
        s = make_tmap_tokens(&tv, a.v, a.H, a.S, a.B, rs, ss, bs);
        if (s != KDA_OK) return s;
        if (a.log_decay) {
            tz = tq;  // unused
        } else {
            s = make_tmap_tokens(&tz, a.z, a.H, a.S, a.B, rs, ss, bs);
            if (s != KDA_OK) return s;
        }
        PrepArgs pa;
        pa.S = (int)a.S;
        pa.H = a.H;
        pa.Nc = (int)Nc;
        pa.Nv = nv;
        pa.units = Nc * a.H * a.B;
        pa.g_min = a.g_min;
        pa.beta = (const __nv_bfloat16 *)a.beta;
        pa.log_decay = a.log_decay;
        pa.ws = (uint8_t *)a.workspace;
        pa.timeouts = timeouts;
        pa.dev_status = a.dev_status;
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t grid = pa.units < sms ? pa.units : sms;
        cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREP_SMEM);
        chunk_prep_kernel<<<(unsigned)grid, 256, PREP_SMEM, st>>>(tq, tk, tv, tz, pa);
        s = check_launch("chunk_prep_kernel");
        if (s != KDA_OK) return s;
    }
    StateArgs sa;
    sa.S = (int)a.S;
    sa.H = a.H;
    sa.Nc = (int)Nc;
    sa.ws = (const uint8_t *)a.workspace;
    sa.S0 = a.initial_state;
    sa.Sf = a.final_state;
    sa.o = (__nv_bfloat16 *)a.o;
    sa.timeouts = timeouts;
    sa.dev_status = a.dev_status;
    kda_status_t s;
    switch (nv) {
        case 16: s = launch_state<16>(sa, (int)a.B, a.H, st); break;
        case 32: s = launch_state<32>(sa, (int)a.B, a.H, st); break;
        default: s = launch_state<64>(sa, (int)a.B, a.H, st); break;
    }
    if (s != KDA_OK) return s;
    if (a.gate_logits && a.S > 0)
        return launch_norm_gate(a.o, a.gate_logits, a.B * a.S, a.H, DD, a.eps, a.o, KDA_BF16, st);
    return KDA_OK;
}

}  // namespace kda
