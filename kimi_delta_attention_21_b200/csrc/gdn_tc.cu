// Tensor-core chunk prep for the Gated DeltaNet special case: one scalar decay
// per token and head (the DPLR post's GDN form, S_t = alpha_t (I - beta_t k_t
// k_t^T) S_{t-1} + beta_t k_t v_t^T, which is Eq. 1 of the Kimi Linear report
// with Diag(alpha_t) = alpha_t I).
//
// With a channel-independent decay the decayed products of the chunk form
// factor exactly: exp(G_r - G_i) is one number per token pair, so
//
//   A[r, i] = beta_r exp(G_r - G_i) (k_r . k_i)      (i < r)
//   M[r, i] =        exp(G_r - G_i) (q_r . k_i)      (i <= r)
//
// come from one plain tensor-core product of the raw bf16 keys and queries
// (products of bf16 values are exact in the fp32 accumulator) scaled by a
// per-pair factor <= 1 in the readout.  No block references, no per-channel
// tables, no split operands, and no bound on g_min.  The rest of the UT
// transform is the KDA prep's: T = (I + A)^{-1}, W = T Diag(beta)(K e^G),
// U = T Diag(beta) V.  The prep writes the same per-chunk record as the KDA
// prep ([-W; Q e^G], K e^{G_C - G}, M^T, U^T, e^{G_C} broadcast to the 128
// key channels), so the state pass, with its fused RMSNorm and output gate, is
// shared unchanged.
//
// gdn_prep_kernel is persistent (one CTA of 16 warps per SM walks the
// (chunk, head, batch) units).  The q, k and v tiles are double-buffered and
// loaded one unit ahead; k and q sit stacked in one [k; q] image that is both
// operands of the [k; q][k; q]^T MMA (lanes 0-63 of its accumulator hold
// K K^T in columns 0-63 and K Q^T = M^T in columns 64-127) and, once those are
// read, the record's [-W; Q e^G] image.
#include <cstring>

#include "tc_common.cuh"

namespace kda {

namespace {

using namespace tc;

constexpr int GP_THREADS = 512;
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t G_KQ = 0;          // [2 buffers][2 atoms (c / 64)][128 rows: k 0-63, q 64-127][128 B]
constexpr uint32_t G_KQ_BUF = 32768;
constexpr uint32_t G_V = 65536;       // [2 buffers][2 atoms][64 rows][128 B]: v, then beta V in place
constexpr uint32_t G_V_BUF = 16384;
constexpr uint32_t G_KT = 98304;      // K e^{G_C - G} image [2 atoms][64][128 B]
constexpr uint32_t G_RH = 114688;     // beta K e^G image [2 atoms][64][128 B] (MN-major B of the W MMA)
constexpr uint32_t G_MT = 131072;     // M^T image [64 rows i][128 B: r]
constexpr uint32_t G_TI = 139264;     // T image [64 rows][128 B]
constexpr uint32_t G_U = 147456;      // U^T image [128 rows j][128 B: r]
constexpr uint32_t G_SA = 163840;     // A [64][SA_LD] fp32
constexpr uint32_t G_ST = G_SA + 64 * SA_LD * 4;   // T [64][ST_LD] fp32
constexpr uint32_t G_IX = G_ST + 64 * ST_LD * 4;   // inverse scratch, 1536 fp32
constexpr uint32_t G_GV = G_IX + 1536 * 4;         // G [64], e^G [64], beta [64], e^{G_C} [128], warp sums [2],
                                                   // the next unit's log-decay [64] and beta [64] (from 384)
constexpr uint32_t G_BAR = G_GV + 2048;            // mbarriers: inputs [2], A/M MMA, W/U MMA; TMEM slot
constexpr uint32_t G_END = G_BAR + 64;
constexpr size_t GDN_SMEM = G_END + 1024;
static_assert(GDN_SMEM <= 232448, "gdn prep shared memory");

struct GdnArgs {
    int S, H, Nc;
    int64_t units;                 // Nc * H * B
    float g_min;
    const __nv_bfloat16 *beta;     // (B, S, H)
    const __nv_bfloat16 *z;        // (B, S, H) decay logits, or null
    const float *log_decay;        // (B, S, H) log alpha, or null (wins over z)
    uint8_t *ws;
    size_t rec_bytes;              // the records' part of ws (checked builds test the record stores against it)
    unsigned int *bounds;
    float *lbound;                 // per-chunk log-bounds of the transition norm [B*H][Nc] (null: one segment)
    unsigned int *timeouts;
    int *dev_status;
};

__global__ void __launch_bounds__(GP_THREADS, 1)
gdn_prep_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, GdnArgs p) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + G_BAR);  // [2] q, k, v of buffer b landed
    uint64_t *bar_am = bar_in + 2;
    uint64_t *bar_wu = bar_in + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_in + 4);
    float *sG = reinterpret_cast<float *>(sm + G_GV);
    float *seG = sG + 64;
    float *sbeta = sG + 128;
    float *sgam = sG + 192;
    float *wsum = sG + 320;
    float *sgn = sG + 384, *sbn = sG + 448;  // the next unit's log-decay and beta, loaded during the inverse
    __shared__ float s_lf;  // sum over the chunk's tokens of log max(1, |1 - beta |k|^2|)

    auto unit_coords = [&](int64_t u, int &n, int &h, int &b) {  // 32-bit: units < 2^31 (host check)
        const uint32_t uu = (uint32_t)u, nc = (uint32_t)p.Nc, hh = (uint32_t)p.H;
        const uint32_t bh = uu / nc;
        n = (int)(uu - bh * nc);
        b = (int)(bh / hh);
        h = (int)(bh - (uint32_t)b * hh);
    };
    auto load_inputs = [&](int64_t u, int buf) {  // q, k, v of unit u -> buffer buf (thread 0)
        int n, h, b;
        unit_coords(u, n, h, b);
        uint8_t *kq = sm + G_KQ + buf * G_KQ_BUF;
        uint8_t *vv = sm + G_V + buf * G_V_BUF;
        mbar_arrive_expect_tx(&bar_in[buf], 6u * 8192u);
        for (int a = 0; a < 2; ++a) {
            tma_load_4d(kq + a * 16384, &tk, &bar_in[buf], 64 * a, h, n * CH, b);
            tma_load_4d(kq + a * 16384 + 8192, &tq, &bar_in[buf], 64 * a, h, n * CH, b);
            tma_load_4d(vv + a * 8192, &tv, &bar_in[buf], 64 * a, h, n * CH, b);
        }
    };
    // log-decay and beta of row `row` of unit u (0 past the end of the sequence: no decay, no write)
    auto load_decay = [&](int64_t u, int row, float &g, float &bt) {
        int n, h, b;
        unit_coords(u, n, h, b);
        const int t = n * CH + row;
        g = 0.f;
        bt = 0.f;
        if (t < p.S) {
            const int64_t i = ((int64_t)b * p.S + t) * p.H + h;
            g = p.log_decay ? clamp_log_decay(p.log_decay[i], p.g_min) : log_alpha_fast(__bfloat162float(p.z[i]), p.g_min);
            bt = __bfloat162float(p.beta[i]);
        }
    };

    if (tid == 0) {
        mbar_init(&bar_in[0], 1);
        mbar_init(&bar_in[1], 1);
        mbar_init(bar_am, 1);
        mbar_init(bar_wu, 1);
        fence_barrier_init();
        if ((int64_t)blockIdx.x < p.units) load_inputs(blockIdx.x, 0);
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
    float g_cur = 0.f, b_cur = 0.f;
    if (tid < CH && (int64_t)blockIdx.x < p.units) load_decay(blockIdx.x, tid, g_cur, b_cur);

    int it = 0;
    for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++it) {
        int n, h, b;
        unit_coords(u, n, h, b);
        const int64_t u_next = u + gridDim.x;
        const int buf = it & 1;
        const uint32_t par = it & 1, ipar = (it >> 1) & 1;
        uint8_t *kq = sm + G_KQ + buf * G_KQ_BUF;
        uint8_t *vb = sm + G_V + buf * G_V_BUF;
        uint8_t *rec = p.ws + ((size_t)(b * p.H + h) * p.Nc + n) * REC_BYTES;
        // the next unit's inputs into the other buffers, once the previous unit's record stores (its
        // [-W; Q e^G] image came from the buffer now reloaded) have read them
        if (tid == 0 && u_next < p.units) {
            bulk_wait_read_all();
            load_inputs(u_next, buf ^ 1);
        }
        if (it > 0 && tid < CH) {  // this unit's log-decay and beta (loaded during the previous inverse)
            g_cur = sgn[tid];
            b_cur = sbn[tid];
        }
        if (tid == 0) s_lf = 0.f;
        // ---- cumulative log-decay over the chunk (warps 0-1: one token per thread), e^G, beta
        if (tid < CH) {
            float x = g_cur;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, d);
                if (lane >= d) x += y;
            }
            if (lane == 31) wsum[warp] = x;
            sbeta[tid] = b_cur;
            named_sync(2, 64);
            if (warp == 1) x += wsum[0];
            sG[tid] = x;
            seG[tid] = fexp(x);
        }
        ok = mbar_wait(&bar_in[buf], ipar) && ok;
        ok = __syncthreads_and(ok);
        if (!ok) break;
        // ---- A/M MMA: [k; q] [k; q]^T (M = N = 128, K = 128), both operands the stacked image
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t id = idesc_f16(128, 128, 0, 0);
            const uint64_t d = smem_desc(smem_u32(kq), 16, 1024, LAYOUT_SW128);
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                const uint32_t ko = s8 >> 2, kb = (s8 & 3) * 32;
                mma_f16_ss(tmem, dadd(d, ko * 16384 + kb), dadd(d, ko * 16384 + kb), id, s8 > 0);
            }
            mma_commit(bar_am);
        }
        // ---- meanwhile: K e^{G_C - G}, beta K e^G and beta V (reads of the MMA's operands only)
        if (tid == 32) bulk_wait_read_all();  // the previous unit's K~, M^T and e^{G_C} stores
        __syncthreads();
        const float GC = sG[CH - 1];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int item = tid + GP_THREADS * m, r = item >> 4, cc = item & 15, atom = cc >> 3, ch = cc & 7;
            const uint32_t koff = atom * 16384 + sw128(r, ch), off = atom * 8192 + sw128(r, ch);
            float kv[8], vv[8], t[8];
            unpack8(*reinterpret_cast<const uint4 *>(kq + koff), kv);
            unpack8(*reinterpret_cast<const uint4 *>(vb + off), vv);
            const float fk = fexp(GC - sG[r]), fr = sbeta[r] * seG[r], bt = sbeta[r];
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = kv[e] * fk;
            *reinterpret_cast<uint4 *>(sm + G_KT + off) = pack8(t);
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = kv[e] * fr;
            *reinterpret_cast<uint4 *>(sm + G_RH + off) = pack8(t);
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = vv[e] * bt;
            *reinterpret_cast<uint4 *>(vb + off) = pack8(t);
        }
        if (tid < 128) sgam[tid] = fexp(GC);
        ok = mbar_wait(bar_am, par) && ok;
        tc_fence_after();
        // ---- readout (lanes 0-63 of the accumulator = key rows i): warps 0-1 A (row r = lane, fp32),
        //      warps 4-5 M^T (row i = lane, bf16 image); the other warps write Q e^G over the q rows
        if (warp < 2 || warp == 4 || warp == 5) {
            const int row = 32 * (warp & 1) + lane;
            const uint32_t base = tmem + ((uint32_t)(32 * (warp & 1)) << 16) + (warp < 2 ? 0u : 64u);
            const float Gr = sG[row];
            uint32_t v[64];
            tmem_ld_32x32b_x32(base, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld_32x32b_x32(base + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tmem_wait_ld();
            // Every entry is computed and the masked ones multiplied by zero (no branch per entry, so the
            // exponential chains overlap); the exponent is capped at 0, which only the masked entries
            // reach (G never increases along the chunk), so that they stay finite.
            if (warp < 2) {  // A[r, i] = beta_r e^{G_r - G_i} k_r . k_i for i < r
                float *sA = reinterpret_cast<float *>(sm + G_SA) + row * SA_LD;
                const float br = sbeta[row];
                float kk = 0.f;  // |k_row|^2, the diagonal entry
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    sA[i] = br * (fexp(fminf(Gr - sG[i], 0.f)) * (i < row ? 1.f : 0.f)) * __uint_as_float(v[i]);
                    if (i == row) kk = __uint_as_float(v[i]);
                }
                if (p.lbound) {  // this token's log max(1, |1 - beta |k|^2|), |k|^2 widened by 2^-7;
                                 // summed over the warp, one shared add per warp
                    const float lo = kk * (1.f - 0.0078125f), hi = kk * (1.f + 0.0078125f);
                    float lf = __logf(fmaxf(1.f, fmaxf(fabsf(1.f - br * lo), fabsf(1.f - br * hi))));
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) lf += __shfl_xor_sync(0xffffffffu, lf, off);
                    if (lane == 0 && lf != 0.f) atomicAdd(&s_lf, lf);
                }
            } else {         // M^T[i, r] = e^{G_r - G_i} q_r . k_i for i <= r (row = i)
#pragma unroll
                for (int k8 = 0; k8 < 8; ++k8) {
                    float t[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int r = 8 * k8 + e;
                        t[e] = (fexp(fminf(sG[r] - Gr, 0.f)) * (row <= r ? 1.f : 0.f)) * __uint_as_float(v[r]);
                    }
                    *reinterpret_cast<uint4 *>(sm + G_MT + sw128(row, k8)) = pack8(t);
                }
            }
        } else {
            const int t2 = (warp < 4 ? tid - 64 : tid - 128);  // warps 2-3: 0 .. 63, warps 6-15: 64 .. 383
            for (int item = t2; item < 1024; item += 384) {   // Q e^G over the q rows of the stacked image
                const int r = item >> 4, cc = item & 15, atom = cc >> 3, ch = cc & 7;
                uint8_t *qp = kq + atom * 16384 + 8192 + sw128(r, ch);
                float qv[8];
                unpack8(*reinterpret_cast<const uint4 *>(qp), qv);
                const float f = seG[r];
#pragma unroll
                for (int e = 0; e < 8; ++e) qv[e] *= f;
                *reinterpret_cast<uint4 *>(qp) = pack8(qv);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok);
        if (!ok) break;
        if (tid == 256 && p.lbound)  // (warp 8, idle in the inverse) the chunk's log-bound: its exact log-decay
                                     // sum (one alpha per token) and the |k| terms
            p.lbound[((size_t)b * p.H + h) * p.Nc + n] = sG[CH - 1] + s_lf;
        if (tid == 32 && in_bounds(rec, REC_BYTES, p.ws, p.rec_bytes, p.bounds)) {
            bulk_store(rec + REC_KT, sm + G_KT, 16384);
            bulk_store(rec + REC_MT, sm + G_MT, 8192);
            bulk_store(rec + REC_GAM, sgam, 512);
            bulk_commit();
        }
        // ---- T = (I + A)^{-1} (warps 0-3); meanwhile warps 4-5 read the next unit's log-decay and beta
        //      (global loads still in flight would hold up a barrier: these have the inverse to land)
        if (warp < 4) {
            invert_unit_lower64(reinterpret_cast<const float *>(sm + G_SA), reinterpret_cast<float *>(sm + G_ST),
                                reinterpret_cast<float *>(sm + G_IX), sm + G_TI, tid);
        } else if (warp < 6 && u_next < p.units) {
            float g, bt;
            load_decay(u_next, tid - 128, g, bt);
            sgn[tid - 128] = g;
            sbn[tid - 128] = bt;
        }
        tc_fence_before();
        __syncthreads();
        // ---- W = T (beta K e^G) (M = 64, N = 128, K = 64) and U^T = (beta V)^T T^T (M = 128, N = 64, K = 64)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idw = idesc_f16(64, 128, 0, 1);
            constexpr uint32_t idu = idesc_f16(128, 64, 1, 0);
            const uint64_t ti = smem_desc(smem_u32(sm + G_TI), 16, 1024, LAYOUT_SW128);
            const uint64_t rw = smem_desc(smem_u32(sm + G_RH), 8192, 1024, LAYOUT_SW128);
            const uint64_t vt = smem_desc(smem_u32(vb), 8192, 1024, LAYOUT_SW128);
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                mma_f16_ss(tmem, dadd(ti, s4 * 32), dadd(rw, s4 * 2048), idw, s4 > 0);
                mma_f16_ss(tmem + 128, dadd(vt, s4 * 2048), dadd(ti, s4 * 32), idu, s4 > 0);
            }
            mma_commit(bar_wu);
        }
        ok = mbar_wait(bar_wu, par) && ok;
        ok = __syncthreads_and(ok);
        tc_fence_after();
        if (!ok) break;
        // ---- -W over the k rows of the stacked image (warp groups 0 and 2: the M = 64 accumulator's rows
        //      16 q4 + lane, half the columns each) and the U^T image (warp groups 1 and 3)
        {
            const int q4 = warp & 3, wg = warp >> 2;
            if ((wg & 1) == 0) {
                const int r = 16 * q4 + lane;
#pragma unroll 1
                for (int cb = 0; cb < 2; ++cb) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q4) << 16) + 64 * (wg >> 1) + 32 * cb, v);
                    tmem_wait_ld();
                    if (lane < 16) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            float t[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) t[e] = -__uint_as_float(v[8 * g + e]);
                            const int j = 8 * (wg >> 1) + 4 * cb + g;  // 8-column group
                            *reinterpret_cast<uint4 *>(kq + (j >> 3) * 16384 + sw128(r, j & 7)) = pack8(t);
                        }
                    }
                }
            } else {
                const int jv = 32 * q4 + lane;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q4) << 16) + 128 + 32 * (wg >> 1), v);
                tmem_wait_ld();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float t[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = __uint_as_float(v[8 * g + e]);
                    *reinterpret_cast<uint4 *>(sm + G_U + sw128(jv, 4 * (wg >> 1) + g)) = pack8(t);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && in_bounds(rec, REC_BYTES, p.ws, p.rec_bytes, p.bounds)) {
            bulk_store(rec + REC_WQ, kq, 32768);
            bulk_store(rec + REC_U, sm + G_U, 16384);
            bulk_commit();
        }
    }

    if (tid == 0 || tid == 32) bulk_wait_all();
    if (tid == 0 && !ok) report_timeout(p.timeouts, p.dev_status);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace

bool gdn_tc_supported(const kda_chunk_args &a, int chunk) {
    return a.dtype == KDA_BF16 && a.D_k == DD && a.D_v == DD && chunk == CH && a.B <= 65535 && a.H <= 65535 &&
           a.S <= 0x7fffffffLL - CH;
}

bool gdn_tc_aligned(const kda_chunk_args &a) {
    auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    return al(a.q) && al(a.k) && al(a.v) && al(a.o) && al(a.initial_state) && al(a.final_state) && al(a.gate_logits);
}

kda_status_t launch_gdn_tc(const kda_chunk_args &a, cudaStream_t st) {
    const int64_t Nc = (a.S + CH - 1) / CH;
    if (Nc > 0) {
        CUtensorMap tq, tk, tv;
        const uint64_t rs = (uint64_t)DD, ss = (uint64_t)a.H * DD, bs = (uint64_t)a.S * a.H * DD;
        kda_status_t s = make_tmap_tokens(&tq, a.q, a.H, a.S, a.B, rs, ss, bs);
        if (s != KDA_OK) return s;
        s = make_tmap_tokens(&tk, a.k, a.H, a.S, a.B, rs, ss, bs);
        if (s != KDA_OK) return s;
        s = make_tmap_tokens(&tv, a.v, a.H, a.S, a.B, rs, ss, bs);
        if (s != KDA_OK) return s;
        GdnArgs ga;
        ga.S = (int)a.S;
        ga.H = a.H;
        ga.Nc = (int)Nc;
        ga.units = Nc * a.H * a.B;
        if (ga.units > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "GDN chunk engine: more than 2^31 chunks");
        ga.g_min = a.g_min;
        ga.beta = (const __nv_bfloat16 *)a.beta;
        ga.z = (const __nv_bfloat16 *)a.z;
        ga.log_decay = a.log_decay;
        ga.ws = (uint8_t *)a.workspace;
        ga.rec_bytes = (size_t)ga.units * REC_BYTES;
        ga.bounds = device_bounds_counter();
        ga.lbound = tc::chunk_log_bounds(a);
        ga.timeouts = device_timeout_counter();
        ga.dev_status = a.dev_status;
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int64_t grid = ga.units < sms ? ga.units : sms;
        cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GDN_SMEM);
        cudaError_t e = launch_pdl(gdn_prep_kernel, dim3((unsigned)grid), dim3(GP_THREADS), GDN_SMEM, st, tq, tk, tv,
                                   ga);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "gdn_prep_kernel: %s", cudaGetErrorString(e));
        s = check_launch("gdn_prep_kernel");
        if (s != KDA_OK) return s;
    }
    return tc::launch_chunk_state_pass(a, st);
}

}  // namespace kda
