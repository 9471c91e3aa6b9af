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
// Kernels:
//  * chunk_prep_kernel, persistent (one CTA per SM walks the (chunk, head,
//    batch) units; all chunks are independent): TMA loads of q, k, v; the
//    cumulative log-decay (from z or the log-decay input, read directly);
//    decay-scaled operands; A^T and M^T on tcgen05; the inverse T in fp32 SIMT;
//    [W | U^T] = T [beta K e^G | beta V] on tcgen05.  It writes one workspace
//    record per chunk holding [-W; Q*e^G], K*e^{G_C-G}, M^T and U^T as
//    ready-made 128-byte-swizzled shared-memory images, and e^{G_C}.
//  * the state pass.  A long sequence is cut into G segments:
//    chunk_map_pair_kernel gives every segment but the last its affine map
//    S_end = A_g S_start + Y_g (both chains in one CTA), chunk_combine_kernel
//    chains the maps into each segment's entering state, and
//    chunk_state_kernel, one CTA per (head, batch, segment), walks the
//    segment's chunks in order with the state resident in TMEM, streaming the
//    records with bulk copies, and writes the gated, normalised output and the
//    final state.
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
// sum_c |q_c k_c| in every product, which can be a large part of a token's
// o~ when o~ is small (the state decayed away, small writes), and the per-head
// RMS normalisation then turns it into a large output error.  M is therefore
// computed with split operands, x = hi + lo (both bf16): every block adds
// hi(k) lo(q) (the low q rows are part of the stacked B operand), and the
// diagonal 16x16 blocks, where no decay shrinks the terms, add lo(k) hi(q)
// too (the low part of the diagonal column operand is part of the A operand).
#include <cstring>

#include <cuda_fp16.h>

#include "tc_common.cuh"

namespace kda {

namespace {

using namespace sm100;
using namespace tc;


// ================================================================ K2a: chunk_prep_kernel
// Persistent: one CTA per SM walks (chunk, head, batch) units.  The next unit's
// q and k tiles are loaded by TMA as soon as the record stores have read this
// unit's copies (while the A/M MMAs run), its z tile once the A/M MMAs have
// read their operands, v after the W/U MMAs; the workspace bulk stores drain
// while the next unit is computed.
// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t P_QI = 0;         // q image; becomes Q e^G (stored as soon as P2 ends)
constexpr uint32_t P_KI = 16384;     // k image; becomes K e^{G_C - G}
constexpr uint32_t P_VI = 32768;     // v image; becomes beta V (operand of the W and U^T MMAs)
constexpr uint32_t P_ZI = 49152;     // beta K e^G (MN-major B operand of the W MMA)
constexpr uint32_t P_A = 65536;      // A operand of the A/M MMAs [2 atoms][224 rows][128 B]: the column operand
                                     // in its 4 block versions (rows 0-159) and the low part of the diagonal
                                     // one (rows 160-223); later -W, U^T and the M^T image
constexpr uint32_t P_B = 122880;     // B operand [2 atoms][192 rows][128 B]: row operands from k, q and the low
                                     // part of the q one; later the T image and the diagonal residues
constexpr uint32_t P_SG = 172032;    // G fp32 [64][132] (the next unit's, written beside this unit's inverse)
constexpr uint32_t P_TAB = 206080;   // per-channel block constants [26][128] fp32 (likewise)
constexpr uint32_t P_XS = 219392;    // quarter sums of the cumulative log-decay [4][128] fp32
constexpr uint32_t P_BETA = 222464;  // beta [64] fp32
constexpr uint32_t P_GAM = 222720;   // e^{G_C} [128] fp32
constexpr uint32_t P_BAR = 223232;   // mbarriers: q/k, A/M MMAs, W/U MMAs; TMEM slot (+24); z tile (+32); v (+40)
constexpr uint32_t P_END = 223312;
constexpr size_t PREP_SMEM = P_END + 1024;
constexpr uint32_t P_RH = P_ZI;
constexpr uint32_t P_WI = P_A, P_UI = P_A + 16384, P_MT = P_A + 32768;
constexpr uint32_t P_ZT = P_A + 40960;  // the next unit's z tile [2 atoms][64 rows][128 B], between the A/M MMAs
                                        // and the next unit's P2 (nothing else uses these 16 KB then)
constexpr uint32_t A_ATOM = 224 * 128;  // bytes per atom column of the A/M MMAs' A operand
constexpr uint32_t B_ATOM = 192 * 128;  // ... and of their B operand
constexpr uint32_t B_ATOM_BYTES = B_ATOM;
// During P3 and P4 the A/M operands are dead: the T image, A and T (fp32) live in the B operand's
// space, the low-part hand-off and the inverse's scratch in the first 10 KB of the A operand's (the
// W and U^T images only take it in P5), so that G, the tables, beta and e^{G_C} are free for the next
// unit's decay, which runs beside the inverse.
constexpr uint32_t P_TI = P_B;                        // T image (bf16)
constexpr uint32_t P_SA = P_B + 8192;                 // A [64][65] fp32
constexpr uint32_t P_ST = P_SA + 16640;               // T [64][68] fp32
constexpr uint32_t P_LOHI = P_A;                      // [64][16] fp32
constexpr uint32_t P_IX = P_A + 4096;                 // inverse scratch [512 + 1024] fp32
static_assert(P_ST + 64 * 68 * 4 <= P_B + 2 * B_ATOM_BYTES, "A and T fit in the B operand's space");
constexpr int SG_LD = 132;
constexpr uint32_t A_KLO = 160;         // first row of the low part of the diagonal column operand

// table rows: b_R (0-3), F_R = e^{b_{R-1} - m_R} (4-7), E_R = e^{b_{R-1}} (8-11),
// D_R = e^{b_3 - b_R} (12-15), C_{V,R} = e^{m_V - b_R} for R <= V (16 + V(V+1)/2 + R)
__device__ __forceinline__ int tab_c(int V, int R) { return 16 + V * (V + 1) / 2 + R; }
__device__ __forceinline__ int kc_row0(int V) { return 8 * V * (V + 1); }  // 0, 16, 48, 96

struct PrepArgs {
    int S, H, Nc;
    int64_t units;  // Nc * H * B
    float g_min;
    const __nv_bfloat16 *beta;
    const float *log_decay;
    uint8_t *ws;
    size_t rec_bytes;        // the records' part of ws (checked builds test the record stores against it)
    unsigned int *bounds;
    float *lbound;           // per-chunk log-bounds of the transition norm [B*H][Nc] (null: one segment)
    unsigned int *timeouts;
    int *dev_status;
};

constexpr int PREP_THREADS = 512;

__global__ void __launch_bounds__(PREP_THREADS, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tz, PrepArgs p) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + P_BAR);
    uint64_t *bar_am = bar_in + 1;
    uint64_t *bar_wu = bar_in + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + P_BAR + 24);
    uint64_t *bar_z = reinterpret_cast<uint64_t *>(sm + P_BAR + 32);
    uint64_t *bar_v = reinterpret_cast<uint64_t *>(sm + P_BAR + 40);
    float *sG = reinterpret_cast<float *>(sm + P_SG);
    float *tab = reinterpret_cast<float *>(sm + P_TAB);
    float *sbeta = reinterpret_cast<float *>(sm + P_BETA);
    float *sgam = reinterpret_cast<float *>(sm + P_GAM);
    const uint32_t in_bytes = 4u * 8192u;  // q, k
    // the chunk's log-bound of the transition norm: the largest log(alpha) of its tokens (from the decay
    // group, per warp then per unit) and beta |k|^2 of each token (from the readout)
    __shared__ float s_gmax_w[8], s_unit_gmax, s_bk[CH];

    auto unit_coords = [&](int64_t u, int &n, int &h, int &b) {  // 32-bit: units < 2^31 (host check)
        const uint32_t uu = (uint32_t)u, nc = (uint32_t)p.Nc, hh = (uint32_t)p.H;
        const uint32_t bh = uu / nc;
        n = (int)(uu - bh * nc);
        b = (int)(bh / hh);
        h = (int)(bh - (uint32_t)b * hh);
    };
    auto load_qk = [&](int64_t u) {
        int n, h, b;
        unit_coords(u, n, h, b);
        mbar_arrive_expect_tx(bar_in, in_bytes);
        for (int a = 0; a < 2; ++a) {
            tma_load_4d(sm + P_QI + a * 8192, &tq, bar_in, 64 * a, h, n * CH, b);
            tma_load_4d(sm + P_KI + a * 8192, &tk, bar_in, 64 * a, h, n * CH, b);
        }
    };
    auto load_z = [&](int64_t u) {  // z tile of unit u -> P_ZT (bf16 decay logits only)
        int n, h, b;
        unit_coords(u, n, h, b);
        mbar_arrive_expect_tx(bar_z, 16384u);
        for (int a = 0; a < 2; ++a) tma_load_4d(sm + P_ZT + a * 8192, &tz, bar_z, 64 * a, h, n * CH, b);
    };
    auto load_v = [&](int64_t u) {
        int n, h, b;
        unit_coords(u, n, h, b);
        mbar_arrive_expect_tx(bar_v, 16384u);
        for (int a = 0; a < 2; ++a) tma_load_4d(sm + P_VI + a * 8192, &tv, bar_v, 64 * a, h, n * CH, b);
    };

    // P1 and the per-channel tables of unit u: beta, G = in-chunk cumulative log-decay (rows past the
    // sequence end: no decay, beta 0), the block constants and e^{G_C}.  The decay input is z (the tile
    // at P_ZT, loaded one unit ahead, landed on bar_z with parity zpar) or the log-decay (read from
    // global memory, prefetched into L2 one unit ahead).  Beta is read from global memory here, its
    // load issued first and its value stored last (a load still in flight holds up the next barrier).
    // Run by the decay group, warps 4-11 (t = tid - 128, named barrier 3): for the first unit before
    // the loop, for every later one beside the previous unit's inverse.  Returns false if the z tile
    // never landed.
    constexpr int DT0 = 128, DTN = 256;
    auto load_beta = [&](int64_t u, int row) -> float {  // beta of row `row` of unit u; 0 past the end
        int n, h, b;
        unit_coords(u, n, h, b);
        const int t0 = n * CH;
        return (t0 + row < p.S) ? __bfloat162float(p.beta[((int64_t)b * p.S + t0 + row) * p.H + h]) : 0.f;
    };
    auto decay_tables = [&](int64_t u, uint32_t zpar) -> bool {
        int n, h, b;
        unit_coords(u, n, h, b);
        const int t = tid - DT0;
        const int t0 = n * CH, len = min(CH, p.S - t0);
        bool landed = true;
        const float beta_row = t < CH ? load_beta(u, t) : 0.f;
        {   // one thread per channel c and 32 rows (half hv); the half sums through a scratch
            const int c = t & 127, hv = t >> 7;
            float *qsum = reinterpret_cast<float *>(sm + P_XS);
            const int64_t i0 = (((int64_t)b * p.S + t0) * p.H + h) * DD + c, rstr = (int64_t)p.H * DD;
            // Rows past the end are computed (from a row inside, or the zero-filled tile rows) and then
            // multiplied by zero: no branch per element, so the 32 exponential chains overlap.
            float g[32];
            if (p.log_decay) {
#pragma unroll
                for (int rr = 0; rr < 32; ++rr) {
                    const int r = hv * 32 + rr;
                    const float lv = p.log_decay[i0 + (int64_t)min(r, len - 1) * rstr];
                    g[rr] = clamp_log_decay(lv, p.g_min) * (r < len ? 1.f : 0.f);
                }
            } else {
                if (!mbar_wait(bar_z, zpar)) landed = false;
                const uint8_t *zc = sm + P_ZT + (c >> 6) * 8192 + (c & 7) * 2;
                const uint32_t ch = (c & 63) >> 3;
#pragma unroll
                for (int rr = 0; rr < 32; ++rr) {
                    const int r = hv * 32 + rr;
                    const float zv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(zc + sw128(r, ch)));
                    g[rr] = log_alpha_fast(zv, p.g_min) * (r < len ? 1.f : 0.f);
                }
            }
            // the largest log(alpha) among this thread's rows (rows past the end, 0, only occur in the
            // sequence's last chunk, in the last segment, whose bound no map reads)
            float gm = g[0];
#pragma unroll
            for (int rr = 1; rr < 32; ++rr) gm = fmaxf(gm, g[rr]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, off));
            if ((t & 31) == 0) s_gmax_w[t >> 5] = gm;
            float acc = 0.f;
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) {
                acc += g[rr];
                g[rr] = acc;
            }
            qsum[hv * 128 + c] = acc;
            named_sync(3, DTN);
            if (t == 0) {
                float m = s_gmax_w[0];
#pragma unroll
                for (int w = 1; w < 8; ++w) m = fmaxf(m, s_gmax_w[w]);
                s_unit_gmax = m;  // read by this unit's readout, one iteration later
            }
            const float base = hv ? qsum[c] : 0.f;
#pragma unroll
            for (int rr = 0; rr < 32; ++rr) sG[(hv * 32 + rr) * SG_LD + c] = g[rr] + base;
        }
        named_sync(3, DTN);
        {  // per-channel block constants, two threads per channel, each two of the four parts
            const int c = t & 127;
            float bb[4], mm[4];
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                bb[R] = sG[(16 * R + 15) * SG_LD + c];
                mm[R] = sG[(16 * R + 7) * SG_LD + c];
            }
#pragma unroll
            for (int part = t >> 7; part < 4; part += 2) {
            if (part == 0) {
#pragma unroll
                for (int R = 0; R < 4; ++R) {
                    const float bm1 = R ? bb[R - 1] : 0.f;
                    tab[R * 128 + c] = bb[R];
                    tab[(4 + R) * 128 + c] = fexp(bm1 - mm[R]);
                    tab[(8 + R) * 128 + c] = fexp(bm1);
                }
            } else if (part == 1) {
#pragma unroll
                for (int R = 0; R < 4; ++R) tab[(12 + R) * 128 + c] = fexp(bb[3] - bb[R]);
                tab[tab_c(0, 0) * 128 + c] = fexp(mm[0] - bb[0]);
                sgam[c] = fexp(bb[3]);
            } else if (part == 2) {
#pragma unroll
                for (int R = 0; R <= 1; ++R) tab[tab_c(1, R) * 128 + c] = fexp(mm[1] - bb[R]);
#pragma unroll
                for (int R = 0; R <= 2; ++R) tab[tab_c(2, R) * 128 + c] = fexp(mm[2] - bb[R]);
            } else {
#pragma unroll
                for (int R = 0; R <= 3; ++R) tab[tab_c(3, R) * 128 + c] = fexp(mm[3] - bb[R]);
            }
            }
        }
        if (t < CH) sbeta[t] = beta_row;
        return landed;
    };

    if (tid == 0) {
        mbar_init(bar_in, 1);
        mbar_init(bar_am, 1);
        mbar_init(bar_wu, 1);
        mbar_init(bar_z, 1);
        mbar_init(bar_v, 1);
        fence_barrier_init();
        if ((int64_t)blockIdx.x < p.units) {
            load_qk(blockIdx.x);
            load_v(blockIdx.x);
            if (!p.log_decay) load_z(blockIdx.x);
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    if (warp >= 4 && warp < 12 && (int64_t)blockIdx.x < p.units) {  // the first unit's decay and tables
        ok = decay_tables(blockIdx.x, 0u);
    }

    int it = 0;
    for (int64_t u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++it) {
        int n, h, b;
        unit_coords(u, n, h, b);
        const int64_t u_next = u + gridDim.x;
        const uint32_t par = it & 1;
        if (u_next < p.units && tid < 256 && p.log_decay) {  // the next unit's log-decay input -> L2
            int n2, h2, b2;
            unit_coords(u_next, n2, h2, b2);
            const int64_t row0 = ((int64_t)b2 * p.S + n2 * CH) * p.H + h2;
            const int row = tid >> 2;
            if (p.log_decay && n2 * CH + row < p.S)
                prefetch_l2(p.log_decay + (row0 + (int64_t)row * p.H) * DD + (tid & 3) * 32);
        }
        // (this unit's decay and tables ran beside the previous unit's inverse)
        ok = mbar_wait(bar_in, par) && ok;
        ok = __syncthreads_and(ok);
        if (!ok) break;

        // ---------------- P2: decay-scaled operands.  A thread takes one row and 8 channels in block R0 =
        // warp % 4 and one in block 3 - R0, so that every warp writes 4 - R0 + 1 + R0 = 5 block versions
        // of the column operand (and no warp diverges on the version count).
        {
            const int R0 = warp & 3, jj = 2 * (warp >> 2) + (lane >> 4);
            float ke3s[2][8];  // k e^{b_R - G} of both items, for the column versions written last
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
                const int R = mi ? 3 - R0 : R0, r = 16 * R + (lane & 15);
                const float beta_r = sbeta[r];
                const int j = jj + 8 * mi, atom = mi, c0 = 8 * j;
                const uint32_t img = atom * 8192 + sw128(r, jj);
                const uint32_t bimg = P_B + atom * B_ATOM;
                float qv[8], kv[8], G[8], bR[8], bRm1[8], F[8], E[8], Dd[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + P_QI + img), qv);
                unpack8(*reinterpret_cast<const uint4 *>(sm + P_KI + img), kv);
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
                // fr = e^{G - m_R} (row factor), fg = e^G, ke3 = k e^{b_R - G} (column factors follow from
                // it by per-channel constants)
                float fr[8], fg[8], ke3[8], t[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float e1 = fexp(G[e] - bRm1[e]);
                    fr[e] = e1 * F[e];
                    fg[e] = e1 * E[e];
                    ke3[e] = kv[e] * fexp(bR[e] - G[e]);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = kv[e] * fr[e];
                *reinterpret_cast<uint4 *>(sm + bimg + sw128(r, jj)) = pack8(t);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = qv[e] * fr[e];
                {
                    const uint4 hi = pack8(t);
                    *reinterpret_cast<uint4 *>(sm + bimg + sw128(64 + r, jj)) = hi;
                    float hf[8], lo[8];
                    unpack8(hi, hf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) lo[e] = t[e] - hf[e];
                    *reinterpret_cast<uint4 *>(sm + bimg + sw128(128 + r, jj)) = pack8(lo);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) ke3s[mi][e] = ke3[e];
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = qv[e] * fg[e];
                *reinterpret_cast<uint4 *>(sm + P_QI + img) = pack8(t);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = ke3[e] * Dd[e];
                *reinterpret_cast<uint4 *>(sm + P_KI + img) = pack8(t);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = (beta_r * kv[e]) * fg[e];
                *reinterpret_cast<uint4 *>(sm + P_RH + img) = pack8(t);
            }
            // beta V last: the v tile is loaded after the previous unit's W/U MMAs and lands meanwhile
            if (!mbar_wait(bar_v, par)) ok = false;
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
                const int R = mi ? 3 - R0 : R0, r = 16 * R + (lane & 15);
                const uint32_t img = mi * 8192 + sw128(r, jj);
                const float beta_r = sbeta[r];
                float vv[8], t[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + P_VI + img), vv);
#pragma unroll
                for (int e = 0; e < 8; ++e) t[e] = beta_r * vv[e];
                *reinterpret_cast<uint4 *>(sm + P_VI + img) = pack8(t);
            }
            // the column versions go into the A operand's space, which the previous unit's bulk stores
            // (W, U^T and M^T images) read from: wait for those reads to finish first
            if (tid == 0) bulk_wait_read_all();
            __syncthreads();
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
                const int R = mi ? 3 - R0 : R0, r = 16 * R + (lane & 15);
                const int c0 = 8 * (jj + 8 * mi);
                const uint32_t aimg = P_A + mi * A_ATOM;
                for (int V = R; V < 4; ++V) {
                    float Cv[8], t[8];
                    load8f(tab + tab_c(V, R) * 128 + c0, Cv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = ke3s[mi][e] * Cv[e];
                    const uint4 hi = pack8(t);
                    *reinterpret_cast<uint4 *>(sm + aimg + sw128(kc_row0(V) + r, jj)) = hi;
                    if (V == R) {  // diagonal block: keep the rounding residue
                        float hf[8], lo[8];
                        unpack8(hi, hf);
#pragma unroll
                        for (int e = 0; e < 8; ++e) lo[e] = t[e] - hf[e];
                        *reinterpret_cast<uint4 *>(sm + aimg + sw128(A_KLO + r, jj)) = pack8(lo);
                    }
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        ok = __syncthreads_and(ok);
        if (!ok) break;

        uint8_t *rec = p.ws + ((size_t)(b * p.H + h) * p.Nc + n) * REC_BYTES;
        // ---------------- tcgen05: A^T (cols 0-63), M^T (64-127), residues of M's diagonal blocks (128-191);
        // meanwhile Q e^G, K e^{G_C - G} and e^{G_C} leave (thread 96; once the stores have read them,
        // during P3, the next unit's q and k tiles take their place: they are not operands of these MMAs)
        if (tid == 96 && in_bounds(rec, REC_BYTES, p.ws, p.rec_bytes, p.bounds)) {
            // Q e^G fills rows 64-127 of each atom of the stacked [W; Q e^G] image
            bulk_store(rec + REC_WQ + 8192, sm + P_QI, 8192);
            bulk_store(rec + REC_WQ + 16384 + 8192, sm + P_QI + 8192, 8192);
            bulk_store(rec + REC_KT, sm + P_KI, 16384);
            bulk_store(rec + REC_GAM, sgam, 512);
            bulk_commit();
        }
        if (tid == 0) {
            tc_fence_after();
            // all block versions at once: D1 = rows 0-127 of the A operand, D2 = rows 96-223 (version 3 and
            // the low part of the diagonal operand), each against [k rows | q rows | low q rows]; every
            // entry read afterwards pairs a row of version V with a column of block V
            constexpr uint32_t id = idesc_f16(128, 192, 0, 0);
            const uint64_t da = smem_desc(smem_u32(sm + P_A), 16, 1024, LAYOUT_SW128);
            const uint64_t db = smem_desc(smem_u32(sm + P_B), 16, 1024, LAYOUT_SW128);
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                const uint32_t ko = s8 >> 2, kb = (s8 & 3) * 32;
                mma_f16_ss(tmem, dadd(da, ko * A_ATOM + kb), dadd(db, ko * B_ATOM + kb), id, s8 > 0);
                mma_f16_ss(tmem + 192, dadd(da, ko * A_ATOM + 96 * 128 + kb), dadd(db, ko * B_ATOM + kb), id, s8 > 0);
            }
            mma_commit(bar_am);
        }
        ok = mbar_wait(bar_am, par);
        ok = __syncthreads_and(ok);
        tc_fence_after();
        if (!ok) break;
        if (tid == 0 && !p.log_decay && u_next < p.units) load_z(u_next);  // the A/M MMAs have read P_A
        if (tid == 96) {
            bulk_wait_read_all();
            if (u_next < p.units) load_qk(u_next);
        }

        // ---------------- P3: A (masked, beta-weighted, fp32) and the M^T image.
        // Lanes of D1 (warps 0-2) and D2 (warps 4-7) are rows of the A operand: version V, row i gives
        // A[r, i] and M[r, i] for r in block V; rows 160-223 (warps 6-7) give the low-part products for
        // the diagonal blocks, handed over through shared memory.
        {
            const int q4 = warp & 3;
            const uint32_t lq = (uint32_t)(32 * q4) << 16;
            float *lohi = reinterpret_cast<float *>(sm + P_LOHI);
            // the readout warps load their accumulator rows and write A first (neither needs the
            // low-part hand-off below); only the M^T image waits for it
            const bool rd = warp != 3 && warp < 6;
            const int prow = warp < 3 ? 32 * warp + lane : 96 + 32 * (warp - 4) + lane;
            const int V = prow < 16 ? 0 : (prow < 48 ? 1 : (prow < 96 ? 2 : 3));
            const int i = prow - kc_row0(V);
            const bool diag = (i >> 4) == V;
            uint32_t m_[16], r_[16];
            if (rd) {
                const uint32_t cb = tmem + lq + (warp < 3 ? 0u : 192u);
                // column block V differs between lanes of a warp: each warp's rows span at most two
                // versions, so load the block of every version present and select
                uint32_t a_[16];
                const int Vlo = (warp < 3 ? (32 * warp < 16 ? 0 : (32 * warp < 48 ? 1 : 2)) : 3);
                const int Vhi = (warp < 3 ? ((32 * warp + 31) < 16 ? 0 : ((32 * warp + 31) < 48 ? 1 : 2)) : 3);
                {
                    uint32_t x[16], y[16], z[16];
                    tmem_ld_32x32b_x16(cb + 16 * Vlo, x);
                    tmem_ld_32x32b_x16(cb + 64 + 16 * Vlo, y);
                    tmem_ld_32x32b_x16(cb + 128 + 16 * Vlo, z);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) { a_[e] = x[e]; m_[e] = y[e]; r_[e] = z[e]; }
                }
                if (Vhi != Vlo) {
                    uint32_t x[16], y[16], z[16];
                    tmem_ld_32x32b_x16(cb + 16 * Vhi, x);
                    tmem_ld_32x32b_x16(cb + 64 + 16 * Vhi, y);
                    tmem_ld_32x32b_x16(cb + 128 + 16 * Vhi, z);
                    tmem_wait_ld();
                    if (V == Vhi) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) { a_[e] = x[e]; m_[e] = y[e]; r_[e] = z[e]; }
                    }
                }
                float *sA = reinterpret_cast<float *>(sm + P_SA);
                float kk = 0.f;  // |k_i|^2: the diagonal entry (r = i), whose row and column factors cancel
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int r = 16 * V + e;
                    sA[r * SA_LD + i] = (i < r) ? sbeta[r] * __uint_as_float(a_[e]) : 0.f;
                    if (r == i) kk = __uint_as_float(a_[e]);
                }
                if (diag) s_bk[i] = sbeta[i] * kk;  // beta_i |k_i|^2, for the chunk's log-bound
            }
            if (warp == 6 || warp == 7) {  // low part of the diagonal column operand x q: row i, block R = i / 16
                const int il = 32 * (warp - 6) + lane, R = il >> 4;
                uint32_t v[16];
                // lanes of one warp span two blocks: load both candidate column blocks, keep the own one
                uint32_t w0[16], w1[16];
                tmem_ld_32x32b_x16(tmem + lq + 192 + 64 + 32 * (warp - 6), w0);
                tmem_ld_32x32b_x16(tmem + lq + 192 + 64 + 32 * (warp - 6) + 16, w1);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = (R & 1) ? w1[e] : w0[e];
#pragma unroll
                for (int e = 0; e < 16; e += 4)
                    *reinterpret_cast<float4 *>(lohi + il * 16 + e) =
                        make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                                    __uint_as_float(v[e + 3]));
            }
            __syncthreads();
            if (rd) {
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    float t[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int ee = 8 * hc + e, r = 16 * V + ee;
                        // hi(k) lo(q) for every block; lo(k) hi(q) on the diagonal block
                        float v = __uint_as_float(m_[ee]) + __uint_as_float(r_[ee]);
                        if (diag) v += lohi[i * 16 + ee];
                        t[e] = (i <= r) ? v : 0.f;
                    }
                    *reinterpret_cast<uint4 *>(sm + P_MT + sw128(i, 2 * V + hc)) = pack8(t);
                }
                if (diag)  // columns of earlier blocks: masked (i > r)
                    for (int cc = 0; cc < 2 * V; ++cc)
                        *reinterpret_cast<uint4 *>(sm + P_MT + sw128(i, cc)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        const float gmax_u = s_unit_gmax;  // (this unit's: the next unit's decay rewrites it only below)
        tc_fence_before();
        __syncthreads();
        if (warp == 12 && p.lbound) {  // (idle in P4) the chunk's log-bound: len tokens of at most gmax_u, and
                                       // each token's log max(1, |1 - beta |k|^2|), |k|^2 widened by 2^-7 (bf16)
            float lf = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const float bk = s_bk[lane + 32 * k2];
                lf += __logf(fmaxf(1.f, fmaxf(fabsf(1.f - bk * (1.f - 0.0078125f)), fabsf(1.f - bk * (1.f + 0.0078125f)))));
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) lf += __shfl_xor_sync(0xffffffffu, lf, off);
            if (lane == 0) p.lbound[((size_t)b * p.H + h) * p.Nc + n] = (float)min(CH, p.S - n * CH) * gmax_u + lf;
        }

        // ---------------- P4: T = (I + A)^{-1} (fp32) by block doubling: the four diagonal 16x16 blocks by
        // forward substitution, then T_{R,R-1} = -T_RR A_{R,R-1} T_{R-1,R-1} for R = 1, 3, then the lower-left
        // 32x32 block the same way from the two diagonal 32x32 blocks.  Blocks above the diagonal are written
        // as zeros where a later product reads them; the T image zero-fills the upper-right 32x32 block.
        // Warps 0-3 only (named barrier 1); warps 4-11 meanwhile compute the next unit's decay and tables.
        if (warp < 4) {
            invert_unit_lower64(reinterpret_cast<const float *>(sm + P_SA), reinterpret_cast<float *>(sm + P_ST),
                                reinterpret_cast<float *>(sm + P_IX), sm + P_TI, tid);
        } else if (warp < 12 && u_next < p.units) {
            ok = decay_tables(u_next, (uint32_t)(it + 1) & 1u) && ok;
        }
        tc_fence_before();
        ok = __syncthreads_and(ok);
        if (!ok) break;

        // ---------------- tcgen05: W = T (beta K e^G)            (M=64, N=128, K=64: A = T, B MN-major)
        //                   U^T = (beta V)^T T^T              (M=128, N=64, K=64: A MN-major, B = T K-major)
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idw = idesc_f16(64, 128, 0, 1);
            constexpr uint32_t idu = idesc_f16(128, 64, 1, 0);
            const uint64_t ti = smem_desc(smem_u32(sm + P_TI), 16, 1024, LAYOUT_SW128);
            const uint64_t rw = smem_desc(smem_u32(sm + P_RH), 8192, 1024, LAYOUT_SW128);
            const uint64_t vt = smem_desc(smem_u32(sm + P_VI), 8192, 1024, LAYOUT_SW128);
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
        if (tid == 0 && u_next < p.units) load_v(u_next);  // beta K e^G and beta V have been consumed

        // ---------------- P5: -W image (warp groups 0 and 2: M = 64 accumulator rows, half the columns
        // each) and U^T image (warp groups 1 and 3: one value column j per lane, half the rows each)
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
                            *reinterpret_cast<uint4 *>(sm + P_WI + (j >> 3) * 8192 + sw128(r, j & 7)) = pack8(t);
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
                    *reinterpret_cast<uint4 *>(sm + P_UI + sw128(jv, 4 * (wg >> 1) + g)) = pack8(t);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && in_bounds(rec, REC_BYTES, p.ws, p.rec_bytes, p.bounds)) {
            bulk_store(rec + REC_WQ, sm + P_WI, 8192);
            bulk_store(rec + REC_WQ + 16384, sm + P_WI + 8192, 8192);
            bulk_store(rec + REC_MT, sm + P_MT, 8192);
            bulk_store(rec + REC_U, sm + P_UI, 16384);
            bulk_commit();
        }
    }

    if (tid == 0 || tid == 96) bulk_wait_all();
    if (tid == 0 && !ok) report_timeout(p.timeouts, p.dev_status);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ================================================================ K2b: chunk_state_kernel
// One CTA per (head, batch, segment) walks the chunks in order.  The state is
// kept transposed in TMEM: lane j (value column) holds S[:, j] in fp32, so
// every per-chunk product takes its A operand straight from TMEM and the
// register work of the chain is spread over all 128 lanes.  Warp roles:
//   warps 0-7   the chain's register work (lane quarter = warp % 4, column
//               half = warp / 4);
//   warp 8      issues the chain's MMAs and the record copies (one thread);
//   warps 9-12  the output stage; its
//               first thread issues the output's transposition MMA itself, so
//               the output never waits on the chain's MMA issue order.
// Per chunk n:
//   chain warps:  S^T -> bf16 copy in TMEM; S^T <- S^T Diag(e^{G_C})
//   MMA:          PO  = S^T [-W; Q e^G]^T        PO[j, r] = -(W S)[r, j],  PO[j, 64 + r] = (Q e^G S)[r, j]
//   chain warps:  V'^T = U^T + PO[:, 0:64] -> bf16 copy in TMEM
//   MMA:          S^T += V'^T K~,  PO[:, 64:128] += V'^T M^T      (= O^T of chunk n)
// and, off the chain's critical path, the output warps write O^T (bf16) as an
// operand image, one MMA with [I; I] turns it back into token rows (into the
// same PO buffer; lanes 64-127 repeat lanes 0-63), and the output warps, 32
// rows x 64 columns each, apply the RMS normalisation over the head and the
// sigmoid of the output-gate logits (a bf16 tile loaded by TMA one chunk
// ahead) and store the tile with a TMA tensor store.  PO is double-buffered;
// a buffer is reused for chunk n + 2 once the output warps have read chunk n.
// Records stream in by bulk copies, two stages deep.
struct StateArgs {
    int S, H, Nc;
    int L, G;              // chunks per segment, segments per sequence
    const uint8_t *ws;
    bool gated;            // apply RMSNorm and sigmoid(gate logits) (tensor map tgl); else write o~
    const float *S0;
    float *Sf;
    const float *seg_init; // state entering segment g >= 1, [B*H][G][128][128] (after the combine pass)
    uint8_t *xt;           // map pass: A_g^T as bf16 operand images [B*H][G-1][32 KB]
    float *yt;             // map pass: Y_g [B*H][G-1][128][128]
    size_t sf_bytes, xt_bytes, yt_bytes;  // sizes of Sf, xt, yt (checked builds test the writes against them)
    const float *lbound;   // map pass: per-chunk log-bounds of the transition norm [B*H][Nc], or null
    unsigned int *bounds;
    float eps;
    unsigned int *timeouts;
    int *dev_status;
};

constexpr int ST_THREADS_MAP = 288;            // warps 0-7 chain register work, warp 8 MMA + copies
constexpr int ST_THREADS_CHAIN = 416;          // ... and warps 9-12 the output stage
constexpr int ST_OUT_WARP0 = 9;
constexpr uint32_t ST_STAGE = REC_GAM;         // the image part of a record (73728 B)
constexpr uint32_t ST_GAM = 2 * ST_STAGE;      // e^{G_C} [2 stages][128] fp32 (the map pass: 3, into OIMG)
constexpr uint32_t ST_OIMG = ST_GAM + 1024;    // output tile [2 atoms (j / 64)][64 rows r][128 B]
constexpr uint32_t ST_SIGT = ST_OIMG + 16384;  // output-gate logits tile (TMA), same layout, bf16
constexpr uint32_t ST_OT = ST_SIGT + 16384;    // O^T image, K-major B [128 rows j][128 B: 64 r]
constexpr uint32_t ST_ID = ST_OT + 16384;      // [I_64; I_64], K-major A [128 rows][128 B: 64 k]
constexpr uint32_t ST_RED = ST_ID + 16384;     // per-row partial sums of squares [64][2] fp32
constexpr uint32_t ST_BAR = ST_RED + 1024;     // mbarriers + TMEM slot
constexpr uint32_t ST_END = ST_BAR + 128;
constexpr size_t STATE_SMEM = ST_END + 1024;
static_assert(STATE_SMEM <= 232448, "state kernel shared memory");
// TMEM columns
constexpr uint32_t T_S32 = 0;     // S^T fp32 [j][c]
constexpr uint32_t T_S16 = 128;   // S^T bf16 pairs (A operand, K = c)
constexpr uint32_t T_PO = 192;    // two [128][128] accumulators
constexpr uint32_t T_V16 = 448;   // V'^T bf16 pairs (A operand, K = r)
constexpr uint32_t ST_TCOLS = 512;

// sigmoid(x) = (1 + tanh(x / 2)) / 2 with the hardware tanh approximation (|error| < 2^-11 of the result)
__device__ __forceinline__ float sigmoid_fast(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}

// The chain over segment blockIdx.z from its entering state, with outputs.
__global__ void __launch_bounds__(ST_THREADS_CHAIN, 1)
chunk_state_kernel(const __grid_constant__ CUtensorMap tmo, const __grid_constant__ CUtensorMap tgl, StateArgs p) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, hf = (warp >> 2) & 1;  // TMEM lane quarter, column half (warps 0-7)
    const int h = blockIdx.x, b = blockIdx.y;
    const int bh = b * p.H + h;
    const int g = (int)blockIdx.z;
    const int n0 = g * p.L;
    const int nc = max(0, min(p.L, p.Nc - n0));  // chunks of this segment
    // Record stages: whole records, two deep; the e^{G_C} of each stage sits after the stages.
    constexpr int STG = 2;
    constexpr uint32_t STB = ST_STAGE;
    constexpr uint32_t O_W_ATOM = 16384u;  // atom stride of the [-W; Q e^G] B operand
    constexpr uint32_t O_KT = REC_KT;
    constexpr uint32_t O_U = REC_U;
    static_assert(STG * STB == ST_GAM, "record stages end where e^{G_C} starts");
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ST_BAR);
    uint64_t *full = bars;           // [STG] record stage landed
    uint64_t *bar_p = bars + 3;      // PO group done
    uint64_t *bar_s = bars + 4;      // S^T += V'^T K~ done (and every earlier group)
    uint64_t *bar_o = bars + 5;      // PO += V'^T M^T done, [2] by PO buffer (slots 5 and 13): chunk n on
                                     // bar_o[n & 1] phase n >> 1, so the output warps, which may trail the
                                     // chain by a chunk, never see a barrier two phases ahead
    uint64_t *bar_t = bars + 6;      // transposition of O done
    uint64_t *bar_simg = bars + 7;   // bf16 copy of S^T written (8 chain warps)
    uint64_t *bar_vimg = bars + 8;   // bf16 copy of V'^T written (8 chain warps)
    uint64_t *bar_ot = bars + 9;     // O^T image written (4 output warps)
    uint64_t *bar_sig = bars + 10;   // gate-logits tile landed
    uint64_t *pofree = bars + 11;    // [2] PO buffer read by the output warps (4 output warps)
    uint64_t *bar_o1 = bars + 13;
    auto bar_of = [&](int n) { return (n & 1) ? bar_o1 : bar_o; };
    auto par_of = [](int n) { return (uint32_t)((n >> 1) & 1); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 14);
    float *sgam = reinterpret_cast<float *>(sm + ST_GAM);
    float *red = reinterpret_cast<float *>(sm + ST_RED);
    const uint8_t *rec0 = p.ws + ((size_t)bh * p.Nc + n0) * REC_BYTES;
    __shared__ volatile int s_fail;

    if (tid == 0) {
        s_fail = 0;
        for (int i = 0; i < 7; ++i) mbar_init(&bars[i], 1);
        mbar_init(bar_simg, 8);
        mbar_init(bar_vimg, 8);
        mbar_init(bar_ot, 4);
        mbar_init(bar_sig, 1);
        mbar_init(&pofree[0], 4);
        mbar_init(&pofree[1], 4);
        mbar_init(bar_o1, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, ST_TCOLS);
        tmem_relinquish();
    }
    for (int e = tid; e < 128 * 8; e += blockDim.x) {  // [I_64; I_64]
        const int row = e >> 3, ch = e & 7;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (((row & 63) >> 3) == ch) reinterpret_cast<uint16_t *>(&v)[row & 7] = 0x3F80;  // bf16 1.0
        *reinterpret_cast<uint4 *>(sm + ST_ID + sw128(row, ch)) = v;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    int issued = 0, landed = 0;  // records requested / seen complete (MMA warp)

    if (warp == 8) {
        // ======================================== MMA and copy issue (one thread)
        if (lane == 0) {
            constexpr uint32_t id_kk = idesc_f16(128, 128, 0, 0);  // A, B K-major (A may be in TMEM)
            constexpr uint32_t id_s = idesc_f16(128, 128, 0, 1);   // B MN-major
            constexpr uint32_t id_o = idesc_f16(128, 64, 0, 1);    // B MN-major
            const uint64_t d_k = smem_desc(smem_u32(sm), 16, 1024, LAYOUT_SW128);     // K-major images
            const uint64_t d_mn = smem_desc(smem_u32(sm), 8192, 1024, LAYOUT_SW128);  // K~ and M^T images
            auto issue_record = [&](int n) {
                const int stg = n % STG;
                uint8_t *dst = sm + stg * STB;
                const uint8_t *src = rec0 + (size_t)n * REC_BYTES;
                mbar_arrive_expect_tx(&full[stg], STB + 512);
                bulk_load(dst, src, ST_STAGE, &full[stg]);
                bulk_load(sgam + stg * 128, src + REC_GAM, 512, &full[stg]);
                ++issued;
            };
            for (int n = 0; n < STG && n < nc; ++n) issue_record(n);
            int n = 0;
            for (; n < nc; ++n) {
                if (s_fail) { ok = false; break; }
                const uint32_t sgo = (n % STG) * STB;
                const uint32_t po = tmem + T_PO + (uint32_t)(n & 1) * 128;
                if (!mbar_wait(&full[n % STG], (n / STG) & 1)) { ok = false; break; }
                landed = n + 1;
                // PO = S_n^T [-W; Q e^G]^T, once the output warps have read chunk n - 2
                if (!mbar_wait(bar_simg, n & 1)) { ok = false; break; }
                if (n >= 2 && !mbar_wait(&pofree[n & 1], ((n - 2) >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8) {
                    const uint32_t ko = s8 >> 2, kb = (s8 & 3) * 32;
                    mma_f16_ts(po, tmem + T_S16 + 8 * s8, dadd(d_k, sgo + ko * O_W_ATOM + kb), id_kk, s8 > 0);
                }
                mma_commit(bar_p);
                // the stage of record n - 1 is free once its last group is done: refill it, STG - 1 ahead
                if (n >= 1 && n + STG - 1 < nc) {
                    if (!mbar_wait(bar_of(n - 1), par_of(n - 1))) { ok = false; break; }
                    issue_record(n + STG - 1);
                }
                // S^T += V'^T K~, then PO[:, 64:] += V'^T M^T
                if (!mbar_wait(bar_vimg, n & 1)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4)
                    mma_f16_ts(tmem + T_S32, tmem + T_V16 + 8 * s4, dadd(d_mn, sgo + O_KT + s4 * 2048), id_s, 1);
                mma_commit(bar_s);
#pragma unroll
                for (int s4 = 0; s4 < 4; ++s4)
                    mma_f16_ts(po + 64, tmem + T_V16 + 8 * s4, dadd(d_mn, sgo + REC_MT + s4 * 2048), id_o, 1);
                mma_commit(bar_of(n));
            }
            if (!ok) s_fail = 1;
        }
    } else if (warp >= ST_OUT_WARP0) {
        // ======================================== output stage (warps 9-12, chains only)
        const int otid = tid - ST_OUT_WARP0 * 32;
        const int oq = warp & 3;               // TMEM lane quarter of this warp
        const uint32_t olane = (uint32_t)(32 * oq) << 16;
        const int j = 32 * oq + lane;          // value column (O^T image row) of this thread
        const int r = 32 * (oq & 1) + lane;    // token row (lanes 64-127 repeat lanes 0-63)
        const int cq2 = oq >> 1;               // value columns 64 cq2 .. 64 cq2 + 63
        auto load_sig = [&](int m) {           // gate-logits tile of chunk m -> shared memory
            if (otid == 0 && p.gated && m < nc) {
                mbar_arrive_expect_tx(bar_sig, GATE_TILE_BYTES);
                tma_load_4d(sm + ST_SIGT, &tgl, bar_sig, 0, h, (n0 + m) * CH, b);
                tma_load_4d(sm + ST_SIGT + 8192, &tgl, bar_sig, 64, h, (n0 + m) * CH, b);
            }
        };
        load_sig(0);
        for (int m = 0; m < nc; ++m) {
            if (s_fail) { ok = false; break; }
            const uint32_t pob = tmem + olane + T_PO + (uint32_t)(m & 1) * 128;
            // O^T of chunk m (PO[m & 1][j, 64 + r]) -> bf16 operand image
            if (!mbar_wait(bar_of(m), par_of(m))) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t ov[32];
                tmem_ld_32x32b_x32(pob + 64 + 32 * hh, ov);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(ov[8 * k + e]);
                    *reinterpret_cast<uint4 *>(sm + ST_OT + sw128(j, 4 * hh + k)) = pack8(f);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_ot);
            // O of chunk m back to token rows, PO[m & 1][r, j] = sum_k [I; I][r, k] O^T[j, k], issued by
            // this group's first thread (its commit tracks only its own MMAs)
            if (otid == 0) {
                if (mbar_wait(bar_ot, m & 1)) {
                    tc_fence_after();
                    constexpr uint32_t id_t = idesc_f16(128, 128, 0, 0);
                    const uint64_t d_k = smem_desc(smem_u32(sm), 16, 1024, LAYOUT_SW128);
                    const uint32_t d = tmem + T_PO + (uint32_t)(m & 1) * 128;
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4)
                        mma_f16_ss(d, dadd(d_k, ST_ID + s4 * 32), dadd(d_k, ST_OT + s4 * 32), id_t, s4 > 0);
                    mma_commit(bar_t);
                } else {
                    s_fail = 1;
                }
            }
            // token rows of chunk m (after the [I; I] transposition) -> normalised, gated output tile
            if (!mbar_wait(bar_t, m & 1)) { ok = false; break; }
            tc_fence_after();
            uint32_t ov[64];
            tmem_ld_32x32b_x32(pob + 64 * cq2, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
            tmem_ld_32x32b_x32(pob + 64 * cq2 + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pofree[m & 1]);  // this PO buffer may take chunk m + 2
            if (p.gated) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 64; ++e) ss = fmaf(__uint_as_float(ov[e]), __uint_as_float(ov[e]), ss);
                red[r * 2 + cq2] = ss;
            }
            if (otid == 0) bulk_wait_read_all();  // the previous tile's store has left shared memory
            named_sync(2, 128);
            float inv = 1.f;
            if (p.gated) {
                inv = rsqrtf((red[r * 2] + red[r * 2 + 1]) * (1.0f / 128.0f) + p.eps);
                if (!mbar_wait(bar_sig, m & 1)) ok = false;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = cq2 * 8192 + sw128(r, k);
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(ov[8 * k + e]);
                if (p.gated) {  // RMSNorm, then the sigmoid of the gate logits
                    float gl[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sm + ST_SIGT + off), gl);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] *= inv * sigmoid_fast(gl[e]);
                }
                *reinterpret_cast<uint4 *>(sm + ST_OIMG + off) = pack8(f);
            }
            fence_proxy_async_smem();
            named_sync(2, 128);
            if (otid == 0) {  // rows past the end of the sequence are clipped by the tensor map
                tma_store_4d(&tmo, sm + ST_OIMG, 0, h, (n0 + m) * CH, b);
                tma_store_4d(&tmo, sm + ST_OIMG + 8192, 64, h, (n0 + m) * CH, b);
                bulk_commit();
            }
            load_sig(m + 1);  // every reader of the gate tile is past the barrier above
            if (!ok) break;
        }
        if (!ok) s_fail = 1;
        if (otid == 0) bulk_wait_all();
    } else {
        // ======================================== chain register work (warps 0-7)
        const uint32_t lrow = (uint32_t)(32 * q4) << 16;
        const int j = 32 * q4 + lane;  // value column (TMEM lane) of this thread
        {   // entering state -> TMEM (S^T[j, c] = S[c, j]: a warp reads 128 contiguous bytes per c)
            const float *s_in = (g == 0) ? (p.S0 ? p.S0 + (size_t)bh * DD * DD : nullptr)
                              : (g == 1) ? p.yt + (size_t)bh * (p.G - 1) * DD * DD  // S_1: segment 0's end state
                                         : p.seg_init + ((size_t)bh * p.G + g) * DD * DD;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t su[32];
                if (s_in) {
                    const float *src = s_in + (size_t)(64 * hf + 32 * hh) * DD + j;
#pragma unroll
                    for (int e = 0; e < 32; ++e) su[e] = __float_as_uint(src[(size_t)e * DD]);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) su[e] = 0u;
                }
                tmem_st_32x32b_x32(tmem + lrow + T_S32 + 64 * hf + 32 * hh, su);
            }
            tmem_wait_st();
        }

        for (int n = 0; n < nc; ++n) {
            if (s_fail) { ok = false; break; }
            const uint32_t po = tmem + lrow + T_PO + (uint32_t)(n & 1) * 128;
            // ---------- S_n^T (after the previous chunk's update) -> bf16 copy; S^T <- S^T Diag(e^{G_C})
            if (n >= 1 && !mbar_wait(bar_s, (n - 1) & 1)) { ok = false; break; }
            if (!mbar_wait(&full[n % STG], (n / STG) & 1)) { ok = false; break; }
            tc_fence_after();
            {   // the bf16 copy goes out first (the PO MMA waits for it); the decay is applied after
                const float4 *g4 = reinterpret_cast<const float4 *>(sgam + (n % STG) * 128 + 64 * hf);
                uint32_t sv[64];
                tmem_ld_32x32b_x32(tmem + lrow + T_S32 + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld_32x32b_x32(tmem + lrow + T_S32 + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_wait_ld();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(sv[32 * hh + 2 * e]), __uint_as_float(sv[32 * hh + 2 * e + 1]));
                    tmem_st_32x32b_x16(tmem + lrow + T_S16 + 32 * hf + 16 * hh, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_simg);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float4 gg = g4[e];
                    sv[4 * e] = __float_as_uint(__uint_as_float(sv[4 * e]) * gg.x);
                    sv[4 * e + 1] = __float_as_uint(__uint_as_float(sv[4 * e + 1]) * gg.y);
                    sv[4 * e + 2] = __float_as_uint(__uint_as_float(sv[4 * e + 2]) * gg.z);
                    sv[4 * e + 3] = __float_as_uint(__uint_as_float(sv[4 * e + 3]) * gg.w);
                }
                tmem_st_32x32b_x32(tmem + lrow + T_S32 + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_st_32x32b_x32(tmem + lrow + T_S32 + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_wait_st();
            }
            // ---------- V'^T = U^T - (W S_n)^T -> bf16 copy in TMEM
            {
                const uint8_t *ut = sm + (n % STG) * STB + O_U;
                uint4 uu[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) uu[k] = *reinterpret_cast<const uint4 *>(ut + sw128(j, 4 * hf + k));
                if (!mbar_wait(bar_p, n & 1)) { ok = false; break; }
                tc_fence_after();
                uint32_t pv[32], pk[16];
                tmem_ld_32x32b_x32(po + 32 * hf, pv);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float u[8];
                    unpack8(uu[k], u);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        pk[4 * k + e] = pack_bf16x2(u[2 * e] + __uint_as_float(pv[8 * k + 2 * e]),
                                                    u[2 * e + 1] + __uint_as_float(pv[8 * k + 2 * e + 1]));
                }
                tmem_st_32x32b_x16(tmem + lrow + T_V16 + 16 * hf, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_vimg);
        }
        if (ok && nc > 0) {
            if (!mbar_wait(bar_s, (nc - 1) & 1) || !mbar_wait(bar_of(nc - 1), par_of(nc - 1))) ok = false;
            tc_fence_after();
        }
        if (ok && p.Sf && g == p.G - 1 &&  // (with no chunks TMEM still holds the entering state)
            in_bounds(p.Sf + (size_t)bh * DD * DD, DD * DD * 4, p.Sf, p.sf_bytes, p.bounds)) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t sv[32];
                tmem_ld_32x32b_x32(tmem + lrow + T_S32 + 64 * hf + 32 * hh, sv);
                tmem_wait_ld();
                float *dst = p.Sf + (size_t)bh * DD * DD + (size_t)(64 * hf + 32 * hh) * DD + j;
#pragma unroll
                for (int e = 0; e < 32; ++e) dst[(size_t)e * DD] = __uint_as_float(sv[e]);
            }
        }
        if (!ok) s_fail = 1;
    }
    __syncthreads();
    if (warp == 8 && lane == 0 && s_fail) {
        report_timeout(p.timeouts, p.dev_status);
        // let the bulk copies already issued land before the CTA exits
        for (int m = landed; m < issued; ++m) mbar_wait(&full[m % STG], (m / STG) & 1, 100000000ull);
    }
    if (tid == ST_OUT_WARP0 * 32 && s_fail && p.gated)
        mbar_wait(bar_sig, 0, 100000000ull), mbar_wait(bar_sig, 1, 100000000ull);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, ST_TCOLS);
}

// ================================================================ K2b': chunk_map_pair_kernel
// The map pass, two chains per CTA (H, B, G - 1 CTAs; blockIdx.z = segment g <= G - 2).  Chain Y runs
// segment g with U from its entering state: the initial state for g = 0 (its end state is S_1, the
// entering state of segment 1), zero for g >= 1 (its end state is Y_g).  Chain X runs segment g from the
// identity without U (its end state is A_g; segment 0 needs none, and its slot stays unused).  Both read
// one stream of records (-W, K~, U^T, e^{G_C}), three stages deep.  The chain warps alternate between
// the two chains, so that each chain's register work fills the other's MMA round trips.  Per chain the
// TMEM columns are S^T fp32 (+0), the bf16 copy of S^T (+128) and PO = S^T (-W)^T (+192); the bf16 V'^T
// reuses the copy's first 32 columns (the copy is dead once PO is done, V'^T once the update is done).
//
// Windows.  Each token's transition S -> (I - beta k k^T) Diag(alpha) S has spectral norm at most
// max_c alpha_c max(1, |1 - beta |k|^2|), so the segment's linear part A_g and everything before a chunk
// reach the end state scaled by at most the product of those bounds over the chunks that follow.  The
// prep leaves each chunk's log-bound in p.lbound.  When the bounds of the segment's last chunks [nb, nc)
// add up below -WINDOW_LOG (e^-200: below the smallest fp32 number even for states of 1e38), A_g is zero
// to fp32 and Y_g is the chain over [nb, nc) alone, from zero: chain X is skipped (A_g's image written as
// zeros) and chain Y runs from chunk nb.  Otherwise (slow decay) both chains run the whole segment.
constexpr float WINDOW_LOG = 200.f;
__device__ __forceinline__ constexpr uint32_t mp_base(int c) { return c ? 256u : 0u; }  // chain X, chain Y
constexpr uint32_t MP_S16 = 128, MP_PO = 192;

__global__ void __launch_bounds__(ST_THREADS_MAP, 1) chunk_map_pair_kernel(StateArgs p) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, hf = (warp >> 2) & 1;  // TMEM lane quarter, column half (warps 0-7)
    const int h = blockIdx.x, b = blockIdx.y, g = (int)blockIdx.z;
    const int bh = b * p.H + h;
    const int n0 = g * p.L;
    const int nc = max(0, min(p.L, p.Nc - n0));
    constexpr int STG = 3;
    constexpr uint32_t STB = 49152u;  // -W rows of both atoms (16 KB), K~ (16 KB), U^T (16 KB)
    constexpr uint32_t O_KT = 16384u, O_U = 32768u;
    static_assert(STG * STB == ST_GAM, "record stages end where e^{G_C} starts");
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ST_BAR);
    uint64_t *full = bars;       // [3] record stage landed
    uint64_t *bar_p = bars + 3;  // [2] PO of chain c done
    uint64_t *bar_s = bars + 5;  // [2] S^T += V'^T K~ of chain c done
    uint64_t *simg = bars + 7;   // [2] bf16 copy of chain c's S^T written (8 chain warps)
    uint64_t *vimg = bars + 9;   // [2] bf16 copy of chain c's V'^T written (8 chain warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 11);
    float *sgam = reinterpret_cast<float *>(sm + ST_GAM);
    const uint8_t *rec0 = p.ws + ((size_t)bh * p.Nc + n0) * REC_BYTES;
    __shared__ volatile int s_fail;
    __shared__ int s_nb, s_win;  // first chunk the chains run (within the segment); whether it is a window

    if (tid == 0) {
        s_fail = 0;
        for (int i = 0; i < 7; ++i) mbar_init(&bars[i], 1);
        for (int i = 7; i < 11; ++i) mbar_init(&bars[i], 8);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, ST_TCOLS);
        tmem_relinquish();
        // the shortest suffix [nb, nc) whose log-bounds add up below -WINDOW_LOG: lane l of a pass takes
        // chunk top - 1 - l, so a prefix over lanes plus the later passes' sum is a suffix sum
        int nb = -1;
        if (p.lbound) {
            const float *lb = p.lbound + (size_t)bh * p.Nc + n0;
            float carry = 0.f;
            for (int top = nc; top > 0 && nb < 0; top -= 32) {
                const int idx = top - 1 - lane;
                float v = idx >= 0 ? lb[idx] : 0.f;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, v, off);
                    if (lane >= off) v += y;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, idx >= 0 && carry + v < -WINDOW_LOG);
                if (hit) nb = top - 1 - (__ffs(hit) - 1);
                carry += __shfl_sync(0xffffffffu, v, 31);
            }
        }
        if (lane == 0) {
            s_win = nb >= 0;
            s_nb = nb >= 0 ? nb : 0;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool windowed = s_win != 0;
    const int nb = s_nb, nrun = nc - nb;  // chunks the chains run: nb .. nc - 1
    const int c0 = windowed ? 1 : 0;      // first chain that runs (chain X only without a window)
    bool ok = true;
    int issued = 0, landed = 0;  // records requested / seen complete (MMA warp)

    if (warp == 8) {
        // ======================================== MMA and copy issue (one thread)
        if (lane == 0) {
            constexpr uint32_t id_po = idesc_f16(128, 64, 0, 0);  // A (TMEM) and B K-major
            constexpr uint32_t id_s = idesc_f16(128, 128, 0, 1);  // B MN-major
            const uint64_t d_k = smem_desc(smem_u32(sm), 16, 1024, LAYOUT_SW128);
            const uint64_t d_mn = smem_desc(smem_u32(sm), 8192, 1024, LAYOUT_SW128);
            // (m counts the chunks run, from chunk nb: stages and barrier phases follow m)
            auto issue_record = [&](int m) {
                const int stg = m % STG;
                uint8_t *dst = sm + stg * STB;
                const uint8_t *src = rec0 + (size_t)(nb + m) * REC_BYTES;
                mbar_arrive_expect_tx(&full[stg], STB + 512);
                bulk_load(dst, src + REC_WQ, 8192, &full[stg]);
                bulk_load(dst + 8192, src + REC_WQ + 16384, 8192, &full[stg]);
                bulk_load(dst + O_KT, src + REC_KT, 16384, &full[stg]);
                bulk_load(dst + O_U, src + REC_U, 16384, &full[stg]);
                bulk_load(sgam + stg * 128, src + REC_GAM, 512, &full[stg]);
                ++issued;
            };
            for (int m = 0; m < STG && m < nrun; ++m) issue_record(m);
            for (int m = 0; m < nrun; ++m) {
                if (s_fail) { ok = false; break; }
                const uint32_t sgo = (m % STG) * STB;
                if (!mbar_wait(&full[m % STG], (m / STG) & 1)) { ok = false; break; }
                landed = m + 1;
#pragma unroll
                for (int c = c0; c < 2; ++c) {  // PO_c = S_c^T (-W)^T
                    if (!mbar_wait(&simg[c], m & 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t base = tmem + mp_base(c);
#pragma unroll
                    for (int s8 = 0; s8 < 8; ++s8) {
                        const uint32_t ko = s8 >> 2, kb = (s8 & 3) * 32;
                        mma_f16_ts(base + MP_PO, base + MP_S16 + 8 * s8, dadd(d_k, sgo + ko * 8192 + kb), id_po, s8 > 0);
                    }
                    mma_commit(&bar_p[c]);
                }
                if (!ok) break;
                // the stage of record m - 1 is free once chain Y's update of it is done (the chain warps
                // read its U^T and e^{G_C} before they signal that update's V')
                if (m >= 1 && m + STG - 1 < nrun) {
                    if (!mbar_wait(&bar_s[1], (m - 1) & 1)) { ok = false; break; }
                    issue_record(m + STG - 1);
                }
#pragma unroll
                for (int c = c0; c < 2; ++c) {  // S_c^T += V'_c^T K~
                    if (!mbar_wait(&vimg[c], m & 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t base = tmem + mp_base(c);
#pragma unroll
                    for (int s4 = 0; s4 < 4; ++s4)
                        mma_f16_ts(base, base + MP_S16 + 8 * s4, dadd(d_mn, sgo + O_KT + s4 * 2048), id_s, 1);
                    mma_commit(&bar_s[c]);
                }
                if (!ok) break;
            }
            if (!ok) s_fail = 1;
        }
    } else {
        // ======================================== chain register work (warps 0-7), both chains
        const uint32_t lrow = (uint32_t)(32 * q4) << 16;
        const int j = 32 * q4 + lane;  // value column (TMEM lane) of this thread
        {   // entering states -> TMEM: X = identity, Y = S_0 (segment 0 without a window) or zero
            const float *s_in = (g == 0 && p.S0 && !windowed) ? p.S0 + (size_t)bh * DD * DD : nullptr;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t su[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) su[e] = (64 * hf + 32 * hh + e == j) ? 0x3F800000u : 0u;
                tmem_st_32x32b_x32(tmem + lrow + mp_base(0) + 64 * hf + 32 * hh, su);
                if (s_in) {
                    const float *src = s_in + (size_t)(64 * hf + 32 * hh) * DD + j;
#pragma unroll
                    for (int e = 0; e < 32; ++e) su[e] = __float_as_uint(src[(size_t)e * DD]);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) su[e] = 0u;
                }
                tmem_st_32x32b_x32(tmem + lrow + mp_base(1) + 64 * hf + 32 * hh, su);
            }
            tmem_wait_st();
        }

        for (int m = 0; m < nrun && ok; ++m) {  // chunk nb + m
            if (s_fail) { ok = false; break; }
            const int stg = m % STG;
            if (!mbar_wait(&full[stg], (m / STG) & 1)) { ok = false; break; }
            const float4 *g4 = reinterpret_cast<const float4 *>(sgam + stg * 128 + 64 * hf);
#pragma unroll
            for (int c = c0; c < 2; ++c) {  // S^T -> bf16 copy; S^T <- S^T Diag(e^{G_C})
                const uint32_t base = tmem + lrow + mp_base(c);
                if (m >= 1 && !mbar_wait(&bar_s[c], (m - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                uint32_t sv[64];
                tmem_ld_32x32b_x32(base + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld_32x32b_x32(base + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_wait_ld();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = pack_bf16x2(__uint_as_float(sv[32 * hh + 2 * e]), __uint_as_float(sv[32 * hh + 2 * e + 1]));
                    tmem_st_32x32b_x16(base + MP_S16 + 32 * hf + 16 * hh, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&simg[c]);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float4 gg = g4[e];
                    sv[4 * e] = __float_as_uint(__uint_as_float(sv[4 * e]) * gg.x);
                    sv[4 * e + 1] = __float_as_uint(__uint_as_float(sv[4 * e + 1]) * gg.y);
                    sv[4 * e + 2] = __float_as_uint(__uint_as_float(sv[4 * e + 2]) * gg.z);
                    sv[4 * e + 3] = __float_as_uint(__uint_as_float(sv[4 * e + 3]) * gg.w);
                }
                tmem_st_32x32b_x32(base + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_st_32x32b_x32(base + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_wait_st();
            }
            if (!ok) break;
#pragma unroll
            for (int c = c0; c < 2; ++c) {  // V'^T = [U^T] - (W S)^T -> bf16, over the dead S copy
                const uint32_t base = tmem + lrow + mp_base(c);
                uint4 uu[4];
                if (c == 1) {
                    const uint8_t *ut = sm + stg * STB + O_U;
#pragma unroll
                    for (int k = 0; k < 4; ++k) uu[k] = *reinterpret_cast<const uint4 *>(ut + sw128(j, 4 * hf + k));
                }
                if (!mbar_wait(&bar_p[c], m & 1)) { ok = false; break; }
                tc_fence_after();
                uint32_t pv[32], pk[16];
                tmem_ld_32x32b_x32(base + MP_PO + 32 * hf, pv);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float u[8];
                    if (c == 1) {
                        unpack8(uu[k], u);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) u[e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        pk[4 * k + e] = pack_bf16x2(u[2 * e] + __uint_as_float(pv[8 * k + 2 * e]),
                                                    u[2 * e + 1] + __uint_as_float(pv[8 * k + 2 * e + 1]));
                }
                tmem_st_32x32b_x16(base + MP_S16 + 16 * hf, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&vimg[c]);
            }
        }
        if (ok && nrun > 0) {
            if ((!windowed && !mbar_wait(&bar_s[0], (nrun - 1) & 1)) || !mbar_wait(&bar_s[1], (nrun - 1) & 1))
                ok = false;
            tc_fence_after();
        }
        if (ok && in_bounds(p.yt + ((size_t)bh * (p.G - 1) + g) * DD * DD, DD * DD * 4, p.yt, p.yt_bytes, p.bounds)) {
            // Y_g (S_1 for segment 0), laid out like a state
            float *dst0 = p.yt + ((size_t)bh * (p.G - 1) + g) * DD * DD;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t sv[32];
                tmem_ld_32x32b_x32(tmem + lrow + mp_base(1) + 64 * hf + 32 * hh, sv);
                tmem_wait_ld();
                float *dst = dst0 + (size_t)(64 * hf + 32 * hh) * DD + j;
#pragma unroll
                for (int e = 0; e < 32; ++e) dst[(size_t)e * DD] = __uint_as_float(sv[e]);
            }
            if (g >= 1 && windowed &&
                in_bounds(p.xt + ((size_t)bh * (p.G - 1) + g) * 32768, 32768, p.xt, p.xt_bytes, p.bounds)) {
                // A_g = 0 to fp32 (the window's bound): its image is zeros, 128 bytes a thread
                uint4 *img = reinterpret_cast<uint4 *>(p.xt + ((size_t)bh * (p.G - 1) + g) * 32768) + tid * 8;
#pragma unroll
                for (int k = 0; k < 8; ++k) img[k] = make_uint4(0u, 0u, 0u, 0u);
            } else if (g >= 1 &&
                       in_bounds(p.xt + ((size_t)bh * (p.G - 1) + g) * 32768, 32768, p.xt, p.xt_bytes, p.bounds)) {
                // A_g^T as the combine pass's MN-major B operand: image row j = lane j
                uint8_t *img = p.xt + ((size_t)bh * (p.G - 1) + g) * 32768;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t sv[32];
                    tmem_ld_32x32b_x32(tmem + lrow + mp_base(0) + 64 * hf + 32 * hh, sv);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(sv[8 * k + e]);
                        *reinterpret_cast<uint4 *>(img + hf * 16384 + sw128(j, 4 * hh + k)) = pack8(f);
                    }
                }
            }
        }
        if (!ok) s_fail = 1;
    }
    __syncthreads();
    if (warp == 8 && lane == 0 && s_fail) {
        report_timeout(p.timeouts, p.dev_status);
        // let the bulk copies already issued land before the CTA exits
        for (int m = landed; m < issued; ++m) mbar_wait(&full[m % STG], (m / STG) & 1, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, ST_TCOLS);
}

// ================================================================ K2c: chunk_combine_kernel
// The segment maps chained in order, one CTA per (head, batch): S_1 is segment 0's end state (the map
// pass ran it from the initial state, its Y slot; segment 1's chain reads it there), then
//   S_{g+1} = A_g S_g + Y_g,   g = 1 .. G-2,
// with the state transposed in TMEM (lane j): S_{g+1}^T = S_g^T A_g^T + Y_g^T, one M = 128 MMA per
// segment (A = bf16 copy of S_g^T in TMEM, B = the A_g^T image).  Writes S_2 .. S_{G-1} for the
// segment chains.
struct CombineArgs {
    int H, G;
    const uint8_t *xt;
    const float *yt;
    float *seg_init;
    size_t seg_bytes;  // size of seg_init (checked builds test the writes against it)
    unsigned int *bounds;
    unsigned int *timeouts;
    int *dev_status;
};

constexpr size_t COMB_SMEM = 2 * (32768 + 65536) + 64 + 1024;  // 2 stages of [A_g^T image | Y_g]

__global__ void __launch_bounds__(128, 1) chunk_combine_kernel(CombineArgs p) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ uint8_t smraw[];
    uint8_t *sm = align1024(smraw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y * p.H + blockIdx.x;
    const int j = tid;
    constexpr uint32_t CST = 32768 + 65536;                         // stage: A_g^T image, then Y_g fp32
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + 2 * CST);  // [2]
    uint64_t *bar_m = full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(full + 3);
    const int nseg = p.G - 1;  // entering states S_1 .. S_{G-1}
    auto issue = [&](int g) {   // A_g^T image and Y_g (g >= 1) -> stage (g - 1) & 1
        const int k = (g - 1) & 1;
        mbar_arrive_expect_tx(&full[k], CST);
        bulk_load(sm + k * CST, p.xt + ((size_t)bh * nseg + g) * 32768, 32768, &full[k]);
        bulk_load(sm + k * CST + 32768, p.yt + ((size_t)bh * nseg + g) * DD * DD, 65536, &full[k]);
    };
    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(bar_m, 1);
        fence_barrier_init();
        for (int g = 1; g < 3 && g < nseg; ++g) issue(g);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lrow = (uint32_t)(32 * warp) << 16;
    constexpr uint32_t C_S32 = 0, C_S16 = 128, C_D = 256;
    float sv[128];
    {   // S_1 (segment 0's end state, in Y slot 0)
        const float *src = p.yt + (size_t)bh * nseg * DD * DD + j;
#pragma unroll
        for (int c = 0; c < 128; ++c) sv[c] = src[(size_t)c * DD];
    }
    bool ok = true;
    int g = 1;
    for (; g < nseg; ++g) {
        const int k = (g - 1) & 1;
        const uint32_t kph = ((g - 1) >> 1) & 1;
        // bf16 copy of S_g^T (A operand)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(sv[32 * q + 2 * e], sv[32 * q + 2 * e + 1]);
            tmem_st_32x32b_x16(tmem + lrow + C_S16 + 16 * q, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            ok = mbar_wait(&full[k], kph);
            if (ok) {
                tc_fence_after();
                constexpr uint32_t id = idesc_f16(128, 128, 0, 1);
                const uint64_t d = smem_desc(smem_u32(sm + k * CST), 16384, 1024, LAYOUT_SW128);
#pragma unroll
                for (int s8 = 0; s8 < 8; ++s8) mma_f16_ts(tmem + C_D, tmem + C_S16 + 8 * s8, dadd(d, s8 * 2048), id, s8 > 0);
                mma_commit(bar_m);
            }
        }
        // while the MMA runs: S_g leaves for its segment chain (S_1 is read where the map pass left it)
        // and Y_g comes into registers
        if (g > 1 && in_bounds(p.seg_init + ((size_t)bh * p.G + g) * DD * DD, DD * DD * 4, p.seg_init, p.seg_bytes,
                               p.bounds)) {
            float *dst = p.seg_init + ((size_t)bh * p.G + g) * DD * DD + j;
#pragma unroll
            for (int c = 0; c < 128; ++c) dst[(size_t)c * DD] = sv[c];
        }
        ok = __syncthreads_and(ok) && mbar_wait(&full[k], kph);
        if (ok) {  // S_{g+1}^T = D + Y_g^T (Y_g in shared memory, [c][j])
            const float *y = reinterpret_cast<const float *>(sm + k * CST + 32768) + j;
#pragma unroll
            for (int c = 0; c < 128; ++c) sv[c] = y[c * DD];
        }
        ok = __syncthreads_and(ok && mbar_wait(bar_m, (g - 1) & 1));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t dv[32];
            tmem_ld_32x32b_x32(tmem + lrow + C_D + 32 * q, dv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[32 * q + e] += __uint_as_float(dv[e]);
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0 && g + 2 < nseg) issue(g + 2);  // this stage has been read
    }
    if (ok && nseg > 0) {  // the last entering state
        float *dst = p.seg_init + ((size_t)bh * p.G + nseg) * DD * DD + j;
#pragma unroll
        for (int c = 0; c < 128; ++c) dst[(size_t)c * DD] = sv[c];
    }
    if (!ok && tid == 0) {
        report_timeout(p.timeouts, p.dev_status);
        for (int m = g; m < nseg && m < g + 2; ++m) mbar_wait(&full[(m - 1) & 1], ((m - 1) >> 1) & 1, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// Segments per sequence: as many as let the chain pass (BH G CTAs), and so the map pass (BH (G - 1)
// CTAs), run in one wave, with at least 4 chunks per segment; 1 when (batch x heads) alone fills the GPU.
int pick_segments(int64_t BH, int64_t Nc, int sms) {
    int64_t G = sms / BH;
    if (G > Nc / 4) G = Nc / 4;
    return (int)(G < 1 ? 1 : G);
}

int device_sms() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

kda_status_t launch_state(const CUtensorMap &tmo, const CUtensorMap &tgl, const StateArgs &sa, int B, int H,
                          cudaStream_t st) {
    if (sa.G > 1) {
        cudaFuncSetAttribute(chunk_map_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)STATE_SMEM);
        cudaError_t e = launch_pdl(chunk_map_pair_kernel, dim3(H, B, sa.G - 1), dim3(ST_THREADS_MAP), STATE_SMEM, st,
                                   sa);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "chunk_map_pair_kernel: %s", cudaGetErrorString(e));
        kda_status_t s = check_launch("chunk_map_pair_kernel");
        if (s != KDA_OK) return s;
    }
    if (sa.G > 2) {  // (with two segments, segment 1 starts from S_1 itself)
        CombineArgs ca;
        ca.H = H;
        ca.G = sa.G;
        ca.xt = sa.xt;
        ca.yt = sa.yt;
        ca.seg_init = const_cast<float *>(sa.seg_init);
        ca.seg_bytes = (size_t)B * H * sa.G * DD * DD * 4;
        ca.bounds = sa.bounds;
        ca.timeouts = sa.timeouts;
        ca.dev_status = sa.dev_status;
        cudaFuncSetAttribute(chunk_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)COMB_SMEM);
        cudaError_t e = launch_pdl(chunk_combine_kernel, dim3(H, B), dim3(128), COMB_SMEM, st, ca);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "chunk_combine_kernel: %s", cudaGetErrorString(e));
        kda_status_t s = check_launch("chunk_combine_kernel");
        if (s != KDA_OK) return s;
    }
    cudaFuncSetAttribute(chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)STATE_SMEM);
    cudaError_t e = launch_pdl(chunk_state_kernel, dim3(H, B, sa.G), dim3(ST_THREADS_CHAIN), STATE_SMEM, st, tmo, tgl,
                               sa);
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "chunk_state_kernel: %s", cudaGetErrorString(e));
    return check_launch("chunk_state_kernel");
}

}  // namespace

kda_status_t tc::make_tmap_tokens(CUtensorMap *m, const void *base, int H, int64_t S, int64_t B, uint64_t rs,
                                  uint64_t ss, uint64_t bs) {
    const uint64_t dims[4] = {(uint64_t)DD, (uint64_t)H, (uint64_t)S, (uint64_t)B};
    const uint64_t strides[3] = {rs, ss, bs};
    const uint32_t box[4] = {64, 1, CH, 1};
    return make_tmap_nd(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 4, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

bool chunk_tc_supported(const kda_chunk_args &a, int chunk) {
    return a.dtype == KDA_BF16 && a.D_k == DD && a.D_v == DD && chunk == CH && a.g_min >= TC_GMIN_LIMIT &&
           a.B <= 65535 && a.H <= 65535 && a.S <= 0x7fffffffLL - CH;
}

bool chunk_tc_aligned(const kda_chunk_args &a) {
    auto al = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    bool okp = al(a.q) && al(a.k) && al(a.v) && al(a.o) && al(a.initial_state) && al(a.final_state) &&
               al(a.gate_logits);
    if (!a.log_decay) okp = okp && al(a.z);
    return okp;
}

namespace {

// Workspace: one record per chunk, then (with several segments) the segment maps
// A_g^T (bf16 images) and Y_g, and the segments' entering states.
struct TcLayout {
    int G, L;
    size_t xt, yt, seg, lb, total;
};

TcLayout tc_layout(const kda_chunk_args &a) {
    TcLayout t;
    const int64_t Nc = (a.S + CH - 1) / CH, BH = (int64_t)a.B * a.H;
    t.G = pick_segments(BH, Nc, device_sms());
    t.L = (int)((Nc + t.G - 1) / t.G);
    if (Nc > 0) t.G = (int)((Nc + t.L - 1) / t.L);  // no empty segment
    t.xt = (size_t)BH * Nc * REC_BYTES;
    const size_t nmap = t.G > 1 ? (size_t)BH * (t.G - 1) : 0;
    t.yt = t.xt + nmap * 32768;
    t.seg = t.yt + nmap * DD * DD * 4;
    t.lb = t.seg + (t.G > 1 ? (size_t)BH * t.G * DD * DD * 4 : 0);
    t.total = t.lb + (t.G > 1 ? (size_t)BH * Nc * 4 : 0);  // per-chunk log-bounds, for the map pass's windows
    return t;
}

}  // namespace

size_t chunk_tc_workspace(const kda_chunk_args &a) { return tc_layout(a).total; }

float *tc::chunk_log_bounds(const kda_chunk_args &a) {
    const TcLayout lay = tc_layout(a);
    return lay.G > 1 ? reinterpret_cast<float *>((uint8_t *)a.workspace + lay.lb) : nullptr;
}

kda_status_t tc::launch_chunk_state_pass(const kda_chunk_args &a, cudaStream_t st) {
    const int64_t Nc = (a.S + CH - 1) / CH;
    CUtensorMap to, tgl;
    memset(&to, 0, sizeof(to));  // (no chunks: never read)
    memset(&tgl, 0, sizeof(tgl));  // (no gate: never read)
    const TcLayout lay = tc_layout(a);
    uint8_t *ws = (uint8_t *)a.workspace;
    if (Nc > 0) {
        const uint64_t rs = (uint64_t)DD, ss = (uint64_t)a.H * DD, bs = (uint64_t)a.S * a.H * DD;
        kda_status_t s = make_tmap_tokens(&to, a.o, a.H, a.S, a.B, rs, ss, bs);
        if (s != KDA_OK) return s;
        if (a.gate_logits) {
            s = make_tmap_tokens(&tgl, a.gate_logits, a.H, a.S, a.B, rs, ss, bs);
            if (s != KDA_OK) return s;
        }
    }
    StateArgs sa;
    sa.S = (int)a.S;
    sa.H = a.H;
    sa.Nc = (int)Nc;
    sa.ws = (const uint8_t *)a.workspace;
    sa.S0 = a.initial_state;
    sa.Sf = a.final_state;
    sa.gated = a.gate_logits != nullptr && Nc > 0;
    sa.L = Nc > 0 ? lay.L : 1;
    sa.G = Nc > 0 ? lay.G : 1;
    sa.xt = ws + lay.xt;
    sa.yt = reinterpret_cast<float *>(ws + lay.yt);
    sa.seg_init = reinterpret_cast<const float *>(ws + lay.seg);
    {
        const size_t BH = (size_t)a.B * a.H, nmap = sa.G > 1 ? BH * (sa.G - 1) : 0;
        sa.sf_bytes = BH * DD * DD * 4;
        sa.xt_bytes = nmap * 32768;
        sa.yt_bytes = nmap * DD * DD * 4;
        sa.bounds = device_bounds_counter();
    }
    sa.lbound = (Nc > 0 && lay.G > 1) ? reinterpret_cast<const float *>(ws + lay.lb) : nullptr;
    sa.eps = a.eps;
    sa.timeouts = device_timeout_counter();
    sa.dev_status = a.dev_status;
    return launch_state(to, tgl, sa, (int)a.B, a.H, st);
}

kda_status_t launch_chunk_tc(const kda_chunk_args &a, cudaStream_t st) {
    const int64_t Nc = (a.S + CH - 1) / CH;
    unsigned int *timeouts = device_timeout_counter();
    if (Nc > 0) {
        CUtensorMap tq, tk, tv, tz;
        const uint64_t rs = (uint64_t)DD, ss = (uint64_t)a.H * DD, bs = (uint64_t)a.S * a.H * DD;
        kda_status_t s = make_tmap_tokens(&tq, a.q, a.H, a.S, a.B, rs, ss, bs);
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
        pa.units = Nc * a.H * a.B;
        if (pa.units > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "chunk engine: more than 2^31 chunks");
        pa.g_min = a.g_min;
        pa.beta = (const __nv_bfloat16 *)a.beta;
        pa.log_decay = a.log_decay;
        pa.ws = (uint8_t *)a.workspace;
        pa.rec_bytes = (size_t)pa.units * REC_BYTES;
        pa.bounds = device_bounds_counter();
        pa.lbound = tc::chunk_log_bounds(a);
        pa.timeouts = timeouts;
        pa.dev_status = a.dev_status;
        const int sms = device_sms();
        const int64_t grid = pa.units < sms ? pa.units : sms;
        cudaFuncSetAttribute(chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PREP_SMEM);
        cudaError_t e = launch_pdl(chunk_prep_kernel, dim3((unsigned)grid), dim3(PREP_THREADS), PREP_SMEM, st, tq, tk,
                                   tv, tz, pa);
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "chunk_prep_kernel: %s", cudaGetErrorString(e));
        s = check_launch("chunk_prep_kernel");
        if (s != KDA_OK) return s;
    }
    return tc::launch_chunk_state_pass(a, st);
}

}  // namespace kda
