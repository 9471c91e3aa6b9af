// The general DPLR recurrence of the "Diagonal-Plus-Low-Rank Matrices and Kimi
// Delta Attention" post (sections 1 and 3) in chunk form, exact fp32 (SIMT):
//
//   S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,    o_t = S_t^T q_t.
//
// Inside a chunk of C tokens with G_r = sum_{i<=r} log alpha_i per key channel
// (G_{-1} = 0) and y_r = b_r^T S_{r-1} (the row the rank-1 erase removes):
//   S_r = Diag(e^{G_r}) S + sum_{i<=r} Diag(e^{G_r - G_i}) (k_i v_i^T - a_i y_i)
// (S: the state entering the chunk), so that, with the decayed products
//   Bk[r,i] = sum_c b_rc k_ic e^{G_{r-1,c} - G_ic},  Ba[r,i] = the same with a   (i < r)
//   Mk[r,i] = sum_c q_rc k_ic e^{G_rc - G_ic},       Ma[r,i] = the same with a   (i <= r),
// the erased rows solve a unit-lower-triangular system and everything follows:
//   (I + Ba) Y = (b * e^{G_{r-1}}) S + Bk V     ->  Y = Wy S + Uy,  Wy = T (b * e^{G_{r-1}}),
//                                                   Uy = T Bk V,  T = (I + Ba)^{-1}
//   O      = (Q * e^G) S + Mk V - Ma Y
//   S_next = Diag(e^{G_last}) S + (K * e^{G_last - G})^T V - (A * e^{G_last - G})^T Y.
// KDA is the case a = beta k, b = alpha * k (write key beta k), where Bk = Ba
// up to the beta of the column and the system is the WY/UT one of the KDA
// engines; here the erase and write directions are free, so four decayed
// products instead of two, and the chain carries Y as well as the state.
//
// Kernels: dc_prep_kernel (one CTA per (b, h, chunk), all chunks at once)
// forms the chunk's Wy, Uy, Q e^G, A e^{G_last - G}, Ma, Mk V and Kd^T V in a
// workspace record; dc_chain_kernel (one CTA per (b, h, 16 value columns))
// walks the chunks in order with the state slice in shared memory and writes
// the outputs and the final state.  Every decay factor is the exponential of
// a difference <= 0.
#include "simt_chunk.cuh"

namespace kda {

namespace {

using namespace simt;

// One (b, h, chunk) record; offsets in floats.
struct DcRec {
    int64_t Gl;    // [Dk] last row of G
    int64_t Qg;    // [C][Dk] Q e^G
    int64_t Ad;    // [C][Dk] A e^{G_last - G}
    int64_t Wy;    // [C][Dk] T (b e^{G_{r-1}})
    int64_t Ma;    // [C][C]  Ma (i <= r)
    int64_t Uy;    // [C][Dv] T Bk V
    int64_t MkV;   // [C][Dv] Mk V
    int64_t KdV;   // [Dk][Dv] (K e^{G_last - G})^T V
    int64_t size;
};

__host__ __device__ inline DcRec dc_rec(int Dk, int Dv) {
    const int64_t C = CB_C;
    DcRec r;
    r.Gl = 0;
    r.Qg = (Dk + 3) & ~3;
    r.Ad = r.Qg + C * Dk;
    r.Wy = r.Ad + C * Dk;
    r.Ma = r.Wy + C * Dk;
    r.Uy = r.Ma + C * C;
    r.MkV = r.Uy + C * Dv;
    r.KdV = r.MkV + C * Dv;
    r.size = (r.KdV + (int64_t)Dk * Dv + 3) & ~(int64_t)3;
    return r;
}

struct DcArgs {
    int64_t S;
    int H, Dk, Dv, Nc;
    const void *q, *k, *v, *a, *b, *z;
    const float *log_decay;
    float g_min;
    const float *S0;
    void *o;
    float *Sf;
    float *ws;  // records [B*H][Nc]
    size_t ws_bytes, sf_bytes;  // (checked builds test the writes against them)
    unsigned int *bounds;
};

// ---------------------------------------------------------------- per chunk
// Pitch of the token-row blocks, and the size each of the five takes (one of them later holds T).
__host__ __device__ inline int dc_lx(int Dk, int Dv) { return cb_max(cb_pad8(Dk), cb_pad8(Dv)) + 1; }
__host__ __device__ inline int dc_region(int Dk, int Dv) { return CB_C * cb_max(dc_lx(Dk, Dv), CB_C + 1); }
__host__ __device__ inline size_t dc_prep_smem(int Dk, int Dv) {
    return sizeof(float) * ((size_t)5 * dc_region(Dk, Dv) + 3 * CB_C * (CB_C + 1));
}

template <typename T>
__global__ void __launch_bounds__(CB_NTC) dc_prep_kernel(DcArgs p) {
    extern __shared__ __align__(16) float cb_sm[];
    const int tid = threadIdx.x;
    const int64_t u = blockIdx.x, bh = u / p.Nc;
    const int n = (int)(u - bh * p.Nc), b = (int)(bh / p.H), h = (int)(bh - (int64_t)b * p.H);
    const int C = CB_C, Dk = p.Dk, Dv = p.Dv, Dkp = cb_pad8(Dk), Dvp = cb_pad8(Dv);
    const int LX = dc_lx(Dk, Dv), LC = C + 1, XR = dc_region(Dk, Dv);
    const int64_t t0 = (int64_t)n * C;
    const int len = (int)min((int64_t)C, p.S - t0);
    // five [C][LX] regions: k (later K e^{G_last - G}), q (later T), a (later V), b (later b e^{G_{r-1}},
    // then Bk V), log alpha (then G); three [C][LC]: Bk, Ba, Mk
    float *sK = cb_sm, *sQ = sK + XR, *sA = sQ + XR, *sB = sA + XR, *sG = sB + XR;
    float *sBk = sG + XR, *sBa = sBk + C * LC, *sMk = sBa + C * LC;
    const DcRec R = dc_rec(Dk, Dv);
    float *rec = p.ws + u * R.size;
    const bool ok = in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds);
    const int64_t row0 = (((int64_t)b * p.S + t0) * p.H + h), rk = (int64_t)p.H * Dk;

    cb_load_rows(sK, LX, (const T *)p.k + row0 * Dk, rk, C, len, Dk, Dkp);
    cb_load_rows(sQ, LX, (const T *)p.q + row0 * Dk, rk, C, len, Dk, Dkp);
    cb_load_rows(sA, LX, (const T *)p.a + row0 * Dk, rk, C, len, Dk, Dkp);
    cb_load_rows(sB, LX, (const T *)p.b + row0 * Dk, rk, C, len, Dk, Dkp);
    if (p.log_decay)
        cb_load_rows(sG, LX, p.log_decay + row0 * Dk, rk, C, len, Dk, Dk);
    else
        cb_load_rows(sG, LX, (const T *)p.z + row0 * Dk, rk, C, len, Dk, Dk);
    __syncthreads();
    for (int c = tid; c < Dk; c += CB_NTC) {  // G: cumulative sum of log(alpha); rows past the end: no decay
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            const float x = sG[r * LX + c];
            acc += r < len ? (p.log_decay ? clamp_log_decay(x, p.g_min) : log_alpha_of(x, p.g_min)) : 0.f;
            sG[r * LX + c] = acc;
        }
        if (ok) rec[R.Gl + c] = acc;
    }
    __syncthreads();
    for (int idx = tid; ok && idx < C * Dk; idx += CB_NTC) {  // Q e^G and A e^{G_last - G}
        const int r = idx / Dk, c = idx - r * Dk;
        const float G = sG[r * LX + c];
        rec[R.Qg + idx] = sQ[r * LX + c] * cb_exp(G);
        rec[R.Ad + idx] = sA[r * LX + c] * cb_exp(sG[(C - 1) * LX + c] - G);
    }
    // the four decayed products over the triangle of pairs (i <= r): the b rows decay from token r - 1,
    // the q rows from token r
    for (int pi = tid; pi < C * (C + 1) / 2; pi += CB_NTC) {
        int r = (int)((sqrtf(8.f * (float)pi + 1.f) - 1.f) * 0.5f);
        while (r > 0 && r * (r + 1) / 2 > pi) --r;
        while ((r + 1) * (r + 2) / 2 <= pi) ++r;
        const int i = pi - r * (r + 1) / 2;
        const float *gr = sG + r * LX, *gi = sG + i * LX, *br = sB + r * LX, *qr = sQ + r * LX;
        const float *ki = sK + i * LX, *ai = sA + i * LX;
        float bk = 0.f, ba = 0.f, mk = 0.f, ma = 0.f;
        for (int c = 0; c < Dk; ++c) {
            const float grp = r > 0 ? gr[c - LX] : 0.f;  // G_{r-1}
            const float e1 = cb_exp(grp - gi[c]), e2 = cb_exp(gr[c] - gi[c]);
            const float bb = br[c] * e1, qq = qr[c] * e2;
            bk = fmaf(bb, ki[c], bk);
            ba = fmaf(bb, ai[c], ba);
            mk = fmaf(qq, ki[c], mk);
            ma = fmaf(qq, ai[c], ma);
        }
        sBk[r * LC + i] = i < r ? bk : 0.f;
        sBa[r * LC + i] = i < r ? ba : 0.f;
        sMk[r * LC + i] = mk;
        if (ok) rec[R.Ma + r * C + i] = ma;
    }
    for (int idx = tid; idx < C * C; idx += CB_NTC) {  // the upper triangles
        const int r = idx / C, i = idx - r * C;
        if (i > r) {
            sBk[r * LC + i] = 0.f;
            sBa[r * LC + i] = 0.f;
            sMk[r * LC + i] = 0.f;
            if (ok) rec[R.Ma + idx] = 0.f;
        }
    }
    __syncthreads();
    // T = (I + Ba)^{-1} over q's space (column j by forward substitution, thread j); meanwhile
    // b e^{G_{r-1}} in place and K e^{G_last - G} in place
    float *sT = sQ;
    if (tid < C) {
        const int j = tid;
        for (int r = 0; r < C; ++r) {
            const float *pr = sBa + r * LC;
            float a0 = r == j ? 1.f : 0.f, a1 = 0.f;
            int m = 0;
            for (; m + 1 < r; m += 2) {
                a0 = fmaf(-pr[m], sT[m * LC + j], a0);
                a1 = fmaf(-pr[m + 1], sT[(m + 1) * LC + j], a1);
            }
            if (m < r) a0 = fmaf(-pr[m], sT[m * LC + j], a0);
            sT[r * LC + j] = a0 + a1;
        }
    }
    for (int idx = tid; idx < C * Dkp; idx += CB_NTC) {
        const int r = idx / Dkp, c = idx - r * Dkp;
        if (c < Dk) {
            sB[r * LX + c] *= r > 0 ? cb_exp(sG[(r - 1) * LX + c]) : 1.f;
            sK[r * LX + c] *= cb_exp(sG[(C - 1) * LX + c] - sG[r * LX + c]);
        }
    }
    __syncthreads();
    // V over a's space
    cb_load_rows(sA, LX, (const T *)p.v + row0 * Dv, (int64_t)p.H * Dv, C, len, Dv, Dvp);
    __syncthreads();
    float *sV = sA;
    if (ok) {
        // Wy = T (b e^{G_{r-1}}),  Mk V,  (K e^{G_last - G})^T V -> record
        cb_mm<false, true>(sT, LC, sB, LX, C, Dkp, C, [&](int r, int c, float x) {
            if (c < Dk) rec[R.Wy + (int64_t)r * Dk + c] = x;
        });
        cb_mm<false, true>(sMk, LC, sV, LX, C, Dvp, C, [&](int r, int j, float x) {
            if (j < Dv) rec[R.MkV + (int64_t)r * Dv + j] = x;
        });
        cb_mm<true, true>(sK, LX, sV, LX, Dkp, Dvp, C, [&](int c, int j, float x) {
            if (c < Dk && j < Dv) rec[R.KdV + (int64_t)c * Dv + j] = x;
        });
    }
    __syncthreads();
    // Bk V over b's space (its padding columns come out zero), then Uy = T Bk V -> record
    float *sBkV = sB;
    cb_mm<false, true>(sBk, LC, sV, LX, C, Dvp, C, [&](int r, int j, float x) { sBkV[r * LX + j] = x; });
    __syncthreads();
    if (ok)
        cb_mm<false, true>(sT, LC, sBkV, LX, C, Dvp, C, [&](int r, int j, float x) {
            if (j < Dv) rec[R.Uy + (int64_t)r * Dv + j] = x;
        });
}

// ---------------------------------------------------------------- the chain, per 16 value columns
// Group A (Y): Wy [C][LK], Uy columns [C][16].  Group B (outputs and state): Q e^G, A e^{G_last - G}
// [C][LK], Ma [C][LC], Mk V columns [C][16], Kd^T V columns [Dk][16], last row of G [Dk].  Then the
// state slice twice (old and new) [Dk][16] and Y [C][16].
__host__ __device__ inline int dc_lk(int Dk) { return cb_pad8(Dk) + 4; }
constexpr int DC_LC = CB_C + 4;

__host__ __device__ inline size_t dc_chain_smem(int Dk) {
    const int LK = dc_lk(Dk), Dk4 = (Dk + 3) & ~3;
    return sizeof(float) * ((size_t)3 * CB_C * LK + CB_C * DC_LC + 2 * CB_C * CB_VS + (size_t)Dk * CB_VS + Dk4 +
                            (size_t)2 * Dk * CB_VS + CB_C * CB_VS + CB_C * CB_VS);
}

template <typename T>
__global__ void __launch_bounds__(CB_NT) dc_chain_kernel(DcArgs p) {
    extern __shared__ __align__(16) float cb_sm[];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int j0 = blockIdx.y * CB_VS;
    const int C = CB_C, Dk = p.Dk, Dv = p.Dv, LK = dc_lk(Dk), LC = DC_LC, Dk4 = (Dk + 3) & ~3;
    const int b = (int)(bh / p.H), h = (int)(bh - (int64_t)b * p.H);
    float *sWy = cb_sm, *sUy = sWy + C * LK;
    float *sQg = sUy + C * CB_VS, *sAd = sQg + C * LK, *sMa = sAd + C * LK, *sMkV = sMa + C * LC;
    float *sKdV = sMkV + C * CB_VS, *sGl = sKdV + Dk * CB_VS;
    float *sS = sGl + Dk4, *sS2 = sS + Dk * CB_VS, *sY = sS2 + Dk * CB_VS, *sO = sY + C * CB_VS;
    const DcRec R = dc_rec(Dk, Dv);
    auto rec_of = [&](int n) { return p.ws + (bh * p.Nc + n) * R.size; };
    auto stage_a = [&](int n) {
        const float *rec = rec_of(n);
        if (in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds)) {
            cb_copy(sWy, LK, rec + R.Wy, C, Dk, C, Dk);
            cb_copy_cols(sUy, rec + R.Uy, C, Dv, j0);
        }
        cp_async_commit_group();
    };
    auto stage_b = [&](int n) {
        const float *rec = rec_of(n);
        if (in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds)) {
            cb_copy(sQg, LK, rec + R.Qg, C, Dk, C, Dk);
            cb_copy(sAd, LK, rec + R.Ad, C, Dk, C, Dk);
            cb_copy(sMa, LC, rec + R.Ma, C, C, C, C);
            cb_copy_cols(sMkV, rec + R.MkV, C, Dv, j0);
            cb_copy_cols(sKdV, rec + R.KdV, Dk, Dv, j0);
            cb_copy(sGl, Dk, rec + R.Gl, 1, Dk, 1, Dk);
        }
        cp_async_commit_group();
    };
    for (int idx = tid; idx < Dk * CB_VS; idx += CB_NT) {
        const int c = idx / CB_VS, j = idx - c * CB_VS;
        sS[idx] = (p.S0 && j0 + j < Dv) ? p.S0[(bh * Dk + c) * Dv + j0 + j] : 0.f;
    }
    stage_a(0);
    stage_b(0);
    for (int n = 0; n < p.Nc; ++n) {
        const int64_t t0 = (int64_t)n * C;
        const int len = (int)min((int64_t)C, p.S - t0);
        cp_async_wait<1>();  // Wy and Uy of chunk n
        __syncthreads();
        {  // Y = Uy + Wy S: thread (row r, four columns)
            const int r = tid >> 2, jq = (tid & 3) * 4;
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) y[e] = sUy[r * CB_VS + jq + e];
            for (int c = 0; c < Dk; ++c) {
                const float wv = sWy[r * LK + c];
                const float4 s = *reinterpret_cast<const float4 *>(sS + c * CB_VS + jq);
                y[0] = fmaf(wv, s.x, y[0]);
                y[1] = fmaf(wv, s.y, y[1]);
                y[2] = fmaf(wv, s.z, y[2]);
                y[3] = fmaf(wv, s.w, y[3]);
            }
            *reinterpret_cast<float4 *>(sY + r * CB_VS + jq) = make_float4(y[0], y[1], y[2], y[3]);
        }
        __syncthreads();  // Wy and Uy of chunk n are read: the next chunk's come in
        if (n + 1 < p.Nc) stage_a(n + 1);
        else cp_async_commit_group();
        cp_async_wait<1>();  // group B of chunk n
        __syncthreads();
        {  // O = Q e^G S + Mk V - Ma Y: thread (row r, four columns)
            const int r = tid >> 2, jq = (tid & 3) * 4;
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = sMkV[r * CB_VS + jq + e];
            for (int c = 0; c < Dk; ++c) {
                const float qg = sQg[r * LK + c];
                const float4 s = *reinterpret_cast<const float4 *>(sS + c * CB_VS + jq);
                o[0] = fmaf(qg, s.x, o[0]);
                o[1] = fmaf(qg, s.y, o[1]);
                o[2] = fmaf(qg, s.z, o[2]);
                o[3] = fmaf(qg, s.w, o[3]);
            }
            for (int i = 0; i <= r; ++i) {
                const float m = sMa[r * LC + i];
                const float4 yv = *reinterpret_cast<const float4 *>(sY + i * CB_VS + jq);
                o[0] = fmaf(-m, yv.x, o[0]);
                o[1] = fmaf(-m, yv.y, o[1]);
                o[2] = fmaf(-m, yv.z, o[2]);
                o[3] = fmaf(-m, yv.w, o[3]);
            }
            *reinterpret_cast<float4 *>(sO + r * CB_VS + jq) = make_float4(o[0], o[1], o[2], o[3]);
        }
        if (tid < 2 * Dk) {  // S_next = Diag(gamma) S + Kd^T V - Ad^T Y: thread (key row c, eight columns)
            const int c = tid >> 1, jh = (tid & 1) * 8;
            const float gam = cb_exp(sGl[c]);
            float s[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) s[e] = fmaf(gam, sS[c * CB_VS + jh + e], sKdV[c * CB_VS + jh + e]);
            for (int r = 0; r < C; ++r) {
                const float ad = sAd[r * LK + c];
                const float4 y0 = *reinterpret_cast<const float4 *>(sY + r * CB_VS + jh);
                const float4 y1 = *reinterpret_cast<const float4 *>(sY + r * CB_VS + jh + 4);
                s[0] = fmaf(-ad, y0.x, s[0]);
                s[1] = fmaf(-ad, y0.y, s[1]);
                s[2] = fmaf(-ad, y0.z, s[2]);
                s[3] = fmaf(-ad, y0.w, s[3]);
                s[4] = fmaf(-ad, y1.x, s[4]);
                s[5] = fmaf(-ad, y1.y, s[5]);
                s[6] = fmaf(-ad, y1.z, s[6]);
                s[7] = fmaf(-ad, y1.w, s[7]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) sS2[c * CB_VS + jh + e] = s[e];
        }
        __syncthreads();  // group B of chunk n, S and Y are read
        if (n + 1 < p.Nc) stage_b(n + 1);
        else cp_async_commit_group();
        for (int idx = tid; idx < len * CB_VS; idx += CB_NT) {  // the chunk's outputs, 16 columns a row
            const int r = idx / CB_VS, j = idx - r * CB_VS;
            if (j0 + j < Dv)
                store_elem((T *)p.o, (((int64_t)b * p.S + t0 + r) * p.H + h) * Dv + j0 + j, sO[idx]);
        }
        float *t = sS;
        sS = sS2;
        sS2 = t;
    }
    __syncthreads();
    if (p.Sf && in_bounds(p.Sf + bh * Dk * Dv, (size_t)Dk * Dv * 4, p.Sf, p.sf_bytes, p.bounds))
        for (int idx = tid; idx < Dk * CB_VS; idx += CB_NT) {
            const int c = idx / CB_VS, j = idx - c * CB_VS;
            if (j0 + j < Dv) p.Sf[(bh * Dk + c) * Dv + j0 + j] = sS[idx];
        }
}

}  // namespace

// ================================================================ host side
size_t dplr_chunk_workspace(int64_t B, int64_t S, int H, int Dk, int Dv) {
    const int64_t Nc = (S + CB_C - 1) / CB_C;
    return (size_t)B * H * Nc * (size_t)dc_rec(Dk, Dv).size * sizeof(float);
}

kda_status_t launch_dplr_chunk(const kda_dplr_args &a, void *workspace, cudaStream_t st) {
    DcArgs p;
    p.S = a.S;
    p.H = a.H;
    p.Dk = a.D_k;
    p.Dv = a.D_v;
    p.Nc = (int)((a.S + CB_C - 1) / CB_C);
    p.q = a.q; p.k = a.k; p.v = a.v; p.a = a.a; p.b = a.b; p.z = a.z;
    p.log_decay = a.log_decay;
    p.g_min = a.g_min;
    p.S0 = a.initial_state;
    p.o = a.o;
    p.Sf = a.final_state;
    p.ws = reinterpret_cast<float *>(workspace);
    p.ws_bytes = dplr_chunk_workspace(a.B, a.S, a.H, a.D_k, a.D_v);
    p.sf_bytes = (size_t)a.B * a.H * a.D_k * a.D_v * 4;
    p.bounds = device_bounds_counter();
    const int64_t nbh = a.B * a.H, units = nbh * p.Nc;
    if (units > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "chunked DPLR: B*H*chunks too large");
    const int nslice = (a.D_v + CB_VS - 1) / CB_VS;
    const size_t s1 = dc_prep_smem(a.D_k, a.D_v), s2 = dc_chain_smem(a.D_k);
    auto go = [&](auto prep, auto chain) -> kda_status_t {
        cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
        cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
        kda_status_t s;
        prep<<<(unsigned)units, CB_NTC, s1, st>>>(p);
        if ((s = check_launch("dc_prep_kernel")) != KDA_OK) return s;
        chain<<<dim3((unsigned)nbh, (unsigned)nslice), CB_NT, s2, st>>>(p);
        return check_launch("dc_chain_kernel");
    };
    if (a.dtype == KDA_F32) return go(dc_prep_kernel<float>, dc_chain_kernel<float>);
    return go(dc_prep_kernel<__nv_bfloat16>, dc_chain_kernel<__nv_bfloat16>);
}

}  // namespace kda
