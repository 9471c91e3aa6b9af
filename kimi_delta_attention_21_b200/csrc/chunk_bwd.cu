// Chunkwise backward of the KDA recurrence (exact fp32, SIMT).
//
// The forward's chunk form (Kimi Linear report, section 3.1 and appendix B,
// Props. 1-2, with beta_r multiplying the whole bracket of Eqs. 17 and 19):
// inside a chunk of C tokens, G_r = sum_{i<=r} log alpha_i per key channel and
// E[r,i,c] = exp(G_rc - G_ic) for i <= r;
//   P[r,i] = sum_c k_rc k_ic E[r,i,c]  (i < r),   A = Diag(beta) P,   T = (I + A)^{-1}
//   W = T Diag(beta)(K * e^G),   U = T Diag(beta) V,   V' = U - W S
//   M[r,i] = sum_c q_rc k_ic E[r,i,c]  (i <= r),  O = (Q * e^G) S + M V'
//   S_next = Diag(gamma) S + Kd^T V',   gamma = e^{G_last},  Kd = K * e^{G_last - G}
// (S: the state entering the chunk, O: the outputs read after each update).
// Reverse-mode differentiation of those lines, with dS_next = dL/dS_next:
//   dV' = M^T dO + Kd dS_next
//   dS  = (Q e^G)^T dO + Diag(gamma) dS_next - W^T dV'          (serial over chunks)
//   dQg = dO S^T,  dKd = V' dS_next^T,  dgamma_c = sum_j dS_next[c,j] S[c,j]
//   dM  = dO V'^T (i <= r),  dW = -dV' S^T
//   dT  = (dV' V^T + dW (K e^G)^T) Diag(beta),  dBv = T^T dV',  dBk = T^T dW
//   dA  = -T^T dT T^T (i < r),  dv = Diag(beta) dBv
//   dbeta_r = sum_j dBv[r,j] v_rj + sum_c dBk[r,c] (k e^G)_rc + sum_i dA[r,i] P[r,i]
// and through the decayed products, each E in a row role (r) and a column role (i):
//   dq_rc = dQg_rc e^{G_rc} + sum_i dM[r,i] k_ic E[r,i,c]
//   dk_rc = beta_r dBk_rc e^{G_rc} + dKd_rc e^{G_last,c - G_rc} + beta_r sum_i dA[r,i] k_ic E[r,i,c]
//           + sum_{r' >= r} (beta_r' dA[r',r] k_r'c + dM[r',r] q_r'c) E[r',r,c]
//   dG_rc = the same terms times their own factor's exponent sign (+ for the row role, - for the
//           column role and for e^{-G} in Kd), plus dgamma_c gamma_c and sum_r dKd Kd on the last row,
// then dlog(alpha) is the reverse cumulative sum of dG over the chunk, and dz follows from
// log(alpha) = g_min sigmoid(z).
//
// Kernels: cb_prep_kernel (one CTA per (b, h, chunk)) forms G, P, M, T, W, U,
// Q e^G and Kd; cb_fwd_chain_kernel (one CTA per (b, h, 16 value columns))
// walks the chunks forward and keeps each chunk's entering state and V';
// cb_bwd_chain_kernel walks them backwards for dS_next, dV' and dgamma;
// cb_grad_mat_kernel and cb_grad_pair_kernel (one CTA per chunk) form the
// chunk's gradients.  Every chunk's intermediates live in a workspace record.
// Every decay factor is the exponential of a difference <= 0, so any g_min is
// safe; all arithmetic is fp32.
#include "simt_chunk.cuh"

namespace kda {

namespace {

using namespace simt;

// One (b, h, chunk) record of the workspace; offsets in floats, row-major blocks.
struct CbRec {
    int64_t G;     // [C][Dk] in-chunk cumulative log-decay
    int64_t P;     // [C][C]  P (strictly lower)
    int64_t T;     // [C][C]  T; after the matrix gradients: dA
    int64_t W;     // [C][Dk] W; after the matrix gradients: dKg = beta dBk
    int64_t U;     // [C][Dv] U
    int64_t M;     // [C][C]  M (i <= r); after the matrix gradients: dM
    int64_t Qg;    // [C][Dk] Q e^G; after the matrix gradients: dQg
    int64_t Kd;    // [C][Dk] K e^{G_last - G}; after the matrix gradients: dKd
    int64_t S;     // [Dk][Dv] the state entering the chunk
    int64_t Vp;    // [C][Dv] V'
    int64_t dS;    // [Dk][Dv] dL/dS leaving the chunk
    int64_t dVp;   // [C][Dv] dV'
    int64_t dgam;  // [nslice][Dk] dgamma, one partial sum per chain CTA
    int64_t size;
};

__host__ __device__ inline CbRec cb_rec(int Dk, int Dv, int nslice) {
    const int64_t C = CB_C;
    CbRec r;
    r.G = 0;
    r.P = r.G + C * Dk;
    r.T = r.P + C * C;
    r.W = r.T + C * C;
    r.U = r.W + C * Dk;
    r.M = r.U + C * Dv;
    r.Qg = r.M + C * C;
    r.Kd = r.Qg + C * Dk;
    r.S = r.Kd + C * Dk;
    r.Vp = r.S + (int64_t)Dk * Dv;
    r.dS = r.Vp + C * Dv;
    r.dVp = r.dS + (int64_t)Dk * Dv;
    r.dgam = r.dVp + C * Dv;
    r.size = (r.dgam + (int64_t)nslice * Dk + 3) & ~(int64_t)3;
    return r;
}

struct CbArgs {
    int64_t S;
    int H, Dk, Dv, Nc, nslice;
    const void *q, *k, *v, *z, *beta, *dO;
    const float *log_decay;
    float g_min;
    const float *S0, *dST;
    float *dq, *dk, *dv, *dbeta, *dz, *dS0;
    float *ws;        // records [B*H][Nc]
    size_t ws_bytes;  // buffer sizes in bytes (checked builds test the writes against them)
    size_t nk_bytes, nv_bytes, nb_bytes, ns_bytes;
    unsigned int *bounds;
};

struct CbUnit {
    int64_t u, bh;
    int n, b, h, len;
    int64_t t0;
};

__device__ __forceinline__ CbUnit cb_unit(const CbArgs &p, int64_t u) {
    CbUnit w;
    w.u = u;
    w.bh = u / p.Nc;
    w.n = (int)(u - w.bh * p.Nc);
    w.b = (int)(w.bh / p.H);
    w.h = (int)(w.bh - (int64_t)w.b * p.H);
    w.t0 = (int64_t)w.n * CB_C;
    w.len = (int)min((int64_t)CB_C, p.S - w.t0);
    return w;
}

// index of element c of token row r of unit w in a (B, S, H, D) tensor
__device__ __forceinline__ int64_t cb_idx(const CbArgs &p, const CbUnit &w, int r, int D, int c) {
    return (((int64_t)w.b * p.S + w.t0 + r) * p.H + w.h) * D + c;
}

// ---------------------------------------------------------------- per chunk: G, P, M, T, W, U, Q e^G, Kd
__host__ __device__ inline size_t cb_prep_smem(int Dk, int Dv) {
    const int LK = cb_pad8(Dk) + 1, LV = cb_pad8(Dv) + 1, LC = CB_C + 1;
    return sizeof(float) * ((size_t)3 * CB_C * LK + (size_t)CB_C * LV + 2 * CB_C * LC + CB_C);
}

template <typename T>
__global__ void __launch_bounds__(CB_NTC) cb_prep_kernel(CbArgs p) {
    extern __shared__ __align__(16) float cb_sm[];
    const int tid = threadIdx.x;
    const CbUnit w = cb_unit(p, blockIdx.x);
    const int C = CB_C, Dk = p.Dk, Dv = p.Dv, len = w.len;
    const int LK = cb_pad8(Dk) + 1, LV = cb_pad8(Dv) + 1, LC = C + 1;
    float *sK = cb_sm, *sQ = sK + C * LK, *sG = sQ + C * LK, *sV = sG + C * LK;
    float *sP = sV + C * LV, *sT = sP + C * LC, *sb = sT + C * LC;
    const CbRec R = cb_rec(Dk, Dv, p.nslice);
    float *rec = p.ws + w.u * R.size;
    const bool ok = in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds);

    // inputs; rows past the sequence end: zero, no decay (the raw decay input first, log(alpha) below)
    const int64_t rk = (int64_t)p.H * Dk, rv = (int64_t)p.H * Dv;
    cb_load_rows(sK, LK, (const T *)p.k + cb_idx(p, w, 0, Dk, 0), rk, C, len, Dk, Dk);
    cb_load_rows(sQ, LK, (const T *)p.q + cb_idx(p, w, 0, Dk, 0), rk, C, len, Dk, Dk);
    if (p.log_decay)
        cb_load_rows(sG, LK, p.log_decay + cb_idx(p, w, 0, Dk, 0), rk, C, len, Dk, Dk);
    else
        cb_load_rows(sG, LK, (const T *)p.z + cb_idx(p, w, 0, Dk, 0), rk, C, len, Dk, Dk);
    cb_load_rows(sV, LV, (const T *)p.v + cb_idx(p, w, 0, Dv, 0), rv, C, len, Dv, Dv);
    if (tid < C) sb[tid] = tid < len ? load_elem((const T *)p.beta, cb_idx(p, w, tid, 1, 0)) : 0.f;
    __syncthreads();
    for (int c = tid; c < Dk; c += CB_NTC) {  // G: cumulative sum of log(alpha) over the chunk's rows
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            const float x = sG[r * LK + c];
            acc += r < len ? (p.log_decay ? clamp_log_decay(x, p.g_min) : log_alpha_of(x, p.g_min)) : 0.f;
            sG[r * LK + c] = acc;
        }
    }
    __syncthreads();
    for (int idx = tid; ok && idx < C * Dk; idx += CB_NTC) {
        const int r = idx / Dk, c = idx - r * Dk;
        const float G = sG[r * LK + c];
        rec[R.G + idx] = G;
        rec[R.Qg + idx] = sQ[r * LK + c] * cb_exp(G);
        rec[R.Kd + idx] = sK[r * LK + c] * cb_exp(sG[(C - 1) * LK + c] - G);
    }
    // P (i < r) and M (i <= r) over the triangle of pairs; neighbouring threads take neighbouring i
    for (int pi = tid; pi < C * (C + 1) / 2; pi += CB_NTC) {
        int r = (int)((sqrtf(8.f * (float)pi + 1.f) - 1.f) * 0.5f);
        while (r > 0 && r * (r + 1) / 2 > pi) --r;
        while ((r + 1) * (r + 2) / 2 <= pi) ++r;
        const int i = pi - r * (r + 1) / 2;
        const float *kr = sK + r * LK, *ki = sK + i * LK, *qr = sQ + r * LK, *gr = sG + r * LK, *gi = sG + i * LK;
        float pk = 0.f, mq = 0.f;
        for (int c = 0; c < Dk; ++c) {
            const float e = cb_exp(gr[c] - gi[c]) * ki[c];
            pk = fmaf(kr[c], e, pk);
            mq = fmaf(qr[c], e, mq);
        }
        pk = i < r ? pk : 0.f;
        sP[r * LC + i] = pk;
        if (ok) {
            rec[R.P + r * C + i] = pk;
            rec[R.M + r * C + i] = mq;
        }
    }
    for (int idx = tid; idx < C * C; idx += CB_NTC) {  // the upper triangles
        const int r = idx / C, i = idx - r * C;
        if (i > r) {
            sP[r * LC + i] = 0.f;
            if (ok) {
                rec[R.P + idx] = 0.f;
                rec[R.M + idx] = 0.f;
            }
        }
    }
    __syncthreads();
    // T = (I + Diag(beta) P)^{-1}: column j by forward substitution (thread j; entries above the
    // diagonal come out as exact zeros)
    if (tid < C) {
        const int j = tid;
        for (int r = 0; r < C; ++r) {
            const float br = sb[r];
            const float *pr = sP + r * LC;
            float a0 = r == j ? 1.f : 0.f, a1 = 0.f;
            int m = 0;
            for (; m + 1 < r; m += 2) {
                a0 = fmaf(-br * pr[m], sT[m * LC + j], a0);
                a1 = fmaf(-br * pr[m + 1], sT[(m + 1) * LC + j], a1);
            }
            if (m < r) a0 = fmaf(-br * pr[m], sT[m * LC + j], a0);
            sT[r * LC + j] = a0 + a1;
        }
    }
    __syncthreads();
    for (int idx = tid; ok && idx < C * C; idx += CB_NTC) {
        const int r = idx / C, m = idx - r * C;
        rec[R.T + idx] = sT[r * LC + m];
    }
    // beta K e^G and beta V in place: the right-hand sides of W and U
    for (int idx = tid; idx < C * Dk; idx += CB_NTC) {
        const int r = idx / Dk, c = idx - r * Dk;
        sK[r * LK + c] = sb[r] * sK[r * LK + c] * cb_exp(sG[r * LK + c]);
    }
    for (int idx = tid; idx < C * Dv; idx += CB_NTC) {
        const int r = idx / Dv, j = idx - r * Dv;
        sV[r * LV + j] *= sb[r];
    }
    __syncthreads();
    // [W | U] = T [beta K e^G | beta V]: a thread per column (D_k + D_v <= 256) and every other group of
    // four rows (the two halves of the CTA take alternate groups, so that both get short and long ones)
    static_assert(CB_NTC == 512, "two threads per column");
    const int col = tid & 255, half = tid >> 8;
    if (ok && col < Dk + Dv) {
        const bool isw = col < Dk;
        const float *Bc = isw ? sK + col : sV + (col - Dk);
        const int ldb = isw ? LK : LV, ldd = isw ? Dk : Dv;
        float *dst = isw ? rec + R.W + col : rec + R.U + (col - Dk);
        for (int g = 0; g < C / 8; ++g) {
            const int r0 = 4 * (2 * g + half);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            for (int m = 0; m <= r0 + 3; ++m) {
                const float x = Bc[m * ldb];
                a0 = fmaf(sT[r0 * LC + m], x, a0);
                a1 = fmaf(sT[(r0 + 1) * LC + m], x, a1);
                a2 = fmaf(sT[(r0 + 2) * LC + m], x, a2);
                a3 = fmaf(sT[(r0 + 3) * LC + m], x, a3);
            }
            dst[(int64_t)r0 * ldd] = a0;
            dst[(int64_t)(r0 + 1) * ldd] = a1;
            dst[(int64_t)(r0 + 2) * ldd] = a2;
            dst[(int64_t)(r0 + 3) * ldd] = a3;
        }
    }
}

// ---------------------------------------------------------------- the state chains, per 16 value columns
// Row pitches of the chain kernels: multiples of 4 floats (16-byte copies) that are 4 mod 8, so that the
// eight rows a warp reads at one column fall in different banks.
__host__ __device__ inline int cb_lk(int Dk) { return cb_pad8(Dk) + 4; }
constexpr int CB_LCC = CB_C + 4;
// forward stages: {W, Kd [C][LK], U columns [C][16], last row of G [Dk]}, two of them
__host__ __device__ inline int cb_fstage(int Dk) {
    return (2 * CB_C * cb_lk(Dk) + CB_C * CB_VS + Dk + 3) & ~3;
}
__host__ __device__ inline size_t cb_chain_smem(int Dk) {
    const int LK = cb_lk(Dk), LC = CB_LCC, Dk4 = (Dk + 3) & ~3;
    // forward: two stages, V' [C][16], S [Dk][16];  backward: M [C][LC], Kd [C][LK], S [Dk][16] (one copy
    // group), Q e^G, W [C][LK], last row of G (the other), dO, dV' [C][16], dS [Dk][16]
    const size_t fwd = (size_t)2 * cb_fstage(Dk) + CB_C * CB_VS + (size_t)Dk * CB_VS;
    const size_t bwd = (size_t)CB_C * LC + (size_t)3 * CB_C * LK + (size_t)2 * Dk * CB_VS + Dk4 + 2 * CB_C * CB_VS;
    return sizeof(float) * (fwd > bwd ? fwd : bwd);
}

// Forward over the chunks of one (b, h) for value columns j0 .. j0 + 15: the state entering every chunk
// and V' go to the chunk's record.  The next chunk's blocks are copied in while this one is computed.
__global__ void __launch_bounds__(CB_NT) cb_fwd_chain_kernel(CbArgs p) {
    extern __shared__ __align__(16) float cb_sm[];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int j0 = blockIdx.y * CB_VS;
    const int C = CB_C, Dk = p.Dk, Dv = p.Dv, LK = cb_lk(Dk), FS = cb_fstage(Dk);
    float *sVp = cb_sm + 2 * FS, *sS = sVp + C * CB_VS;
    const CbRec R = cb_rec(Dk, Dv, p.nslice);
    auto stage = [&](int n) {  // chunk n's blocks into stage n & 1, one copy group
        const float *rec = p.ws + (bh * p.Nc + n) * R.size;
        float *st = cb_sm + (n & 1) * FS;
        if (in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds)) {
            cb_copy(st, LK, rec + R.W, C, Dk, C, Dk);
            cb_copy(st + C * LK, LK, rec + R.Kd, C, Dk, C, Dk);
            cb_copy_cols(st + 2 * C * LK, rec + R.U, C, Dv, j0);
            cb_copy(st + 2 * C * LK + C * CB_VS, Dk, rec + R.G + (int64_t)(C - 1) * Dk, 1, Dk, 1, Dk);
        }
        cp_async_commit_group();
    };
    for (int idx = tid; idx < Dk * CB_VS; idx += CB_NT) {
        const int c = idx / CB_VS, j = idx - c * CB_VS;
        sS[idx] = (p.S0 && j0 + j < Dv) ? p.S0[(bh * Dk + c) * Dv + j0 + j] : 0.f;
    }
    stage(0);
    for (int n = 0; n < p.Nc; ++n) {
        if (n + 1 < p.Nc) stage(n + 1);
        else cp_async_commit_group();
        cp_async_wait<1>();  // chunk n's copies
        __syncthreads();
        const float *st = cb_sm + (n & 1) * FS;
        const float *sW = st, *sKd = st + C * LK, *sU = st + 2 * C * LK, *sGl = sU + C * CB_VS;
        float *rec = p.ws + (bh * p.Nc + n) * R.size;
        const bool ok = in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds);
        for (int idx = tid; ok && idx < Dk * CB_VS; idx += CB_NT) {  // the state entering chunk n
            const int c = idx / CB_VS, j = idx - c * CB_VS;
            if (j0 + j < Dv) rec[R.S + (int64_t)c * Dv + j0 + j] = sS[idx];
        }
        {  // V' = U - W S: thread (row r, four columns)
            const int r = tid >> 2, jq = (tid & 3) * 4;
            float a[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) a[e] = sU[r * CB_VS + jq + e];
            for (int c = 0; c < Dk; ++c) {
                const float wv = sW[r * LK + c];
                const float4 s = *reinterpret_cast<const float4 *>(sS + c * CB_VS + jq);
                a[0] = fmaf(-wv, s.x, a[0]);
                a[1] = fmaf(-wv, s.y, a[1]);
                a[2] = fmaf(-wv, s.z, a[2]);
                a[3] = fmaf(-wv, s.w, a[3]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sVp[r * CB_VS + jq + e] = a[e];
                if (ok && j0 + jq + e < Dv) rec[R.Vp + (int64_t)r * Dv + j0 + jq + e] = a[e];
            }
        }
        __syncthreads();
        if (tid < 2 * Dk) {  // S <- Diag(gamma) S + Kd^T V': thread (key row c, eight columns)
            const int c = tid >> 1, jh = (tid & 1) * 8;
            const float gam = cb_exp(sGl[c]);
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = gam * sS[c * CB_VS + jh + e];
            for (int r = 0; r < C; ++r) {
                const float kd = sKd[r * LK + c];
                const float4 v0 = *reinterpret_cast<const float4 *>(sVp + r * CB_VS + jh);
                const float4 v1 = *reinterpret_cast<const float4 *>(sVp + r * CB_VS + jh + 4);
                a[0] = fmaf(kd, v0.x, a[0]);
                a[1] = fmaf(kd, v0.y, a[1]);
                a[2] = fmaf(kd, v0.z, a[2]);
                a[3] = fmaf(kd, v0.w, a[3]);
                a[4] = fmaf(kd, v1.x, a[4]);
                a[5] = fmaf(kd, v1.y, a[5]);
                a[6] = fmaf(kd, v1.z, a[6]);
                a[7] = fmaf(kd, v1.w, a[7]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) sS[c * CB_VS + jh + e] = a[e];
        }
        __syncthreads();  // stage n & 1 takes chunk n + 2 next
    }
}

// Backward over the chunks of one (b, h) for value columns j0 .. j0 + 15: dS_next, dV' and the
// partial dgamma of every chunk go to its record; dL/dS_0 to the output.  The blocks the first half of
// a step reads (M, Kd, S) and those of its second half (Q e^G, W, G) are two copy groups, each refilled
// with the previous chunk's as soon as its half is done.
template <typename T>
__global__ void __launch_bounds__(CB_NT) cb_bwd_chain_kernel(CbArgs p) {
    extern __shared__ __align__(16) float cb_sm[];
    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int sl = blockIdx.y, j0 = sl * CB_VS;
    const int C = CB_C, Dk = p.Dk, Dv = p.Dv, LK = cb_lk(Dk), LC = CB_LCC, Dk4 = (Dk + 3) & ~3;
    const int b = (int)(bh / p.H), h = (int)(bh - (int64_t)b * p.H);
    float *sM = cb_sm, *sKd = sM + C * LC, *sSn = sKd + C * LK;
    float *sQg = sSn + Dk * CB_VS, *sW = sQg + C * LK, *sGl = sW + C * LK;
    float *sdO = sGl + Dk4, *sdV = sdO + C * CB_VS, *sdS = sdV + C * CB_VS;
    const CbRec R = cb_rec(Dk, Dv, p.nslice);
    auto rec_of = [&](int n) { return p.ws + (bh * p.Nc + n) * R.size; };
    auto stage_a = [&](int n) {
        const float *rec = rec_of(n);
        if (in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds)) {
            cb_copy(sM, LC, rec + R.M, C, C, C, C);
            cb_copy(sKd, LK, rec + R.Kd, C, Dk, C, Dk);
            cb_copy_cols(sSn, rec + R.S, Dk, Dv, j0);
        }
        cp_async_commit_group();
    };
    auto stage_b = [&](int n) {
        const float *rec = rec_of(n);
        if (in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds)) {
            cb_copy(sQg, LK, rec + R.Qg, C, Dk, C, Dk);
            cb_copy(sW, LK, rec + R.W, C, Dk, C, Dk);
            cb_copy(sGl, Dk, rec + R.G + (int64_t)(C - 1) * Dk, 1, Dk, 1, Dk);
        }
        cp_async_commit_group();
    };
    float pre[C * CB_VS / CB_NT];  // this thread's dO elements of a chunk: element tid + CB_NT u of [C][16]
    auto load_do = [&](int n) {
        const int64_t t0 = (int64_t)n * C;
        const int len = (int)min((int64_t)C, p.S - t0);
#pragma unroll
        for (int u = 0; u < C * CB_VS / CB_NT; ++u) {
            const int idx = tid + u * CB_NT, r = idx / CB_VS, j = idx - r * CB_VS;
            pre[u] = (r < len && j0 + j < Dv)
                         ? load_elem((const T *)p.dO, (((int64_t)b * p.S + t0 + r) * p.H + h) * Dv + j0 + j)
                         : 0.f;
        }
    };
    auto store_do = [&]() {
#pragma unroll
        for (int u = 0; u < C * CB_VS / CB_NT; ++u) sdO[tid + u * CB_NT] = pre[u];
    };
    for (int idx = tid; idx < Dk * CB_VS; idx += CB_NT) {
        const int c = idx / CB_VS, j = idx - c * CB_VS;
        sdS[idx] = (p.dST && j0 + j < Dv) ? p.dST[(bh * Dk + c) * Dv + j0 + j] : 0.f;
    }
    stage_a(p.Nc - 1);
    stage_b(p.Nc - 1);
    load_do(p.Nc - 1);
    store_do();
    for (int n = p.Nc - 1; n >= 0; --n) {
        float *rec = rec_of(n);
        const bool ok = in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds);
        cp_async_wait<1>();  // M, Kd and S of chunk n
        __syncthreads();
        for (int idx = tid; ok && idx < Dk * CB_VS; idx += CB_NT) {  // dS_next of chunk n
            const int c = idx / CB_VS, j = idx - c * CB_VS;
            if (j0 + j < Dv) rec[R.dS + (int64_t)c * Dv + j0 + j] = sdS[idx];
        }
        for (int c = tid; ok && c < Dk; c += CB_NT) {  // this slice's part of dgamma = rowsum(dS_next * S)
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < CB_VS; ++j) s = fmaf(sdS[c * CB_VS + j], sSn[c * CB_VS + j], s);
            rec[R.dgam + (int64_t)sl * Dk + c] = s;
        }
        {  // dV' = M^T dO + Kd dS_next: thread (row r, four columns)
            const int r = tid >> 2, jq = (tid & 3) * 4;
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int i = r; i < C; ++i) {
                const float mv = sM[i * LC + r];
                const float4 d = *reinterpret_cast<const float4 *>(sdO + i * CB_VS + jq);
                a[0] = fmaf(mv, d.x, a[0]);
                a[1] = fmaf(mv, d.y, a[1]);
                a[2] = fmaf(mv, d.z, a[2]);
                a[3] = fmaf(mv, d.w, a[3]);
            }
            for (int c = 0; c < Dk; ++c) {
                const float kd = sKd[r * LK + c];
                const float4 d = *reinterpret_cast<const float4 *>(sdS + c * CB_VS + jq);
                a[0] = fmaf(kd, d.x, a[0]);
                a[1] = fmaf(kd, d.y, a[1]);
                a[2] = fmaf(kd, d.z, a[2]);
                a[3] = fmaf(kd, d.w, a[3]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sdV[r * CB_VS + jq + e] = a[e];
                if (ok && j0 + jq + e < Dv) rec[R.dVp + (int64_t)r * Dv + j0 + jq + e] = a[e];
            }
        }
        __syncthreads();  // M, Kd and S of chunk n are read: the previous chunk's come in
        if (n > 0) {
            stage_a(n - 1);
            load_do(n - 1);
        } else {
            cp_async_commit_group();
        }
        cp_async_wait<1>();  // Q e^G, W and G of chunk n
        __syncthreads();
        if (tid < 2 * Dk) {  // dS <- Diag(gamma) dS_next + (Q e^G)^T dO - W^T dV'
            const int c = tid >> 1, jh = (tid & 1) * 8;
            const float gam = cb_exp(sGl[c]);
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = gam * sdS[c * CB_VS + jh + e];
            for (int r = 0; r < C; ++r) {
                const float qg = sQg[r * LK + c], wv = sW[r * LK + c];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    a[e] = fmaf(qg, sdO[r * CB_VS + jh + e], fmaf(-wv, sdV[r * CB_VS + jh + e], a[e]));
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) sdS[c * CB_VS + jh + e] = a[e];
        }
        __syncthreads();  // Q e^G, W, G and dO of chunk n are read
        if (n > 0) {
            stage_b(n - 1);
            store_do();
        } else {
            cp_async_commit_group();
        }
    }
    __syncthreads();
    if (p.dS0 && in_bounds(p.dS0 + bh * Dk * Dv, (size_t)Dk * Dv * 4, p.dS0, p.ns_bytes, p.bounds))
        for (int idx = tid; idx < Dk * CB_VS; idx += CB_NT) {
            const int c = idx / CB_VS, j = idx - c * CB_VS;
            if (j0 + j < Dv) p.dS0[(bh * Dk + c) * Dv + j0 + j] = sdS[idx];
        }
}

// ---------------------------------------------------------------- per chunk: the matrix gradients
// dQg, dW, dKd, dM, dT, dBv (-> dv), dBk (-> dKg), dA and dbeta.
__host__ __device__ inline size_t cb_mat_smem(int Dk, int Dv) {
    const int Dkp = cb_pad8(Dk), LK = Dkp + 1, LV = cb_pad8(Dv) + 1, LC = CB_C + 1;
    const int LVC = cb_max(LV, LC);
    // S or dS_next [Dk][Dv]; later V and K e^G [C][LV + LK]; later P [C][LC]
    const size_t big = cb_max(cb_max(Dkp * LV, CB_C * (LV + LK)), CB_C * LC);
    return sizeof(float) * (big + (size_t)CB_C * LVC      // dO, later T
                            + (size_t)CB_C * LV            // dV'
                            + (size_t)CB_C * LVC           // V', later dT
                            + (size_t)CB_C * LK            // dW
                            + (size_t)CB_C * LC            // dM, later dT T^T
                            + 2 * CB_C);                   // beta, dbeta
}

template <typename T>
__global__ void __launch_bounds__(CB_NTC) cb_grad_mat_kernel(CbArgs p) {
    extern __shared__ __align__(16) float cb_sm[];
    const int tid = threadIdx.x;
    const CbUnit w = cb_unit(p, blockIdx.x);
    const int C = CB_C, Dk = p.Dk, Dv = p.Dv, len = w.len;
    const int Dkp = cb_pad8(Dk), Dvp = cb_pad8(Dv), LK = Dkp + 1, LV = Dvp + 1, LC = C + 1;
    const int LVC = cb_max(LV, LC);
    float *sX = cb_sm;
    float *sdO = sX + cb_max(cb_max(Dkp * LV, C * (LV + LK)), C * LC);
    float *sdV = sdO + C * LVC, *sV = sdV + C * LV, *sdW = sV + C * LVC, *sdM = sdW + C * LK;
    float *sb = sdM + C * LC, *sdb = sb + C;
    const CbRec R = cb_rec(Dk, Dv, p.nslice);
    float *rec = p.ws + w.u * R.size;
    const bool ok = in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds);
    if (!ok) return;

    // S [c][j], dV' [r][j], V' [r][j] (copies), dO [r][j] (zero padding to multiples of 8)
    cb_copy(sX, LV, rec + R.S, Dk, Dv, Dkp, Dvp);
    cb_copy(sdV, LV, rec + R.dVp, C, Dv, C, Dvp);
    cb_copy(sV, LV, rec + R.Vp, C, Dv, C, Dvp);
    cp_async_commit_group();
    cb_load_rows(sdO, LV, (const T *)p.dO + cb_idx(p, w, 0, Dv, 0), (int64_t)p.H * Dv, C, len, Dv, Dvp);
    if (tid < C) {
        sb[tid] = tid < len ? load_elem((const T *)p.beta, cb_idx(p, w, tid, 1, 0)) : 0.f;
        sdb[tid] = 0.f;
    }
    cp_async_wait<0>();
    __syncthreads();
    // dQg = dO S^T -> record (Q e^G's place);  dW = -dV' S^T -> shared
    cb_mm<false, false>(sdO, LV, sX, LV, C, Dkp, Dvp, [&](int r, int c, float v) {
        if (c < Dk) rec[R.Qg + (int64_t)r * Dk + c] = v;
    });
    cb_mm<false, false>(sdV, LV, sX, LV, C, Dkp, Dvp, [&](int r, int c, float v) { sdW[r * LK + c] = -v; });
    __syncthreads();
    // dS_next [c][j] over S
    cb_copy(sX, LV, rec + R.dS, Dk, Dv, Dkp, Dvp);
    cp_async_commit_group();
    cp_async_wait<0>();
    __syncthreads();
    // dKd = V' dS_next^T -> record (Kd's place);  dM = dO V'^T (i <= r) -> shared and record (M's place)
    cb_mm<false, false>(sV, LV, sX, LV, C, Dkp, Dvp, [&](int r, int c, float v) {
        if (c < Dk) rec[R.Kd + (int64_t)r * Dk + c] = v;
    });
    cb_mm<false, false>(sdO, LV, sV, LV, C, C, Dvp, [&](int r, int i, float v) {
        v = i <= r ? v : 0.f;
        sdM[r * LC + i] = v;
        rec[R.M + r * C + i] = v;
    });
    __syncthreads();
    // V [m][j] and K e^G [m][c] over S's space; T [r][m] over dO's
    float *sVin = sX, *sKg = sX + C * LV, *sT = sdO, *sdT = sV;
    cb_copy(sT, LC, rec + R.T, C, C, C, C);
    cp_async_commit_group();
    cb_load_rows(sVin, LV, (const T *)p.v + cb_idx(p, w, 0, Dv, 0), (int64_t)p.H * Dv, C, len, Dv, Dvp);
    cb_load_rows(sKg, LK, (const T *)p.k + cb_idx(p, w, 0, Dk, 0), (int64_t)p.H * Dk, C, len, Dk, Dkp, rec + R.G);
    cp_async_wait<0>();
    __syncthreads();
    // dT = (dV' V^T + dW (K e^G)^T) Diag(beta), in two passes over the same threads' elements
    cb_mm<false, false>(sdV, LV, sVin, LV, C, C, Dvp, [&](int r, int m, float v) { sdT[r * LC + m] = v; });
    cb_mm<false, false>(sdW, LK, sKg, LK, C, C, Dkp, [&](int r, int m, float v) {
        sdT[r * LC + m] = (sdT[r * LC + m] + v) * sb[m];
    });
    __syncthreads();
    // dBv^T = dV'^T T: dv = beta dBv; dbeta += rowsum(dBv * V).  dBk^T = dW^T T: dKg = beta dBk -> record
    // (W's place); dbeta += rowsum(dBk * K e^G).  (Threads next to each other take neighbouring rows m.)
    cb_mm<true, true>(sdV, LV, sT, LC, Dvp, C, C, [&](int j, int m, float v) {
        if (j < Dv) {
            if (m < len) p.dv[cb_idx(p, w, m, Dv, j)] = sb[m] * v;
            atomicAdd(sdb + m, v * sVin[m * LV + j]);
        }
    });
    cb_mm<true, true>(sdW, LK, sT, LC, Dkp, C, C, [&](int c, int m, float v) {
        if (c < Dk) {
            rec[R.W + (int64_t)m * Dk + c] = sb[m] * v;
            atomicAdd(sdb + m, v * sKg[m * LK + c]);
        }
    });
    __syncthreads();
    // P over S's space (V and K e^G are read) while X = dT T^T goes to dM's
    float *sP = sX, *sX1 = sdM;
    cb_copy(sP, LC, rec + R.P, C, C, C, C);
    cp_async_commit_group();
    cb_mm<false, false>(sdT, LC, sT, LC, C, C, C, [&](int r, int m, float v) { sX1[r * LC + m] = v; });
    cp_async_wait<0>();
    __syncthreads();
    // dA^T = -X^T T (dA[r][i], i < r) -> record (T's place); dbeta += rowsum(dA * P)
    cb_mm<true, true>(sX1, LC, sT, LC, C, C, C, [&](int i, int r, float v) {
        const float a = i < r ? -v : 0.f;
        rec[R.T + r * C + i] = a;
        atomicAdd(sdb + r, a * sP[r * LC + i]);
    });
    __syncthreads();
    if (tid < len) p.dbeta[cb_idx(p, w, tid, 1, 0)] = sdb[tid];
}

// ---------------------------------------------------------------- per chunk: the decayed-product gradients
__host__ __device__ inline size_t cb_pair_smem(int Dk) {
    const int LK = cb_pad8(Dk) + 1, LC = CB_C + 1;
    return sizeof(float) * ((size_t)5 * CB_C * LK + 2 * CB_C * LC + CB_C);
}

template <typename T>
__global__ void __launch_bounds__(CB_NTC) cb_grad_pair_kernel(CbArgs p) {
    extern __shared__ __align__(16) float cb_sm[];
    const int tid = threadIdx.x;
    const CbUnit w = cb_unit(p, blockIdx.x);
    const int C = CB_C, Dk = p.Dk, len = w.len;
    const int LK = cb_pad8(Dk) + 1, LC = C + 1;
    float *sG = cb_sm, *sK = sG + C * LK, *sQ = sK + C * LK, *sdk = sQ + C * LK, *sdG = sdk + C * LK;
    float *sdA = sdG + C * LK, *sdM = sdA + C * LC, *sb = sdM + C * LC;
    const CbRec R = cb_rec(Dk, p.Dv, p.nslice);
    const float *rec = p.ws + w.u * R.size;
    if (!in_bounds(rec, (size_t)R.size * 4, p.ws, p.ws_bytes, p.bounds)) return;

    const int64_t rk = (int64_t)p.H * Dk, row0 = cb_idx(p, w, 0, Dk, 0);
    cb_copy(sG, LK, rec + R.G, C, Dk, C, Dk);
    cb_copy(sdA, LC, rec + R.T, C, C, C, C);
    cb_copy(sdM, LC, rec + R.M, C, C, C, C);
    cp_async_commit_group();
    cb_load_rows(sK, LK, (const T *)p.k + row0, rk, C, len, Dk, Dk);
    cb_load_rows(sQ, LK, (const T *)p.q + row0, rk, C, len, Dk, Dk);
    if (tid < C) sb[tid] = tid < len ? load_elem((const T *)p.beta, cb_idx(p, w, tid, 1, 0)) : 0.f;
    cp_async_wait<0>();
    __syncthreads();
    // row roles: token r against the earlier tokens i <= r; dq is final here
    for (int idx = tid; idx < C * Dk; idx += CB_NTC) {
        const int r = idx / Dk, c = idx - r * Dk;
        const float dQg = rec[R.Qg + idx], dKg = rec[R.W + idx], dKd = rec[R.Kd + idx];  // (in flight meanwhile)
        const float Gr = sG[r * LK + c];
        float xa = 0.f, y = 0.f;
        for (int i = 0; i <= r; ++i) {
            const float e = cb_exp(Gr - sG[i * LK + c]) * sK[i * LK + c];
            xa = fmaf(sdA[r * LC + i], e, xa);
            y = fmaf(sdM[r * LC + i], e, y);
        }
        const float eG = cb_exp(Gr), eD = cb_exp(sG[(C - 1) * LK + c] - Gr);
        const float kv = sK[r * LK + c], qv = sQ[r * LK + c], bxa = sb[r] * xa;
        if (r < len) p.dq[cb_idx(p, w, r, Dk, c)] = fmaf(dQg, eG, y);
        sdk[r * LK + c] = dKg * eG + dKd * eD + bxa;
        sdG[r * LK + c] = qv * (dQg * eG + y) + kv * (dKg * eG - dKd * eD + bxa);
    }
    __syncthreads();
    // column roles: token i against the later tokens r >= i
    for (int idx = tid; idx < C * Dk; idx += CB_NTC) {
        const int i = idx / Dk, c = idx - i * Dk;
        const float Gi = sG[i * LK + c];
        float x = 0.f;
        for (int r = i; r < C; ++r) {
            const float e = cb_exp(sG[r * LK + c] - Gi);
            x = fmaf(fmaf(sb[r] * sdA[r * LC + i], sK[r * LK + c], sdM[r * LC + i] * sQ[r * LK + c]), e, x);
        }
        sdk[i * LK + c] += x;
        sdG[i * LK + c] -= sK[i * LK + c] * x;
    }
    __syncthreads();
    // dKd over dA's and dM's space, the raw decay input over Q's
    float *sdKd = sdA, *sZ = sQ;
    cb_copy(sdKd, LK, rec + R.Kd, C, Dk, C, Dk);
    cp_async_commit_group();
    if (p.log_decay)
        cb_load_rows(sZ, LK, p.log_decay + row0, rk, C, len, Dk, Dk);
    else
        cb_load_rows(sZ, LK, (const T *)p.z + row0, rk, C, len, Dk, Dk);
    cp_async_wait<0>();
    __syncthreads();
    // per channel: the last row's gamma and Kd terms, the reverse cumulative sum, dz and dk
    for (int c = tid; c < Dk; c += CB_NTC) {
        const float Gl = sG[(C - 1) * LK + c];
        float s = 0.f;
        for (int r = 0; r < C; ++r) s = fmaf(sdKd[r * LK + c] * sK[r * LK + c], cb_exp(Gl - sG[r * LK + c]), s);
        float dgam = 0.f;
        for (int sl = 0; sl < p.nslice; ++sl) dgam += rec[R.dgam + (int64_t)sl * Dk + c];
        float acc = s + dgam * cb_exp(Gl);
        for (int r = C - 1; r >= 0; --r) {
            acc += sdG[r * LK + c];
            if (r < len) {
                const int64_t i = cb_idx(p, w, r, Dk, c);
                const float raw = sZ[r * LK + c];
                float dz;
                if (p.log_decay) {
                    dz = (raw >= p.g_min && raw <= 0.f) ? acc : 0.f;  // a clamped input has no gradient
                } else {  // g = g_min sigmoid(z): dg/dz = g (1 - g / g_min)
                    const float g = log_alpha_of(raw, p.g_min);
                    dz = acc * g * (1.0f - g / p.g_min);
                }
                p.dz[i] = dz;
                p.dk[i] = sdk[r * LK + c];
            }
        }
    }
}

}  // namespace

// ================================================================ host side
size_t chunk_bwd_workspace(int64_t B, int64_t S, int H, int Dk, int Dv) {
    const int nslice = (Dv + CB_VS - 1) / CB_VS;
    const int64_t Nc = (S + CB_C - 1) / CB_C;
    return (size_t)B * H * Nc * (size_t)cb_rec(Dk, Dv, nslice).size * sizeof(float);
}

kda_status_t launch_chunk_bwd(const kda_recurrent_bwd_args &a, cudaStream_t st) {
    CbArgs p;
    p.S = a.S;
    p.H = a.H;
    p.Dk = a.D_k;
    p.Dv = a.D_v;
    p.Nc = (int)((a.S + CB_C - 1) / CB_C);
    p.nslice = (a.D_v + CB_VS - 1) / CB_VS;
    p.q = a.q; p.k = a.k; p.v = a.v; p.z = a.z; p.beta = a.beta; p.dO = a.d_o;
    p.log_decay = a.log_decay;
    p.g_min = a.g_min;
    p.S0 = a.initial_state;
    p.dST = a.d_final_state;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv; p.dbeta = a.dbeta; p.dz = a.dz; p.dS0 = a.d_initial_state;
    const int64_t nbh = a.B * a.H;
    p.ws = reinterpret_cast<float *>(a.workspace);
    p.ws_bytes = chunk_bwd_workspace(a.B, a.S, a.H, a.D_k, a.D_v);
    p.nk_bytes = (size_t)nbh * a.S * a.D_k * 4;
    p.nv_bytes = (size_t)nbh * a.S * a.D_v * 4;
    p.nb_bytes = (size_t)nbh * a.S * 4;
    p.ns_bytes = (size_t)nbh * a.D_k * a.D_v * 4;
    p.bounds = device_bounds_counter();
    if (a.S == 0) {
        if (a.d_initial_state) {
            if (a.d_final_state)
                cudaMemcpyAsync(a.d_initial_state, a.d_final_state, p.ns_bytes, cudaMemcpyDeviceToDevice, st);
            else
                cudaMemsetAsync(a.d_initial_state, 0, p.ns_bytes, st);
        }
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? KDA_OK : fail(KDA_ERR_CUDA, "chunk backward: %s", cudaGetErrorString(e));
    }
    const int64_t units = nbh * p.Nc;
    if (units > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "chunk backward: B*H*chunks too large");
    const dim3 gu((unsigned)units), gc((unsigned)nbh, (unsigned)p.nslice);
    const size_t s1 = cb_prep_smem(a.D_k, a.D_v), s2 = cb_chain_smem(a.D_k), s4 = cb_mat_smem(a.D_k, a.D_v),
                 s5 = cb_pair_smem(a.D_k);
    auto go = [&](auto prep, auto bchain, auto mat, auto pair) -> kda_status_t {
        cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
        cudaFuncSetAttribute(cb_fwd_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
        cudaFuncSetAttribute(bchain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
        cudaFuncSetAttribute(mat, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s4);
        cudaFuncSetAttribute(pair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s5);
        kda_status_t s;
        prep<<<gu, CB_NTC, s1, st>>>(p);
        if ((s = check_launch("cb_prep_kernel")) != KDA_OK) return s;
        cb_fwd_chain_kernel<<<gc, CB_NT, s2, st>>>(p);
        if ((s = check_launch("cb_fwd_chain_kernel")) != KDA_OK) return s;
        bchain<<<gc, CB_NT, s2, st>>>(p);
        if ((s = check_launch("cb_bwd_chain_kernel")) != KDA_OK) return s;
        mat<<<gu, CB_NTC, s4, st>>>(p);
        if ((s = check_launch("cb_grad_mat_kernel")) != KDA_OK) return s;
        pair<<<gu, CB_NTC, s5, st>>>(p);
        return check_launch("cb_grad_pair_kernel");
    };
    if (a.dtype == KDA_F32)
        return go(cb_prep_kernel<float>, cb_bwd_chain_kernel<float>, cb_grad_mat_kernel<float>,
                  cb_grad_pair_kernel<float>);
    return go(cb_prep_kernel<__nv_bfloat16>, cb_bwd_chain_kernel<__nv_bfloat16>,
              cb_grad_mat_kernel<__nv_bfloat16>, cb_grad_pair_kernel<__nv_bfloat16>);
}

}  // namespace kda
