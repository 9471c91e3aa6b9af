// Gradient of the KDA recurrence (exact fp32, recurrent form) for training.
//
// The token step of Eq. 1 (Kimi Linear report, section 3) with the readout
// from the updated state ("KDA Recurrence" page) is
//   X_t = Diag(alpha_t) S_{t-1},  p_t = X_t^T k_t,  u_t = v_t - p_t,
//   S_t = X_t + beta_t k_t u_t^T,  o_t = S_t^T q_t,
// and reverse-mode differentiation of those lines, from the last token back,
// is (dS = dL/dS_t, accumulated):
//   dS += q_t do_t^T;  dq_t = S_t do_t
//   dr = dS^T k_t;  dk_t = dS (beta_t u_t);  dbeta_t = dr . u_t;  dv_t = beta_t dr
//   dX = dS - beta_t k_t dr^T;  dk_t += X_t (-beta_t dr)
//   dalpha_t = rowsum(dX * S_{t-1});  dS <- Diag(alpha_t) dX
// with dlog(alpha) = dalpha alpha and dz = dlog(alpha) g_min sigmoid(z)(1 - sigmoid(z)).
//
// Value columns are independent in every line except the sums over them (dq,
// dk, dbeta, dalpha), so a CTA owns one (b, h) and 16 value columns, and those
// sums are added across the CTAs of a (b, h) with fp32 atomics.  The state
// slice lives in registers: thread t holds key row c = t / 2 and 8 columns.
// rec_ckpt_kernel runs the recurrence forward and stores the state entering
// every chunk of 64 tokens; rec_bwd_kernel walks the chunks backwards,
// recomputes the chunk's states from its checkpoint into a per-CTA stash, and
// applies the reverse steps token by token.  The sums over key rows (p, dr)
// are warp shuffles plus one shared-memory pass.
#include "rec_common.cuh"

namespace kda {

namespace {

using rec::rowsum16;
constexpr int RB_THREADS = rec::THREADS;
constexpr int RB_VS = rec::VS;
constexpr int RB_C = 64;         // tokens per checkpoint interval

struct RbArgs {
    int64_t S;
    int H, Dk, Dv, nslice, Nc;
    const void *q, *k, *v, *z, *beta, *dO;
    const float *log_decay;
    float g_min;
    const float *S0, *dST;
    float *dq, *dk, *dv, *dbeta, *dz, *dS0;
    float *ckpt;   // [B*H][nslice][Nc][Dk][16]
    float *stash;  // [B*H][nslice][64][Dk][16]
};

template <typename T>
struct Step {  // per-thread view of one token's inputs
    float a, kc, qc, b, g;  // alpha_c, k_c, q_c, beta, log alpha_c
};

template <typename T>
__device__ __forceinline__ Step<T> load_step(const RbArgs &p, int b, int h, int64_t t, int c) {
    Step<T> s;
    const int64_t row = ((int64_t)b * p.S + t) * p.H + h;
    s.b = load_elem((const T *)p.beta, row);
    if (c < p.Dk) {
        const int64_t i = row * p.Dk + c;
        s.kc = load_elem((const T *)p.k, i);
        s.qc = load_elem((const T *)p.q, i);
        s.g = p.log_decay ? clamp_log_decay(p.log_decay[i], p.g_min) : log_alpha_of(load_elem((const T *)p.z, i), p.g_min);
        s.a = expf(s.g);
    } else {
        s.kc = s.qc = s.g = 0.f;
        s.a = 1.f;
    }
    return s;
}

// One forward token step on the register slice S (S_{t-1} -> S_t); u_t of the 16 columns goes to su.
template <typename T>
__device__ __forceinline__ void fwd_step(const RbArgs &p, int b, int h, int64_t t, int c, int half, int j0,
                                         float (&S)[8], float *red, float *su, int tid) {
    const Step<T> st = load_step<T>(p, b, h, t, c);
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        S[e] *= st.a;
        x[e] = st.kc * S[e];
    }
    const float pj = rowsum16(x, red, tid);
    if (tid < 16) {
        const int j = j0 + tid;
        su[tid] = (j < p.Dv) ? load_elem((const T *)p.v, (((int64_t)b * p.S + t) * p.H + h) * p.Dv + j) - pj : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = fmaf(st.kc * st.b, su[8 * half + e], S[e]);
}

template <typename T>
__global__ void __launch_bounds__(RB_THREADS) rec_ckpt_kernel(RbArgs p) {
    __shared__ float red[RB_THREADS / 32 * 16];
    __shared__ float su[16];
    const int tid = threadIdx.x, c = tid >> 1, half = tid & 1;
    const int bh = blockIdx.x, slice = blockIdx.y, b = bh / p.H, h = bh % p.H, j0 = slice * RB_VS;
    const int jc = j0 + 8 * half;
    float S[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        S[e] = (p.S0 && c < p.Dk && jc + e < p.Dv) ? p.S0[((int64_t)bh * p.Dk + c) * p.Dv + jc + e] : 0.f;
    float *ck = p.ckpt + ((int64_t)bh * p.nslice + slice) * p.Nc * p.Dk * RB_VS;
    for (int n = 0; n < p.Nc; ++n) {
        if (c < p.Dk)
#pragma unroll
            for (int e = 0; e < 8; ++e) ck[((int64_t)n * p.Dk + c) * RB_VS + 8 * half + e] = S[e];
        const int64_t t1 = min(p.S, (int64_t)(n + 1) * RB_C);
        for (int64_t t = (int64_t)n * RB_C; t < t1; ++t) fwd_step<T>(p, b, h, t, c, half, j0, S, red, su, tid);
    }
}

template <typename T>
__global__ void __launch_bounds__(RB_THREADS) rec_bwd_kernel(RbArgs p) {
    __shared__ float red[RB_THREADS / 32 * 16];
    __shared__ float su[16];
    __shared__ float su_all[RB_C][16];  // u_t of the chunk's tokens
    __shared__ float sdr[16];
    const int tid = threadIdx.x, c = tid >> 1, half = tid & 1;
    const int bh = blockIdx.x, slice = blockIdx.y, b = bh / p.H, h = bh % p.H, j0 = slice * RB_VS;
    const int jc = j0 + 8 * half;
    const bool row_ok = c < p.Dk;
    float dS[8], S[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        dS[e] = (p.dST && row_ok && jc + e < p.Dv) ? p.dST[((int64_t)bh * p.Dk + c) * p.Dv + jc + e] : 0.f;
    const int64_t cta = (int64_t)bh * p.nslice + slice;
    const float *ck = p.ckpt + cta * p.Nc * p.Dk * RB_VS;
    float *stash = p.stash + cta * RB_C * p.Dk * RB_VS;
    for (int n = p.Nc - 1; n >= 0; --n) {
        const int64_t t0 = (int64_t)n * RB_C, t1 = min(p.S, t0 + RB_C);
        // recompute the chunk forward from its checkpoint, keeping S_{t-1} and u_t of every token
#pragma unroll
        for (int e = 0; e < 8; ++e) S[e] = row_ok ? ck[((int64_t)n * p.Dk + c) * RB_VS + 8 * half + e] : 0.f;
        for (int64_t t = t0; t < t1; ++t) {
            if (row_ok)
#pragma unroll
                for (int e = 0; e < 8; ++e) stash[((t - t0) * p.Dk + c) * RB_VS + 8 * half + e] = S[e];
            fwd_step<T>(p, b, h, t, c, half, j0, S, red, su, tid);
            if (tid < 16) su_all[t - t0][tid] = su[tid];
        }
        __syncthreads();  // u_t of the last token is read by every thread below
        // reverse steps; S holds S_t
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const Step<T> st = load_step<T>(p, b, h, t, c);
            const int64_t row = ((int64_t)b * p.S + t) * p.H + h;
            float Sp[8], dO[8], u[8], dSt[8], x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                Sp[e] = row_ok ? stash[((t - t0) * p.Dk + c) * RB_VS + 8 * half + e] : 0.f;
                dO[e] = (jc + e < p.Dv) ? load_elem((const T *)p.dO, row * p.Dv + jc + e) : 0.f;
                u[e] = su_all[t - t0][8 * half + e];
            }
            float dq = 0.f, dk = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                dSt[e] = fmaf(st.qc, dO[e], dS[e]);
                dq = fmaf(S[e], dO[e], dq);
                dk = fmaf(dSt[e], st.b * u[e], dk);
                x[e] = dSt[e] * st.kc;
            }
            const float drj = rowsum16(x, red, tid);
            if (tid < 16) {
                sdr[tid] = drj;
                if (j0 + tid < p.Dv) p.dv[row * p.Dv + j0 + tid] = st.b * drj;
            }
            __syncthreads();
            if (tid == 0) {
                float db = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) db = fmaf(sdr[j], su_all[t - t0][j], db);
                atomicAdd(p.dbeta + row, db);
            }
            float da = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float dp = -st.b * sdr[8 * half + e];
                const float dX = fmaf(st.kc, dp, dSt[e]);
                dk = fmaf(st.a * Sp[e], dp, dk);
                da = fmaf(dX, Sp[e], da);
                dS[e] = st.a * dX;
                S[e] = Sp[e];
            }
            dq += __shfl_xor_sync(0xffffffffu, dq, 1);
            dk += __shfl_xor_sync(0xffffffffu, dk, 1);
            da += __shfl_xor_sync(0xffffffffu, da, 1);
            if (half == 0 && row_ok) {
                const int64_t i = row * p.Dk + c;
                atomicAdd(p.dq + i, dq);
                atomicAdd(p.dk + i, dk);
                float dg = da * st.a;  // d/dlog(alpha)
                if (p.log_decay) {
                    const float raw = p.log_decay[i];
                    if (!(raw >= p.g_min && raw <= 0.f)) dg = 0.f;  // clamped input: no gradient
                } else {
                    const float sz = 1.0f / (1.0f + expf(-load_elem((const T *)p.z, i)));
                    dg *= p.g_min * sz * (1.0f - sz);
                }
                atomicAdd(p.dz + i, dg);
            }
        }
    }
    if (p.dS0 && row_ok)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (jc + e < p.Dv) p.dS0[((int64_t)bh * p.Dk + c) * p.Dv + jc + e] = dS[e];
}

}  // namespace

size_t rec_bwd_workspace(int64_t B, int64_t S, int H, int Dk, int Dv) {
    const int64_t nslice = (Dv + RB_VS - 1) / RB_VS, Nc = (S + RB_C - 1) / RB_C;
    const size_t per_cta = (size_t)(Nc + RB_C) * Dk * RB_VS * sizeof(float);
    return (size_t)B * H * nslice * per_cta;
}

kda_status_t launch_rec_bwd(const kda_recurrent_bwd_args &a, cudaStream_t st) {
    RbArgs p;
    p.S = a.S;
    p.H = a.H;
    p.Dk = a.D_k;
    p.Dv = a.D_v;
    p.nslice = (a.D_v + RB_VS - 1) / RB_VS;
    p.Nc = (int)((a.S + RB_C - 1) / RB_C);
    p.q = a.q; p.k = a.k; p.v = a.v; p.z = a.z; p.beta = a.beta; p.dO = a.d_o;
    p.log_decay = a.log_decay;
    p.g_min = a.g_min;
    p.S0 = a.initial_state;
    p.dST = a.d_final_state;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv; p.dbeta = a.dbeta; p.dz = a.dz; p.dS0 = a.d_initial_state;
    const int64_t nbh = a.B * a.H;
    const size_t nk = (size_t)nbh * a.S * a.D_k * sizeof(float), nb = (size_t)nbh * a.S * sizeof(float);
    // the per-row gradients are sums over the column slices: start them from zero
    cudaMemsetAsync(a.dq, 0, nk, st);
    cudaMemsetAsync(a.dk, 0, nk, st);
    cudaMemsetAsync(a.dz, 0, nk, st);
    cudaMemsetAsync(a.dbeta, 0, nb, st);
    if (a.S == 0) {
        if (a.d_initial_state) {
            const size_t ns = (size_t)nbh * a.D_k * a.D_v * sizeof(float);
            if (a.d_final_state) cudaMemcpyAsync(a.d_initial_state, a.d_final_state, ns, cudaMemcpyDeviceToDevice, st);
            else cudaMemsetAsync(a.d_initial_state, 0, ns, st);
        }
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? KDA_OK : fail(KDA_ERR_CUDA, "recurrent backward: %s", cudaGetErrorString(e));
    }
    uint8_t *ws = (uint8_t *)a.workspace;
    p.ckpt = reinterpret_cast<float *>(ws);
    p.stash = reinterpret_cast<float *>(ws + (size_t)nbh * p.nslice * p.Nc * a.D_k * RB_VS * sizeof(float));
    const dim3 grid((unsigned)nbh, (unsigned)p.nslice);
    if (a.dtype == KDA_F32) {
        rec_ckpt_kernel<float><<<grid, RB_THREADS, 0, st>>>(p);
        kda_status_t s = check_launch("rec_ckpt_kernel");
        if (s != KDA_OK) return s;
        rec_bwd_kernel<float><<<grid, RB_THREADS, 0, st>>>(p);
        return check_launch("rec_bwd_kernel");
    }
    rec_ckpt_kernel<__nv_bfloat16><<<grid, RB_THREADS, 0, st>>>(p);
    kda_status_t s = check_launch("rec_ckpt_kernel");
    if (s != KDA_OK) return s;
    rec_bwd_kernel<__nv_bfloat16><<<grid, RB_THREADS, 0, st>>>(p);
    return check_launch("rec_bwd_kernel");
}

}  // namespace kda
