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
// are warp shuffles plus one shared-memory pass.  A chunk's inputs are staged
// in shared memory once, so that no token step waits on a global load.
#include "rec_common.cuh"
#include "sm100_ptx.cuh"

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
    // buffer sizes in bytes (checked builds test the workspace accesses and the writes against them)
    size_t ckpt_bytes, stash_bytes, nk_bytes, nv_bytes, nb_bytes, ns_bytes;
    unsigned int *bounds;
};

// The inputs of one 64-token chunk, staged in shared memory by coalesced loads once per chunk (the
// recompute and the reverse pass both read them): k, q and log alpha [64][D_k], the CTA's 16 columns of
// v and dO [64][16], beta [64].  Then the ring the stash of S_{t-1} is prefetched into, RB_NR tokens
// ahead, each thread by cp.async for its own 8 floats (so no barrier orders it).
constexpr int RB_NR = 4;

struct Staged {
    float *k, *q, *g, *v, *dO, *b, *ring;
};

__device__ __forceinline__ Staged staged_at(float *base, int Dk) {
    Staged s;
    s.k = base;
    s.q = s.k + RB_C * Dk;
    s.g = s.q + RB_C * Dk;
    s.v = s.g + RB_C * Dk;
    s.dO = s.v + RB_C * RB_VS;
    s.b = s.dO + RB_C * RB_VS;
    s.ring = s.b + RB_C;  // 16-byte aligned: every array before it is a multiple of 4 floats long
    return s;
}

size_t rec_smem_bytes(int Dk) { return (size_t)(3 * RB_C * Dk + 2 * RB_C * RB_VS + RB_C + RB_NR * Dk * RB_VS) * 4; }

template <typename T>
__device__ void stage_chunk(const RbArgs &p, const Staged &s, int b, int h, int64_t t0, int len, int j0, bool with_q,
                            bool with_dO, int tid) {
    const int64_t row0 = (int64_t)b * p.S + t0;
    for (int idx = tid; idx < len * p.Dk; idx += RB_THREADS) {
        const int r = idx / p.Dk, c = idx - r * p.Dk;
        const int64_t i = ((row0 + r) * p.H + h) * p.Dk + c;
        s.k[idx] = load_elem((const T *)p.k, i);
        if (with_q) s.q[idx] = load_elem((const T *)p.q, i);
        s.g[idx] = p.log_decay ? clamp_log_decay(p.log_decay[i], p.g_min)
                               : log_alpha_of(load_elem((const T *)p.z, i), p.g_min);
    }
    for (int idx = tid; idx < len * RB_VS; idx += RB_THREADS) {
        const int r = idx / RB_VS, j = idx - r * RB_VS;
        const int64_t i = ((row0 + r) * p.H + h) * p.Dv + j0 + j;
        const bool in = j0 + j < p.Dv;
        s.v[idx] = in ? load_elem((const T *)p.v, i) : 0.f;
        if (with_dO) s.dO[idx] = in ? load_elem((const T *)p.dO, i) : 0.f;
    }
    for (int r = tid; r < len; r += RB_THREADS) s.b[r] = load_elem((const T *)p.beta, (row0 + r) * p.H + h);
}

// One forward token step (token r of the staged chunk) on the register slice S (S_{t-1} -> S_t); u_t of
// the 16 columns goes to su.
__device__ __forceinline__ void fwd_step(const RbArgs &p, const Staged &s, int r, int c, int half, float (&S)[8],
                                         float *red, float *su, int tid) {
    const bool row_ok = c < p.Dk;
    const float a = row_ok ? expf(s.g[r * p.Dk + c]) : 1.f, kc = row_ok ? s.k[r * p.Dk + c] : 0.f, bt = s.b[r];
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        S[e] *= a;
        x[e] = kc * S[e];
    }
    const float pj = rowsum16(x, red, tid);
    if (tid < 16) su[tid] = s.v[r * RB_VS + tid] - pj;  // (columns past D_v: v = 0 and S = 0)
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = fmaf(kc * bt, su[8 * half + e], S[e]);
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_ring() { asm volatile("cp.async.wait_group %0;" ::"n"(RB_NR - 1) : "memory"); }

template <typename T>
__global__ void __launch_bounds__(RB_THREADS) rec_ckpt_kernel(RbArgs p) {
    extern __shared__ __align__(16) float smf[];
    __shared__ float red[RB_THREADS / 32 * 16];
    __shared__ float su[16];
    const Staged st = staged_at(smf, p.Dk);
    const int tid = threadIdx.x, c = tid >> 1, half = tid & 1;
    const int bh = blockIdx.x, slice = blockIdx.y, b = bh / p.H, h = bh % p.H, j0 = slice * RB_VS;
    const int jc = j0 + 8 * half;
    float S[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        S[e] = (p.S0 && c < p.Dk && jc + e < p.Dv) ? p.S0[((int64_t)bh * p.Dk + c) * p.Dv + jc + e] : 0.f;
    float *ck = p.ckpt + ((int64_t)bh * p.nslice + slice) * p.Nc * p.Dk * RB_VS;
    for (int n = 0; n < p.Nc; ++n) {
        if (c < p.Dk && in_bounds(ck + (int64_t)n * p.Dk * RB_VS, (size_t)p.Dk * RB_VS * 4, p.ckpt, p.ckpt_bytes, p.bounds))
#pragma unroll
            for (int e = 0; e < 8; ++e) ck[((int64_t)n * p.Dk + c) * RB_VS + 8 * half + e] = S[e];
        const int64_t t0 = (int64_t)n * RB_C;
        const int len = (int)min((int64_t)RB_C, p.S - t0);
        __syncthreads();  // the previous chunk's steps are done with the staged inputs
        stage_chunk<T>(p, st, b, h, t0, len, j0, false, false, tid);
        __syncthreads();
        for (int r = 0; r < len; ++r) fwd_step(p, st, r, c, half, S, red, su, tid);
    }
}

template <typename T>
__global__ void __launch_bounds__(RB_THREADS) rec_bwd_kernel(RbArgs p) {
    extern __shared__ __align__(16) float smf[];
    __shared__ float red[RB_THREADS / 32 * 16];
    __shared__ float su[16];
    __shared__ float su_all[RB_C][16];  // u_t of the chunk's tokens
    __shared__ float sdr[16];
    const Staged st = staged_at(smf, p.Dk);
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
    const int soff = c * RB_VS + 8 * half;  // this thread's 8 floats within a token's [D_k][16] slice
    const bool stash_ok = in_bounds(stash, (size_t)RB_C * p.Dk * RB_VS * 4, p.stash, p.stash_bytes, p.bounds);
    for (int n = p.Nc - 1; n >= 0; --n) {
        const int64_t t0 = (int64_t)n * RB_C;
        const int len = (int)min((int64_t)RB_C, p.S - t0);
        __syncthreads();  // the later chunk's steps are done with the staged inputs
        stage_chunk<T>(p, st, b, h, t0, len, j0, true, true, tid);
        __syncthreads();
        // recompute the chunk forward from its checkpoint, keeping S_{t-1} (stash) and u_t of every token
        const bool ck_ok =
            in_bounds(ck + (int64_t)n * p.Dk * RB_VS, (size_t)p.Dk * RB_VS * 4, p.ckpt, p.ckpt_bytes, p.bounds);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            S[e] = (row_ok && ck_ok) ? ck[((int64_t)n * p.Dk + c) * RB_VS + 8 * half + e] : 0.f;
        for (int r = 0; r < len; ++r) {
            if (row_ok && stash_ok)
#pragma unroll
                for (int e = 0; e < 8; ++e) stash[(size_t)r * p.Dk * RB_VS + soff + e] = S[e];
            fwd_step(p, st, r, c, half, S, red, su, tid);
            if (tid < 16) su_all[r][tid] = su[tid];
        }
        __threadfence();  // this thread's stash stores are performed before its cp.async reads them back
        __syncthreads();  // u_t of the last token is read by every thread below
        // the stash of the last RB_NR tokens into the ring (slot r % RB_NR for token r of the chunk)
        auto prefetch = [&](int r) {
            if (r >= 0 && row_ok && stash_ok) {
                float *dst = st.ring + (r % RB_NR) * p.Dk * RB_VS + soff;
                const float *src = stash + (size_t)r * p.Dk * RB_VS + soff;
                cp_async16(dst, src);
                cp_async16(dst + 4, src + 4);
            }
            cp_async_commit();  // one group per token, empty ones included, so the wait count holds
        };
#pragma unroll
        for (int i = 0; i < RB_NR; ++i) prefetch(len - 1 - i);
        // reverse steps; S holds S_t
        for (int r = len - 1; r >= 0; --r) {
            const int64_t row = ((int64_t)b * p.S + t0 + r) * p.H + h;
            const float a = row_ok ? expf(st.g[r * p.Dk + c]) : 1.f;
            const float kc = row_ok ? st.k[r * p.Dk + c] : 0.f, qc = row_ok ? st.q[r * p.Dk + c] : 0.f;
            const float bt = st.b[r];
            float Sp[8], dO[8], u[8], dSt[8], x[8];
            cp_async_wait_ring();  // this thread's copy of token r's stash has landed
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                Sp[e] = row_ok ? st.ring[(r % RB_NR) * p.Dk * RB_VS + soff + e] : 0.f;
                dO[e] = st.dO[r * RB_VS + 8 * half + e];
                u[e] = su_all[r][8 * half + e];
            }
            prefetch(r - RB_NR);  // into the slot just read
            float dq = 0.f, dk = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                dSt[e] = fmaf(qc, dO[e], dS[e]);
                dq = fmaf(S[e], dO[e], dq);
                dk = fmaf(dSt[e], bt * u[e], dk);
                x[e] = dSt[e] * kc;
            }
            const float drj = rowsum16(x, red, tid);
            if (tid < 16) {
                sdr[tid] = drj;
                st.v[r * RB_VS + tid] = bt * drj;
            }
            __syncthreads();
            if (tid == 0) {
                float db = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) db = fmaf(sdr[j], su_all[r][j], db);
                st.b[r] = db;
            }
            float da = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float dp = -bt * sdr[8 * half + e];
                const float dX = fmaf(kc, dp, dSt[e]);
                dk = fmaf(a * Sp[e], dp, dk);
                da = fmaf(dX, Sp[e], da);
                dS[e] = a * dX;
                S[e] = Sp[e];
            }
            dq += __shfl_xor_sync(0xffffffffu, dq, 1);
            dk += __shfl_xor_sync(0xffffffffu, dk, 1);
            da += __shfl_xor_sync(0xffffffffu, da, 1);
            if (half == 0 && row_ok) {  // this token's k, q and log alpha are dead: their slots take the gradients
                float dg = da * a;  // d/dlog(alpha)
                if (p.log_decay) {
                    const float raw = p.log_decay[row * p.Dk + c];
                    if (!(raw >= p.g_min && raw <= 0.f)) dg = 0.f;  // clamped input: no gradient
                } else {  // g = g_min sigmoid(z): dg/dz = g_min sigmoid (1 - sigmoid) = g (1 - g / g_min)
                    const float g = st.g[r * p.Dk + c];
                    dg *= g * (1.0f - g / p.g_min);
                }
                st.q[r * p.Dk + c] = dq;
                st.k[r * p.Dk + c] = dk;
                st.g[r * p.Dk + c] = dg;
            }
        }
        // the chunk's gradients leave together: dv and, summed over the value-column slices of this (b, h)
        // with fp32 atomics, dq, dk, dz and dbeta (no global access in the token steps above)
        __syncthreads();
        const int64_t row0 = (int64_t)b * p.S + t0;
        // the chunk's rows of each output span [(row0 H + h) D, ((row0 + len - 1) H + h) D + D)
        const int64_t k_lo = (row0 * p.H + h) * p.Dk, k_n = ((int64_t)(len - 1) * p.H) * p.Dk + p.Dk;
        const int64_t v_lo = (row0 * p.H + h) * p.Dv, v_n = ((int64_t)(len - 1) * p.H) * p.Dv + p.Dv;
        const int64_t b_lo = row0 * p.H + h, b_n = (int64_t)(len - 1) * p.H + 1;
        const bool k_ok = in_bounds(p.dq + k_lo, k_n * 4, p.dq, p.nk_bytes, p.bounds) &&
                          in_bounds(p.dk + k_lo, k_n * 4, p.dk, p.nk_bytes, p.bounds) &&
                          in_bounds(p.dz + k_lo, k_n * 4, p.dz, p.nk_bytes, p.bounds);
        const bool v_ok = in_bounds(p.dv + v_lo, v_n * 4, p.dv, p.nv_bytes, p.bounds);
        const bool b_ok = in_bounds(p.dbeta + b_lo, b_n * 4, p.dbeta, p.nb_bytes, p.bounds);
        for (int idx = tid; k_ok && idx < len * p.Dk; idx += RB_THREADS) {
            const int r = idx / p.Dk, cc = idx - r * p.Dk;
            const int64_t i = ((row0 + r) * p.H + h) * p.Dk + cc;
            atomicAdd(p.dq + i, st.q[idx]);
            atomicAdd(p.dk + i, st.k[idx]);
            atomicAdd(p.dz + i, st.g[idx]);
        }
        for (int idx = tid; v_ok && idx < len * RB_VS; idx += RB_THREADS) {
            const int r = idx / RB_VS, j = idx - r * RB_VS;
            if (j0 + j < p.Dv) p.dv[((row0 + r) * p.H + h) * p.Dv + j0 + j] = st.v[idx];
        }
        for (int r = tid; b_ok && r < len; r += RB_THREADS) atomicAdd(p.dbeta + (row0 + r) * p.H + h, st.b[r]);
    }
    if (p.dS0 && row_ok && in_bounds(p.dS0 + (int64_t)bh * p.Dk * p.Dv, (size_t)p.Dk * p.Dv * 4, p.dS0, p.ns_bytes, p.bounds))
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
    p.ckpt_bytes = (size_t)nbh * p.nslice * p.Nc * a.D_k * RB_VS * sizeof(float);
    p.stash_bytes = (size_t)nbh * p.nslice * RB_C * a.D_k * RB_VS * sizeof(float);
    p.nk_bytes = nk;
    p.nv_bytes = (size_t)nbh * a.S * a.D_v * sizeof(float);
    p.nb_bytes = nb;
    p.ns_bytes = (size_t)nbh * a.D_k * a.D_v * sizeof(float);
    p.bounds = device_bounds_counter();
    const dim3 grid((unsigned)nbh, (unsigned)p.nslice);
    const size_t smem = rec_smem_bytes(a.D_k);
    if (a.dtype == KDA_F32) {
        cudaFuncSetAttribute(rec_ckpt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cudaFuncSetAttribute(rec_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        rec_ckpt_kernel<float><<<grid, RB_THREADS, smem, st>>>(p);
        kda_status_t s = check_launch("rec_ckpt_kernel");
        if (s != KDA_OK) return s;
        rec_bwd_kernel<float><<<grid, RB_THREADS, smem, st>>>(p);
        return check_launch("rec_bwd_kernel");
    }
    cudaFuncSetAttribute(rec_ckpt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(rec_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    rec_ckpt_kernel<__nv_bfloat16><<<grid, RB_THREADS, smem, st>>>(p);
    kda_status_t s = check_launch("rec_ckpt_kernel");
    if (s != KDA_OK) return s;
    rec_bwd_kernel<__nv_bfloat16><<<grid, RB_THREADS, smem, st>>>(p);
    return check_launch("rec_bwd_kernel");
}

}  // namespace kda
