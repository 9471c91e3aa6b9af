// The general diagonal-plus-low-rank recurrence of the "Diagonal-Plus-Low-Rank
// Matrices and Kimi Delta Attention" post (sections 1 and 3), token by token:
//
//   S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,    o_t = S_t^T q_t
//
// with free erase directions a_t, b_t, evaluated as
//   w = b_t^T S_{t-1};  S_t = Diag(alpha_t) S_{t-1} - a_t w^T + k_t v_t^T;  o_t = S_t^T q_t.
// It is the comparator of the KDA engines: without KDA's binding (a = beta k,
// b = k * alpha) the chunkwise UT/WY form does not apply as is, and this is the
// form every such transition has.  Exact fp32; a block owns one (b, h) and 16
// value columns with the state slice in registers (two sums over the key rows
// per token).
#include "rec_common.cuh"

namespace kda {

namespace {

struct DplrParams {
    int64_t S;
    int H, Dk, Dv;
    const void *q, *k, *v, *a, *b, *z;
    const float *log_decay;
    float g_min;
    const float *S0;
    void *o;
    float *Sf;
};

template <typename T>
__global__ void __launch_bounds__(rec::THREADS) dplr_recurrent_kernel(DplrParams p) {
    __shared__ float red[rec::THREADS / 32 * 16];
    __shared__ float sw[16], sv[16];
    const int tid = threadIdx.x, c = tid >> 1, half = tid & 1;
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H, j0 = blockIdx.y * rec::VS, jc = j0 + 8 * half;
    const bool row_ok = c < p.Dk;
    float S[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        S[e] = (p.S0 && row_ok && jc + e < p.Dv) ? p.S0[((int64_t)bh * p.Dk + c) * p.Dv + jc + e] : 0.f;
    for (int64_t t = 0; t < p.S; ++t) {
        const int64_t row = ((int64_t)b * p.S + t) * p.H + h;
        float al = 1.f, ac = 0.f, bc = 0.f, kc = 0.f, qc = 0.f;
        if (row_ok) {
            const int64_t i = row * p.Dk + c;
            const float g = p.log_decay ? clamp_log_decay(p.log_decay[i], p.g_min)
                                        : log_alpha_of(load_elem((const T *)p.z, i), p.g_min);
            al = expf(g);
            ac = load_elem((const T *)p.a, i);
            bc = load_elem((const T *)p.b, i);
            kc = load_elem((const T *)p.k, i);
            qc = load_elem((const T *)p.q, i);
        }
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = bc * S[e];
        const float wj = rec::rowsum16(x, red, tid);  // w = b^T S_{t-1}
        if (tid < 16) {
            sw[tid] = wj;
            sv[tid] = (j0 + tid < p.Dv) ? load_elem((const T *)p.v, row * p.Dv + j0 + tid) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            S[e] = fmaf(al, S[e], fmaf(-ac, sw[8 * half + e], kc * sv[8 * half + e]));
            x[e] = qc * S[e];
        }
        const float oj = rec::rowsum16(x, red, tid);  // o = S_t^T q
        if (tid < 16 && j0 + tid < p.Dv) store_elem((T *)p.o, row * p.Dv + j0 + tid, oj);
        __syncthreads();  // the next token's first sum reuses `red`
    }
    if (p.Sf && row_ok)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (jc + e < p.Dv) p.Sf[((int64_t)bh * p.Dk + c) * p.Dv + jc + e] = S[e];
}

}  // namespace

kda_status_t launch_dplr(const kda_dplr_args &a, cudaStream_t st) {
    DplrParams p;
    p.S = a.S;
    p.H = a.H;
    p.Dk = a.D_k;
    p.Dv = a.D_v;
    p.q = a.q; p.k = a.k; p.v = a.v; p.a = a.a; p.b = a.b; p.z = a.z;
    p.log_decay = a.log_decay;
    p.g_min = a.g_min;
    p.S0 = a.initial_state;
    p.o = a.o;
    p.Sf = a.final_state;
    const dim3 grid((unsigned)(a.B * a.H), (unsigned)((a.D_v + rec::VS - 1) / rec::VS));
    if (a.dtype == KDA_F32) dplr_recurrent_kernel<float><<<grid, rec::THREADS, 0, st>>>(p);
    else dplr_recurrent_kernel<__nv_bfloat16><<<grid, rec::THREADS, 0, st>>>(p);
    return check_launch("dplr_recurrent_kernel");
}

}  // namespace kda
