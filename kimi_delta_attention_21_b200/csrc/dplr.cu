// The general diagonal-plus-low-rank recurrence of the "Diagonal-Plus-Low-Rank
// Matrices and Kimi Delta Attention" post (sections 1 and 3), token by token:
//
//   S_t = (Diag(alpha_t) - a_t b_t^T) S_{t-1} + k_t v_t^T,    o_t = S_t^T q_t
//
// with free erase directions a_t, b_t, evaluated as
//   w = b_t^T S_{t-1};  S_t = Diag(alpha_t) S_{t-1} - a_t w^T + k_t v_t^T;  o_t = S_t^T q_t.
// It is the comparator of the KDA engines: without KDA's binding (a = beta k,
// b = k * alpha) the KDA engines' chunkwise UT/WY form does not apply as is;
// this is the form every such transition has, and dplr_chunk.cu the chunk form
// of the general case.  Exact fp32; a block owns one (b, h) and 16
// value columns with the state slice in registers (two sums over the key rows
// per token, one block barrier each).
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
    size_t o_bytes, sf_bytes;  // (checked builds test the writes against them)
    unsigned int *bounds;
};

// A chunk of 64 tokens is staged in shared memory by coalesced loads (k, q, a, b and log alpha [64][D_k],
// the block's 16 columns of v [64][16]) and its outputs leave together (o [64][16]), so that no token
// step waits on global memory; the two sums per token take one block barrier each.
constexpr int DP_C = 64;

size_t dplr_smem_bytes(int Dk) { return (size_t)(5 * DP_C * Dk + 2 * DP_C * rec::VS) * 4; }

template <typename T>
__global__ void __launch_bounds__(rec::THREADS) dplr_recurrent_kernel(DplrParams p) {
    extern __shared__ __align__(16) float smf[];
    __shared__ __align__(16) float red[2][rec::THREADS / 32 * 16];
    float *sk = smf, *sq = sk + DP_C * p.Dk, *sa = sq + DP_C * p.Dk, *sbv = sa + DP_C * p.Dk;
    float *sg = sbv + DP_C * p.Dk, *sv = sg + DP_C * p.Dk, *so = sv + DP_C * rec::VS;
    const int tid = threadIdx.x, c = tid >> 1, half = tid & 1;
    const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H, j0 = blockIdx.y * rec::VS, jc = j0 + 8 * half;
    const bool row_ok = c < p.Dk;
    float S[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        S[e] = (p.S0 && row_ok && jc + e < p.Dv) ? p.S0[((int64_t)bh * p.Dk + c) * p.Dv + jc + e] : 0.f;
    int par = 0;  // which of the two partial-sum buffers the next sum uses
    for (int64_t t0 = 0; t0 < p.S; t0 += DP_C) {
        const int len = (int)min((int64_t)DP_C, p.S - t0);
        const int64_t row0 = (int64_t)b * p.S + t0;
        __syncthreads();  // the previous chunk's steps and output flush are done with the staged arrays
        for (int idx = tid; idx < len * p.Dk; idx += rec::THREADS) {
            const int r = idx / p.Dk, cc = idx - r * p.Dk;
            const int64_t i = ((row0 + r) * p.H + h) * p.Dk + cc;
            sk[idx] = load_elem((const T *)p.k, i);
            sq[idx] = load_elem((const T *)p.q, i);
            sa[idx] = load_elem((const T *)p.a, i);
            sbv[idx] = load_elem((const T *)p.b, i);
            sg[idx] = p.log_decay ? clamp_log_decay(p.log_decay[i], p.g_min)
                                  : log_alpha_of(load_elem((const T *)p.z, i), p.g_min);
        }
        for (int idx = tid; idx < len * rec::VS; idx += rec::THREADS) {
            const int r = idx / rec::VS, j = idx - r * rec::VS;
            sv[idx] = (j0 + j < p.Dv) ? load_elem((const T *)p.v, ((row0 + r) * p.H + h) * p.Dv + j0 + j) : 0.f;
        }
        __syncthreads();
        for (int r = 0; r < len; ++r) {
            const int ri = r * p.Dk + c;
            const float al = row_ok ? expf(sg[ri]) : 1.f, ac = row_ok ? sa[ri] : 0.f, bc = row_ok ? sbv[ri] : 0.f;
            const float kc = row_ok ? sk[ri] : 0.f, qc = row_ok ? sq[ri] : 0.f;
            float x[8], w[8], o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = bc * S[e];
            rec::rowsum16_all(x, red[par], tid, w);  // w = b^T S_{t-1}
            par ^= 1;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                S[e] = fmaf(al, S[e], fmaf(-ac, w[e], kc * sv[r * rec::VS + 8 * half + e]));
                x[e] = qc * S[e];
            }
            rec::rowsum16_all(x, red[par], tid, o);  // o = S_t^T q
            par ^= 1;
            if (tid < 2)
#pragma unroll
                for (int e = 0; e < 8; ++e) so[r * rec::VS + 8 * half + e] = o[e];
        }
        __syncthreads();
        const int64_t o_lo = (row0 * p.H + h) * p.Dv, o_n = ((int64_t)(len - 1) * p.H) * p.Dv + p.Dv;
        const bool o_ok = in_bounds((const T *)p.o + o_lo, (size_t)o_n * sizeof(T), p.o, p.o_bytes, p.bounds);
        for (int idx = tid; o_ok && idx < len * rec::VS; idx += rec::THREADS) {
            const int r = idx / rec::VS, j = idx - r * rec::VS;
            if (j0 + j < p.Dv) store_elem((T *)p.o, ((row0 + r) * p.H + h) * p.Dv + j0 + j, so[idx]);
        }
    }
    if (p.Sf && row_ok && in_bounds(p.Sf + (int64_t)bh * p.Dk * p.Dv, (size_t)p.Dk * p.Dv * 4, p.Sf, p.sf_bytes, p.bounds))
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
    p.o_bytes = (size_t)a.B * a.S * a.H * a.D_v * (a.dtype == KDA_F32 ? 4 : 2);
    p.sf_bytes = (size_t)a.B * a.H * a.D_k * a.D_v * 4;
    p.bounds = device_bounds_counter();
    const dim3 grid((unsigned)(a.B * a.H), (unsigned)((a.D_v + rec::VS - 1) / rec::VS));
    const size_t smem = dplr_smem_bytes(a.D_k);
    if (a.dtype == KDA_F32) {
        cudaFuncSetAttribute(dplr_recurrent_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        dplr_recurrent_kernel<float><<<grid, rec::THREADS, smem, st>>>(p);
    } else {
        cudaFuncSetAttribute(dplr_recurrent_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        dplr_recurrent_kernel<__nv_bfloat16><<<grid, rec::THREADS, smem, st>>>(p);
    }
    return check_launch("dplr_recurrent_kernel");
}

}  // namespace kda
