// Single-token decode step (Kimi Linear report, section 3, Eq. 1; the fused
// recurrent update order of the "Kimi Delta Attention" DeltaNet blog summary):
//
//   S'   = Diag(alpha) S                    (decay)
//   p    = S'^T k                            (prediction)
//   r    = beta (v - p)                      (residual)
//   S    = S' + k r^T                        (write, in place)
//   o~   = S^T q = S'^T q + (q . k) r        (read from the updated state)
//
// The second form of o~ lets one read of S produce both reductions, so the
// fp32 state crosses HBM exactly once in each direction: the kernel is
// bandwidth-bound on 2 * D_k * D_v * 4 bytes per (sequence, head).
#include "kda_internal.cuh"

namespace kda {

namespace {

// ------------------------------------------------------------------ D_k = D_v = 128
// One CTA (8 warps) per (b, h).  Lane l owns value columns 4l..4l+3; warp w owns
// key rows w, w+8, ..., w+120.  Each warp reads whole 512-byte state rows.
constexpr int DK = 128, DV = 128, NW = 8, RPW = DK / NW;

template <typename T>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? 2 : 1)
decode128_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                 const T *__restrict__ z, const float *__restrict__ log_decay, float g_min,
                 const T *__restrict__ beta, float *__restrict__ state,
                 const T *__restrict__ gate, float eps, T *__restrict__ o) {
    using AT = typename AccT<T>::type;
    __shared__ float s_q[DK], s_k[DK], s_a[DK];
    __shared__ AT s_red[2][NW][DV];
    __shared__ AT s_qk;
    const int bh = blockIdx.x;
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    float4 *S = reinterpret_cast<float4 *>(state + (int64_t)bh * DK * DV);

    // issue the state loads first: they are the whole cost of the kernel
    float4 s[RPW];
#pragma unroll
    for (int i = 0; i < RPW; ++i) s[i] = S[(w + NW * i) * (DV / 4) + l];

    if (tid < DK) {
        const int64_t off = (int64_t)bh * DK + tid;
        s_q[tid] = load_elem(q, off);
        s_k[tid] = load_elem(k, off);
        const float g = log_decay ? log_decay[off] : log_alpha_of(load_elem(z, off), g_min);
        s_a[tid] = expf(g);
    }
    __syncthreads();
    if (w == 0) {
        AT t = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) t += (AT)s_q[4 * l + j] * (AT)s_k[4 * l + j];
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) t += __shfl_xor_sync(0xffffffffu, t, m);
        if (l == 0) s_qk = t;
    }
    AT p[4] = {0, 0, 0, 0}, qs[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int c = w + NW * i;
        const float a = s_a[c];
        const AT kc = s_k[c], qc = s_q[c];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        p[0] += kc * s[i].x; p[1] += kc * s[i].y; p[2] += kc * s[i].z; p[3] += kc * s[i].w;
        qs[0] += qc * s[i].x; qs[1] += qc * s[i].y; qs[2] += qc * s[i].z; qs[3] += qc * s[i].w;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        s_red[0][w][4 * l + j] = p[j];
        s_red[1][w][4 * l + j] = qs[j];
    }
    __syncthreads();
    const AT b = load_elem(beta, (int64_t)bh);
    AT r[4], ot[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        AT pp = 0, qq = 0;
#pragma unroll
        for (int u = 0; u < NW; ++u) {
            pp += s_red[0][u][4 * l + j];
            qq += s_red[1][u][4 * l + j];
        }
        r[j] = b * ((AT)load_elem(v, (int64_t)bh * DV + 4 * l + j) - pp);
        ot[j] = qq + s_qk * r[j];
    }
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const AT kc = s_k[w + NW * i];
        s[i].x = (float)(s[i].x + kc * r[0]); s[i].y = (float)(s[i].y + kc * r[1]);
        s[i].z = (float)(s[i].z + kc * r[2]); s[i].w = (float)(s[i].w + kc * r[3]);
        S[(w + NW * i) * (DV / 4) + l] = s[i];
    }
    if (w == 0) {
        const int64_t ob = (int64_t)bh * DV + 4 * l;
        if (gate) {
            AT ss = ot[0] * ot[0] + ot[1] * ot[1] + ot[2] * ot[2] + ot[3] * ot[3];
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            const AT inv = AT(1) / sqrt(ss / (AT)DV + (AT)eps);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                store_elem(o, ob + j, (float)(ot[j] * inv * (AT)sigmoid_precise(load_elem(gate, ob + j))));
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) store_elem(o, ob + j, (float)ot[j]);
        }
    }
}

// ------------------------------------------------------------------ any D_k, D_v <= 128
// One CTA of 128 threads per (b, h); thread j owns value column j.
template <typename T>
__global__ void __launch_bounds__(128)
decode_generic_kernel(int Dk, int Dv, const T *__restrict__ q, const T *__restrict__ k,
                      const T *__restrict__ v, const T *__restrict__ z,
                      const float *__restrict__ log_decay, float g_min, const T *__restrict__ beta,
                      float *__restrict__ state, const T *__restrict__ gate, float eps,
                      T *__restrict__ o) {
    using AT = typename AccT<T>::type;
    __shared__ float s_q[128], s_k[128], s_a[128];
    __shared__ AT s_red[128];
    const int bh = blockIdx.x, j = threadIdx.x;
    float *S = state + (int64_t)bh * Dk * Dv;
    if (j < Dk) {
        const int64_t off = (int64_t)bh * Dk + j;
        s_q[j] = load_elem(q, off);
        s_k[j] = load_elem(k, off);
        const float g = log_decay ? log_decay[off] : log_alpha_of(load_elem(z, off), g_min);
        s_a[j] = expf(g);
    }
    __syncthreads();
    AT qk = 0;
    for (int c = 0; c < Dk; ++c) qk += (AT)s_q[c] * (AT)s_k[c];
    AT ot = 0;
    if (j < Dv) {
        AT p = 0, qs = 0;
        for (int c = 0; c < Dk; ++c) {
            const float sc = s_a[c] * S[c * Dv + j];
            p += (AT)s_k[c] * sc;
            qs += (AT)s_q[c] * sc;
        }
        const AT r = (AT)load_elem(beta, (int64_t)bh) * ((AT)load_elem(v, (int64_t)bh * Dv + j) - p);
        for (int c = 0; c < Dk; ++c) S[c * Dv + j] = (float)(s_a[c] * S[c * Dv + j] + (AT)s_k[c] * r);
        ot = qs + qk * r;
    }
    const int64_t ob = (int64_t)bh * Dv + j;
    if (gate) {
        s_red[j] = (j < Dv) ? ot * ot : 0.f;
        __syncthreads();
        for (int m = 64; m > 0; m >>= 1) {
            if (j < m) s_red[j] += s_red[j + m];
            __syncthreads();
        }
        const AT inv = AT(1) / sqrt(s_red[0] / (AT)Dv + (AT)eps);
        if (j < Dv) store_elem(o, ob, (float)(ot * inv * (AT)sigmoid_precise(load_elem(gate, ob))));
    } else if (j < Dv) {
        store_elem(o, ob, (float)ot);
    }
}

template <typename T>
kda_status_t launch_typed(const kda_decode_args &a, cudaStream_t st) {
    const int64_t nbh = a.B * a.H;
    if (nbh > 0x7fffffffLL) return fail(KDA_ERR_UNSUPPORTED, "B*H too large");
    const T *q = (const T *)a.q, *k = (const T *)a.k, *v = (const T *)a.v, *z = (const T *)a.z;
    const T *beta = (const T *)a.beta, *gate = (const T *)a.gate_logits;
    T *o = (T *)a.o;
    if (a.D_k == DK && a.D_v == DV && (reinterpret_cast<uintptr_t>(a.state) & 15u) == 0) {
        decode128_kernel<T><<<(unsigned)nbh, 256, 0, st>>>(q, k, v, z, a.log_decay, a.g_min, beta,
                                                            a.state, gate, a.eps, o);
        return check_launch("decode128_kernel");
    }
    decode_generic_kernel<T><<<(unsigned)nbh, 128, 0, st>>>(a.D_k, a.D_v, q, k, v, z, a.log_decay,
                                                             a.g_min, beta, a.state, gate, a.eps, o);
    return check_launch("decode_generic_kernel");
}

}  // namespace

kda_status_t launch_decode(const kda_decode_args &a, cudaStream_t st) {
    if (a.dtype == KDA_F32) return launch_typed<float>(a, st);
    return launch_typed<__nv_bfloat16>(a, st);
}

}  // namespace kda
