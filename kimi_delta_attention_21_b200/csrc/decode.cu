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
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

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
        const float g = log_decay ? clamp_log_decay(log_decay[off], g_min) : log_alpha_of(load_elem(z, off), g_min);
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

// ------------------------------------------------------------------ D_k = D_v = 128, bf16, streamed
// Persistent: one CTA per SM walks (b, h) tasks.  Each task's 64 KiB state arrives by a bulk copy into
// one of three shared-memory stages, three tasks ahead, and its stage is refilled as soon as the state
// is in registers; the token's q, k, v, z (or log-decay) and gate come the same way into small stages
// of their own.  The updated state goes straight from registers to HBM (each warp writes whole 512-byte
// rows), so the read stream never waits for the arithmetic or the writes.  Same arithmetic and thread
// layout as decode128_kernel.
constexpr int DSTAGES = 3;
constexpr uint32_t DS_VEC = 2048;  // per stage: q, k, v, z, gate 256 B each; log-decay 512 B at 1024
constexpr size_t DS_SMEM = DSTAGES * (65536 + DS_VEC) + 128;

__global__ void __launch_bounds__(256, 1)
decode128_stream_kernel(int nbh, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                        const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ z,
                        const float *__restrict__ log_decay, float g_min, const __nv_bfloat16 *__restrict__ beta,
                        float *__restrict__ state, const __nv_bfloat16 *__restrict__ gate, float eps,
                        __nv_bfloat16 *__restrict__ o, unsigned int *timeouts) {
    using namespace sm100;
    pdl_trigger();
    pdl_wait();
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ uint64_t fullS[DSTAGES], fullV[DSTAGES];
    __shared__ float s_a[DK], s_qk;
    __shared__ float s_red[2][NW][DV];
    const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
    uint8_t *vecs = dsm + DSTAGES * 65536;
    const uint32_t vec_bytes = 3 * 256 + (log_decay ? 512 : 256) + (gate ? 256 : 0);
    auto issue_state = [&](int t, int stg) {
        mbar_arrive_expect_tx(&fullS[stg], 65536);
        bulk_load(dsm + stg * 65536, state + (size_t)t * DK * DV, 65536, &fullS[stg]);
    };
    auto issue_vec = [&](int t, int stg) {
        uint8_t *vb = vecs + stg * DS_VEC;
        mbar_arrive_expect_tx(&fullV[stg], vec_bytes);
        bulk_load(vb, q + (size_t)t * DK, 256, &fullV[stg]);
        bulk_load(vb + 256, k + (size_t)t * DK, 256, &fullV[stg]);
        bulk_load(vb + 512, v + (size_t)t * DV, 256, &fullV[stg]);
        if (log_decay) bulk_load(vb + 1024, log_decay + (size_t)t * DK, 512, &fullV[stg]);
        else bulk_load(vb + 768, z + (size_t)t * DK, 256, &fullV[stg]);
        if (gate) bulk_load(vb + 1536, gate + (size_t)t * DV, 256, &fullV[stg]);
    };
    if (tid == 0) {
        for (int i = 0; i < DSTAGES; ++i) {
            mbar_init(&fullS[i], 1);
            mbar_init(&fullV[i], 1);
        }
        fence_barrier_init();
        for (int i = 0; i < DSTAGES; ++i) {
            const int t = blockIdx.x + i * gridDim.x;
            if (t < nbh) {
                issue_state(t, i);
                issue_vec(t, i);
            }
        }
    }
    __syncthreads();
    bool ok = true;
    int it = 0;
    for (int t = blockIdx.x; t < nbh; t += gridDim.x, ++it) {
        const int stg = it % DSTAGES;
        const uint32_t par = (it / DSTAGES) & 1;
        const int tn = t + DSTAGES * (int)gridDim.x;  // the task that reuses this task's stages
        const float bt = __bfloat162float(beta[t]);
        if (!mbar_wait(&fullV[stg], par)) { ok = false; break; }
        const __nv_bfloat16 *sq = reinterpret_cast<const __nv_bfloat16 *>(vecs + stg * DS_VEC);
        const __nv_bfloat16 *sk = sq + 128, *sv = sq + 256, *sz = sq + 384;
        const float *sld = reinterpret_cast<const float *>(vecs + stg * DS_VEC + 1024);
        const __nv_bfloat16 *sg = sq + 768;
        if (tid < DK) s_a[tid] = expf(log_decay ? clamp_log_decay(sld[tid], g_min) : log_alpha_of(__bfloat162float(sz[tid]), g_min));
        if (w == 0) {
            float tq = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) tq += __bfloat162float(sq[4 * l + j]) * __bfloat162float(sk[4 * l + j]);
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) tq += __shfl_xor_sync(0xffffffffu, tq, m);
            if (l == 0) s_qk = tq;
        }
        if (!mbar_wait(&fullS[stg], par)) { ok = false; break; }
        float4 s[RPW];
        {
            const float4 *S = reinterpret_cast<const float4 *>(dsm + stg * 65536);
#pragma unroll
            for (int i = 0; i < RPW; ++i) s[i] = S[(w + NW * i) * (DV / 4) + l];
        }
        __syncthreads();  // the state stage has been read; s_a and s_qk are ready
        if (tid == 0 && tn < nbh) issue_state(tn, stg);
        float p[4] = {0.f, 0.f, 0.f, 0.f}, qs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int c = w + NW * i;
            const float a = s_a[c], kc = __bfloat162float(sk[c]), qc = __bfloat162float(sq[c]);
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
        float r[4], ot[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float pp = 0.f, qq = 0.f;
#pragma unroll
            for (int u = 0; u < NW; ++u) {
                pp += s_red[0][u][4 * l + j];
                qq += s_red[1][u][4 * l + j];
            }
            r[j] = bt * (__bfloat162float(sv[4 * l + j]) - pp);
            ot[j] = qq + s_qk * r[j];
        }
        float4 *Sg = reinterpret_cast<float4 *>(state + (size_t)t * DK * DV);
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const float kc = __bfloat162float(sk[w + NW * i]);
            s[i].x += kc * r[0]; s[i].y += kc * r[1]; s[i].z += kc * r[2]; s[i].w += kc * r[3];
            Sg[(w + NW * i) * (DV / 4) + l] = s[i];
        }
        if (w == 0) {
            float f[4] = {ot[0], ot[1], ot[2], ot[3]};
            if (gate) {
                float ss = ot[0] * ot[0] + ot[1] * ot[1] + ot[2] * ot[2] + ot[3] * ot[3];
#pragma unroll
                for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                const float inv = 1.0f / sqrtf(ss / (float)DV + eps);
#pragma unroll
                for (int j = 0; j < 4; ++j) f[j] = ot[j] * inv * sigmoid_precise(__bfloat162float(sg[4 * l + j]));
            }
            __nv_bfloat162 h0 = __floats2bfloat162_rn(f[0], f[1]), h1 = __floats2bfloat162_rn(f[2], f[3]);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t *>(&h0);
            pk.y = *reinterpret_cast<uint32_t *>(&h1);
            *reinterpret_cast<uint2 *>(o + (size_t)t * DV + 4 * l) = pk;
        }
        __syncthreads();  // every read of this task's vectors is done
        if (tid == 0 && tn < nbh) issue_vec(tn, stg);
    }
    if (!ok && tid == 0) {
        if (timeouts) atomicAdd(timeouts, 1u);
        for (int i = 0; i < DSTAGES; ++i) {  // let copies in flight land before the CTA exits
            mbar_wait(&fullS[i], 0, 100000000ull);
            mbar_wait(&fullV[i], 0, 100000000ull);
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
        const float g = log_decay ? clamp_log_decay(log_decay[off], g_min) : log_alpha_of(load_elem(z, off), g_min);
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
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (sizeof(T) == 2 && a.D_k == DK && a.D_v == DV && al16(a.state) && al16(a.q) && al16(a.k) && al16(a.v) &&
        al16(a.o) && al16(a.gate_logits) && (a.log_decay ? al16(a.log_decay) : al16(a.z))) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int grid = (int)(nbh < sms ? nbh : sms);
        cudaFuncSetAttribute(decode128_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DS_SMEM);
        cudaError_t e = launch_pdl(
            decode128_stream_kernel, dim3(grid), dim3(256), DS_SMEM, st, (int)nbh, (const __nv_bfloat16 *)q,
            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, (const __nv_bfloat16 *)z, a.log_decay, a.g_min,
            (const __nv_bfloat16 *)beta, a.state, (const __nv_bfloat16 *)gate, a.eps, (__nv_bfloat16 *)o,
            device_timeout_counter());
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "decode128_stream_kernel: %s", cudaGetErrorString(e));
        return check_launch("decode128_stream_kernel");
    }
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
