// Shared pieces of the tensor-core chunk engines (the KDA prep, the GDN prep and
// the state pass): the per-chunk workspace record both preps write and the
// state pass reads, bf16/swizzle helpers, and the 64 x 64 unit-lower-triangular
// inverse of the UT transform.
#pragma once

#include <cuda_bf16.h>

#include "kda_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int CH = 64;   // chunk length
constexpr int DD = 128;  // D_k = D_v
constexpr float TC_GMIN_LIMIT = -5.5f;

// ---------------------------------------------------------------- workspace record (per b, h, chunk)
// All images are 128-byte-swizzled bf16 tiles in the layout the state kernel's
// MMAs read them in, so a record is one contiguous bulk copy away from use.
constexpr uint32_t REC_WQ = 0;        // [2 atoms (c / 64)][128 rows: -W rows 0-63, Q e^G rows 64-127][128 B]
                                      //   K-major A operand of [-W; Q e^G] S (M = 128)
constexpr uint32_t REC_KT = 32768;    // K e^{G_C - G}  [2 atoms (c / 64)][64 rows i][128 B], MN-major A of K~^T V'
constexpr uint32_t REC_MT = 49152;    // M^T            [64 rows i][128 B: r]; with the K~ atom in front of it,
                                      //   the MN-major A operand of [*; M] V' (M = 128, rows 64-127 = M)
constexpr uint32_t REC_U = 57344;     // U^T            [128 rows j][128 B: r]
constexpr uint32_t REC_GAM = 73728;   // e^{G_C}        128 fp32
constexpr uint32_t REC_BYTES = 74240;
constexpr uint32_t GATE_TILE_BYTES = CH * 128 * 2;  // one chunk of output-gate logits, [2 atoms][64 rows][128 B] bf16

__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 u;
    u.x = pack_bf16x2(f[0], f[1]);
    u.y = pack_bf16x2(f[2], f[3]);
    u.z = pack_bf16x2(f[4], f[5]);
    u.w = pack_bf16x2(f[6], f[7]);
    return u;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 x = __bfloat1622float2(h[j]);
        f[2 * j] = x.x;
        f[2 * j + 1] = x.y;
    }
}

__device__ __forceinline__ void load8f(const float *p, float (&f)[8]) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0];
    const float4 b = reinterpret_cast<const float4 *>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// The tensor-core engine works on bf16 data and every exponent it takes is
// bounded (|x| <= 8 |g_min| + |g_min| * 64), so the hardware exp2 approximation
// (a few ulp of fp32) is far below the bf16 rounding it feeds.
__device__ __forceinline__ float fexp(float x) { return __expf(x); }
__device__ __forceinline__ float log_alpha_fast(float z, float g_min) {
    return g_min * __fdividef(1.0f, 1.0f + __expf(-z));
}

// A descriptor for base + off: the start-address field holds address >> 4 in 14
// bits, which cannot carry for shared-memory addresses below 256 KB.
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t off_bytes) { return d + (off_bytes >> 4); }

// The first 1024-byte boundary at or after the dynamic shared-memory base p.  Pointer arithmetic on p
// itself (not an integer round trip), so that the compiler still knows every access through the
// result is a shared-memory access (ld.shared / st.shared, 32-bit addresses).
__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void report_timeout(unsigned int *timeouts, int *dev_status) {
    if (timeouts) atomicAdd(timeouts, 1u);
    if (dev_status) atomicExch(dev_status, (int)KDA_ERR_TIMEOUT);
}

constexpr int SA_LD = 65, ST_LD = 68;  // row strides (floats) of A and T in the inverse

// T = (I + A)^{-1} for a strictly lower triangular 64 x 64 A (fp32, row stride SA_LD), by block
// doubling: the four diagonal 16x16 blocks by forward substitution, then T_{R,R-1} = -T_RR A_{R,R-1}
// T_{R-1,R-1} for R = 1, 3, then the lower-left 32x32 block the same way from the two diagonal 32x32
// blocks.  Blocks above the diagonal are written as zeros where a later product reads them; the
// image zero-fills the upper-right 32x32 block.  Run by threads 0-127 (tid), named barrier 1.
// Writes T (fp32, row stride ST_LD) and its bf16 image `ti` (K-major, 64 rows x 64 columns, 128-byte
// swizzle); xs is 1536 floats of scratch.  The image is fenced for the async proxy.
__device__ __forceinline__ void invert_unit_lower64(const float *sA, float *sT, float *xs, uint8_t *ti, int tid) {
        if (tid < 64) {  // diagonal block R, column jc: (I + A_RR) x = e_jc, right-looking
            const int R = tid >> 4, jc = tid & 15, o = 16 * R;
            float x[16];
    #pragma unroll
            for (int a = 0; a < 16; ++a) x[a] = (a == jc) ? 1.f : 0.f;
            // once x[m] is final, every later row subtracts its term: one FMA per step on the
            // critical path (entries above jc stay exact zeros)
    #pragma unroll
            for (int m = 0; m < 15; ++m)
    #pragma unroll
                for (int a = m + 1; a < 16; ++a) x[a] = fmaf(-sA[(o + a) * SA_LD + o + m], x[m], x[a]);
    #pragma unroll
            for (int a = 0; a < 16; ++a) sT[(o + a) * ST_LD + o + jc] = x[a];
        }
        named_sync(1, 128);
        // The products below give each thread rows (p, p + h) and four adjacent columns, so that one
        // float4 of the right operand feeds eight FMAs (shared-memory wavefronts, not FMAs, bound them).
        float *x2 = xs + 512;  // X = A[32:64, 0:32] T[0:32, 0:32] for the 32 -> 64 step, [32][32]
        if (tid < 64) {  // 16 -> 32: X = A_{R,R-1} T_{R-1,R-1}, R = 1 + 2 hb
            const int hb = tid >> 5, R = 1 + 2 * hb, pr = (tid >> 2) & 7, c4 = 4 * (tid & 3), o = 16 * (R - 1);
            const float *a0 = sA + (16 * R + pr) * SA_LD + o, *a1 = a0 + 8 * SA_LD;
            const float *tb = sT + o * ST_LD + o + c4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
    #pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float u = a0[m], v = a1[m];
                const float4 t = *reinterpret_cast<const float4 *>(tb + m * ST_LD);
                x.x += u * t.x; x.y += u * t.y; x.z += u * t.z; x.w += u * t.w;
                y.x += v * t.x; y.y += v * t.y; y.z += v * t.z; y.w += v * t.w;
            }
            *reinterpret_cast<float4 *>(xs + hb * 256 + pr * 16 + c4) = x;
            *reinterpret_cast<float4 *>(xs + hb * 256 + (pr + 8) * 16 + c4) = y;
        } else {  // meanwhile the part of the 32 -> 64 product that needs only the diagonal blocks:
                  // X[:, 16 B + c] = A[32:64, 16 B : 16 B + 16] T_BB  (B = 0, 1)
            const int t2 = tid - 64, pr = t2 >> 2, c8 = 8 * (t2 & 3), blk = c8 >> 4;
            const float *a0 = sA + (32 + pr) * SA_LD + 16 * blk, *a1 = a0 + 16 * SA_LD;
            const float *tb = sT + 16 * blk * ST_LD + c8;
            float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0, y0 = x0, y1 = x0;
    #pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float u = a0[m], v = a1[m];
                const float4 t0 = *reinterpret_cast<const float4 *>(tb + m * ST_LD);
                const float4 t1 = *reinterpret_cast<const float4 *>(tb + m * ST_LD + 4);
                x0.x += u * t0.x; x0.y += u * t0.y; x0.z += u * t0.z; x0.w += u * t0.w;
                x1.x += u * t1.x; x1.y += u * t1.y; x1.z += u * t1.z; x1.w += u * t1.w;
                y0.x += v * t0.x; y0.y += v * t0.y; y0.z += v * t0.z; y0.w += v * t0.w;
                y1.x += v * t1.x; y1.y += v * t1.y; y1.z += v * t1.z; y1.w += v * t1.w;
            }
            *reinterpret_cast<float4 *>(x2 + pr * 32 + c8) = x0;
            *reinterpret_cast<float4 *>(x2 + pr * 32 + c8 + 4) = x1;
            *reinterpret_cast<float4 *>(x2 + (pr + 16) * 32 + c8) = y0;
            *reinterpret_cast<float4 *>(x2 + (pr + 16) * 32 + c8 + 4) = y1;
        }
        named_sync(1, 128);
        if (tid < 64) {  //       T_{R,R-1} = -T_RR X  (T_RR is zero above its diagonal); zero block (R-1, R)
            const int hb = tid >> 5, R = 1 + 2 * hb, pr = (tid >> 2) & 7, c4 = 4 * (tid & 3);
            const float *t0 = sT + (16 * R + pr) * ST_LD + 16 * R, *t1 = t0 + 8 * ST_LD;
            const float *xb = xs + hb * 256 + c4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
    #pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float u = t0[m], v = t1[m];
                const float4 t = *reinterpret_cast<const float4 *>(xb + m * 16);
                x.x += u * t.x; x.y += u * t.y; x.z += u * t.z; x.w += u * t.w;
                y.x += v * t.x; y.y += v * t.y; y.z += v * t.z; y.w += v * t.w;
            }
            float *d0 = sT + (16 * R + pr) * ST_LD + 16 * (R - 1) + c4;
            *reinterpret_cast<float4 *>(d0) = make_float4(-x.x, -x.y, -x.z, -x.w);
            *reinterpret_cast<float4 *>(d0 + 8 * ST_LD) = make_float4(-y.x, -y.y, -y.z, -y.w);
            float *z0 = sT + (16 * (R - 1) + pr) * ST_LD + 16 * R + c4;
            *reinterpret_cast<float4 *>(z0) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4 *>(z0 + 8 * ST_LD) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        named_sync(1, 128);
        if (tid < 64) {  // 32 -> 64: the rest of X, X[:, 0:16] += A[32:64, 16:32] T_10
            const int pr = tid >> 2, c4 = 4 * (tid & 3);
            const float *a0 = sA + (32 + pr) * SA_LD + 16, *a1 = a0 + 16 * SA_LD;
            const float *tb = sT + 16 * ST_LD + c4;
            float4 x = *reinterpret_cast<const float4 *>(x2 + pr * 32 + c4);
            float4 y = *reinterpret_cast<const float4 *>(x2 + (pr + 16) * 32 + c4);
    #pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float u = a0[m], v = a1[m];
                const float4 t = *reinterpret_cast<const float4 *>(tb + m * ST_LD);
                x.x += u * t.x; x.y += u * t.y; x.z += u * t.z; x.w += u * t.w;
                y.x += v * t.x; y.y += v * t.y; y.z += v * t.z; y.w += v * t.w;
            }
            *reinterpret_cast<float4 *>(x2 + pr * 32 + c4) = x;
            *reinterpret_cast<float4 *>(x2 + (pr + 16) * 32 + c4) = y;
        }
        named_sync(1, 128);
        if (tid < 128) {  //       T[32:64, 0:32] = -T[32:64, 32:64] X  (rows 32-47: T_22 only, T_23 = 0)
            const int pr = tid >> 3, c4 = 4 * (tid & 7);
            const float *t0 = sT + (32 + pr) * ST_LD + 32, *t1 = t0 + 16 * ST_LD;
            const float *xb = x2 + c4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
    #pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float u = t0[m], v = t1[m];
                const float4 t = *reinterpret_cast<const float4 *>(xb + m * 32);
                x.x += u * t.x; x.y += u * t.y; x.z += u * t.z; x.w += u * t.w;
                y.x += v * t.x; y.y += v * t.y; y.z += v * t.z; y.w += v * t.w;
            }
    #pragma unroll
            for (int m = 16; m < 32; ++m) {
                const float v = t1[m];
                const float4 t = *reinterpret_cast<const float4 *>(xb + m * 32);
                y.x += v * t.x; y.y += v * t.y; y.z += v * t.z; y.w += v * t.w;
            }
            float *d0 = sT + (32 + pr) * ST_LD + c4;
            *reinterpret_cast<float4 *>(d0) = make_float4(-x.x, -x.y, -x.z, -x.w);
            *reinterpret_cast<float4 *>(d0 + 16 * ST_LD) = make_float4(-y.x, -y.y, -y.z, -y.w);
        }
        named_sync(1, 128);
        for (int k = 0; k < 4; ++k) {  // T image (K-major, 64 rows x 64 cols), 8-column chunks
            const int r = (tid >> 3) + 16 * k, cc = tid & 7;
            float t[8];
            const bool upper = r < 32 && cc >= 4;
    #pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = upper ? 0.f : sT[r * ST_LD + 8 * cc + e];
            *reinterpret_cast<uint4 *>(ti + sw128(r, cc)) = pack8(t);
        }
        fence_proxy_async_smem();
}

// (B, S, H, 128) bf16 tensor as a 4-D TMA map (channel, head, token, batch): boxes of 64 channels x
// 1 head x 64 tokens x 1 batch row, 128-byte swizzled; tokens past the end of a sequence read as zero.
kda_status_t make_tmap_tokens(CUtensorMap *m, const void *base, int H, int64_t S, int64_t B, uint64_t rs,
                              uint64_t ss, uint64_t bs);

// The state pass (segment maps, combine, segment chains with the fused RMSNorm and output gate) over
// the per-chunk records in a.workspace, which a prep kernel has written for every (b, h, chunk).
kda_status_t launch_chunk_state_pass(const kda_chunk_args &a, cudaStream_t st);

// Where a prep leaves each chunk's log-bound of the transition norm ([B*H][Nc] fp32 in a.workspace: the
// sum over its tokens of log(max_c alpha_c) + log(max(1, |1 - beta |k|^2|)), or an upper bound of it),
// or null when the sequence is one segment (the map pass, which reads them, does not run).
float *chunk_log_bounds(const kda_chunk_args &a);

}  // namespace tc
}  // namespace kda
