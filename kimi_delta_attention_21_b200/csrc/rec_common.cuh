// Shared by the token-by-token kernels (the recurrent backward and the DPLR
// comparator): a block of 256 threads holds a D_k x 16 slice of the state in
// registers, thread t owning key row t / 2 and 8 of the 16 value columns.
#pragma once

#include "kda_internal.cuh"

namespace kda {
namespace rec {

constexpr int THREADS = 256;  // thread t: key row c = t >> 1, columns 8 (t & 1) .. 8 (t & 1) + 7 of the slice
constexpr int VS = 16;        // value columns per block

// Sum over the key rows (threads) of x[8] for this thread's 8 columns; thread j < 16 gets column j's
// total back (the return value; 0 elsewhere).  Warp shuffles, then one pass through `red`
// (THREADS / 32 * 16 floats) after one block barrier.
__device__ __forceinline__ float rowsum16(const float (&x)[8], float *red, int tid) {
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = x[e];
#pragma unroll
    for (int off = 2; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] += __shfl_xor_sync(0xffffffffu, y[e], off);
    const int lane = tid & 31, warp = tid >> 5;
    if (lane < 2)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp * 16 + 8 * lane + e] = y[e];
    __syncthreads();
    float s = 0.f;
    if (tid < 16)
#pragma unroll
        for (int w = 0; w < THREADS / 32; ++w) s += red[w * 16 + tid];
    return s;
}

// The same sum, but every thread gets the totals of its own 8 columns (columns 8 (t & 1) .. + 7 of the
// slice) in s[8], summed over the warps in the same order as rowsum16.  One block barrier and no second
// one: `red` (THREADS / 32 * 16 floats) must alternate between two buffers from one call to the next, so
// that a thread writing the next call's partial sums never meets a thread still reading this call's.
__device__ __forceinline__ void rowsum16_all(const float (&x)[8], float *red, int tid, float (&s)[8]) {
    // (red: 16-byte aligned)
    float y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] = x[e];
#pragma unroll
    for (int off = 2; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] += __shfl_xor_sync(0xffffffffu, y[e], off);
    const int lane = tid & 31, warp = tid >> 5, half = tid & 1;
    if (lane < 2)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp * 16 + 8 * lane + e] = y[e];
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = 0.f;
#pragma unroll
    for (int w = 0; w < THREADS / 32; ++w) {
        const float4 lo = *reinterpret_cast<const float4 *>(red + w * 16 + 8 * half);
        const float4 hi = *reinterpret_cast<const float4 *>(red + w * 16 + 8 * half + 4);
        s[0] += lo.x; s[1] += lo.y; s[2] += lo.z; s[3] += lo.w;
        s[4] += hi.x; s[5] += hi.y; s[6] += hi.z; s[7] += hi.w;
    }
}

}  // namespace rec
}  // namespace kda
