// TMA tensor-map encoding and the device wait-timeout counter.
#include <atomic>
#include <mutex>

#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "tma_host.cuh"

namespace kda {

// Counts bounded device-side waits that ran out (all kernels of this library).
__device__ unsigned int g_kda_wait_timeouts;
__device__ unsigned int g_kda_bounds_errors;  // writes a checked build skipped (always 0 otherwise)

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

kda_status_t make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                          uint64_t rows, uint64_t cols, uint64_t row_stride, uint32_t box_rows, uint32_t box_cols,
                          CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (!fn) return fail(KDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_stride * (uint64_t)elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KDA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return KDA_OK;
}

kda_status_t make_tmap_3d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                          uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0,
                          uint32_t box1, uint32_t box2, CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (!fn) return fail(KDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1 * (uint64_t)elem_bytes, stride2 * (uint64_t)elem_bytes};
    cuuint32_t box[3] = {box0, box1, box2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, dtype, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KDA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return KDA_OK;
}

kda_status_t make_tmap_nd(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes, int rank,
                          const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                          CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (!fn) return fail(KDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    if (rank < 1 || rank > 5) return fail(KDA_ERR_INVALID_ARG, "tensor map rank %d", rank);
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
    }
    for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i] * (uint64_t)elem_bytes;
    CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KDA_ERR_CUDA, "cuTensorMapEncodeTiled (rank %d) failed (%d)", rank, (int)r);
    return KDA_OK;
}

unsigned int *device_timeout_counter() {
    static std::atomic<unsigned int *> ptrs[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    unsigned int *p = ptrs[dev].load();
    if (!p) {
        void *q = nullptr;
        if (cudaGetSymbolAddress(&q, g_kda_wait_timeouts) != cudaSuccess) return nullptr;
        p = static_cast<unsigned int *>(q);
        ptrs[dev].store(p);
    }
    return p;
}

unsigned int *device_bounds_counter() {
    static std::atomic<unsigned int *> ptrs[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    unsigned int *p = ptrs[dev].load();
    if (!p) {
        void *q = nullptr;
        if (cudaGetSymbolAddress(&q, g_kda_bounds_errors) != cudaSuccess) return nullptr;
        p = static_cast<unsigned int *>(q);
        ptrs[dev].store(p);
    }
    return p;
}

}  // namespace kda

extern "C" kda_status_t kda_device_bounds_errors(uint32_t *count, int reset, int *checked_build) {
    using namespace kda;
    if (!count) return fail(KDA_ERR_INVALID_ARG, "count is NULL");
#ifdef KDA_CHECKED
    if (checked_build) *checked_build = 1;
#else
    if (checked_build) *checked_build = 0;
#endif
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_kda_bounds_errors, sizeof(v));
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "reading the bounds counter: %s", cudaGetErrorString(e));
    *count = v;
    if (reset) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_kda_bounds_errors, &zero, sizeof(zero));
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "resetting the bounds counter: %s", cudaGetErrorString(e));
    }
    return KDA_OK;
}

extern "C" kda_status_t kda_device_timeouts(uint32_t *count, int reset) {
    using namespace kda;
    if (!count) return fail(KDA_ERR_INVALID_ARG, "count is NULL");
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_kda_wait_timeouts, sizeof(v));
    if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "reading the timeout counter: %s", cudaGetErrorString(e));
    *count = v;
    if (reset) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_kda_wait_timeouts, &zero, sizeof(zero));
        if (e != cudaSuccess) return fail(KDA_ERR_CUDA, "resetting the timeout counter: %s", cudaGetErrorString(e));
    }
    return KDA_OK;
}
