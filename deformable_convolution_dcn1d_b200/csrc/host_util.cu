// Host helpers shared by the tensor-core kernels: the tensor-map encoder, the SM
// count and the kernels' shared-memory limits, each queried or set once per process /
// device.
#include <atomic>
#include <mutex>

#include "sm100.cuh"

namespace dcn1d {

EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

void *current_context() {
    using GetCtxFn = CUresult (*)(CUcontext *);
    static const GetCtxFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<GetCtxFn>(p);
        return static_cast<GetCtxFn>(nullptr);
    }();
    CUcontext ctx = nullptr;
    if (!fn || fn(&ctx) != CUDA_SUCCESS)
        return nullptr;
    return ctx;
}

int sm_count() {
    static std::atomic<int> counts[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 0;
    if (counts[dev].load(std::memory_order_relaxed) == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        counts[dev].store(n, std::memory_order_relaxed);
    }
    return counts[dev].load(std::memory_order_relaxed);
}

cudaError_t ensure_smem(const void *kernel, int bytes) {
    struct Entry {
        const void *fn;
        int dev, bytes;
    };
    static std::mutex mu;
    static Entry table[256];
    static int n = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(mu);
    int i = 0;
    while (i < n && !(table[i].fn == kernel && table[i].dev == dev))
        ++i;
    if (i < n && table[i].bytes >= bytes)
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
        return e;
    if (i < n)
        table[i].bytes = bytes;
    else if (n < 256)
        table[n++] = Entry{kernel, dev, bytes};
    return cudaSuccess;
}

bool encode_2d_ld(CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t cols,
                  uint64_t rows, uint64_t ld, uint32_t elem_bytes, uint32_t box_cols,
                  uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_2d(CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t cols,
               uint64_t rows, uint32_t elem_bytes, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle swizzle) {
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * elem_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dcn1d
