// dcn1d_forward_noalloc: the forward for callers that cannot allocate device
// memory -- code running where cudaMalloc is not allowed or not wanted, such
// as a real-time loop that must not allocate, an embedding runtime that owns
// every allocation, or a host that reserved all device memory up front.
//
// A path that needs scratch gets it here from a file-scope device array of fixed
// size; the kernels receive its device address.  (No forward path needs scratch at
// present -- the fp32 tensor-core path forms the weight's low tf32 part in shared
// memory and adds its split-K partial sums on chip -- so every valid call runs as
// dcn1d_forward without touching the array.)  Host code must not pass the array's
// name itself to a kernel: on the host it is a stand-in symbol, not a device
// address, so the address is looked up once per device with cudaGetSymbolAddress.
#include <mutex>

#include "sm100.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(48) << 20;   // 48 MiB

// Shared by every call on a device; it keeps the last call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device (NULL on failure).  It is
// looked up once per device and context: a device reset (cudaDeviceReset) ends the
// context the cached address belongs to, so a new context triggers a new lookup.
void *scratch_address() {
    static std::mutex mu;
    static void *addr[64] = {};
    static void *ctx_of[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    // The first runtime call above made the device's primary context current.
    void *ctx = dcn1d::current_context();
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || ctx_of[dev] != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess)
            return nullptr;
        addr[dev] = p;
        ctx_of[dev] = ctx;
    }
    return addr[dev];
}

}  // namespace

extern "C" int dcn1d_forward_noalloc(const dcn1d_tensor *x, const dcn1d_tensor *offsets,
                                     const dcn1d_tensor *mask, const dcn1d_tensor *weight,
                                     const dcn1d_tensor *bias, int64_t stride, int64_t padding,
                                     int64_t dilation, int64_t groups, int64_t offset_groups,
                                     int unconstrained, dcn1d_tensor *out, void *stream) {
    const int64_t need = dcn1d_forward_workspace_size(x, offsets, mask, weight, bias, stride,
                                                      padding, dilation, groups, offset_groups,
                                                      unconstrained, out);
    if (need < 0)
        return (int)-need;   // invalid arguments: the status code
    if ((uint64_t)need > kNoAllocScratchBytes)
        return DCN1D_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0) {
        ws = scratch_address();
        if (!ws)
            return DCN1D_ERR_CUDA;
    }
    return dcn1d_forward_ws(x, offsets, mask, weight, bias, stride, padding, dilation, groups,
                            offset_groups, unconstrained, out, ws,
                            need > 0 ? kNoAllocScratchBytes : 0, stream);
}
