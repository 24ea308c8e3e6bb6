// Scratch-free variant of the W4A16 layer forward, for callers that cannot allocate device memory
// where they run the layer (a plugin or custom-op host that only hands over its input and output
// buffers, a runtime that plans all device memory up front and forbids allocation while serving).
//
// The scratch that moe_w4a16_forward takes from its caller lives here instead, in one file-scope
// static device array. In host code the array's name is only a host-side stand-in for the
// symbol, never a device address: the device address is looked up with cudaGetSymbolAddress
// once per device, with that device current, on the first call made on it. Nothing here
// allocates; every later step is the ordinary forward given that address as its workspace.
#include <mutex>

#include "common.cuh"

namespace moeq {
namespace {

constexpr size_t kNoAllocScratchBytes = MOEQ_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

// Shared by every call on a device; holds the last call's contents. Nothing in it has to start
// at zero: within a call every scratch value is written before it is read.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

int scratch_address(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return set_error(MOEQ_ERR_CUDA, "moe_w4a16_forward_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return set_error(MOEQ_ERR_UNSUPPORTED, "moe_w4a16_forward_noalloc: device %d out of range", dev);
    std::lock_guard<std::mutex> g(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // the current device is `dev`
        if (e != cudaSuccess || p == nullptr)
            return set_error(MOEQ_ERR_CUDA, "moe_w4a16_forward_noalloc: cudaGetSymbolAddress: %s",
                             cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOEQ_OK;
}

}  // namespace
}  // namespace moeq

extern "C" int moe_w4a16_forward_noalloc(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                                         const int32_t *w13_q, const uint16_t *w13_s, const int32_t *w2_q,
                                         const uint16_t *w2_s, uint16_t *out, int32_t *topk_ids_out,
                                         float *topk_w_out, void *stream)
{
    using namespace moeq;
    const size_t need = moe_w4a16_workspace_size(T, H, I, E, k);
    if (need == 0) return moe_w4a16_forward(x, logits, T, H, I, E, k, w13_q, w13_s, w2_q, w2_s, out, topk_ids_out,
                                            topk_w_out, nullptr, 0, stream);  // reports the shape error
    if (T == 0) return MOEQ_OK;
    if (need > kNoAllocScratchBytes)
        return set_error(MOEQ_ERR_WORKSPACE,
                         "moe_w4a16_forward_noalloc: this shape needs %zu bytes of scratch, more than the "
                         "library's built-in %zu bytes; use moe_w4a16_forward with a caller workspace",
                         need, kNoAllocScratchBytes);
    void *ws = nullptr;
    const int rc = scratch_address(&ws);
    if (rc != MOEQ_OK) return rc;
    return moe_w4a16_forward(x, logits, T, H, I, E, k, w13_q, w13_s, w2_q, w2_s, out, topk_ids_out, topk_w_out, ws,
                             kNoAllocScratchBytes, stream);
}
