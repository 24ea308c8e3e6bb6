// Host utilities of the tensor-core kernels: TMA tensor maps (encoded through the driver entry
// point, so the library needs no link-time dependency on libcuda) and the device status word that
// kernels with bounded waits write when a wait gives up.
#include <atomic>
#include <mutex>

#include "tc_common.cuh"

namespace moeq {

__device__ int g_device_status = 0;

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
int *g_status_addr[64] = {};
}  // namespace

// Memo of encoded tensor maps. A tensor map is a pure function of its parameters (address,
// type, extents, pitch, box, swizzle), so a repeated call with the same buffers reuses the
// encoding instead of going through the driver again ("vLLM x Novita AI: Chord W4A16 INT4 MoE
// Kernel for Kimi K2.x", section "SM90 grouped kernels": descriptors memoized per shape, about
// 30 us of host work per small decode launch saved). A small ring, most recent first.
namespace {
struct TmapKey {
    const void *base;
    int dtype, elem_bytes;
    uint64_t rows, cols;
    uint32_t box_rows, box_cols;
    bool swizzle128;
    bool operator==(const TmapKey &o) const
    {
        return base == o.base && dtype == o.dtype && elem_bytes == o.elem_bytes && rows == o.rows && cols == o.cols &&
               box_rows == o.box_rows && box_cols == o.box_cols && swizzle128 == o.swizzle128;
    }
};
constexpr int kTmapMemo = 64;
std::mutex g_memo_mu;
TmapKey g_memo_key[kTmapMemo];
CUtensorMap g_memo_map[kTmapMemo];
int g_memo_n = 0, g_memo_next = 0;
std::atomic<long long> g_memo_hits{0}, g_memo_misses{0};
}  // namespace

int make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes, uint64_t rows,
                 uint64_t cols, uint32_t box_rows, uint32_t box_cols, bool swizzle128)
{
    const TmapKey key{base, (int)dtype, elem_bytes, rows, cols, box_rows, box_cols, swizzle128};
    {
        std::lock_guard<std::mutex> g(g_memo_mu);
        for (int i = 0; i < g_memo_n; ++i) {
            const int j = (g_memo_next - 1 - i + kTmapMemo) % kTmapMemo;
            if (g_memo_key[j] == key) {
                *map = g_memo_map[j];
                g_memo_hits.fetch_add(1, std::memory_order_relaxed);
                return MOEQ_OK;
            }
        }
    }
    {
        std::lock_guard<std::mutex> g(g_mu);
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
                return set_error(MOEQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable: %s", cudaGetErrorString(e));
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
    }
    if (reinterpret_cast<uintptr_t>(base) % 16 || (cols * elem_bytes) % 16)
        return set_error(MOEQ_ERR_UNSUPPORTED, "tensor map: base and row pitch must be 16-byte aligned");
    if ((box_cols * (uint64_t)elem_bytes) % 16 || (swizzle128 && box_cols * (uint64_t)elem_bytes != 128))
        return set_error(MOEQ_ERR_UNSUPPORTED, "tensor map: box inner extent %u x %d bytes not supported", box_cols,
                         elem_bytes);
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estride,
                                CU_TENSOR_MAP_INTERLEAVE_NONE,
                                swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(MOEQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    g_memo_misses.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> g(g_memo_mu);
    g_memo_key[g_memo_next] = key;
    g_memo_map[g_memo_next] = *map;
    g_memo_next = (g_memo_next + 1) % kTmapMemo;
    if (g_memo_n < kTmapMemo) ++g_memo_n;
    return MOEQ_OK;
}

void tmap_memo_stats(long long *hits, long long *misses)
{
    if (hits) *hits = g_memo_hits.load(std::memory_order_relaxed);
    if (misses) *misses = g_memo_misses.load(std::memory_order_relaxed);
}

// A wait that can never complete (nothing arrives on the barrier), given a short poll limit: the
// bounded-wait helper every tensor-core kernel uses must give up and flag the status word.
__global__ void selftest_bounded_wait_kernel(uint32_t polls, int *status)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        abort_flag = 0;
        tc::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) tc::mbar_wait(&bar, 0, &abort_flag, status, polls);
}

int launch_selftest_bounded_wait(cudaStream_t s)
{
    int *status = device_status_ptr();
    if (!status) return set_error(MOEQ_ERR_CUDA, "moe_selftest_bounded_wait: no device status word");
    selftest_bounded_wait_kernel<<<1, 32, 0, s>>>(4096u, status);
    return MOEQ_OK;
}

int *device_status_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_status_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_addr[dev] = static_cast<int *>(p);
    }
    return g_status_addr[dev];
}

}  // namespace moeq
