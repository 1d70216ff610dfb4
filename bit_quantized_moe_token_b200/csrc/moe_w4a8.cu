// moe_w4a8.cu — the single translation unit of libmoe_w4a8.so (sm_100a).
//
// Every kernel of the library is compiled here so that the device-status word below is one
// symbol without relocatable device code.
#include <algorithm>
#include <atomic>

#include "common.cuh"

namespace moe {
// The library's sticky device-status word (one per device, per loaded library), a set of
// flags: kStatusTimeout from kernels with bounded waits when a wait gives up, kStatusBadRecord
// from the expert-parallel receive path when a record names an expert outside the receiver's
// range.  moe_last_device_status() reads and clears it.
constexpr int kStatusTimeout = 1;
constexpr int kStatusBadRecord = 2;
__device__ int g_device_status = 0;
}

#include "pack.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "forward.cuh"
#include "ep.cuh"
#include "router.cuh"
#include "tc_ptx.cuh"

namespace moe {
// An mbarrier that nothing arrives on: the bounded wait must give up after `limit_ns`.
__global__ void k_selftest_bounded_wait(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
        if (!tc::mbar_wait(&bar, 0, limit_ns)) atomicOr(&g_device_status, kStatusTimeout);
    }
}
}  // namespace moe

extern "C" int moe_selftest_bounded_wait(int64_t limit_ns, moe_stream_t stream) {
    if (limit_ns < 1000 || limit_ns > 1000000000) return MOE_ERR_INVALID_ARG;
    moe::k_selftest_bounded_wait<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_ns));
    return moe::launch_status();
}

extern "C" int moe_last_device_status(moe_stream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, moe::g_device_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(moe::g_device_status, &zero, sizeof(int)) != cudaSuccess)
            return MOE_ERR_CUDA;
        return (v & moe::kStatusTimeout) ? MOE_ERR_TIMEOUT : MOE_ERR_INVALID_ARG;
    }
    return MOE_OK;
}

extern "C" const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_MISALIGNED: return "misaligned pointer";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_NO_DEVICE: return "no sm_100 device";
        default: return "unknown status";
    }
}

// ---------------------------------------------------------------------------------------------
// Allocation-free routing.  Some callers cannot allocate device memory at all (an engine whose
// own allocator has reserved every byte of the GPU up front, a C caller with no device allocator
// to link), so this variant of moe_route_topk takes its permutation scratch from a fixed array
// compiled into the library instead of a caller buffer.
// ---------------------------------------------------------------------------------------------
namespace moe {

// Per-chunk expert counts of the multi-chunk permutation: (ceil(T*k / 1024) * E) int32 words.
constexpr size_t kRouteStaticBytes = 256 * 1024;
static __device__ __align__(256) int32_t g_route_static_scratch[kRouteStaticBytes / sizeof(int32_t)];

// Device address of the array on the current device, looked up on the first call made with that
// device current and kept per device.  Host code may not pass `g_route_static_scratch` itself to a
// kernel: on the host that name is only a stand-in.  The slots are atomics, so host threads making
// their first calls at the same time only repeat the lookup (each stores the same address).  A
// cudaDeviceReset() unloads the library's module on that device; the cached address is then
// stale, and a process that resets a device must not call this entry point on it again.
static int route_static_scratch(int32_t** out) {
    static std::atomic<int32_t*> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED_SHAPE;
    int32_t* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        void* q = nullptr;
        if (cudaGetSymbolAddress(&q, g_route_static_scratch) != cudaSuccess || !q) return MOE_ERR_CUDA;
        p = static_cast<int32_t*>(q);
        cache[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return MOE_OK;
}

}  // namespace moe

extern "C" size_t moe_route_noalloc_max_scratch_bytes(void) { return moe::kRouteStaticBytes; }

extern "C" int moe_route_topk_noalloc(const float* logits, int64_t T, int E, int k,
                                      int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                                      int32_t* sorted_pairs, int32_t* row_of_pair,
                                      moe_stream_t stream) {
    using namespace moe;
    int st = route_args_ok(T, E, k);
    if (st != MOE_OK) return st;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!logits || !topk_ids || !topk_w || !sorted_pairs || !row_of_pair))
        return MOE_ERR_INVALID_ARG;
    if (route_ws_bytes(T, E, k) > kRouteStaticBytes) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_w, 4) ||
        !aligned(expert_offsets, 4) || !aligned(sorted_pairs, 4) || !aligned(row_of_pair, 4))
        return MOE_ERR_MISALIGNED;
    int32_t* scratch = nullptr;
    if ((st = route_static_scratch(&scratch)) != MOE_OK) return st;
    if (T == 0) {
        if (cudaMemsetAsync(expert_offsets, 0, (E + 1) * sizeof(int32_t), stream) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    // every count the permutation reads is written earlier in the same call: nothing to clear
    st = launch_topk(logits, T, E, k, topk_ids, topk_w, stream);
    if (st != MOE_OK) return st;
    return launch_permute(topk_ids, T, E, k, expert_offsets, sorted_pairs, row_of_pair, scratch, stream);
}
