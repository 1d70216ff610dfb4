// moe_w4a8.cu — the single translation unit of libmoe_w4a8.so (sm_100a).
//
// Every kernel of the library is compiled here so that the device-status word below is one
// symbol without relocatable device code.
#include <algorithm>

#include "common.cuh"

namespace moe {
// The library's sticky device-status word (one per device, per loaded library): kernels
// with bounded waits set it when a wait gives up; moe_last_device_status() reads and clears it.
__device__ int g_device_status = 0;
}

#include "pack.cuh"
#include "quant.cuh"
#include "route.cuh"
#include "forward.cuh"
#include "tc_ptx.cuh"

namespace moe {
// An mbarrier that nothing arrives on: the bounded wait must give up after `limit_ns`.
__global__ void k_selftest_bounded_wait(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
        if (!tc::mbar_wait(&bar, 0, limit_ns)) atomicExch(&g_device_status, 1);
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
        return MOE_ERR_TIMEOUT;
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
