/*
 * synth_dev.cu — device filler for the seeded workload generator.  The values
 * are those of synth_core.h, computed on the GPU so that full-size inputs
 * (gigabytes of expert weights) are built in HBM in milliseconds.  Built with
 * -fmad=false so that no multiply-add is contracted and every value matches
 * the host filler bit for bit.  Returns 0 on success, else the CUDA error.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include "synth_core.h"

namespace {

__global__ void k_fill_normal_bf16(uint64_t key, int64_t start, int64_t n, double sigma,
                                   uint16_t* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < n;
         j += (int64_t)gridDim.x * blockDim.x)
        out[j] = syn_f32_to_bf16((float)(sigma * syn_normal(key, (uint64_t)(start + j))));
}

__global__ void k_fill_tokens_bf16(uint64_t key, int64_t t0, int64_t nt, int64_t H,
                                   const uint8_t* mask, double gain, uint16_t* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < nt * H;
         j += (int64_t)gridDim.x * blockDim.x) {
        double z = syn_normal(key, (uint64_t)(t0 * H + j));
        if (mask && mask[j % H]) z = z * gain;
        out[j] = syn_f32_to_bf16((float)z);
    }
}

__global__ void k_fill_logits(uint64_t key, int64_t t0, int64_t nt, int64_t E,
                              const double* bias, float* out) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < nt * E;
         j += (int64_t)gridDim.x * blockDim.x) {
        double z = syn_normal(key, (uint64_t)(t0 * E + j));
        if (bias) z = z + bias[j % E];
        out[j] = (float)z;
    }
}

int grid_for(int64_t n) {
    int64_t g = (n + 255) / 256;
    if (g > 148 * 64) g = 148 * 64;
    if (g < 1) g = 1;
    return (int)g;
}

}  // namespace

extern "C" {

int syn_dev_fill_normal_bf16(uint64_t seed, uint64_t stream, int64_t start, int64_t n,
                             double sigma, uint16_t* out, cudaStream_t s) {
    if (n <= 0) return 0;
    k_fill_normal_bf16<<<grid_for(n), 256, 0, s>>>(syn_stream_key(seed, stream), start, n,
                                                    sigma, out);
    return (int)cudaGetLastError();
}

int syn_dev_fill_tokens_bf16(uint64_t seed, uint64_t stream, int64_t t0, int64_t nt, int64_t H,
                             const uint8_t* mask, double gain, uint16_t* out, cudaStream_t s) {
    if (nt * H <= 0) return 0;
    k_fill_tokens_bf16<<<grid_for(nt * H), 256, 0, s>>>(syn_stream_key(seed, stream), t0, nt, H,
                                                        mask, gain, out);
    return (int)cudaGetLastError();
}

int syn_dev_fill_logits(uint64_t seed, uint64_t stream, int64_t t0, int64_t nt, int64_t E,
                        const double* bias, float* out, cudaStream_t s) {
    if (nt * E <= 0) return 0;
    k_fill_logits<<<grid_for(nt * E), 256, 0, s>>>(syn_stream_key(seed, stream), t0, nt, E, bias,
                                                   out);
    return (int)cudaGetLastError();
}

}  // extern "C"
