// harness.cu -- kernels a test or benchmark puts around the MoE layer; not
// part of the method.  The residual + RMS step makes layer l+1's input (and
// so its routing) depend on layer l's output, as in the model, where the
// routing of a layer is only known once the layers below it have run.
#include "common.cuh"
#include "launch.cuh"

namespace moe {

// r[t] += y[t];  x_next[t] = bf16(r[t] / sqrt(mean(r[t]^2) + 1e-6)).  One CTA per token.
__global__ void __launch_bounds__(256) residual_rmsnorm_kernel(float* __restrict__ r, const float* __restrict__ y,
                                                               uint16_t* __restrict__ x_next, int D) {
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x;
    float* rr = r + size_t(t) * D;
    const float* yy = y + size_t(t) * D;
    float ss = 0.f;
    for (int k = threadIdx.x; k < D; k += blockDim.x) {
        const float v = rr[k] + yy[k];
        rr[k] = v;
        ss = fmaf(v, v, ss);
    }
    __shared__ float part[8];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < int(blockDim.x >> 5); ++i) tot += part[i];
    const float inv = rsqrtf(tot / float(D) + 1e-6f);
    for (int k = threadIdx.x; k < D; k += blockDim.x) x_next[size_t(t) * D + k] = f32_to_bf16_rn(rr[k] * inv);
}

cudaError_t launch_residual_rmsnorm(float* r, const float* y, uint16_t* x_next, int T, int D, bool pdl,
                                    cudaStream_t s) {
    return launch_kernel(residual_rmsnorm_kernel, dim3(T), dim3(256), 0, s, pdl, 1, r, y, x_next, D);
}

__global__ void bf16_to_f32_kernel(const uint16_t* __restrict__ x, float* __restrict__ out, size_t n) {
    pdl_wait();
    pdl_trigger();
    for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x)
        out[i] = bf16_to_f32(x[i]);
}

cudaError_t launch_bf16_to_f32(const uint16_t* x, float* out, size_t n, bool pdl, cudaStream_t s) {
    const int blocks = int(n / 256 + 1 < 1024 ? n / 256 + 1 : 1024);
    return launch_kernel(bf16_to_f32_kernel, dim3(blocks), dim3(256), 0, s, pdl, 1, x, out, n);
}

}  // namespace moe
