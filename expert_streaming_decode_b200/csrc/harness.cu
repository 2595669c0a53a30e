// harness.cu -- kernels a test or benchmark puts around the MoE layer; not
// part of the method.  The residual + RMS step makes layer l+1's input (and
// so its routing) depend on layer l's output, as in the model, where the
// routing of a layer is only known once the layers below it have run.
#include "common.cuh"
#include "launch.cuh"

namespace moe {

// r[t] += y[t];  x_next[t] = bf16(r[t] / sqrt(mean(r[t]^2) + 1e-6)).  One CTA per token;
// rows of up to kRmsRegs * 4 * 256 values are read once, with all loads in
// flight together, and kept in registers.
constexpr int kRmsRegs = 4;
__global__ void __launch_bounds__(256) residual_rmsnorm_kernel(float* __restrict__ r, const float* __restrict__ y,
                                                               uint16_t* __restrict__ x_next, int D) {
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x;
    float4* rr = reinterpret_cast<float4*>(r + size_t(t) * D);
    const float4* yy = reinterpret_cast<const float4*>(y + size_t(t) * D);
    uint2* xo = reinterpret_cast<uint2*>(x_next + size_t(t) * D);
    const int n4 = D / 4;
    const bool in_regs = n4 <= kRmsRegs * int(blockDim.x);
    float4 v[kRmsRegs];
    float ss = 0.f;
    if (in_regs) {
        float4 a[kRmsRegs], b[kRmsRegs];
#pragma unroll
        for (int i = 0; i < kRmsRegs; ++i) {
            const int c = threadIdx.x + i * blockDim.x;
            if (c < n4) { a[i] = rr[c]; b[i] = yy[c]; }
        }
#pragma unroll
        for (int i = 0; i < kRmsRegs; ++i) {
            const int c = threadIdx.x + i * blockDim.x;
            if (c >= n4) continue;
            v[i] = make_float4(a[i].x + b[i].x, a[i].y + b[i].y, a[i].z + b[i].z, a[i].w + b[i].w);
            rr[c] = v[i];
            ss = fmaf(v[i].x, v[i].x, ss); ss = fmaf(v[i].y, v[i].y, ss);
            ss = fmaf(v[i].z, v[i].z, ss); ss = fmaf(v[i].w, v[i].w, ss);
        }
    } else {
        for (int c = threadIdx.x; c < n4; c += blockDim.x) {
            const float4 a = rr[c], b = yy[c];
            const float4 w = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
            rr[c] = w;
            ss = fmaf(w.x, w.x, ss); ss = fmaf(w.y, w.y, ss); ss = fmaf(w.z, w.z, ss); ss = fmaf(w.w, w.w, ss);
        }
    }
    __shared__ float part[8];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < int(blockDim.x >> 5); ++i) tot += part[i];
    const float inv = rsqrtf(tot / float(D) + 1e-6f);
    auto put = [&](int c, float4 w) {
        xo[c] = make_uint2(uint32_t(f32_to_bf16_rn(w.x * inv)) | (uint32_t(f32_to_bf16_rn(w.y * inv)) << 16),
                           uint32_t(f32_to_bf16_rn(w.z * inv)) | (uint32_t(f32_to_bf16_rn(w.w * inv)) << 16));
    };
    if (in_regs) {
#pragma unroll
        for (int i = 0; i < kRmsRegs; ++i) {
            const int c = threadIdx.x + i * blockDim.x;
            if (c < n4) put(c, v[i]);
        }
    } else {
        for (int c = threadIdx.x; c < n4; c += blockDim.x) put(c, rr[c]);
    }
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
