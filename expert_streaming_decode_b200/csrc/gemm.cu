// gemm.cu -- K6: tcgen05 tensor-core grouped GEMM over dequantised expert
// tiles, for the prefill chunk.
//
// Method: the prompt is prefilled in chunks of up to 128 tokens so that an
// expert fetched once is applied to every row routed to it ("TurboFieldfare:
// motor open source ...", section "Proceso de generacion de tokens").  With
// the chunk's (token, k) pairs grouped by expert, each expert is a small dense
// GEMM: H = gelu_tanh(X W_g^T) * (X W_u^T) [M_e x F], Y = H W_d^T [M_e x D],
// y[t] += w * Y[t] -- the one dense contraction on the path.
//
// B200 mapping (one CTA per (entry, 128 output rows), 4 warps):
//   * D[128 x N] = A[128 x K] * B[N x K]^T with tcgen05.mma kind::f16, M = 128
//     weight rows, N = the entry's token rows rounded up to 16 (experts carry
//     ~11 rows on average, so the weights sit in the M slot), fp32 accumulator
//     in tensor memory.
//   * K runs in groups of 64 (one quantisation group).  For each group all
//     threads dequantise the 128 x 64 weight tile (w = s*q + b rounded to fp16)
//     and convert the N x 64 activation tile (bf16 x or fp32 h) to fp16, both
//     in the no-swizzle K-major core-matrix layout (8 rows x 16 bytes per core
//     matrix; K-direction core stride 128 B, 8-row stride 1024 B); one thread
//     issues 4 MMAs of K = 16 and commits them to an mbarrier.  Two stages:
//     the next group is prepared while the tensor core works on this one.
//   * gate/up epilogue: warp w holds one 32-row blob tile (16 gate rows then the
//     16 matching up rows) in its TMEM lanes: h = gelu(g) * u with one shuffle.
//   * down epilogue: y[token][row] += w * D, fp32 atomics (entries of different
//     experts add into the same output rows).
#include "common.cuh"
#include "ffn.cuh"
#include "launch.cuh"

namespace moe {

constexpr int kGemmThreads = 128;
constexpr int kGemmStageBytes = 128 * 64 * 2;  // one 128 x 64 fp16 tile

struct GemmArgs {
    const WorkList* wl;
    const FfnEntry* entries;
    const FfnRow* rows;
    const uint16_t* x;   // bf16 [T][D]
    float* h;            // activations
    float* y;            // [T][D], accumulated
    int D;
    int* status;
};

// byte offset of element (r, k) of a [rows][64] fp16 tile in the core layout
__device__ __forceinline__ uint32_t core_off(int r, int k) {
    return uint32_t((r >> 3) * 1024 + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2);
}
// shared-memory matrix descriptor: no swizzle, K-direction core stride 128 B
// (leading byte offset), 8-row stride 1024 B (stride byte offset), version 1
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
    uint64_t d = uint64_t((saddr >> 4) & 0x3FFF);
    d |= uint64_t(128 >> 4) << 16;
    d |= uint64_t(1024 >> 4) << 32;
    d |= uint64_t(1) << 46;
    return d;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity, int* status) {
    return mbar_wait(bar, parity, status);
}

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads) grouped_gemm_kernel(GemmArgs A) {
    extern __shared__ __align__(1024) uint8_t gsm[];
    uint8_t* sA = gsm;                                   // [2][128 x 64 fp16]
    uint8_t* sB = gsm + 2 * kGemmStageBytes;             // [2][128 x 64 fp16]
    __shared__ __align__(8) uint64_t mbar[2];
    __shared__ uint32_t tbase;
    __shared__ FfnEntry s_en;
    __shared__ int s_tile;
    __shared__ FfnRow s_rows[128];
    __shared__ int s_bad;

    pdl_wait();
    pdl_trigger();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const WorkList W = *A.wl;
    const int total = MODE == 0 ? W.units_gu : W.units_dn;
    if (int(blockIdx.x) >= total) return;
    const int D = A.D;
    if (tid == 0) {
        // entry of this tile: entries are sorted by their first tile
        int lo = 0, hi = W.n_entries - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            const int b = MODE == 0 ? A.entries[mid].ubase_gu : A.entries[mid].ubase_dn;
            if (b <= int(blockIdx.x)) lo = mid; else hi = mid - 1;
        }
        s_en = A.entries[lo];
        s_tile = int(blockIdx.x) - (MODE == 0 ? s_en.ubase_gu : s_en.ubase_dn);
        s_bad = 0;
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        mbar_fence_init();
    }
    __syncthreads();
    const FfnEntry en = s_en;
    const int tile = s_tile;
    const int M = min(en.n_rows, 128);
    const int N = (M + 15) & ~15;
    if (tid < M) s_rows[tid] = A.rows[en.row0 + tid];
    int ncols = 32;
    while (ncols < N) ncols <<= 1;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tbase)),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tbase;
    // D f32, A/B f16, both K-major, N, M = 128
    const uint32_t idesc = (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(128 >> 4) << 24);

    const int F = en.F;
    const int Kin = MODE == 0 ? D : F;
    const int ngroups = Kin / kGroup;
    const int ks = MODE == 0 ? kGuSlice : down_ks(F);
    const int nsl = MODE == 0 ? D / kGuSlice : F / ks;
    const uint8_t* sec = en.blob + (MODE == 0 ? size_t(0) : gu_section_bytes(D, F));
    bool ok = true;

    for (int g = 0; g < ngroups; ++g) {
        const int st = g & 1;
        if (g >= 2 && ok) ok = gemm_wait(&mbar[st], ((g - 2) >> 1) & 1, A.status);  // stage free again
        uint8_t* a = sA + st * kGemmStageBytes;
        uint8_t* b = sB + st * kGemmStageBytes;
        // A: thread tid dequantises weight row tid (blob tile 4*tile + warp, row lane)
        {
            const int bt = 4 * tile + warp;
            const int s = (g * kGroup) / ks, gg = ((g * kGroup) % ks) / kGroup;
            const uint8_t* chunk = sec + (size_t(bt) * nsl + s) * (18u * ks);
            const uint4 qa = *reinterpret_cast<const uint4*>(chunk + ((2 * gg) * 32 + lane) * 16);
            const uint4 qb = *reinterpret_cast<const uint4*>(chunk + ((2 * gg + 1) * 32 + lane) * 16);
            const uint32_t sbw = *reinterpret_cast<const uint32_t*>(chunk + 16 * ks + (gg * 32 + lane) * 4);
            const float sc = f16_to_f32(uint16_t(sbw & 0xFFFF)), bi = f16_to_f32(uint16_t(sbw >> 16));
            const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // word j = inputs 8j .. 8j+7 of the group
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = fmaf(sc, float((words[j] >> (4 * i)) & 15u), bi);
                *reinterpret_cast<uint4*>(a + core_off(tid, 8 * j)) =
                    make_uint4(pack_half2(v[0], v[1]), pack_half2(v[2], v[3]), pack_half2(v[4], v[5]),
                               pack_half2(v[6], v[7]));
            }
        }
        // B: N rows x 64 inputs (rows >= M are zero)
        for (int idx = tid; idx < N * 8; idx += kGemmThreads) {
            const int j = idx >> 3, kb = idx & 7;
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (j < M) {
                const int k0 = g * kGroup + 8 * kb;
                if (MODE == 0) {
                    const uint4 q = *reinterpret_cast<const uint4*>(A.x + size_t(s_rows[j].x_row) * D + k0);
                    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        v[2 * i] = __uint_as_float(w4[i] << 16);
                        v[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
                    }
                } else {
                    const float* hp = A.h + s_rows[j].h_off + k0;
                    const float4 p0 = *reinterpret_cast<const float4*>(hp);
                    const float4 p1 = *reinterpret_cast<const float4*>(hp + 4);
                    v[0] = p0.x; v[1] = p0.y; v[2] = p0.z; v[3] = p0.w;
                    v[4] = p1.x; v[5] = p1.y; v[6] = p1.z; v[7] = p1.w;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (!(fabsf(v[i]) <= 65504.f)) { s_bad = 1; v[i] = 0.f; }  // beyond fp16 (or NaN)
            }
            *reinterpret_cast<uint4*>(b + core_off(j, 8 * kb)) =
                make_uint4(pack_half2(v[0], v[1]), pack_half2(v[2], v[3]), pack_half2(v[4], v[5]),
                           pack_half2(v[6], v[7]));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (tid == 0 && ok) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = umma_desc(smem_u32(a) + kk * 256);
                const uint64_t bd = umma_desc(smem_u32(b) + kk * 256);
                const uint32_t acc = (g > 0 || kk > 0) ? 1u : 0u;
                asm volatile(
                    "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, "
                    "p;\n}\n" ::"r"(tmem),
                    "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                    : "memory");
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(&mbar[st]))
                         : "memory");
        }
    }
    // all MMAs done (a commit tracks every MMA issued before it)
    const int last = ngroups - 1;
    if (ok) ok = gemm_wait(&mbar[last & 1], (last >> 1) & 1, A.status);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (s_bad && tid == 0) set_status(A.status, MOE_ERR_RANGE);

    if (ok) {
        for (int c0 = 0; c0 < N; c0 += 16) {
            uint32_t v[16];
            const uint32_t ta = tmem + (uint32_t(warp * 32) << 16) + uint32_t(c0);
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                  "=r"(v[15])
                : "r"(ta)
                : "memory");
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const int j = c0 + jj;
                const float d = __uint_as_float(v[jj]);
                if (MODE == 0) {
                    // warp = blob tile 4*tile + warp: lanes 0..15 gate, 16..31 up of outputs 16*bt + lane
                    const float up = __shfl_down_sync(0xffffffffu, d, 16);
                    if (lane < 16 && j < M)
                        A.h[s_rows[j].h_off + 16 * (4 * tile + warp) + lane] = gelu_tanh(d) * up;
                } else if (j < M) {
                    atomicAdd(&A.y[size_t(s_rows[j].y_row) * D + 128 * tile + 32 * warp + lane], s_rows[j].w * d);
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
}

size_t gemm_smem_bytes() { return size_t(4) * kGemmStageBytes; }

cudaError_t gemm_prepare() {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(gemm_smem_bytes()));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(gemm_smem_bytes()));
}

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t s, void (*hook)(void*, int), void* hook_arg) {
    GemmArgs a;
    a.wl = L.wl;
    a.entries = L.entries;
    a.rows = L.rows;
    a.x = L.x;
    a.h = L.h;
    a.y = L.y;
    a.D = L.D;
    a.status = L.status;
    if (hook) hook(hook_arg, 0);
    cudaError_t e = launch_kernel(grouped_gemm_kernel<0>, dim3(L.max_tiles_gu), dim3(kGemmThreads),
                                  gemm_smem_bytes(), s, L.pdl, 1, a);
    if (e != cudaSuccess) return e;
    if (hook) hook(hook_arg, 1);
    e = launch_kernel(grouped_gemm_kernel<1>, dim3(L.max_tiles_dn), dim3(kGemmThreads), gemm_smem_bytes(), s, L.pdl,
                      1, a);
    if (hook) hook(hook_arg, 2);
    return e;
}

// y (fp32) -> bf16, for the prefill path's optional bf16 output
__global__ void f32_to_bf16_kernel(const float* __restrict__ y, uint16_t* __restrict__ out, size_t n) {
    pdl_wait();
    pdl_trigger();
    for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n; i += size_t(gridDim.x) * blockDim.x)
        out[i] = f32_to_bf16_rn(y[i]);
}

cudaError_t launch_f32_to_bf16(const float* y, uint16_t* out, size_t n, bool pdl, cudaStream_t s) {
    const int blocks = int(n / 256 + 1 < 1024 ? n / 256 + 1 : 1024);
    return launch_kernel(f32_to_bf16_kernel, dim3(blocks), dim3(256), 0, s, pdl, 1, y, out, n);
}

}  // namespace moe
