// attn.cu -- decode attention for one token over a binary16 KV cache, split
// along the cached positions and merged exactly.
//
// Method: "TurboFieldfare: motor open source ...", section "Proceso de
// generacion de tokens": decode attention is an exact split-K/V method, and
// the fp16 KV cache is a bounded ring for the sliding-window layers and linear
// storage for the full-attention layers.  Reading: the cached positions of a
// KV head are cut into parts; each part yields its running maximum m, its sum
// of exponentials l and its unnormalised value sum o (the K path gives the
// weights, the V path the sums); parts merge by rescaling with 2^(m_j - M),
// which is exact up to rounding, so the result is softmax attention itself.
//
// Work decomposition (HBM-bound: every cached byte is read once):
//   grid (parts, KV heads); CTA = kAttnWarps warps; a CTA owns a contiguous
//   range of slots of one KV head and serves all query heads of its group,
//   so each K/V row is read once for the whole group.  A warp takes four rows
//   at a time (two at head width 512): each lane loads its 16-byte (or smaller) piece
//   of every row (a row of a head is contiguous, so a warp's load is one
//   coalesced segment), dot products reduce by shuffles, and an online softmax
//   keeps (m, l, o) per query head in registers.  Warps merge in shared
//   memory, parts merge in the last CTA of the KV head to finish (an atomic
//   ticket; no CTA ever waits for another).
#include <cuda_fp16.h>

#include "common.cuh"
#include "launch.cuh"
#include "moe.h"

namespace moe {

namespace {

constexpr int kAttnWarps = 8;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kAttnUnroll = 4;      // rows a warp has in flight
constexpr int kAttnMaxSplits = 64;  // parts per KV head
constexpr int kAttnMaxKvHeads = 64;
constexpr int kAttnCounterBytes = 256;  // kAttnMaxKvHeads tickets
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// A lane's share of one head row: DPL binary16 values in DPL/2 words.
// DPL >= 8: 16-byte pieces at element 8*(lane + 32*i), i < DPL/8, so that each
// load instruction of the warp covers 512 contiguous bytes; DPL < 8: the
// lane's DPL contiguous elements at lane*DPL.
template <int DPL>
struct RowPiece {
    uint32_t w[DPL / 2];
};
template <int DPL>
__device__ __forceinline__ int piece_elem(int lane, int i) {  // first element of word group i
    if constexpr (DPL >= 8) return 8 * (lane + 32 * i);
    else return lane * DPL;
}
template <int DPL>
__device__ __forceinline__ RowPiece<DPL> load_piece(const uint16_t* row, int lane) {
    RowPiece<DPL> r;
    if constexpr (DPL >= 8) {
#pragma unroll
        for (int i = 0; i < DPL / 8; ++i) {
            const uint4 u = ld_stream_v4(row + piece_elem<DPL>(lane, i));
            r.w[4 * i] = u.x; r.w[4 * i + 1] = u.y; r.w[4 * i + 2] = u.z; r.w[4 * i + 3] = u.w;
        }
    } else if constexpr (DPL == 4) {
        const uint2 u = ld_stream_v2(row + piece_elem<DPL>(lane, 0));
        r.w[0] = u.x; r.w[1] = u.y;
    } else {
        r.w[0] = ld_stream_u32(row + piece_elem<DPL>(lane, 0));
    }
    return r;
}
// element index of value j (0..DPL-1) of a lane's piece
template <int DPL>
__device__ __forceinline__ int piece_index(int lane, int j) {
    if constexpr (DPL >= 8) return piece_elem<DPL>(lane, j / 8) + (j % 8);
    else return lane * DPL + j;
}

__device__ __forceinline__ float2 h2_to_f2(uint32_t w) { return __half22float2(*reinterpret_cast<__half2*>(&w)); }

struct AttnArgs {
    const uint16_t* q;  // bf16 [Hq][hd]
    const uint16_t* k;  // binary16 [Hkv][cap][hd]
    const uint16_t* v;
    float* o;           // fp32 [Hq][hd]
    int* tickets;       // [Hkv], zero between calls
    float2* part_ml;    // [Hkv][kAttnMaxSplits][G] (m, l), base-2 exponent units
    float* part_o;      // [Hkv][kAttnMaxSplits][G][hd]
    int hd, cap, L, chunk;
    float qscale;       // scale * log2(e)
};

template <int DPL, int G>
__global__ void __launch_bounds__(kAttnThreads, 2) attn_decode_kernel(AttnArgs A) {
    constexpr int HD = DPL * 32;
    constexpr int U = DPL >= 16 ? 2 : kAttnUnroll;  // rows in flight per warp (register budget)
    __shared__ float s_acc[kAttnWarps][G][HD];
    __shared__ float s_m[kAttnWarps][G], s_l[kAttnWarps][G];
    __shared__ float s_f[G][kAttnMaxSplits];
    __shared__ float s_den[G];
    __shared__ int s_last;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y, part = blockIdx.x, S = gridDim.x;
    const int p0 = part * A.chunk, p1 = min(A.L, p0 + A.chunk);
    const uint16_t* kh = A.k + size_t(h) * A.cap * HD;
    const uint16_t* vh = A.v + size_t(h) * A.cap * HD;

    // Start this part's rows streaming into L2 (a hint: no data is read and
    // nothing waits on it), then wait for the preceding kernel in the stream.
    // Everything the kernel reads or writes comes after the wait, so with
    // programmatic dependent launch the next layer's rows stream in while
    // this kernel's last parts merge.
    if (warp == 0) {
        const size_t off = size_t(p0) * HD, bytes = size_t(p1 - p0) * HD * sizeof(uint16_t);
        bulk_prefetch_l2(kh + off, bytes, lane, 32);
        bulk_prefetch_l2(vh + off, bytes, lane, 32);
    }
    pdl_wait();
    pdl_trigger();

    // the warp's first rows, then the group's queries (pre-scaled so that
    // exp(scale*q.k) = 2^(q'.k)) while those rows are in flight
    RowPiece<DPL> kr[U], vr[U];
    int p = p0 + warp * U;
#pragma unroll
    for (int u = 0; u < U; ++u)
        if (p + u < p1) {
            kr[u] = load_piece<DPL>(kh + size_t(p + u) * HD, lane);
            vr[u] = load_piece<DPL>(vh + size_t(p + u) * HD, lane);
        }
    float qr[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int j = 0; j < DPL; ++j)
            qr[g][j] = bf16_to_f32(A.q[size_t(h * G + g) * HD + piece_index<DPL>(lane, j)]) * A.qscale;

    float m[G], l[G], acc[G][DPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int j = 0; j < DPL; ++j) acc[g][j] = 0.f;
    }

    for (; p < p1; p += kAttnWarps * U) {
        float s[U][G];
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int g = 0; g < G; ++g) s[u][g] = 0.f;
            if (p + u < p1) {
#pragma unroll
                for (int w = 0; w < DPL / 2; ++w) {
                    const float2 kf = h2_to_f2(kr[u].w[w]);
#pragma unroll
                    for (int g = 0; g < G; ++g) s[u][g] = fmaf(qr[g][2 * w + 1], kf.y, fmaf(qr[g][2 * w], kf.x, s[u][g]));
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int g = 0; g < G; ++g) s[u][g] += __shfl_xor_sync(0xffffffffu, s[u][g], off);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float mx = m[g];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (p + u < p1) mx = fmaxf(mx, s[u][g]);
            const float c = exp2f(m[g] - mx);  // 0 while m is -inf; mx is finite (row p is valid)
            l[g] *= c;
#pragma unroll
            for (int j = 0; j < DPL; ++j) acc[g][j] *= c;
            m[g] = mx;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (p + u >= p1) continue;
            float e[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                e[g] = exp2f(s[u][g] - m[g]);
                l[g] += e[g];
            }
#pragma unroll
            for (int w = 0; w < DPL / 2; ++w) {
                const float2 vf = h2_to_f2(vr[u].w[w]);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    acc[g][2 * w] = fmaf(e[g], vf.x, acc[g][2 * w]);
                    acc[g][2 * w + 1] = fmaf(e[g], vf.y, acc[g][2 * w + 1]);
                }
            }
        }
        // the warp's next rows (the registers are free again)
        const int pn = p + kAttnWarps * U;
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (pn + u < p1) {
                kr[u] = load_piece<DPL>(kh + size_t(pn + u) * HD, lane);
                vr[u] = load_piece<DPL>(vh + size_t(pn + u) * HD, lane);
            }
    }

    // warps -> this part
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int j = 0; j < DPL; ++j) s_acc[warp][g][piece_index<DPL>(lane, j)] = acc[g][j];
        if (lane == 0) {
            s_m[warp][g] = m[g];
            s_l[warp][g] = l[g];
        }
    }
    __syncthreads();
    const size_t pbase = size_t(h) * kAttnMaxSplits + part;
    for (int i = tid; i < G * HD; i += kAttnThreads) {
        const int g = i / HD, d = i % HD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_m[w][g]);
        float O = 0.f, Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            const float f = s_m[w][g] == -INFINITY ? 0.f : exp2f(s_m[w][g] - M);
            O = fmaf(f, s_acc[w][g][d], O);
            Ls = fmaf(f, s_l[w][g], Ls);
        }
        A.part_o[(pbase * G + g) * HD + d] = O;
        if (d == 0) A.part_ml[pbase * G + g] = make_float2(M, Ls);
    }

    // the last part of this KV head to finish merges all parts, in part order
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(A.tickets + h, 1) == S - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (warp < G) {
        // per part j (lanes j and j + 32): its factor 2^(m_j - M) and the
        // normaliser sum_j 2^(m_j - M) l_j, reduced in a fixed order
        const int g = warp;
        const float2* ml = A.part_ml + size_t(h) * kAttnMaxSplits * G + g;
        const float2 a0 = lane < S ? __ldcg(ml + size_t(lane) * G) : make_float2(-INFINITY, 0.f);
        const float2 a1 = lane + 32 < S ? __ldcg(ml + size_t(lane + 32) * G) : make_float2(-INFINITY, 0.f);
        float M = fmaxf(a0.x, a1.x);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float f0 = lane < S ? exp2f(a0.x - M) : 0.f;
        const float f1 = lane + 32 < S ? exp2f(a1.x - M) : 0.f;
        s_f[g][lane] = f0;
        s_f[g][lane + 32] = f1;
        float den = fmaf(f0, a0.y, f1 * a1.y);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
        if (lane == 0) s_den[g] = den;
    }
    __syncthreads();
    // each output element: all parts' partial sums loaded together, then summed in part order
    constexpr int kBatch = 16;
    for (int i = tid; i < G * HD; i += kAttnThreads) {
        const int g = i / HD, d = i % HD;
        const float* po = A.part_o + (size_t(h) * kAttnMaxSplits * G + g) * HD + d;
        float num = 0.f;
        for (int j0 = 0; j0 < S; j0 += kBatch) {
            float t[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) t[u] = j0 + u < S ? __ldcg(po + size_t(j0 + u) * G * HD) : 0.f;
#pragma unroll
            for (int u = 0; u < kBatch; ++u) num = fmaf(s_f[g][(j0 + u) & (kAttnMaxSplits - 1)], t[u], num);
        }
        A.o[size_t(h * G + g) * HD + d] = num / s_den[g];
    }
    if (tid == 0) atomicExch(A.tickets + h, 0);  // ready for the next call
}

template <int DPL, int G>
cudaError_t launch_attn(const AttnArgs& a, dim3 grid, cudaStream_t s) {
    return launch_kernel(attn_decode_kernel<DPL, G>, grid, dim3(kAttnThreads), 0, s, true, 1, a);
}

template <int DPL>
cudaError_t launch_attn_g(const AttnArgs& a, int G, dim3 grid, cudaStream_t s) {
    switch (G) {
        case 1: return launch_attn<DPL, 1>(a, grid, s);
        case 2: return launch_attn<DPL, 2>(a, grid, s);
        case 4: if constexpr (DPL * 4 <= 32) return launch_attn<DPL, 4>(a, grid, s); else break;
        case 8: if constexpr (DPL * 8 <= 32) return launch_attn<DPL, 8>(a, grid, s); else break;
        default: break;
    }
    return cudaErrorInvalidValue;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_attn_workspace_bytes(int n_heads_q, int head_dim) {
    if (n_heads_q < 1 || head_dim < 1) return 0;
    return size_t(kAttnCounterBytes) + size_t(n_heads_q) * kAttnMaxSplits * sizeof(float2) +
           size_t(n_heads_q) * kAttnMaxSplits * size_t(head_dim) * sizeof(float);
}

int moe_attn_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache, int n_heads_q,
                    int n_heads_kv, int head_dim, int capacity, int n_tokens, float scale, float* o,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !k_cache || !v_cache || !o || !workspace) return MOE_ERR_ARG;
    if (n_tokens < 1 || capacity < 1 || n_heads_kv < 1 || n_heads_kv > kAttnMaxKvHeads) return MOE_ERR_ARG;
    if (n_heads_q % n_heads_kv != 0) return MOE_ERR_ARG;
    const int G = n_heads_q / n_heads_kv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return MOE_ERR_ARG;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256 && head_dim != 512) return MOE_ERR_ARG;
    if ((head_dim / 32) * G > 32) return MOE_ERR_ARG;
    if (!(scale > 0.f) || !(scale < INFINITY)) return MOE_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(workspace))
        return MOE_ERR_ARG;
    if (workspace_bytes < moe_attn_workspace_bytes(n_heads_q, head_dim)) return MOE_ERR_ARG;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm < 1)
        return MOE_ERR_CUDA;
    // attended slots: the ring holds the newest min(n, capacity) positions
    const int L = n_tokens < capacity ? n_tokens : capacity;
    // about two CTAs per SM: parts per KV head, each a multiple of the unroll
    int want = (2 * nsm + n_heads_kv - 1) / n_heads_kv;
    if (want > kAttnMaxSplits) want = kAttnMaxSplits;
    int chunk = (L + want - 1) / want;
    chunk = (chunk + kAttnUnroll - 1) / kAttnUnroll * kAttnUnroll;
    const int S = (L + chunk - 1) / chunk;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    AttnArgs a;
    a.q = q;
    a.k = k_cache;
    a.v = v_cache;
    a.o = o;
    a.tickets = reinterpret_cast<int*>(ws);
    a.part_ml = reinterpret_cast<float2*>(ws + kAttnCounterBytes);
    a.part_o = reinterpret_cast<float*>(ws + kAttnCounterBytes + size_t(n_heads_q) * kAttnMaxSplits * sizeof(float2));
    a.hd = head_dim;
    a.cap = capacity;
    a.L = L;
    a.chunk = chunk;
    a.qscale = scale * kLog2e;
    const dim3 grid(S, n_heads_kv);
    cudaError_t e;
    switch (head_dim) {
        case 64: e = launch_attn_g<2>(a, G, grid, stream); break;
        case 128: e = launch_attn_g<4>(a, G, grid, stream); break;
        case 256: e = launch_attn_g<8>(a, G, grid, stream); break;
        default: e = launch_attn_g<16>(a, G, grid, stream); break;
    }
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
