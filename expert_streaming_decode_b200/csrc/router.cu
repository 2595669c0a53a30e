// router.cu -- K1: 8-bit router GEMV + top-K + softmax gate weights.
//
// Method: per token the layer's router scores the E experts and keeps the K
// most relevant ("El milagro de la IA de 2GB en Apple Silicon", section "Por
// que la mayor parte de tu modelo de IA es peso muerto"); the router is 8-bit
// ("TurboFieldfare: motor open source ...", section "Estructura de ejecucion
// para reducir memoria").  Gate weights: softmax over the K chosen logits.
//
// B200 mapping: one thread-block cluster of kRouterCtas CTAs per token.  CTA c
// scores experts [c*E/kRouterCtas, (c+1)*E/kRouterCtas): every thread runs the
// fp32 FMA chain of one (expert, group of 64) pair from 16-byte loads of the
// int8 row, then one thread per expert chains the group sums with their
// scales.  Logits land in rank 0's shared memory through distributed shared
// memory; rank 0's first warp selects the top-K with shuffles and writes ids
// and weights.  The FMA order is fixed (below), so ids are bit-reproducible.
#include <cooperative_groups.h>

#include "common.cuh"
#include "decode_wl.cuh"
#include "launch.cuh"

namespace cg = cooperative_groups;

namespace moe {

constexpr int kRouterCtas = 8;
constexpr int kRouterThreads = 256;
constexpr int kMaxE = 1024;

// logit_e = fma-chain_g( s[e][g] * S_g ) + bias_e,
// S_g     = fma-chain_{k in g, ascending}( q[e][k] * x[k] ), both from 0.
__global__ void __launch_bounds__(kRouterThreads) router_topk_kernel(
    const uint16_t* __restrict__ x, const int8_t* __restrict__ wq, const uint16_t* __restrict__ ws,
    const float* __restrict__ bias, int E, int D, int K, int32_t* __restrict__ ids, float* __restrict__ gate_w,
    int* status, DecodeWLTarget wlt, const uint8_t* __restrict__ pf_ptr, size_t pf_bytes) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = int(cluster.block_rank());
    const int t = blockIdx.y;
    const int ng = D / kGroup;
    const int e_per = E / kRouterCtas;
    const int e0 = rank * e_per;

    extern __shared__ float sm[];
    float* xs = sm;                       // [ng][kGroup + 1] hidden state in fp32 (padded rows)
    float* gsum = xs + ng * (kGroup + 1); // [e_per][ng] group sums
    __shared__ float logits[kMaxE];       // rank 0 gathers all logits here

    // prologue (may overlap the previous kernel): pull this CTA's router rows
    // towards L2; they are immutable
    (void)pf_ptr;
    (void)pf_bytes;
    for (int i = threadIdx.x; i < e_per * ng; i += blockDim.x) {
        const int g = i / e_per, el = i % e_per;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(wq + size_t(e0 + el) * D + size_t(g) * kGroup));
    }
    pdl_wait();
    pdl_trigger();
    for (int k = threadIdx.x; k < D; k += blockDim.x)
        xs[(k / kGroup) * (kGroup + 1) + k % kGroup] = bf16_to_f32(x[size_t(t) * D + k]);
    __syncthreads();

    // group chains: work item i = (group g, expert el); neighbouring threads
    // share g, so their hidden-state reads are shared-memory broadcasts
    for (int i = threadIdx.x; i < e_per * ng; i += blockDim.x) {
        const int g = i / e_per, el = i % e_per;
        const int4* row = reinterpret_cast<const int4*>(wq + size_t(e0 + el) * D + size_t(g) * kGroup);
        int4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = __ldg(row + j);
        float S = 0.0f;
        const float* xg = xs + g * (kGroup + 1);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w4[4] = {uint32_t(v[j].x), uint32_t(v[j].y), uint32_t(v[j].z), uint32_t(v[j].w)};
#pragma unroll
            for (int b = 0; b < 16; ++b) {
                const int8_t q = int8_t((w4[b >> 2] >> (8 * (b & 3))) & 0xFF);
                S = __fmaf_rn(float(q), xg[j * 16 + b], S);
            }
        }
        gsum[el * ng + g] = S;
    }
    __syncthreads();

    // expert chains over groups, then publish to rank 0 (DSMEM); the first
    // cluster barrier guarantees every CTA of the cluster is running
    cluster.sync();
    float* logits0 = cluster.map_shared_rank(logits, 0);
    for (int el = threadIdx.x; el < e_per; el += blockDim.x) {
        const int e = e0 + el;
        float acc = 0.0f;
        for (int g = 0; g < ng; ++g) acc = __fmaf_rn(f16_to_f32(ws[size_t(e) * ng + g]), gsum[el * ng + g], acc);
        if (bias) acc = __fadd_rn(acc, bias[e]);
        logits0[e] = acc;
    }
    cluster.sync();
    if (rank != 0 || threadIdx.x >= 32) return;

    // top-K by (logit desc, id asc) with warp shuffles; lane L owns ids L, L+32, ...
    const int lane = threadIdx.x;
    bool nan = false;
    for (int e = lane; e < E; e += 32) nan |= isnan(logits[e]);
    nan = __any_sync(0xffffffffu, nan);
    if (nan) {
        if (lane < K) { ids[size_t(t) * K + lane] = lane; gate_w[size_t(t) * K + lane] = 1.0f / K; }
        if (lane == 0) set_status(status, MOE_ERR_NAN);
        if (wlt.wl) write_decode_worklist(wlt, K, lane, 1.0f / K, true);
        return;
    }
    uint32_t taken = 0;  // bit j: id lane + 32*j already selected (E <= 1024)
    float sel_l = 0.f;
    int sel_id = 0;
    for (int i = 0; i < K; ++i) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int j = 0, e = lane; e < E; ++j, e += 32) {
            if ((taken >> j) & 1u) continue;
            const float v = logits[e];
            if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == i) { sel_l = bv; sel_id = bi; }
    }
    // softmax over the K chosen (lane i holds the i-th largest; lane 0 the max)
    const float m = __shfl_sync(0xffffffffu, sel_l, 0);
    const float ex = lane < K ? expf(sel_l - m) : 0.0f;
    float z = 0.0f;
    for (int i = 0; i < K; ++i) z += __shfl_sync(0xffffffffu, ex, i);
    if (lane < K) {
        ids[size_t(t) * K + lane] = sel_id;
        gate_w[size_t(t) * K + lane] = ex / z;
    }
    // one token, resident experts: the expert FFN work list (slot = expert id)
    if (wlt.wl) write_decode_worklist(wlt, K, sel_id, ex / z, true);
}

cudaError_t launch_router(const uint16_t* x, const int8_t* wq, const uint16_t* ws, const float* bias, int E, int D,
                          int K, int T, int32_t* ids, float* gate_w, int* status, const DecodeWLTarget& wlt,
                          const uint8_t* pf_ptr, size_t pf_bytes, bool pdl, cudaStream_t s) {
    const int ng = D / kGroup;
    const size_t smem = size_t(ng) * (kGroup + 1) * 4 + size_t(E / kRouterCtas) * ng * 4;  // < 48 KB for D <= 8192
    return launch_kernel(router_topk_kernel, dim3(kRouterCtas, T, 1), dim3(kRouterThreads), smem, s, pdl, kRouterCtas,
                         x, wq, ws, bias, E, D, K, ids, gate_w, status, wlt, pf_ptr, pf_bytes);
}

}  // namespace moe
