// router.cu -- K1: 8-bit router GEMV + top-K + softmax gate weights.
//
// Method: per token the layer's router scores the E experts and keeps the K
// most relevant ("El milagro de la IA de 2GB en Apple Silicon", section "Por
// que la mayor parte de tu modelo de IA es peso muerto"); the router is 8-bit
// ("TurboFieldfare: motor open source ...", section "Estructura de ejecucion
// para reducir memoria").  Gate weights: softmax over the K chosen logits.
//
// B200 mapping: one thread-block cluster of kRouterCtas CTAs per token.  CTA c
// scores experts [c*E/kRouterCtas, (c+1)*E/kRouterCtas).  Its int8 rows are
// immutable, so before waiting on the kernel that writes the hidden state the
// CTA starts bulk copies of them (one per row, rows padded by 16 B so that
// neighbouring threads reading neighbouring rows hit different banks) into
// shared memory, and reads their group scales; when many rows do not fit, they
// go in passes through two buffers.  Every thread then runs the fp32 FMA
// chain of one (expert, group of 64) pair; one thread per expert chains the
// group sums with their scales.  Logits land in rank 0's shared memory through
// distributed shared memory; in rank 0 every expert counts the experts that
// rank above it (logit descending, id ascending), the K with fewer than K
// above are the selection, and the first warp writes ids and weights.  The
// FMA order is fixed (below), so ids are bit-reproducible.
#include <cooperative_groups.h>

#include "common.cuh"
#include "decode_wl.cuh"
#include "launch.cuh"

namespace cg = cooperative_groups;

namespace moe {

constexpr int kRouterCtas = 16;  // a non-portable cluster size (B200 allows 16)
constexpr int kRouterThreads = 512;
constexpr int kMaxE = 1024;
constexpr int kMaxK = 16;
constexpr int kRouterRowPad = 16;               // bytes added to every staged row
constexpr size_t kRouterRingBudget = 120 << 10; // shared memory for staged rows
constexpr size_t kRouterSmemMax = 200 << 10;    // dynamic shared memory limit of the kernel

struct RouterShape {
    int e_per, rows, passes, nbuf;
    size_t row_bytes, buf_bytes, smem;
};

__host__ __device__ inline RouterShape router_shape(int E, int D) {
    RouterShape r;
    const int ng = D / kGroup;
    r.e_per = E / kRouterCtas;
    r.row_bytes = size_t(D) + kRouterRowPad;
    if (size_t(r.e_per) * r.row_bytes <= kRouterRingBudget) {  // all rows in one pass
        r.rows = r.e_per;
        r.nbuf = 1;
    } else {  // passes through two buffers of half the budget each
        const int rows = int(kRouterRingBudget / 2 / r.row_bytes);
        r.rows = rows < 1 ? 1 : rows;
        r.nbuf = 2;
    }
    r.passes = (r.e_per + r.rows - 1) / r.rows;
    r.buf_bytes = size_t(r.rows) * r.row_bytes;
    // [nbuf][rows][D + pad] int8 | xs [ng][kGroup + 1] f32 | gsum [rows][ng] f32 | scales [rows][ng] f32
    r.smem = r.nbuf * r.buf_bytes + size_t(ng) * (kGroup + 1) * 4 + 2 * size_t(r.rows) * ng * 4;
    return r;
}

// exact int8 -> fp32 without a conversion instruction: with the byte's sign
// bit flipped, the byte is q + 128 in 0..255; spliced into the mantissa of
// 2^23 it gives 2^23 + q + 128 exactly, and subtracting 2^23 + 128 leaves q.
__device__ __forceinline__ float i8_to_f32(uint32_t flipped_word, int byte) {
    return __uint_as_float(__byte_perm(flipped_word, 0x4B000000u, 0x7540u + uint32_t(byte))) - 8388736.0f;
}

// logit_e = fma-chain_g( s[e][g] * S_g ) + bias_e,
// S_g     = fma-chain_{k in g, ascending}( q[e][k] * x[k] ), both from 0.
__global__ void __launch_bounds__(kRouterThreads) router_topk_kernel(
    const uint16_t* __restrict__ x, const int8_t* __restrict__ wq, const uint16_t* __restrict__ ws,
    const float* __restrict__ bias, int E, int D, int K, int32_t* __restrict__ ids, float* __restrict__ gate_w,
    int* status, DecodeWLTarget wlt) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = int(cluster.block_rank());
    const int t = blockIdx.y;
    const int ng = D / kGroup;
    const RouterShape sh = router_shape(E, D);
    const int e0 = rank * sh.e_per;

    extern __shared__ __align__(16) uint8_t rsm[];
    uint8_t* ring = rsm;                                                    // staged int8 rows
    float* xs = reinterpret_cast<float*>(rsm + sh.nbuf * sh.buf_bytes);     // [ng][kGroup + 1]
    float* gsum = xs + ng * (kGroup + 1);                                   // [rows][ng]
    float* scl = gsum + sh.rows * ng;                                       // [rows][ng]
    __shared__ float logits[kMaxE];  // rank 0 gathers all logits here
    __shared__ float s_bias[kMaxE / kRouterCtas];
    __shared__ int s_sel_id[kMaxK], s_nan;
    __shared__ float s_sel_l[kMaxK];
    __shared__ __align__(8) uint64_t full[2];
    __shared__ int s_ok;

    int issued = 0;  // passes whose copies thread 0 has started
    auto rows_of = [&](int p) { return min(sh.rows, sh.e_per - p * sh.rows); };
    auto issue = [&](int p) {  // thread 0: bulk copies of pass p's rows into buffer p & 1
        issued = p + 1;
        const int nr = rows_of(p);
        uint64_t* bar = &full[p & 1];
        mbar_arrive_expect_tx(bar, uint32_t(nr) * uint32_t(D));
        const uint64_t pol = l2_evict_last();
        uint8_t* dst = ring + size_t(p & 1) * sh.buf_bytes;
        for (int r = 0; r < nr; ++r)
            bulk_g2s(dst + size_t(r) * sh.row_bytes, wq + size_t(e0 + p * sh.rows + r) * D, uint32_t(D), bar, pol);
    };
    auto load_scales = [&](int p) {
        const int nr = rows_of(p);
        for (int i = threadIdx.x; i < nr * ng; i += blockDim.x)
            scl[i] = f16_to_f32(ws[size_t(e0 + p * sh.rows) * ng + i]);
    };

    // prologue (may overlap the previous kernel): only immutable router weights
    if (threadIdx.x == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_fence_init();
        s_ok = 1;
        s_nan = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        issue(0);
        if (sh.passes > 1) issue(1);
    }
    load_scales(0);
    // every CTA of the cluster is running before anyone writes rank 0's logits
    cluster.sync();

    pdl_wait();
    pdl_trigger();
    // hidden state: one 16-byte load (8 inputs of one group) per thread and
    // round, all issued before any is used; the CTA's logit biases likewise
    {
        const uint4* x8 = reinterpret_cast<const uint4*>(x + size_t(t) * D);
        constexpr int kRounds = 2;  // D / 8 <= kRounds * kRouterThreads for D <= 8192
        uint4 v[kRounds];
#pragma unroll
        for (int i = 0; i < kRounds; ++i) {
            const int c = threadIdx.x + i * kRouterThreads;
            if (c < D / 8) v[i] = x8[c];
        }
        if (bias && threadIdx.x < sh.e_per) s_bias[threadIdx.x] = bias[e0 + threadIdx.x];
#pragma unroll
        for (int i = 0; i < kRounds; ++i) {
            const int c = threadIdx.x + i * kRouterThreads;
            if (c >= D / 8) continue;
            float* dst = xs + (c / 8) * (kGroup + 1) + (c % 8) * 8;  // inputs 8c .. 8c+7, one group
            const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                dst[2 * j] = __uint_as_float(w4[j] << 16);
                dst[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
            }
        }
    }
    float* logits0 = cluster.map_shared_rank(logits, 0);

    int consumed = 0;  // passes whose copies have landed
    for (int p = 0; p < sh.passes; ++p) {
        const int nr = rows_of(p);
        if (p > 0) {
            load_scales(p);
            if (threadIdx.x == 0 && p + 1 < sh.passes) {
                // buffer (p + 1) & 1 was last read in pass p - 1 (all threads past the barrier below)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue(p + 1);
            }
        }
        if (threadIdx.x == 0) {
            if (mbar_wait(&full[p & 1], uint32_t((p >> 1) & 1), status)) consumed = p + 1;
            else s_ok = 0;
        }
        __syncthreads();  // staged rows, scales and (first pass) xs are ready
        if (!s_ok) break;
        const uint8_t* buf = ring + size_t(p & 1) * sh.buf_bytes;

        // group chains: work item i = (group g, row r); neighbouring threads
        // share g, so their hidden-state reads are shared-memory broadcasts
        for (int i = threadIdx.x; i < nr * ng; i += blockDim.x) {
            const int g = i / nr, r = i % nr;
            const uint4* row = reinterpret_cast<const uint4*>(buf + size_t(r) * sh.row_bytes + size_t(g) * kGroup);
            const float* xg = xs + g * (kGroup + 1);
            float S = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = row[j];
                const uint32_t w4[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u,
                                        v.w ^ 0x80808080u};
#pragma unroll
                for (int b = 0; b < 16; ++b) S = __fmaf_rn(i8_to_f32(w4[b >> 2], b & 3), xg[j * 16 + b], S);
            }
            gsum[r * ng + g] = S;
        }
        __syncthreads();
        // expert chains over groups, published to rank 0 (DSMEM)
        for (int r = threadIdx.x; r < nr; r += blockDim.x) {
            const int e = e0 + p * sh.rows + r;
            float acc = 0.0f;
            for (int g = 0; g < ng; ++g) acc = __fmaf_rn(scl[r * ng + g], gsum[r * ng + g], acc);
            if (bias) acc = __fadd_rn(acc, s_bias[p * sh.rows + r]);
            logits0[e] = acc;
        }
        __syncthreads();  // gsum and scales are rewritten by the next pass
    }
    // after a failed wait: wait (bounded) for the copies still in flight, so
    // none lands after exit, and mark this CTA's logits NaN so rank 0 reports it
    if (!s_ok && threadIdx.x == 0)
        for (int q = consumed; q < issued; ++q) (void)mbar_wait(&full[q & 1], uint32_t((q >> 1) & 1), status);
    if (!s_ok)
        for (int e = e0 + threadIdx.x; e < e0 + sh.e_per; e += blockDim.x) logits0[e] = __int_as_float(0x7fc00000);
    cluster.sync();
    if (rank != 0) return;

    // top-K by (logit desc, id asc): every expert counts the experts ranked
    // above it, four threads per expert each over every fourth id
    // (shared-memory broadcast reads); ranks 0..K-1 are the selection
    for (int eb = 0; eb < E; eb += kRouterThreads / 4) {
        const int e = eb + int(threadIdx.x >> 2), part = threadIdx.x & 3;
        const float v = e < E ? logits[e] : 0.f;
        int above = 0;
        if (e < E) {
            for (int f = part; f < E; f += 4) {  // the four threads read four neighbouring words
                const float u = logits[f];
                above += (u > v) || (u == v && f < e);
            }
        }
        above += __shfl_xor_sync(0xffffffffu, above, 1);
        above += __shfl_xor_sync(0xffffffffu, above, 2);
        if (e < E && part == 0) {
            if (isnan(v)) s_nan = 1;
            else if (above < K) {
                s_sel_id[above] = e;
                s_sel_l[above] = v;
            }
        }
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    if (s_nan) {
        if (lane < K) { ids[size_t(t) * K + lane] = lane; gate_w[size_t(t) * K + lane] = 1.0f / K; }
        if (lane == 0) set_status(status, MOE_ERR_NAN);
        if (wlt.wl) write_decode_worklist(wlt, K, lane, 1.0f / K, true);
        return;
    }
    const float sel_l = lane < K ? s_sel_l[lane] : 0.f;
    const int sel_id = lane < K ? s_sel_id[lane] : 0;
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

size_t router_smem_bytes(int E, int D) { return router_shape(E, D).smem; }

cudaError_t launch_router(const uint16_t* x, const int8_t* wq, const uint16_t* ws, const float* bias, int E, int D,
                          int K, int T, int32_t* ids, float* gate_w, int* status, const DecodeWLTarget& wlt,
                          bool pdl, cudaStream_t s) {
    const size_t smem = router_smem_bytes(E, D);
    static thread_local int attr_set_for = -1;  // device whose attribute this thread last set
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (attr_set_for != dev) {
        e = cudaFuncSetAttribute(router_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kRouterSmemMax));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(router_topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        attr_set_for = dev;
    }
    if (smem > kRouterSmemMax) return cudaErrorInvalidValue;
    return launch_kernel(router_topk_kernel, dim3(kRouterCtas, T, 1), dim3(kRouterThreads), smem, s, pdl, kRouterCtas,
                         x, wq, ws, bias, E, D, K, ids, gate_w, status, wlt);
}

}  // namespace moe
