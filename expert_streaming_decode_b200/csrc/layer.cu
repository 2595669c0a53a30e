// layer.cu -- the one-token MoE layer as one persistent kernel: router, top-K,
// gate weights, cache plan, shared and routed expert FFNs and the combine, with
// two grid-wide barriers instead of five launches.
//
// Method (per token and layer): the router scores the experts and keeps the K
// best ("El milagro de la IA de 2GB en Apple Silicon", section "Por que la
// mayor parte de tu modelo de IA es peso muerto"); their ids are checked
// against the layer's LFU slot cache, a miss replacing the least frequently
// used resident expert (same page, "Mas inteligente que tu RAM"); the shared
// expert runs while the missed experts are fetched, and shared and routed
// outputs are combined ("TurboFieldfare: motor open source ...", section
// "Proceso de generacion de tokens").  Arithmetic as in router.cu, plan.cu and
// ffn.cu: fixed-order fp32 router logits, rank-count top-K, softmax over the K,
// the LFU rule with its readings, and dequantising GEMVs on a 16-bit
// fixed-point image of the inputs with fp32 accumulation.
//
// B200 mapping.  One CTA per SM (a cooperative launch, so all are resident),
// a producer warp streaming weight chunks into two shared-memory rings (gate/up
// chunks of 4.6 KB, down chunks of up to 12.7 KB) and twelve consumer warps.
//   prologue   before the dependency wait (weights only): each CTA starts the
//              bulk copies of its router rows and of its share of the shared
//              expert's gate/up chunks.
//   phase 1    the cache state and the token's input (16-bit image + fp32
//              copy) into shared memory; each CTA scores its
//              experts (logits to global), arrives at barrier A, then computes
//              its shared-expert chunks while the other CTAs finish.
//   phase 2    after A every CTA reads all logits and computes the same top-K,
//              gate weights and cache plan from its copy of the state (CTA 0
//              alone writes state, ids, gate weights, plan mailbox and
//              counters); the producer then streams the CTA's down chunks (as
//              far as the ring holds them) and its routed gate/up chunks.  A
//              missed expert is read from pinned host memory over the bus with
//              16-byte asynchronous copies and written into its slot by the
//              consumers as they use it (no host round trip, no copy engine).
//   phase 3    after barrier B (every h row complete) the consumers stage the
//              h segments of their down chunks and finish the combine; a
//              32-row output tile split between CTAs is summed by the last CTA
//              to finish it, in CTA order (deterministic).
// Every wait is bounded: mbarriers by iteration count, grid barriers by the
// global timer (1 s); a wait that gives up records MOE_ERR_TIMEOUT, the CTA
// skips its remaining work and returns only after its copies have landed.
#include "common.cuh"
#include "launch.cuh"
#include "layer.cuh"

namespace moe {

namespace {

constexpr int kLNW = 12;                      // consumer warps
constexpr int kLNC = kLNW * 32;               // consumer threads
constexpr int kLThreads = kLNC + 64;          // + producer warps (gate/up ring, down ring)
// Gate/up stages hold up to kLChunksPerStage consecutive chunks of one tile (a
// tile's chunks are contiguous in the blob): one bulk request per stage.  Each
// bulk request costs a CTA a roughly fixed time whatever its size (measured:
// 4.6 KB requests stream at ~12 GB/s per CTA, 18-37 KB requests at 45+), so
// few large requests keep the CTA's share of HBM bandwidth.
constexpr int kLChunk = 18 * kGuSlice;        // 4608 B: 32 rows x 256 inputs
#ifndef MOE_LAYER_GU_CPS
#define MOE_LAYER_GU_CPS 4
#endif
#ifndef MOE_LAYER_GU_STAGES
#define MOE_LAYER_GU_STAGES 5
#endif
constexpr int kLChunksPerStage = MOE_LAYER_GU_CPS;  // compile-time tuning values
constexpr int kLGuStages = MOE_LAYER_GU_STAGES;
constexpr int kLDnStages = 7;  // all of a CTA's down units for the 26B-A4B shapes (7 per CTA)
constexpr int kLGuStage = kLChunksPerStage * kLChunk;  // 18432 B at four chunks
constexpr int kLDnStage = 18 * kDownSliceMax; // 12672 B
constexpr int kLMaxK = 16;
constexpr unsigned long long kGridWaitNs = 1000000000ull;  // 1 s

// Shared-memory carve-up, identical on host (size) and device (pointers).
struct Carve {
    size_t gu, dn, bars, xq, xsx, xX, xs, hq, hsx, hX, rrow, gsum, gsc, logit, cnt, last, slot_of, ein, inwave, total;
};

__host__ __device__ inline size_t up16(size_t b) { return (b + 15) & ~size_t(15); }

__host__ __device__ inline Carve layer_carve(int D, int E, int S, int hvals, int rows) {
    Carve c;
    size_t o = 0;
    auto take = [&](size_t b) { const size_t at = o; o += up16(b); return at; };
    const int ng = D / kGroup;
    c.gu = take(size_t(kLGuStages) * kLGuStage);
    c.dn = take(size_t(kLDnStages) * kLDnStage);
    c.bars = take(sizeof(uint64_t) * (2 * kLGuStages + 2 * kLDnStages + 2));
    c.xq = take(size_t(D) * 2);                        // 16-bit image of x
    c.xsx = take(sizeof(float) * ng);
    c.xX = take(sizeof(float) * ng);
    c.xs = take(sizeof(float) * size_t(ng) * (kGroup + 1));  // fp32 x for the router, padded rows
    c.hq = take(size_t(hvals) * 2);                    // 16-bit image of the staged h segments
    c.hsx = take(sizeof(float) * (hvals / kGroup + 1));
    c.hX = take(sizeof(float) * (hvals / kGroup + 1));
    c.rrow = take(size_t(rows) * D);                   // router rows of this CTA's experts
    c.gsum = take(sizeof(float) * ng);
    c.gsc = take(sizeof(float) * ng);
    c.logit = take(sizeof(float) * E);
    c.cnt = take(sizeof(uint32_t) * E);
    c.last = take(sizeof(uint32_t) * E);
    c.slot_of = take(sizeof(int32_t) * E);
    c.ein = take(sizeof(int32_t) * S);
    c.inwave = take(size_t(E));
    c.total = o;
    return c;
}

__device__ __forceinline__ int range_start(int c, int U, int G) { return int((long long)c * U / G); }
__device__ __forceinline__ int cta_of(int u, int U, int G) { return int(((long long)(u + 1) * G + U - 1) / U) - 1; }

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid barrier over all CTAs (cooperative launch: all resident).  Word 0 counts
// arrivals, word kGenWord is the generation (another 128-byte line, so the
// waiters' polling does not contend with the arrivals' atomics); the last
// arrival resets the count and advances the generation.  Called by one thread
// per CTA after the CTA's writes; arrive returns the generation to wait on.
constexpr int kGenWord = 32;
__device__ __forceinline__ unsigned grid_arrive(unsigned* bar, unsigned G) {
    const unsigned gen = ld_acquire_u32(bar + kGenWord);  // read before arriving
    __threadfence();
    if (atomicAdd(bar, 1u) == G - 1) {
        atomicExch(bar, 0u);
        __threadfence();
        st_release_u32(bar + kGenWord, gen + 1);
    }
    return gen;
}
__device__ __forceinline__ bool grid_wait(const unsigned* bar, unsigned gen, int* status) {
    const unsigned long long t0 = global_ns();
    for (unsigned it = 0;; ++it) {
        if (ld_acquire_u32(bar + kGenWord) != gen) return true;
        if ((it & 63) == 63 && global_ns() - t0 > kGridWaitNs) {
            set_status(status, MOE_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(32);
    }
}

// 16-byte asynchronous copy global (device or mapped host memory) -> shared.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
// The mbarrier tracks this thread's earlier cp.async copies (pending count +1,
// one arrival when they land).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// waits until every cp.async this thread issued has landed
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ bool lwait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, status)) return true;
    *abort_flag = 1;
    return false;
}

// One 8-input task of the 16-bit fixed-point image (all 32 lanes call; `ok`
// marks lanes with a real task).  Per group of 64: s = max|v| / 32767,
// v ~= s * (256*hi + lo), hi a signed and lo an unsigned byte; the 16 bytes of
// inputs k0..k0+7 hold (hi even, lo even, hi odd, lo odd) as byte vectors.
__device__ __forceinline__ void image_task(const float (&v)[8], bool ok, int task, uint4* q, float* sx, float* X) {
    float amax = 0.f, sum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        amax = fmaxf(amax, fabsf(v[j]));
        sum += v[j];
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        sum += __shfl_xor_sync(0xffffffffu, sum, off);
    }
    if (!ok) return;
    const float inv = amax > 0.f ? 32767.f / amax : 0.f;
    uint32_t hi_e = 0, lo_e = 0, hi_o = 0, lo_o = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        int qv = __float2int_rn(v[j] * inv);
        qv = max(-32767, min(32767, qv));
        const uint32_t hb = uint32_t(qv >> 8) & 0xFFu, lb = uint32_t(qv) & 0xFFu;
        const int sh = 8 * (j >> 1);
        if ((j & 1) == 0) { hi_e |= hb << sh; lo_e |= lb << sh; }
        else { hi_o |= hb << sh; lo_o |= lb << sh; }
    }
    q[task] = make_uint4(hi_e, lo_e, hi_o, lo_o);
    if ((task & 7) == 0) {
        sx[task >> 3] = amax / 32767.f;
        X[task >> 3] = sum;
    }
}

// One quantisation group of a chunk (lane = row): s*(sum q*x) + b*(sum x),
// from the staged image of the group's 64 inputs.
__device__ __forceinline__ float group_dot(const uint8_t* chunk, int ks, int g, int lane, const uint4* xq,
                                           float sx, float X, uint4* qa_out, uint4* qb_out, uint32_t* sb_out) {
    const uint4 qa = *reinterpret_cast<const uint4*>(chunk + ((2 * g) * 32 + lane) * 16);
    const uint4 qb = *reinterpret_cast<const uint4*>(chunk + ((2 * g + 1) * 32 + lane) * 16);
    const uint32_t sbw = *reinterpret_cast<const uint32_t*>(chunk + 16 * ks + (g * 32 + lane) * 4);
    *qa_out = qa;
    *qb_out = qb;
    *sb_out = sbw;
    const float s = f16_to_f32(uint16_t(sbw & 0xFFFF)), b = f16_to_f32(uint16_t(sbw >> 16));
    const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
    int shi = 0, shi2 = 0;
    uint32_t slo = 0, slo2 = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t lo = words[j] & 0x0F0F0F0Fu;
        const uint32_t hi = (words[j] >> 4) & 0x0F0F0F0Fu;
        const uint4 xv = xq[j];
        shi = dp4a_us(lo, xv.x, shi);
        slo = dp4a_uu(lo, xv.y, slo);
        shi2 = dp4a_us(hi, xv.z, shi2);
        slo2 = dp4a_uu(hi, xv.w, slo2);
    }
    const int dot = 256 * (shi + shi2) + int(slo + slo2);
    return fmaf(s, float(dot) * sx, b * X);
}

// The group's bytes back to the same place in the blob (a missed expert read
// from host memory is written into its slot as it is used).
__device__ __forceinline__ void group_writeback(uint8_t* wb_chunk, int ks, int g, int lane, uint4 qa, uint4 qb,
                                                uint32_t sbw) {
    *reinterpret_cast<uint4*>(wb_chunk + ((2 * g) * 32 + lane) * 16) = qa;
    *reinterpret_cast<uint4*>(wb_chunk + ((2 * g + 1) * 32 + lane) * 16) = qb;
    *reinterpret_cast<uint32_t*>(wb_chunk + 16 * ks + (g * 32 + lane) * 4) = sbw;
}

struct LEntry {
    const uint8_t* src;  // blob the producer reads (device memory, or the pinned host store)
    uint8_t* wb;         // slot the blob is written into (a miss read from the host), or null
    int F;
    int host;            // src is host memory: 16-byte asynchronous copies
    float w;             // gate weight (1 for the shared expert)
    int h_off;           // float offset of this entry's activation row in h
};

}  // namespace

__global__ void __launch_bounds__(kLThreads, 1) layer_decode_kernel(LayerArgs A) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int D = A.D, E = A.E, K = A.K, S = A.S, F = A.F, FS = A.FS;
    const int G = gridDim.x, c = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ng = D / kGroup, NSg = D / kGuSlice;
    const bool streaming = A.experts == nullptr;
    const int nsh = A.shared_blob ? 1 : 0;
    const int rows = (E + G - 1) / G;  // router rows per CTA (upper bound)
    const Carve cv = layer_carve(D, E, S, A.hvals, rows);
    uint8_t* gu_ring = smem + cv.gu;
    uint8_t* dn_ring = smem + cv.dn;
    uint64_t* full_gu = reinterpret_cast<uint64_t*>(smem + cv.bars);
    uint64_t* empty_gu = full_gu + kLGuStages;
    uint64_t* full_dn = empty_gu + kLGuStages;
    uint64_t* empty_dn = full_dn + kLDnStages;
    uint64_t* rt_bar = empty_dn + kLDnStages;
    uint64_t* plan_bar = rt_bar + 1;
    uint4* xq = reinterpret_cast<uint4*>(smem + cv.xq);
    float* xsx = reinterpret_cast<float*>(smem + cv.xsx);
    float* xX = reinterpret_cast<float*>(smem + cv.xX);
    float* xs = reinterpret_cast<float*>(smem + cv.xs);
    uint4* hq = reinterpret_cast<uint4*>(smem + cv.hq);
    float* hsx = reinterpret_cast<float*>(smem + cv.hsx);
    float* hX = reinterpret_cast<float*>(smem + cv.hX);
    int8_t* rrow = reinterpret_cast<int8_t*>(smem + cv.rrow);
    float* gsum = reinterpret_cast<float*>(smem + cv.gsum);
    float* gsc = reinterpret_cast<float*>(smem + cv.gsc);
    float* lg = reinterpret_cast<float*>(smem + cv.logit);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + cv.cnt);
    uint32_t* last = reinterpret_cast<uint32_t*>(smem + cv.last);
    int32_t* slot_of = reinterpret_cast<int32_t*>(smem + cv.slot_of);
    int32_t* ein = reinterpret_cast<int32_t*>(smem + cv.ein);
    uint8_t* inwave = smem + cv.inwave;

    __shared__ LEntry s_ent[kLMaxK + 1];
    __shared__ float red2[2][kLNW * 32];
    __shared__ int s_sel_id[kLMaxK], s_ulist[kLMaxK], s_uslot[kLMaxK], s_uhit[kLMaxK], s_uvic[kLMaxK];
    __shared__ float s_sel_l[kLMaxK];
    __shared__ int s_nan, s_abort;
    __shared__ float s_upart[kLDnStages * 4][32];  // per unit of the down range: w_e * dot, lane = row
    __shared__ int s_nmiss, s_stop;

    // work ranges: gate/up units (shared tiles, then routed k = 0..K-1), down
    // units (tile-major: per 32-row tile the shared slices, then routed k)
    const int ush = nsh ? (FS / 16) * NSg : 0, urt = (F / 16) * NSg;
    const int ks_sh = nsh ? down_ks(FS) : 1, ks_rt = down_ks(F);
    const int ns_sh = nsh ? FS / ks_sh : 0, ns_rt = F / ks_rt;
    const int upt = ns_sh + K * ns_rt, tiles_dn = D / kChunkRows;
    const int Udn = tiles_dn * upt;
    // gate/up: the shared expert's units and the routed units are two pools,
    // each split evenly over all CTAs, so every CTA streams shared weights
    // during the router phase and routed weights after the plan
    // (whole 16-output tiles per CTA: no tile is split between CTAs, so the
    // gate/up results need no cross-CTA reduction)
    const int TS = nsh ? FS / 16 : 0, TR = K * (F / 16);
    const int sh0 = range_start(c, TS, G) * NSg, sh1 = range_start(c + 1, TS, G) * NSg;
    const int r0 = ush + range_start(c, TR, G) * NSg, r1 = ush + range_start(c + 1, TR, G) * NSg;
    const int d0 = range_start(c, Udn, G), d1 = range_start(c + 1, Udn, G);
    const int n_rows = c < E ? (E - 1 - c) / G + 1 : 0;  // experts c, c+G, ...
    auto gu_entry = [&](int u) { return u < ush ? 0 : nsh + (u - ush) / urt; };
    auto gu_base = [&](int e) { return e < nsh ? 0 : ush + (e - nsh) * urt; };
    auto dn_unit = [&](int u, int& e, int& tile, int& slice) {
        tile = u / upt;
        const int o = u - tile * upt;
        if (o < ns_sh) { e = 0; slice = o; }
        else { e = nsh + (o - ns_sh) / ns_rt; slice = (o - ns_sh) % ns_rt; }
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < kLGuStages; ++i) {
            mbar_init(&full_gu[i], 1);
            mbar_init(&empty_gu[i], kLNW);  // every consumer warp, once per stage
        }
        for (int i = 0; i < kLDnStages; ++i) {
            mbar_init(&full_dn[i], 1);
            mbar_init(&empty_dn[i], 1);  // the one warp that computes the unit
        }
        mbar_init(rt_bar, 1);
        mbar_init(plan_bar, 1);
        mbar_fence_init();
        s_abort = 0;
        s_nan = 0;
        s_nmiss = 0;
    }
    if (threadIdx.x < 32 && nsh) {
        // entry 0 (the shared expert) is known before the plan
        if (threadIdx.x == 0) {
            LEntry en;
            en.src = A.shared_blob;
            en.wb = nullptr;
            en.F = FS;
            en.host = 0;
            en.w = 1.0f;
            en.h_off = 0;
            s_ent[0] = en;
        }
    }
    __syncthreads();

    // ================================================================ producer
    if (warp >= kLNW) {
        const bool gu_warp = warp == kLNW;  // the other producer warp streams the down ring
        const uint64_t pol = l2_evict_first();
        int issued_gu = 0, issued_dn = 0;
        bool ok = true;
        // one chunk into a ring stage: bulk copy (device memory) or 16-byte
        // asynchronous copies by every lane (host memory)
        auto issue = [&](uint8_t* ring, int stage_bytes, uint64_t* full, uint64_t* empty, int nst, int& issued,
                         const uint8_t* src, uint32_t bytes, bool host) {
            const int st = issued % nst;
            if (issued >= nst) {
                bool w = true;
                if (lane == 0) w = lwait(&empty[st], uint32_t((issued / nst) - 1) & 1u, A.status, &s_abort);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) return false;
            }
            uint8_t* dst = ring + size_t(st) * stage_bytes;
            if (host) {
                for (uint32_t o = uint32_t(lane) * 16u; o < bytes; o += 32u * 16u) cp_async16(dst + o, src + o);
                cp_async_commit();
                cp_async_arrive(&full[st]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[st]);
            } else if (lane == 0) {
                mbar_arrive_expect_tx(&full[st], bytes);
                bulk_g2s(dst, src, bytes, &full[st], pol);
            }
            __syncwarp();
            ++issued;
            return true;
        };
        // a chunk source must lie inside the blob its entry names: the host
        // store (host entries) or a slot, a resident expert or the shared blob
        const size_t blob_rt = blob_bytes(D, F), blob_sh = nsh ? blob_bytes(D, FS) : 0;
        auto src_ok = [&](const LEntry& en, const uint8_t* p, uint32_t bytes) {
            if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0 || (bytes & 15u) != 0) return false;
            auto inside = [&](const uint8_t* base, size_t n) { return base && p >= base && p + bytes <= base + n; };
            if (en.host) return inside(A.store, size_t(E) * A.store_stride);
            return inside(A.shared_blob, blob_sh) ||
                   (streaming ? inside(A.slots, size_t(S) * A.slot_stride)
                              : inside(A.experts, size_t(E) * A.expert_stride));
        };
        auto issue_checked = [&](uint8_t* ring, int stage_bytes, uint64_t* full, uint64_t* empty, int nst,
                                 int& issued, const LEntry& en, const uint8_t* src, uint32_t bytes) {
            if (!src_ok(en, src, bytes) || (en.wb && en.host == 0)) {
                // never copy from outside: report, stop, and complete nothing more
                if (lane == 0) {
                    set_status(A.status, MOE_ERR_RANGE);
                    s_abort = 1;
                }
                __syncwarp();
                return false;
            }
            return issue(ring, stage_bytes, full, empty, nst, issued, src, bytes, en.host != 0);
        };
        // the stage of units [u, u + n) (consecutive chunks of one tile)
        auto issue_gu = [&](int u, int n) {
            const int e = gu_entry(u);
            const LEntry& en = s_ent[e];
            return issue_checked(gu_ring, kLGuStage, full_gu, empty_gu, kLGuStages, issued_gu, en,
                                 en.src + size_t(u - gu_base(e)) * kLChunk, uint32_t(n) * kLChunk);
        };
        // a pool range [a, b) of whole tiles, stage by stage
        auto issue_gu_range = [&](int a, int b) {
            bool good = true;
            for (int t0 = a; good && t0 < b; t0 += NSg)
                for (int j = 0; good && j < NSg; j += kLChunksPerStage)
                    good = issue_gu(t0 + j, min(kLChunksPerStage, NSg - j));
            return good;
        };
        auto issue_dn = [&](int u) {
            int e, tile, slice;
            dn_unit(u, e, tile, slice);
            const LEntry& en = s_ent[e];
            const int ks = down_ks(en.F);
            return issue_checked(dn_ring, kLDnStage, full_dn, empty_dn, kLDnStages, issued_dn, en,
                                 en.src + gu_section_bytes(D, en.F) + size_t(tile * (en.F / ks) + slice) * (18u * ks),
                                 uint32_t(18u * ks));
        };
        // gate/up warp: router rows of this CTA's experts and its shared-expert
        // tiles (immutable weights, fetched before the dependency wait)
        if (gu_warp) {
            if (lane == 0 && n_rows > 0) {
                mbar_arrive_expect_tx(rt_bar, uint32_t(n_rows) * uint32_t(D));
                const uint64_t keep = l2_evict_last();
                for (int r = 0; r < n_rows; ++r)
                    bulk_g2s(rrow + size_t(r) * D, A.wq + size_t(c + r * G) * D, uint32_t(D), rt_bar, keep);
            }
            ok = ok && issue_gu_range(sh0, sh1);
        }
        // the plan (entries) is ready
        if (ok) {
            bool w = true;
            if (lane == 0) w = mbar_wait(plan_bar, 0, A.status);
            w = __shfl_sync(0xffffffffu, w, 0);
            ok = w && !s_abort;
        }
        // the routed gate/up tiles (the ring is free again: the consumers
        // released the shared tiles before the plan), or the down units (weights
        // only: they land while the gate/up phase runs), each on its own warp
        // so that neither queue waits behind the other's issues
        if (gu_warp) ok = ok && issue_gu_range(r0, r1);
        else
            for (int v = d0; ok && v < d1; ++v) ok = issue_dn(v);
        // every issued copy has landed before the CTA may exit: each lane's own
        // asynchronous copies, then (lane 0) the last uses of every stage
        cp_async_wait_all();
        __syncwarp();
        if (lane == 0) {
            for (int i = issued_gu > kLGuStages ? issued_gu - kLGuStages : 0; i < issued_gu; ++i)
                mbar_wait(&full_gu[i % kLGuStages], uint32_t(i / kLGuStages) & 1u, A.status);
            for (int i = issued_dn > kLDnStages ? issued_dn - kLDnStages : 0; i < issued_dn; ++i)
                mbar_wait(&full_dn[i % kLDnStages], uint32_t(i / kLDnStages) & 1u, A.status);
        }
        return;
    }

    // =============================================================== consumers
    pdl_wait();  // the token's input comes from the preceding launch
    // the cache state (the preceding launch may be this cache's reset): read
    // now, used by the plan after barrier A
    if (streaming) {
        const uint32_t* g_cnt = reinterpret_cast<const uint32_t*>(A.state);
        for (int e = threadIdx.x; e < E; e += kLNC) {
            cnt[e] = g_cnt[e];
            last[e] = g_cnt[E + e];
            slot_of[e] = A.state[2 * E + e];
            inwave[e] = 0;
        }
        for (int s = threadIdx.x; s < S; s += kLNC) ein[s] = A.state[3 * E + s];
    }
    // phase 1a: the input as a 16-bit image (GEMV) and in fp32 (router)
    for (int base = 0; base < D / 8; base += kLNC) {
        const int t = base + int(threadIdx.x);
        const bool okt = t < D / 8;
        float v[8];
        if (okt) {
            const uint4 q = reinterpret_cast<const uint4*>(A.x)[t];
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[2 * j] = __uint_as_float(w4[j] << 16);
                v[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
            }
            float* dst = xs + (t / 8) * (kGroup + 1) + (t % 8) * 8;
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = v[j];
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = 0.f;
        }
        image_task(v, okt, t, xq, xsx, xX);
    }
    named_sync(1, kLNC);

    // phase 1b: this CTA's router logits, same fp32 FMA order as router.cu:
    // S_g = chain over the group's 64 inputs ascending, logit = chain over
    // groups of s_g * S_g, plus the bias
    if (n_rows > 0) {
        // s_stop: one value for all consumers (s_abort may change under them)
        if (threadIdx.x == 0) s_stop = lwait(rt_bar, 0, A.status, &s_abort) ? 0 : 1;
        named_sync(1, kLNC);
        for (int r = 0; r < n_rows && !s_stop; ++r) {
            const int e = c + r * G;
            for (int g = threadIdx.x; g < ng; g += kLNC) {
                const int8_t* q = rrow + size_t(r) * D + g * kGroup;
                const float* xg = xs + g * (kGroup + 1);
                gsc[g] = f16_to_f32(A.ws[size_t(e) * ng + g]);
                float Sg = 0.0f;
                for (int k = 0; k < kGroup; ++k) Sg = __fmaf_rn(float(q[k]), xg[k], Sg);
                gsum[g] = Sg;
            }
            named_sync(1, kLNC);
            if (threadIdx.x == 0) {
                float acc = 0.0f;
                for (int g = 0; g < ng; ++g) acc = __fmaf_rn(gsc[g], gsum[g], acc);
                if (A.bias) acc = __fadd_rn(acc, A.bias[e]);
                A.logits[e] = acc;
            }
            named_sync(1, kLNC);
        }
    }
    // arrive at A (logits written), then the shared-expert chunks while the
    // other CTAs finish their logits
    unsigned gen_a = 0;
    if (threadIdx.x == 0) gen_a = grid_arrive(A.bar, unsigned(G));

    // ---------------------------------------------- gate/up consumer loop
    // Whole tiles (NSg chunks, 16 gate + 16 up rows) stage by stage: a stage
    // holds up to kLChunksPerStage chunks (4 groups of 64 inputs each) and
    // warp w takes the stage's groups w, w + 12, ...: one wait and one release
    // per stage and warp.  At a tile's end the warps' partial sums (lane = row)
    // are added in warp order by one warp (double-buffered by tile parity, so
    // one barrier per tile suffices) and h = gelu(gate) * up is written.
    int tiles_done = 0;
    int q_gu = 0;  // ring position of the next gate/up stage
    auto gu_tiles = [&](int ua, int ub) {
        for (int t0 = ua; t0 < ub; t0 += NSg) {
            const int e = gu_entry(t0);
            const int ul0 = t0 - gu_base(e);  // the tile's first chunk inside its blob
            const int tile = ul0 / NSg;
            const LEntry& en = s_ent[e];
            float a = 0.f;
            for (int c0 = 0; c0 < NSg; c0 += kLChunksPerStage, ++q_gu) {
                const int nc = min(kLChunksPerStage, NSg - c0);
                const int st = q_gu % kLGuStages;
                const bool have = lwait(&full_gu[st], uint32_t(q_gu / kLGuStages) & 1u, A.status, &s_abort);
                if (have) {
                    const uint8_t* stage = gu_ring + size_t(st) * kLGuStage;
                    for (int g = warp; g < 4 * nc; g += kLNW) {
                        const int ch = g >> 2, gw = g & 3;
                        const int gi = 4 * c0 + g;  // input group: chunk c0 + ch, group gw
                        uint4 qa, qb;
                        uint32_t sbw;
                        a += group_dot(stage + size_t(ch) * kLChunk, kGuSlice, gw, lane, xq + gi * 8, xsx[gi], xX[gi],
                                       &qa, &qb, &sbw);
                        if (en.wb) group_writeback(en.wb + size_t(ul0 + c0 + ch) * kLChunk, kGuSlice, gw, lane, qa, qb, sbw);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_gu[st]);
            }
            const int tb = tiles_done & 1;
            red2[tb][warp * 32 + lane] = a;
            named_sync(1, kLNC);
            if (warp == tiles_done % kLNW) {
                float tot = 0.f;
                for (int w = 0; w < kLNW; ++w) tot += red2[tb][w * 32 + lane];
                // lanes 0..15 gate rows, 16..31 up rows of outputs 16*tile + lane
                const float upv = __shfl_down_sync(0xffffffffu, tot, 16);
                if (lane < 16) A.h[en.h_off + 16 * tile + lane] = gelu_tanh(tot) * upv;
            }
            ++tiles_done;
        }
    };
    gu_tiles(sh0, sh1);  // shared-expert tiles (known before the plan)

    // ------------------------------------------------- phase 2: top-K + plan
    bool ok_a = true;
    if (threadIdx.x == 0) ok_a = grid_wait(A.bar, gen_a, A.status);
    if (threadIdx.x == 0 && !ok_a) s_abort = 1;
    named_sync(1, kLNC);
    for (int e = threadIdx.x; e < E; e += kLNC) lg[e] = __ldcg(A.logits + e);
    named_sync(1, kLNC);
    // rank counting: the experts ranked above e (logit descending, id ascending)
    for (int e = threadIdx.x; e < E; e += kLNC) {
        const float v = lg[e];
        int above = 0;
        for (int f = 0; f < E; ++f) {
            const float o = lg[f];
            above += (o > v) || (o == v && f < e);
        }
        if (isnan(v)) s_nan = 1;
        else if (above < K) {
            s_sel_id[above] = e;
            s_sel_l[above] = v;
        }
    }
    named_sync(1, kLNC);
    if (warp == 0) {
        const bool nanl = s_nan != 0;
        int sel = 0;
        float w = 0.f;
        if (nanl) {
            // no order exists: valid indices, uniform weights, reported
            sel = lane < K ? lane : 0;
            w = 1.0f / K;
            if (c == 0 && lane == 0) set_status(A.status, MOE_ERR_NAN);
        } else {
            const float sl_l = lane < K ? s_sel_l[lane] : 0.f;
            sel = lane < K ? s_sel_id[lane] : 0;
            const float m = __shfl_sync(0xffffffffu, sl_l, 0);
            const float ex = lane < K ? expf(sl_l - m) : 0.0f;
            float z = 0.0f;
            for (int i = 0; i < K; ++i) z += __shfl_sync(0xffffffffu, ex, i);
            w = ex / z;
        }
        if (c == 0 && lane < K) {
            if (A.ids) A.ids[lane] = sel;
            if (A.gate_w) A.gate_w[lane] = w;
        }
        // distinct selected experts in ascending id (NaN fallback ids are distinct too)
        int rank = 0;
        for (int i = 0; i < K; ++i) rank += (__shfl_sync(0xffffffffu, sel, i) < sel);
        if (lane < K) s_ulist[rank] = sel;
        __syncwarp();
        int slot_k = sel, hit_k = 1;
        if (streaming) {
            // the cache plan (one wave: K <= S), the rule of plan.cu
            const bool halve = A.policy == MOE_POLICY_LFU_DECAY && A.decay_period > 0u && A.step > 0u &&
                               A.step % A.decay_period == 0u;
            if (halve)
                for (int e = lane; e < E; e += 32) cnt[e] >>= 1;
            __syncwarp();
            if (lane < K) {
                cnt[sel] += 1u;
                inwave[sel] = 1;
            }
            __syncwarp();
            int n_miss = 0, rep1 = 0, rep2 = 0;
            for (int i = 0; i < K; ++i) {
                const int e = s_ulist[i];
                const uint32_t lu = last[e];
                rep1 += (lu != 0u && lu == A.step);
                rep2 += (lu != 0u && lu + 1u >= A.step);
                int victim = -1, slot = slot_of[e];
                if (slot >= S) {
                    if (lane == 0 && c == 0) set_status(A.status, MOE_ERR_STATE);
                    slot = -1;
                }
                const bool hit = slot >= 0;
                if (!hit) {
                    slot = -1;
                    for (int b = 0; b < S && slot < 0; b += 32) {
                        const int s = b + lane;
                        const uint32_t bal = __ballot_sync(0xffffffffu, s < S && ein[s] < 0);
                        if (bal) slot = b + __ffs(bal) - 1;
                    }
                    if (slot < 0) {
                        uint32_t bc = 0xffffffffu, bl = 0xffffffffu;
                        int br = 0x7fffffff;
                        for (int s = lane; s < S; s += 32) {
                            const int r = ein[s];
                            if (r < 0 || r >= E || inwave[r]) continue;
                            const uint32_t cr = A.policy == MOE_POLICY_LRU ? 0u : cnt[r];
                            if (cr < bc || (cr == bc && (last[r] < bl || (last[r] == bl && r < br)))) {
                                bc = cr; bl = last[r]; br = r;
                            }
                        }
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) {
                            const uint32_t oc = __shfl_xor_sync(0xffffffffu, bc, off);
                            const uint32_t ol = __shfl_xor_sync(0xffffffffu, bl, off);
                            const int orr = __shfl_xor_sync(0xffffffffu, br, off);
                            if (oc < bc || (oc == bc && (ol < bl || (ol == bl && orr < br)))) {
                                bc = oc; bl = ol; br = orr;
                            }
                        }
                        if (br < E) {
                            victim = br;
                            slot = slot_of[victim];
                        }
                        if (slot < 0 || slot >= S) {
                            if (lane == 0 && c == 0) set_status(A.status, MOE_ERR_STATE);
                            victim = -1;
                            slot = 0;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) {
                        if (victim >= 0) {
                            slot_of[victim] = -1;
                            if (A.policy == MOE_POLICY_LFU_IN_CACHE) cnt[victim] = 0u;
                        }
                        const int prev = ein[slot];
                        if (prev >= 0 && prev < E && prev != victim) slot_of[prev] = -1;
                        slot_of[e] = slot;
                        ein[slot] = e;
                    }
                    ++n_miss;
                }
                if (lane == 0) {
                    s_uslot[i] = slot;
                    s_uhit[i] = hit ? 1 : 0;
                    s_uvic[i] = victim;
                }
                __syncwarp();
            }
            if (lane < K) last[s_ulist[lane]] = A.step + 1u;
            __syncwarp();
            // selection k's slot and residency
            int pos = 0;
            for (int i = 0; i < K; ++i) pos = (s_ulist[i] == sel) ? i : pos;
            slot_k = s_uslot[pos];
            hit_k = s_uhit[pos];
            if (lane == 0) s_nmiss = n_miss;
            if (c == 0 && lane == 0 && A.stats) {
                A.stats[0] += 1;                                 // layer calls
                A.stats[1] += uint64_t(K - n_miss);              // hits
                A.stats[2] += uint64_t(n_miss);                  // misses
                A.stats[3] += uint64_t(n_miss) * A.blob_bytes;   // bytes read from the host store
                A.stats[4] += uint64_t(rep1);                    // selected at the previous token
                A.stats[5] += uint64_t(rep2);                    // ... or the one before
                A.stats[6] += uint64_t(K);                       // selections
            }
        }
        // the routed entries, in k order
        if (lane < K) {
            LEntry en;
            en.F = F;
            en.w = w;
            en.h_off = FS * nsh + lane * F;
            if (streaming) {
                uint8_t* slotp = A.slots + size_t(slot_k) * A.slot_stride;
                en.src = hit_k ? slotp : A.store + size_t(sel) * A.store_stride;
                en.wb = hit_k ? nullptr : slotp;
                en.host = hit_k ? 0 : 1;
            } else {
                en.src = A.experts + size_t(sel) * A.expert_stride;
                en.wb = nullptr;
                en.host = 0;
            }
            s_ent[nsh + lane] = en;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(plan_bar);  // the producer may stream the routed chunks
    }
    // CTA 0: the cache's new state and the plan for the host
    if (c == 0 && streaming) {
        named_sync(1, kLNC);
        uint32_t* g_cnt = reinterpret_cast<uint32_t*>(A.state);
        for (int e = threadIdx.x; e < E; e += kLNC) {
            g_cnt[e] = cnt[e];
            g_cnt[E + e] = last[e];
            A.state[2 * E + e] = slot_of[e];
        }
        for (int s = threadIdx.x; s < S; s += kLNC) A.state[3 * E + s] = ein[s];
        if (A.mailbox) {
            if (threadIdx.x < K) {
                A.mailbox->expert[threadIdx.x] = s_ulist[threadIdx.x];
                A.mailbox->slot[threadIdx.x] = s_uslot[threadIdx.x];
                A.mailbox->hit[threadIdx.x] = s_uhit[threadIdx.x];
                A.mailbox->victim[threadIdx.x] = s_uvic[threadIdx.x];
                A.mailbox->wave[threadIdx.x] = 0;
            }
            named_sync(1, kLNC);
            if (threadIdx.x == 0) {
                A.mailbox->n_distinct = K;
                A.mailbox->n_waves = 1;
                A.mailbox->n_misses = s_nmiss;
                __threadfence_system();
                *reinterpret_cast<volatile uint32_t*>(&A.mailbox->seq) = A.seq;
            }
        }
    }
    named_sync(1, kLNC);

    // ------------------------------------------- the routed gate/up chunks
    gu_tiles(r0, r1);

    // ------------------------------------------------ phase 3: down + combine
    named_sync(1, kLNC);
    if (threadIdx.x == 0) {
        const unsigned gen_b = grid_arrive(A.bar + 2 * kGenWord, unsigned(G));
        if (!grid_wait(A.bar + 2 * kGenWord, gen_b, A.status)) s_abort = 1;
    }
    // one snapshot of the abort flag for all consumers (the producer warp may
    // still set s_abort; every consumer must take the same branch here)
    if (threadIdx.x == 0) s_stop = s_abort;
    named_sync(1, kLNC);
    // the next launch may start its prologue (weights and the next cache's
    // state) while this CTA finishes
    pdl_trigger();
    if (s_stop) return;
    // Down + combine.  This CTA's units d0..d1 (tile-major: per 32-row output
    // tile the shared expert's slices, then routed k) go to the warps whole:
    // warp w takes units w, w + 12, ...  A warp stages its unit's h segment as
    // a 16-bit image (one slot of kDownSliceMax values per unit), waits for
    // the unit's weights (ring stage i % kLDnStages, consumed by this warp
    // alone), and keeps w_e * (the unit's dot product) per row.  The units of
    // one tile are then added in unit order; a tile split between CTAs goes
    // through the cross-CTA partial slots (first and last tile of the range).
    const int nu = d1 - d0;
    for (int i = warp; i < nu; i += kLNW) {
        int e, tile, slice;
        dn_unit(d0 + i, e, tile, slice);
        const LEntry& en = s_ent[e];
        const int ks = down_ks(en.F);
        const int tb = i * (kDownSliceMax / 8);  // first image task (8 values) of this unit's slot
        const float* hp = A.h + en.h_off + slice * ks;
        // all of the segment's loads first (up to 3 rounds of 32 tasks: one
        // L2 round trip), then the image
        constexpr int kRounds = (kDownSliceMax / 8 + 31) / 32;
        float4 hv[kRounds][2];
#pragma unroll
        for (int r = 0; r < kRounds; ++r) {
            const int t = 32 * r + lane;
            if (t < ks / 8) {
                hv[r][0] = __ldcg(reinterpret_cast<const float4*>(hp + 8 * t));
                hv[r][1] = __ldcg(reinterpret_cast<const float4*>(hp + 8 * t) + 1);
            } else {
                hv[r][0] = make_float4(0.f, 0.f, 0.f, 0.f);
                hv[r][1] = hv[r][0];
            }
        }
#pragma unroll
        for (int r = 0; r < kRounds; ++r) {
            if (32 * r >= ks / 8) break;  // uniform across the warp
            const int t = 32 * r + lane;
            const float v[8] = {hv[r][0].x, hv[r][0].y, hv[r][0].z, hv[r][0].w,
                                hv[r][1].x, hv[r][1].y, hv[r][1].z, hv[r][1].w};
            image_task(v, t < ks / 8, tb + t, hq, hsx, hX);
        }
        __syncwarp();
        const int st = i % kLDnStages;
        float a = 0.f;
        if (lwait(&full_dn[st], uint32_t(i / kLDnStages) & 1u, A.status, &s_abort)) {
            const uint8_t* chunk = dn_ring + size_t(st) * kLDnStage;
            const int gb = tb / 8;  // first group of the unit's slot
            for (int g = 0; g < ks / kGroup; ++g) {
                uint4 qa, qb;
                uint32_t sbw;
                a += group_dot(chunk, ks, g, lane, hq + (gb + g) * 8, hsx[gb + g], hX[gb + g], &qa, &qb, &sbw);
                if (en.wb)
                    group_writeback(en.wb + gu_section_bytes(D, en.F) + size_t(tile * (en.F / ks) + slice) * (18u * ks),
                                    ks, g, lane, qa, qb, sbw);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_dn[st]);
        s_upart[i][lane] = en.w * a;
    }
    named_sync(1, kLNC);
    // tile segments of the range, one warp each
    const int t_first = d0 / upt, t_last = (d1 - 1) / upt;
    for (int tt = t_first + warp; nu > 0 && tt <= t_last; tt += kLNW) {
        const int key_u0 = tt * upt;
        const int ua = max(d0, key_u0), ub = min(d1, key_u0 + upt);
        float tot = 0.f;
        for (int u = ua; u < ub; ++u) tot += s_upart[u - d0][lane];
        const bool whole = ua == key_u0 && ub == key_u0 + upt;
        bool lastc = whole;
        if (!whole) {
            const int sl = (ua == d0) ? 0 : 1;
            A.partials_dn[size_t(2 * c + sl) * 32 + lane] = tot;
            __threadfence();
            __syncwarp();
            int old = 0;
            if (lane == 0) old = atomicAdd(&A.counters_dn[tt], ub - ua);
            old = __shfl_sync(0xffffffffu, old, 0);
            lastc = (old + (ub - ua) == upt);
            if (lastc) {
                __threadfence();
                tot = 0.f;
                const int c0 = cta_of(key_u0, Udn, G), c1 = cta_of(key_u0 + upt - 1, Udn, G);
                for (int cc = c0; cc <= c1; ++cc) {
                    const int rs = range_start(cc, Udn, G);
                    if (rs >= range_start(cc + 1, Udn, G)) continue;
                    tot += __ldcg(A.partials_dn + size_t(2 * cc + (rs >= key_u0 ? 0 : 1)) * 32 + lane);
                }
                if (lane == 0) A.counters_dn[tt] = 0;
            }
        }
        if (lastc) {
            const int r = 32 * tt + lane;
            A.y[r] = tot;
            if (A.y_bf16) A.y_bf16[r] = f32_to_bf16_rn(tot);
        }
    }
}

// ----------------------------------------------------------------- host side
size_t layer_smem_bytes(const LayerArgs& a, int G) {
    return layer_carve(a.D, a.E, a.S, a.hvals, (a.E + G - 1) / G).total;
}

int layer_hvals(int D, int K, int F, int FS, int G) {
    // staged h values of the CTA with the most down units (at most 4 rings' worth)
    const int nsh = FS > 0 ? 1 : 0;
    const int upt = (nsh ? FS / down_ks(FS) : 0) + K * (F / down_ks(F));
    const int Udn = (D / kChunkRows) * upt;
    int most = (Udn + G - 1) / G;
    most = most < kLDnStages * 4 ? most : kLDnStages * 4;
    return most * kDownSliceMax;
}

bool layer_supported(int D, int E, int K, int F, int FS, int S, int G) {
    if (K > kLMaxK || K < 1 || G < 1) return false;
    const int nsh = FS > 0 ? 1 : 0;
    const int upt = (nsh ? FS / down_ks(FS) : 0) + K * (F / down_ks(F));
    const int Udn = (D / kChunkRows) * upt;
    if ((Udn + G - 1) / G > kLDnStages * 4) return false;  // staged h segments
    LayerArgs a{};
    a.D = D;
    a.E = E;
    a.S = S;
    a.hvals = layer_hvals(D, K, F, FS, G);
    // dynamic carve + the kernel's static shared arrays (about 6 KB) within the 227 KB per block
    return layer_smem_bytes(a, G) + (size_t(8) << 10) <= size_t(227) << 10;
}

int layer_threads() { return kLThreads; }

cudaError_t launch_layer(const LayerArgs& a, int G, bool pdl, cudaStream_t s) {
    static thread_local int attr_dev = -1;
    static thread_local size_t attr_smem = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const size_t smem = layer_smem_bytes(a, G);
    if (attr_dev != dev || attr_smem < smem) {
        e = cudaFuncSetAttribute(layer_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        attr_dev = dev;
        attr_smem = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kLThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    int n = 0;
    at[n].id = cudaLaunchAttributeCooperative;
    at[n].val.cooperative = 1;
    ++n;
    if (pdl) {
        at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = at;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, layer_decode_kernel, a);
}

cudaError_t layer_grid(int dev, int* G) {
    int sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    *G = sms;
    return cudaSuccess;
}

}  // namespace moe
