// plan.cu -- K2: per-layer LFU expert-cache plan on the device.
//
// Method ("El milagro de la IA de 2GB en Apple Silicon", section "Mas
// inteligente que tu RAM": each layer keeps 16 of its 128 experts in an LFU
// cache and a miss replaces the least frequently used resident expert;
// "TurboFieldfare: motor open source ...", section "Proceso de generacion de
// tokens": the top-8 ids are checked against the layer's cache and the misses
// become a fetch plan).  Readings where the pages are silent: frequency = all
// selections so far (kept across evictions); ties by older last use, then
// lower id; the experts of the current wave are never evicted; empty slots
// fill lowest first; distinct experts are planned in ascending id, in waves of
// at most S; last_use = step + 1 after a wave.  Variants of the replacement
// rule (MOE_POLICY_*): LRU, LFU with periodic halving, in-cache LFU.
//
// One CTA per call.  State is staged in shared memory, counts are gathered
// with shared atomics, and a single warp walks the distinct experts in order;
// each miss picks its slot with a ballot (empty slot) or a shuffle arg-min
// over the resident slots (victim).  Results: pair -> slot map and pair ->
// wave map in device memory, and the per-expert plan in the pinned mapped
// mailbox for the host, published by writing `seq` last.
#include "common.cuh"
#include "plan.cuh"
#include "decode_wl.cuh"
#include "launch.cuh"

namespace moe {

constexpr int kPlanThreads = 256;

// shared-memory words before the staged mailbox rows: 6 int arrays of E, one
// of S, two byte arrays of E (rounded up to whole words)
__host__ __device__ inline int plan_mb_offset_words(int E, int S) { return 6 * E + S + (2 * E + 3) / 4; }

__global__ void __launch_bounds__(kPlanThreads) cache_plan_kernel(
    const int32_t* __restrict__ ids, int npairs, int E, int S, int policy, uint32_t decay_period,
    int32_t* __restrict__ state, uint32_t step,
    int32_t* __restrict__ pair_slot, int32_t* __restrict__ pair_wave, PlanMailbox* mailbox, uint32_t seq,
    int* status, const float* __restrict__ gate_w, DecodeWLTarget wl_shared, DecodeWLTarget wl_routed,
    uint64_t* stats, uint64_t blob_bytes) {
    extern __shared__ int32_t psm[];
    uint32_t* mult = reinterpret_cast<uint32_t*>(psm);   // [E] selections in this call
    uint32_t* count = mult + E;                           // [E]
    uint32_t* last = count + E;                           // [E]
    int32_t* slot_of = reinterpret_cast<int32_t*>(last + E);  // [E]
    int32_t* expert_in = slot_of + E;                     // [S]
    int32_t* uslot = expert_in + S;                       // [E] slot of expert in its wave
    int32_t* uwave = uslot + E;                           // [E]
    uint8_t* inwave = reinterpret_cast<uint8_t*>(uwave + E);  // [E]
    uint8_t* uhit = inwave + E;                           // [E] 1: the expert was resident
    int32_t* mb = reinterpret_cast<int32_t*>(psm) + plan_mb_offset_words(E, S);  // [5][E] mailbox rows, staged
    __shared__ int32_t ulist[1024];
    __shared__ int s_n;

    uint32_t* g_count = reinterpret_cast<uint32_t*>(state);
    uint32_t* g_last = g_count + E;
    int32_t* g_slot_of = state + 2 * E;
    int32_t* g_expert_in = state + 3 * E;
    pdl_wait();
    pdl_trigger();

    // the first pairs' ids load together with the state: one round trip
    const int id_first = int(threadIdx.x) < npairs ? ids[threadIdx.x] : 0;
    // LFU_DECAY: the counts are halved at the start of a call whose step is a
    // positive multiple of the period, before its selections are added
    const bool halve = policy == MOE_POLICY_LFU_DECAY && decay_period > 0u && step > 0u && step % decay_period == 0u;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        mult[e] = 0;
        count[e] = halve ? (uint32_t(g_count[e]) >> 1) : uint32_t(g_count[e]);
        last[e] = g_last[e];
        slot_of[e] = g_slot_of[e];
        uslot[e] = -1;
        uwave[e] = -1;
        inwave[e] = 0;
        uhit[e] = 0;
    }
    for (int s = threadIdx.x; s < S; s += blockDim.x) expert_in[s] = g_expert_in[s];
    __syncthreads();
    bool bad = false;
    for (int p = threadIdx.x; p < npairs; p += blockDim.x) {
        int e = p == int(threadIdx.x) ? id_first : ids[p];
        if (e < 0 || e >= E) { bad = true; e = 0; }
        atomicAdd(&mult[e], 1u);
    }
    if (bad) set_status(status, MOE_ERR_RANGE);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) count[e] += mult[e];
    __syncthreads();

    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        // distinct experts, ascending id (ballot compaction)
        int n = 0;
        for (int base = 0; base < E; base += 32) {
            const int e = base + lane;
            const bool f = e < E && mult[e] > 0;
            const uint32_t b = __ballot_sync(0xffffffffu, f);
            if (f) ulist[n + __popc(b & ((1u << lane) - 1u))] = e;
            n += __popc(b);
        }
        __syncwarp();
        int n_miss = 0, rep1 = 0, rep2 = 0;
        // experts also chosen by the previous call (last_use == step) or by
        // one of the two previous calls (last_use >= step - 1), before update
        for (int i = lane; i < n; i += 32) {
            const uint32_t lu = last[ulist[i]];
            rep1 += (lu != 0u && lu == step);
            rep2 += (lu != 0u && lu + 1u >= step);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            rep1 += __shfl_xor_sync(0xffffffffu, rep1, off);
            rep2 += __shfl_xor_sync(0xffffffffu, rep2, off);
        }
        const int waves = (n + S - 1) / S;
        for (int w = 0; w < waves; ++w) {
            const int lo = w * S, hi = min(n, (w + 1) * S);
            for (int i = lo + lane; i < hi; i += 32) inwave[ulist[i]] = 1;
            __syncwarp();
            for (int i = lo; i < hi; ++i) {
                const int e = ulist[i];
                int victim = -1, slot = slot_of[e];
                if (slot >= S) {  // corrupted state: treat as not resident, report
                    if (lane == 0) set_status(status, MOE_ERR_STATE);
                    slot = -1;
                }
                const bool hit = slot >= 0;
                if (!hit) {
                    // lowest empty slot
                    slot = -1;
                    for (int base = 0; base < S && slot < 0; base += 32) {
                        const int s = base + lane;
                        const uint32_t b = __ballot_sync(0xffffffffu, s < S && expert_in[s] < 0);
                        if (b) slot = base + __ffs(b) - 1;
                    }
                    if (slot < 0) {
                        // victim: smallest (count, last_use, id) among resident, not in
                        // this wave; LRU drops the count from the key
                        uint32_t bc = 0xffffffffu, bl = 0xffffffffu;
                        int br = 0x7fffffff;
                        for (int s = lane; s < S; s += 32) {
                            const int r = expert_in[s];
                            if (r < 0 || r >= E || inwave[r]) continue;
                            const uint32_t cr = policy == MOE_POLICY_LRU ? 0u : count[r];
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
                        if (br < E) {  // S >= wave size guarantees one exists in a valid state
                            victim = br;
                            slot = slot_of[victim];
                        }
                        if (slot < 0 || slot >= S) {  // corrupted state: stay in bounds, report
                            if (lane == 0) set_status(status, MOE_ERR_STATE);
                            victim = -1;
                            slot = 0;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) {
                        if (victim >= 0) {
                            slot_of[victim] = -1;
                            if (policy == MOE_POLICY_LFU_IN_CACHE) count[victim] = 0u;  // restarts when evicted
                        }
                        const int prev = expert_in[slot];
                        if (prev >= 0 && prev < E && prev != victim) slot_of[prev] = -1;
                        slot_of[e] = slot;
                        expert_in[slot] = e;
                    }
                    ++n_miss;
                }
                if (lane == 0) {
                    uslot[e] = slot;
                    uwave[e] = w;
                    uhit[e] = hit ? 1 : 0;
                    mb[i] = e;  // staged; copied to the host mailbox by all threads at the end
                    mb[E + i] = slot;
                    mb[2 * E + i] = hit ? 1 : 0;
                    mb[3 * E + i] = victim;
                    mb[4 * E + i] = w;
                }
                __syncwarp();
            }
            for (int i = lo + lane; i < hi; i += 32) {
                last[ulist[i]] = step + 1u;
                inwave[ulist[i]] = 0;
            }
            __syncwarp();
        }
        if (lane == 0) {
            s_n = n;
            if (stats) {
                stats[0] += 1;
                stats[1] += uint64_t(n - n_miss);
                stats[2] += uint64_t(n_miss);
                stats[3] += uint64_t(n_miss) * blob_bytes;
                stats[4] += uint64_t(rep1);
                stats[5] += uint64_t(rep2);
                stats[6] += uint64_t(n);
            }
            if (mailbox) {
                mailbox->n_distinct = n;
                mailbox->n_waves = waves;
                mailbox->n_misses = n_miss;
            }
        }
    }
    __syncthreads();
    for (int p = threadIdx.x; p < npairs; p += blockDim.x) {
        int e = ids[p];
        if (e < 0 || e >= E) e = 0;
        pair_slot[p] = uslot[e];
        if (pair_wave) pair_wave[p] = uwave[e];
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        g_count[e] = count[e];
        g_last[e] = last[e];
        g_slot_of[e] = slot_of[e];
    }
    for (int s = threadIdx.x; s < S; s += blockDim.x) g_expert_in[s] = expert_in[s];
    // one token: the work lists of the shared phase and of the routed phase
    if (threadIdx.x < 32 && (wl_shared.wl || wl_routed.wl) && npairs <= 32) {
        const int lane = threadIdx.x;
        int sl = 0;
        float w = 0.f;
        if (lane < npairs) {
            int e = ids[lane];
            if (e < 0 || e >= E) e = 0;
            sl = uslot[e] < 0 ? 0 : uslot[e];
            w = gate_w ? gate_w[lane] : 1.f;
        }
        // list A: shared expert + the selections already resident (runs while
        // the misses are copied); list B: the misses (runs after the copies)
        const bool hit = lane < npairs && uhit[ids[lane] < 0 || ids[lane] >= E ? 0 : ids[lane]];
        if (wl_shared.wl) write_decode_worklist(wl_shared, npairs, sl, w, hit);
        if (wl_routed.wl) write_decode_worklist(wl_routed, npairs, sl, w, !hit);
    }
    // the host's copy of the plan: rows written by all threads at once, then
    // one system-scope fence and `seq`, which the host polls for
    if (mailbox) {
        for (int i = threadIdx.x; i < s_n; i += blockDim.x) {
            mailbox->expert[i] = mb[i];
            mailbox->slot[i] = mb[E + i];
            mailbox->hit[i] = mb[2 * E + i];
            mailbox->victim[i] = mb[3 * E + i];
            mailbox->wave[i] = mb[4 * E + i];
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence_system();
            *reinterpret_cast<volatile uint32_t*>(&mailbox->seq) = seq;
        }
    }
}

size_t plan_smem_bytes(int E, int S) { return (size_t(plan_mb_offset_words(E, S)) + 5 * size_t(E)) * 4; }

cudaError_t launch_plan(const int32_t* ids, int npairs, int E, int S, int policy, uint32_t decay_period,
                        int32_t* state, uint32_t step,
                        int32_t* pair_slot, int32_t* pair_wave, PlanMailbox* mailbox, uint32_t seq, int* status,
                        const float* gate_w, const DecodeWLTarget& wl_shared, const DecodeWLTarget& wl_routed,
                        uint64_t* stats, uint64_t blob_bytes, bool pdl, cudaStream_t s) {
    static thread_local int attr_set_for = -1;  // device whose attribute this thread last set
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (attr_set_for != dev) {  // up to 51 KB for 1024 experts
        e = cudaFuncSetAttribute(cache_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(plan_smem_bytes(1024, 1024)));
        if (e != cudaSuccess) return e;
        attr_set_for = dev;
    }
    return launch_kernel(cache_plan_kernel, dim3(1), dim3(kPlanThreads), plan_smem_bytes(E, S), s, pdl, 1, ids, npairs,
                         E, S, policy, decay_period, state, step, pair_slot, pair_wave, mailbox, seq, status, gate_w,
                         wl_shared, wl_routed, stats, blob_bytes);
}

__global__ void cache_reset_kernel(int32_t* state, int E, int S) {
    pdl_wait();
    pdl_trigger();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < 3 * E + S; i += gridDim.x * blockDim.x)
        state[i] = (i < 2 * E) ? 0 : -1;
}

cudaError_t launch_cache_reset(int32_t* state, int E, int S, bool pdl, cudaStream_t s) {
    return launch_kernel(cache_reset_kernel, dim3(4), dim3(256), 0, s, pdl, 1, state, E, S);
}

}  // namespace moe
