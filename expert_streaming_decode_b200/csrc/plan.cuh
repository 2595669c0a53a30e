// plan.cuh -- the pinned mapped mailbox through which the cache-plan kernel
// hands each call's plan to the host, and the plan launchers (plan.cu).
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kMailboxMax = 1024;  // distinct experts per call (n_experts <= 1024)

struct PlanMailbox {
    uint32_t seq;         // written last by the kernel: the call's sequence number
    int32_t n_distinct;
    int32_t n_waves;
    int32_t n_misses;
    int32_t expert[kMailboxMax];
    int32_t slot[kMailboxMax];
    int32_t hit[kMailboxMax];
    int32_t victim[kMailboxMax];
    int32_t wave[kMailboxMax];
};

size_t plan_smem_bytes(int E, int S);
// `wl_shared` / `wl_routed` (wl == nullptr: skip): one-token work lists of the
// shared-expert phase and of the routed phase, written when npairs <= 32 (T = 1).
// `stats` (or null): the context's counters, updated by the kernel (calls,
// hits, misses, missed bytes at blob_bytes each, repeats, distinct experts).
cudaError_t launch_plan(const int32_t* ids, int npairs, int E, int S, int policy, uint32_t decay_period,
                        int32_t* state, uint32_t step,
                        int32_t* pair_slot, int32_t* pair_wave, PlanMailbox* mailbox, uint32_t seq, int* status,
                        const float* gate_w, const DecodeWLTarget& wl_shared, const DecodeWLTarget& wl_routed,
                        uint64_t* stats, uint64_t blob_bytes, bool pdl, cudaStream_t s);
cudaError_t launch_cache_reset(int32_t* state, int E, int S, bool pdl, cudaStream_t s);

}  // namespace moe
