// layer.cuh -- host interface of the one-token layer kernel (layer.cu).
#pragma once
#include "common.cuh"
#include "plan.cuh"

namespace moe {

struct LayerArgs {
    // the token's input and the layer's resident weights
    const uint16_t* x;           // bf16 [D] (device)
    const int8_t* wq;            // router int8 [E][D], 16-byte aligned
    const uint16_t* ws;          // router binary16 scales [E][D/64]
    const float* bias;           // [E] or null
    const uint8_t* shared_blob;  // shared expert (width FS), or null
    // routed experts: resident (experts + e * expert_stride) when experts is
    // non-null, else the slot cache below
    const uint8_t* experts;
    size_t expert_stride;
    uint8_t* slots;
    size_t slot_stride;
    int32_t* state;              // count[E], last_use[E], slot_of[E], expert_in[S]
    const uint8_t* store;        // pinned host store, device-accessible (misses are read from it)
    size_t store_stride;
    int policy;
    uint32_t decay_period;
    uint32_t step;
    int D, E, K, F, FS, S;
    size_t blob_bytes;           // routed blob size (statistics)
    int hvals;                   // staged h values per CTA (layer_hvals)
    // outputs
    float* y;                    // fp32 [D]
    uint16_t* y_bf16;            // bf16 [D] or null
    int32_t* ids;                // [K] or null
    float* gate_w;               // [K] or null
    PlanMailbox* mailbox;        // plan for the host, or null
    uint32_t seq;
    uint64_t* stats;             // device counters (calls, hits, misses, bytes, repeats, selections) or null
    // scratch
    float* logits;               // [E]
    float* h;                    // [FS + K*F]
    float* partials_gu;          // [4*G][32]: two per CTA and pool (shared, routed)
    int* counters_gu;            // [FS/16 + K*F/16], zero between launches
    float* partials_dn;          // [2*G][32]
    int* counters_dn;            // [D/32], zero between launches
    unsigned* bar;               // [128], zero-initialised (two grid barriers, counter and generation lines apart)
    int* status;
};

// Whether the one-token layer kernel handles these sizes on a grid of G CTAs
// (shared memory, staged down segments, K).
bool layer_supported(int D, int E, int K, int F, int FS, int S, int G);
int layer_hvals(int D, int K, int F, int FS, int G);
cudaError_t layer_grid(int dev, int* G);
// Cooperative launch (all CTAs resident), with programmatic dependent launch
// when pdl is set.
cudaError_t launch_layer(const LayerArgs& a, int G, bool pdl, cudaStream_t s);

}  // namespace moe
