// ffn.cuh -- host-side interface of the expert GEMV kernels (ffn.cu).
#pragma once
#include "common.cuh"

namespace moe {

struct GemvShape {
    int grid;       // persistent CTAs (SMs x resident CTAs per SM)
    size_t smem;    // dynamic shared memory per CTA
};
struct GemvShapes {
    GemvShape gu[2];   // [0]: one-token decode kernel, [1]: up to kMaxRows rows per entry
    GemvShape dn[2];
    int vstride_gu, vstride_dn;
    int stage_dn_decode;  // input values the down decode kernel stages (top_k*F + FS)
};

struct GemvLaunch {
    const WorkList* wl;
    const FfnEntry* entries;
    const FfnRow* rows;
    const uint16_t* x;
    float* h;
    const float* y_in;
    float* y;
    uint16_t* y_bf16;
    float* partials_gu;
    int* counters_gu;
    float* partials_dn;
    int* counters_dn;
    int D;
    int rmax;      // 1 when every entry has one row (T == 1), else kMaxRows
    const GemvShapes* shapes;
    int* status;
    bool pdl = true;  // launch with programmatic dependent launch
    int list_cap = 0;  // entries and rows the work-list buffers hold
    int max_tiles_gu = 0;  // one-token lists: most gate/up output tiles the list can hold (0: unknown)
    // one-token lists whose first entry is the shared expert: its blob, width
    // and h offset, so the gate/up kernel can start it before the work list
    // exists (null: no such entry, or do not start early)
    const uint8_t* shared_blob = nullptr;
    int FS = 0;
    int h_shared_off = 0;
};

struct WorkListArgs {
    int T, K;                   // tokens, selections per token in this call (K may be 0)
    const int32_t* pair_slot;   // [T*K]
    const int32_t* pair_wave;   // [T*K] or null: keep only pairs with pair_wave == wave
    int wave;
    const float* gate_w;        // [T*K]
    const uint8_t* slot_base;
    size_t slot_stride;
    int n_slot_range;
    int F;
    const uint8_t* shared_blob; // or null
    int FS;
    int h_shared_off;           // float offset of the shared rows in the h buffer
    int D;
    WorkList* wl;
    FfnEntry* entries;
    FfnRow* rows;
    int* status;
    int gemm = 0;  // GEMM mode: entries carry up to kGemmMaxRows rows; unit bases count 128-output GEMM tiles
};

// Tensor-core grouped GEMM (gemm.cu) over a work list built in GEMM mode.
struct GemmLaunch {
    const WorkList* wl;
    const FfnEntry* entries;
    const FfnRow* rows;
    const uint16_t* x;  // fp16 bits [T][D] (launch_bf16_to_f16 of the call's hidden states)
    float* h;
    float* y;          // accumulated with atomics: zero it before the first launch
    int D;
    int max_tiles_gu;  // grid bounds (CTAs past the work list's tile count exit)
    int max_tiles_dn;
    int row_cap = 0;   // most token rows any entry carries (the call's T, at most kGemmMaxRows); 0: kGemmMaxRows
    int* status;
    bool pdl = true;
};
cudaError_t gemm_prepare();
cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t s, void (*hook)(void*, int), void* hook_arg);
cudaError_t launch_f32_to_bf16(const float* y, uint16_t* out, size_t n, bool pdl, cudaStream_t s);
// bf16 [n] -> fp16 [n] (n % 8 == 0, 16-byte aligned); out-of-range values -> 0, MOE_ERR_RANGE
cudaError_t launch_bf16_to_f16(const uint16_t* x, uint16_t* out, size_t n, int* status, bool pdl, cudaStream_t s);

cudaError_t ffn_prepare(int D, int F, int FS, int K, int T, int sms, GemvShapes* shapes);
// Launch shapes of the one-token kernels (shapes->gu[0], dn[0]) for inputs up
// to vstride_gu wide (gate/up) and stage_dn staged values (down: top_k*F+FS),
// raising (never lowering) each kernel's dynamic shared-memory limit; the [1]
// entries are left zero.
cudaError_t ffn_shapes_one_row(int vstride_gu, int stage_dn, int T, int sms, GemvShapes* shapes);
// Raises the one-row kernels' shared-memory limits back to what `shapes`
// needs, should another user of the library have lowered them since.
cudaError_t ffn_ensure_one_row_smem(const GemvShapes& shapes);
// Launches K3 (gate/up) then K4 (down); `between` (may be null) is called
// after K3's launch and `after` after K4's (used for timing events).
cudaError_t launch_ffn(const GemvLaunch& L, cudaStream_t s, void (*hook)(void*, int), void* hook_arg);
cudaError_t launch_build_worklist(const WorkListArgs& a, bool pdl, cudaStream_t s);

}  // namespace moe
