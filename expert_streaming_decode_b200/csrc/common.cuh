// common.cuh -- device-side building blocks shared by the kernels of libmoe:
// status reporting, mbarrier + 1-D bulk-copy (TMA engine) wrappers with bounded
// waits, number conversions, and the work-list structures the expert kernels
// consume.  sm_100a only.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "moe.h"

namespace moe {

// ------------------------------------------------------------------ limits
constexpr int kMaxRows = 8;          // token rows one work entry carries (GEMV path)
constexpr int kGemmMaxRows = 64;     // token rows one work entry carries (grouped GEMM: its N)
constexpr int kGroup = 64;           // quantisation group
constexpr int kGuSlice = 256;        // gate/up chunk inputs (KS)
constexpr int kDownSliceMax = 704;   // down chunk inputs (KS) when F > 704
constexpr int kChunkRows = 32;       // rows per chunk
// Iterations of a bounded spin (each try_wait may itself block for a while);
// far beyond any legitimate wait (copies finish in microseconds).
constexpr uint32_t kSpinLimit = 1u << 24;

__host__ __device__ constexpr int down_ks(int F) { return F <= kDownSliceMax ? F : kDownSliceMax; }
__host__ __device__ constexpr size_t gu_section_bytes(int D, int F) {
    return size_t(F / 16) * size_t(D / kGuSlice) * 18u * kGuSlice;
}
__host__ __device__ constexpr size_t blob_bytes(int D, int F) {
    return gu_section_bytes(D, F) + size_t(D / kChunkRows) * size_t(F / down_ks(F)) * 18u * size_t(down_ks(F));
}

// ---------------------------------------------------------------- status
// The context's device status word: 0, or the first MOE_ERR_* a kernel hit.
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ----------------------------------------------------------- shared memory
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// --------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Nanoseconds of the GPU's global timer.
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Longest legitimate wait of any barrier here: copies and peer CTAs finish in
// microseconds (a missed expert read over the host link in well under 1 ms).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Bounded wait for the phase with the given parity to complete: gives up
// after kWaitLimitNs of global time or kSpinLimit tries, whichever comes
// first, and returns false after recording MOE_ERR_TIMEOUT.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
    unsigned long long t0 = 0;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255) == 255) {
            const unsigned long long t = global_ns();
            if (t0 == 0) t0 = t;
            else if (t - t0 > kWaitLimitNs) break;
        }
    }
    set_status(status, MOE_ERR_TIMEOUT);
    return false;
}

// ------------------------------------------------------- 1-D bulk copies
// Global -> shared bulk copy on the TMA engine, completion counted on `bar`
// (complete_tx).  Source and destination 16-byte aligned, bytes % 16 == 0.
// The copy lands in this CTA's own shared memory only.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// Bulk prefetch of [p, p + bytes) into L2 (no destination, no completion to
// wait for), spread over the calling threads: thread `i` of `n` issues pieces
// i, i+n, ...  p 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, size_t bytes, int i, int n) {
    constexpr size_t kPiece = 32768;
    const char* c = static_cast<const char*>(p);
    const size_t pieces = (bytes + kPiece - 1) / kPiece;
    for (size_t k = size_t(i); k < pieces; k += size_t(n)) {
        const size_t off = k * kPiece;
        const uint32_t len = uint32_t(bytes - off < kPiece ? bytes - off : kPiece);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(c + off), "r"(len) : "memory");
    }
}

// L2 policy for small weights read again on every token (kept in L2 ahead of
// the streamed expert weights).
__device__ __forceinline__ uint64_t l2_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// L2 policy for weights streamed exactly once per launch.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while its predecessor in the stream is finishing.
// Discipline used by every kernel here: before pdl_wait() a kernel only reads
// immutable data (weights) or data produced two or more launches back; after
// pdl_wait() (the predecessor has completed and its writes are visible) it may
// read anything and write; pdl_trigger() comes after pdl_wait(), so when a
// kernel starts, its predecessor's predecessor has completed.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Named barrier over a subset of warps (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ----------------------------------------------------------------- numbers
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float f16_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// GELU, tanh form: 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))).
__device__ __forceinline__ float gelu_tanh(float v) {
    const float c = 0.7978845608028654f;  // sqrt(2/pi)
    return 0.5f * v * (1.0f + tanhf(c * fmaf(0.044715f * v, v * v, v)));
}

// --------------------------------------------------------------- work lists
// One expert stream of the GEMV kernels: an expert blob and up to kMaxRows
// token rows that use it.
struct FfnEntry {
    const uint8_t* blob;   // expert blob (device, 256-byte aligned)
    // null, or a word that holds ready_val once the blob has landed (a miss
    // copied in by the copy engine while this list already runs)
    const uint32_t* ready;
    uint32_t ready_val;
    int F;                 // FFN width of this expert
    int n_rows;            // 1..kMaxRows
    int row0;              // first row in FfnRow[]
    int ubase_gu;          // first gate/up unit of this entry (global)
    int ubase_dn;          // first down unit of this entry (global)
};
struct FfnRow {
    int x_row;   // token whose hidden state is the input
    int h_off;   // float offset of this row's FFN activation in the h buffer
    int y_row;   // token whose output receives the result
    float w;     // gate weight (1 for the shared expert)
};
struct WorkList {
    int n_entries;
    int units_gu;     // total gate/up units (32-row x 256-input chunks)
    int units_dn;     // total down units (32-row x KS chunks)
    int T;            // tokens (rows of x and y)
    int units_per_tile_dn;  // down units per 32-row output tile
    int max_rows;     // largest n_rows of any entry
    // entries are the shared expert's (width FS) first, then routed ones
    // (width F): this is enough to map a unit to its entry in O(1)
    int n_shared;     // shared entries
    int ush_gu;       // gate/up units of one shared entry
    int urt_gu;       // gate/up units of one routed entry
    int ns_sh_dn;     // down slices per tile of a shared entry
    int ns_rt_dn;     // down slices per tile of a routed entry
    int F, FS;        // widths
};

// Where a one-token work list is written by the router or plan kernel (so no
// separate builder launch is needed); wl == nullptr: not requested.
struct DecodeWLTarget {
    WorkList* wl;
    FfnEntry* entries;
    FfnRow* rows;
    const uint8_t* slot_base;   // routed blob of slot s at slot_base + s*slot_stride
    size_t slot_stride;
    const uint8_t* shared_blob; // or null
    int F, FS, D;
    int h_shared_off;           // float offset of the shared row's activation
    size_t blob_bytes;          // routed blob size (for L2 prefetch)
    // routed entries of slot s wait until ready[s] == ready_val (null: no wait;
    // the default, so a target built field by field never waits on garbage)
    const uint32_t* ready = nullptr;
    uint32_t ready_val = 0;
};

}  // namespace moe
