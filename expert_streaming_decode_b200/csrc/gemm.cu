// gemm.cu -- K6: tcgen05 tensor-core grouped GEMM over dequantised expert
// tiles, for batches of tokens (a batched decode step, a prefill chunk).
//
// Method: the prompt is prefilled in chunks of up to 128 tokens so that an
// expert fetched once is applied to every row routed to it ("TurboFieldfare:
// motor open source ...", section "Proceso de generacion de tokens").  With
// the call's (token, k) pairs grouped by expert, each expert is a small dense
// GEMM: H = gelu_tanh(X W_g^T) * (X W_u^T) [M_e x F], Y = H W_d^T [M_e x D],
// y[t] += w * Y[t] -- the one dense contraction on the path.
//
// B200 mapping (one CTA per (entry, 128 output rows); an entry is an expert
// and up to 64 of its token rows):
//   * D[128 x N] = A[128 x K] * B[N x K]^T with tcgen05.mma kind::f16, M = 128
//     weight rows, N = the entry's token rows rounded up to 16 (experts carry
//     a few rows each, so the weights sit in the M slot), fp32 accumulator in
//     tensor memory.
//   * A producer warp streams the raw 4-bit weights of the CTA's four blob
//     tiles into a shared-memory ring with 1-D bulk copies (mbarrier
//     transaction counts, L2 evict-first); the down GEMM starts streaming
//     before it waits on the gate/up GEMM, since its weights do not depend on it.
//   * K runs in groups of 64 (one quantisation group).  Per group eight math
//     warps dequantise the 128 x 64 weight tile from the ring (w = s*q + b
//     rounded to fp16, two weights per half2 instruction) and write it, with
//     the N x 64 activation tile (loaded into registers four groups ahead: x
//     as bf16, h as the fp16 the gate/up epilogue stored), in
//     the no-swizzle K-major core-matrix layout (8 rows x 16 bytes per core
//     matrix; K-direction core stride 128 B, 8-row stride 1024 B).  An MMA
//     warp issues 4 MMAs of K = 16 per group and commits them to an mbarrier;
//     two fp16 buffer sets let the math warps run a group ahead of the tensor
//     core, and the raw-weight ring holds 12 groups per CTA.
//   * gate/up epilogue: TMEM lanes 32w..32w+31 hold one 32-row blob tile (16
//     gate rows then the 16 matching up rows): h = gelu(g) * u with one
//     shuffle, stored as fp16 (the down GEMM's operand type; the rounding is
//     the one the down GEMM applied to fp32 h before).
//   * down epilogue: y[token][row] += w * D, fp32 atomics (entries of different
//     experts add into the same output rows).
#include "common.cuh"
#include "ffn.cuh"
#include "launch.cuh"

namespace moe {


struct GemmArgs {
    const WorkList* wl;
    const FfnEntry* entries;
    const FfnRow* rows;
    const uint16_t* x;   // fp16 bits [T][D] (the call's hidden states, converted once per call)
    float* h;            // activations
    float* y;            // [T][D], accumulated
    int D;
    int b_bytes;         // bytes of one B (activation) tile buffer: the call's row cap (<= 64, a multiple of 16) x 128
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

// bounded wait that gives up at once once any warp of the CTA timed out
__device__ __forceinline__ bool ring_wait_gemm(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, status)) return true;
    *abort_flag = 1;
    return false;
}

// Raw weight stages.  A stage is GPS consecutive quantisation groups of the
// CTA's four blob tiles; per blob tile its nibble block (GPS x 1 KB: two
// 16-byte word-quads per row and group) and its scale/bias block (GPS x
// 128 B) are each contiguous inside one chunk, so a stage is 8 bulk copies.
// Ring layout: [NST stages][4 blob tiles][GPS KB nibbles | GPS x 128 B s,b].
template <int MODE>
struct GemmRing;
#ifndef MOE_GEMM_GU_STAGES
#define MOE_GEMM_GU_STAGES 3
#endif
template <>
struct GemmRing<0> {  // gate/up: 4 groups per 256-input chunk, take 2 at a time
    static constexpr int kGroupsPerStage = 2;
    static constexpr int kStages = MOE_GEMM_GU_STAGES;
};
template <>
struct GemmRing<1> {  // down: chunk widths need not be even in groups
    static constexpr int kGroupsPerStage = 1;
    static constexpr int kStages = 2 * MOE_GEMM_GU_STAGES;
};
template <int MODE>
__host__ __device__ constexpr int ring_bt_bytes() { return GemmRing<MODE>::kGroupsPerStage * 1152; }
template <int MODE>
__host__ __device__ constexpr int ring_stage_bytes() { return 4 * ring_bt_bytes<MODE>(); }

constexpr int kOpBufs = 2;                          // fp16 operand buffer sets (A and B tiles of one group)
constexpr int kABytes = 128 * 64 * 2;               // A: 128 weight rows x 64 inputs
constexpr int kBBytes = kGemmMaxRows * 64 * 2;      // B: up to kGemmMaxRows token rows x 64 inputs
// Shared memory of one CTA when the B buffers hold b_bytes each (sized by the
// call's row cap, so that small batches fit three CTAs per SM).
template <int MODE>
constexpr size_t gemm_smem(int b_bytes = kBBytes) {
    return size_t(kOpBufs) * (kABytes + size_t(b_bytes)) + size_t(GemmRing<MODE>::kStages) * ring_stage_bytes<MODE>() +
           128;
}

constexpr int kMathWarps = 8;               // thread = (weight row, half of the group's 64 inputs)
constexpr int kMathThreads = kMathWarps * 32;
constexpr int kProducerWarp = kMathWarps;   // bulk copies of raw weights
constexpr int kMmaWarp = kMathWarps + 1;    // issues the tensor-core MMAs
constexpr int kGemmWarps = kMathWarps + 2;
constexpr int kBTasks = kGemmMaxRows * 8 / kMathThreads;  // (row, 8-input block) tasks of the B tile per thread
constexpr int kAhead = 4;  // groups whose activations are in flight (registers) ahead of their use

// Inside every 8-input block the fp16 tiles hold the inputs in the order
// 0,4,1,5,2,6,3,7 (A and B alike, so the contraction is unchanged): that is
// the order in which two nibbles at a time come out of a 32-bit word below.

// 8 weights w = s*q + b of one 32-bit word (nibble i = input i) as fp16, in the
// block order above.  A 4-bit field placed in a binary16 mantissa reads as an
// exact integer offset from a power of two: in the low bits of 1024.0
// (0x6400, unit 1) as 1024 + q, and in bits 4..7 of 64.0 (0x5400, unit 1/16)
// as 64 + q.  So nibbles i and i+4 (bits 4i and 16+4i) come out of the word
// with one logic operation each for i = 0, 1, and of the word shifted by 8 for
// i = 2, 3; subtracting the power of two is exact, and the fused multiply-add
// rounds s*q + b once.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t s2, uint32_t b2) {
    const uint32_t w8 = w >> 8;
    const uint32_t m[4] = {(w & 0x000F000Fu) | 0x64006400u, (w & 0x00F000F0u) | 0x54005400u,
                           (w8 & 0x000F000Fu) | 0x64006400u, (w8 & 0x00F000F0u) | 0x54005400u};
    const uint32_t base[4] = {0x64006400u, 0x54005400u, 0x64006400u, 0x54005400u};
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t q;
        asm("sub.f16x2 %0, %1, %2;" : "=r"(q) : "r"(m[i]), "r"(base[i]));
        asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r[i]) : "r"(q), "r"(s2), "r"(b2));
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// Warp roles.  Producer warp: bulk copies of raw weight stages into the ring
// (full/empty barriers).  Math warps: per group, wait for the ring stage and a
// free operand buffer set, write the fp16 B tile (activations, loaded one
// group ahead) and the dequantised A tile, arrive on `ready`.  MMA warp: per
// group, wait for `ready`, issue 4 MMAs (K = 16 each) into the tensor-memory
// accumulator and commit them to `freed` (the buffer set may be rewritten);
// a last commit on `done` releases the epilogue.  No CTA-wide barrier runs
// per group.
template <int MODE>
__global__ void __launch_bounds__(kGemmWarps * 32, 3) grouped_gemm_kernel(GemmArgs A) {
    constexpr int GPS = GemmRing<MODE>::kGroupsPerStage;
    constexpr int NST = GemmRing<MODE>::kStages;
    constexpr int BT_BYTES = ring_bt_bytes<MODE>();
    constexpr int ST_BYTES = ring_stage_bytes<MODE>();
    extern __shared__ __align__(128) uint8_t gsm[];
    uint8_t* sA = gsm;                                   // [kOpBufs][128 x 64 fp16]
    uint8_t* sB = gsm + kOpBufs * kABytes;               // [kOpBufs][b_bytes: row cap x 64 fp16]
    uint8_t* ring = sB + kOpBufs * A.b_bytes;            // [NST][ST_BYTES]
    __shared__ __align__(8) uint64_t full[NST], empty[NST];
    __shared__ __align__(8) uint64_t ready[kOpBufs], freed[kOpBufs], done;
    __shared__ uint32_t tbase;
    __shared__ FfnEntry s_en;
    __shared__ int s_tile;
    __shared__ FfnRow s_rows[kGemmMaxRows];
    __shared__ int s_bad, s_abort;

    // gate/up: the work list is the previous launch's output; down: it is two
    // launches back, so the weights start streaming before the wait
    if (MODE == 0) {
        pdl_wait();
        pdl_trigger();
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const WorkList W = *A.wl;
    const int total = MODE == 0 ? W.units_gu : W.units_dn;
    if (int(blockIdx.x) >= total) return;
    const int D = A.D;
    if (tid == 0) {
        int lo = 0, hi = W.n_entries - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            const int b = MODE == 0 ? A.entries[mid].ubase_gu : A.entries[mid].ubase_dn;
            if (b <= int(blockIdx.x)) lo = mid; else hi = mid - 1;
        }
        s_en = A.entries[lo];
        s_tile = int(blockIdx.x) - (MODE == 0 ? s_en.ubase_gu : s_en.ubase_dn);
        s_bad = 0;
        s_abort = 0;
        for (int i = 0; i < NST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kMathWarps);
        }
        for (int i = 0; i < kOpBufs; ++i) {
            mbar_init(&ready[i], kMathWarps);
            mbar_init(&freed[i], 1);
        }
        mbar_init(&done, 1);
        mbar_fence_init();
    }
    __syncthreads();
    const FfnEntry en = s_en;
    const int tile = s_tile;
    const int M = min(en.n_rows, kGemmMaxRows);
    const int N = (M + 15) & ~15;
    if (N * 128 > A.b_bytes) {  // more rows than the launch's B buffers hold: report, touch nothing
        if (tid == 0) set_status(A.status, MOE_ERR_RANGE);
        return;
    }
    const int F = en.F;
    const int Kin = MODE == 0 ? D : F;
    const int ngroups = Kin / kGroup;
    const int ks = MODE == 0 ? kGuSlice : down_ks(F);
    const int nsl = MODE == 0 ? D / kGuSlice : F / ks;
    const int gpc = ks / kGroup;  // groups per chunk (a multiple of GPS)
    const uint8_t* sec = en.blob + (MODE == 0 ? size_t(0) : gu_section_bytes(D, F));
    const int nstages = ngroups / GPS;
    const int ncols = N <= 32 ? 32 : 64;  // tensor-memory columns: fp32 accumulator [128 lanes][N]

    if (warp == kProducerWarp) {
        // -------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            int issued = 0;
            bool ok = true;
            for (int si = 0; si < nstages && ok; ++si, ++issued) {
                const int st = si % NST;
                if (si >= NST) ok = ring_wait_gemm(&empty[st], ((si / NST) - 1) & 1, A.status, &s_abort);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[st], ST_BYTES);
                uint8_t* dst = ring + size_t(st) * ST_BYTES;
                const int g0 = si * GPS, c = g0 / gpc, gg = g0 % gpc;  // chunk and first group in it
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const uint8_t* chunk = sec + (size_t(4 * tile + w) * nsl + c) * (18u * ks);
                    bulk_g2s(dst + w * BT_BYTES, chunk + gg * 1024, GPS * 1024, &full[st], pol);
                    bulk_g2s(dst + w * BT_BYTES + GPS * 1024, chunk + 16 * ks + gg * 128, GPS * 128, &full[st], pol);
                }
            }
            // no copy may land after the CTA exits
            const int first = issued > NST ? issued - NST : 0;
            for (int i = first; i < issued; ++i) mbar_wait(&full[i % NST], (i / NST) & 1, A.status);
        }
        return;
    }

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tbase)),
                     "r"(ncols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid < M) s_rows[tid] = A.rows[en.row0 + tid];
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    named_sync(2, kMathThreads + 32);  // math warps + MMA warp
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tbase;

    if (warp == kMmaWarp) {
        // ----------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(128 >> 4) << 24);
            for (int g = 0; g < ngroups; ++g) {
                const int b = g % kOpBufs;
                if (!ring_wait_gemm(&ready[b], (g / kOpBufs) & 1, A.status, &s_abort)) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t a_addr = smem_u32(sA + b * kABytes), b_addr = smem_u32(sB + b * A.b_bytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t ad = umma_desc(a_addr + kk * 256);
                    const uint64_t bd = umma_desc(b_addr + kk * 256);
                    const uint32_t acc = (g > 0 || kk > 0) ? 1u : 0u;
                    asm volatile(
                        "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, "
                        "%3, p;\n}\n" ::"r"(tmem),
                        "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                        : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&freed[b]))
                             : "memory");
            }
            // completes when every MMA issued above has (also after an early stop)
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             smem_u32(&done))
                         : "memory");
        }
        return;
    }

    // ------------------------------------------------------------ math warps
    if (MODE == 1) {
        pdl_wait();  // h is the gate/up GEMM's output
        pdl_trigger();
    }
    // Activation tile tasks: task idx = tid + kMathThreads*i covers row j,
    // inputs 8*kb .. +7 of the group, with j = 8*(idx/64) + idx%8 and
    // kb = (idx/8)%8: a warp's 16-byte stores then hit 8 different rows of a
    // core matrix (no bank conflicts) and its loads still fill whole sectors.
    // Rows M..N-1 are zero padding.  Raw loads are kept in registers, two
    // groups ahead (two register sets, alternating), and converted when used.
    // MODE 0 reads x (as fp16, converted once per call), MODE 1 the h rows the
    // gate/up GEMM stored as fp16 (at the same element offsets): 8 fp16 per task
    const int ntasks = 8 * N;
    using Raw = uint4;
    const uint16_t* bsrc[kBTasks];  // row base of each task (nullptr: padding row)
#pragma unroll
    for (int i = 0; i < kBTasks; ++i) {
        const int idx = tid + kMathThreads * i;
        const int j = 8 * (idx >> 6) + (idx & 7);
        bsrc[i] = nullptr;
        if (idx < ntasks && j < M)
            bsrc[i] = MODE == 0 ? A.x + size_t(s_rows[j].x_row) * D
                                : reinterpret_cast<const uint16_t*>(A.h) + s_rows[j].h_off;
    }
    auto load_b = [&](int g, Raw (&braw)[kBTasks]) {
#pragma unroll
        for (int i = 0; i < kBTasks; ++i) {
            const int idx = tid + kMathThreads * i;
            if (idx >= ntasks) break;
            const int k0 = g * kGroup + 8 * ((idx >> 3) & 7);
            braw[i] = bsrc[i] ? *reinterpret_cast<const uint4*>(bsrc[i] + k0) : make_uint4(0, 0, 0, 0);
        }
    };
    // this thread's weights: row r of the 128 (blob tile 4*tile + r/32, row r%32), inputs 32*hk .. +31 of each group
    const int r = tid & 127, hk = tid >> 7;
    const int bt_row = r >> 5, row = r & 31;
    // one group: wait for its ring stage and a free buffer set, write B (from
    // braw, then reload braw with group g + 2) and the dequantised A, arrive
    auto step = [&](int g, Raw (&braw)[kBTasks]) -> bool {
        const int si = g / GPS, gl = g % GPS, st = si % NST;
        const int b = g % kOpBufs;
        // the buffer set's previous MMAs are done; the ring stage has landed
        if (g >= kOpBufs && !ring_wait_gemm(&freed[b], ((g / kOpBufs) - 1) & 1, A.status, &s_abort)) return false;
        if (gl == 0 && !ring_wait_gemm(&full[st], (si / NST) & 1, A.status, &s_abort)) return false;
        uint8_t* a = sA + b * kABytes;
        uint8_t* bt = sB + b * A.b_bytes;
#pragma unroll
        for (int i = 0; i < kBTasks; ++i) {
            const int idx = tid + kMathThreads * i;
            if (idx >= ntasks) break;
            const uint4 q = braw[i];
            // fp16 already (range checked when written): reorder (0,1)(2,3)(4,5)(6,7)
            // into the block order (0,4)(1,5)(2,6)(3,7)
            const uint4 out = make_uint4(__byte_perm(q.x, q.z, 0x5410), __byte_perm(q.x, q.z, 0x7632),
                                         __byte_perm(q.y, q.w, 0x5410), __byte_perm(q.y, q.w, 0x7632));
            const int j = 8 * (idx >> 6) + (idx & 7);
            *reinterpret_cast<uint4*>(bt + core_off(j, 8 * ((idx >> 3) & 7))) = out;
        }
        if (g + kAhead < ngroups) load_b(g + kAhead, braw);
        // A: dequantise this thread's 32 weights of the group from the raw stage
        {
            const uint8_t* raw = ring + size_t(st) * ST_BYTES + bt_row * BT_BYTES;
            const uint4 q = *reinterpret_cast<const uint4*>(raw + ((2 * gl + hk) * 32 + row) * 16);
            const uint32_t sbw = *reinterpret_cast<const uint32_t*>(raw + GPS * 1024 + (gl * 32 + row) * 4);
            const uint32_t s2 = __byte_perm(sbw, 0, 0x1010), b2 = __byte_perm(sbw, 0, 0x3232);  // (s,s), (b,b)
            const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)  // word j: inputs 32*hk + 8j .. +7 of the group
                *reinterpret_cast<uint4*>(a + core_off(r, 32 * hk + 8 * j)) = dequant_word(words[j], s2, b2);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&ready[b]);
            if (gl == GPS - 1) mbar_arrive(&empty[st]);  // this warp is done with the raw stage
        }
        return true;
    };
    Raw braw0[kBTasks], braw1[kBTasks], braw2[kBTasks], braw3[kBTasks];
    load_b(0, braw0);
    if (ngroups > 1) load_b(1, braw1);
    if (ngroups > 2) load_b(2, braw2);
    if (ngroups > 3) load_b(3, braw3);
    bool ok = true;
    for (int g = 0; g < ngroups && ok; g += kAhead) {
        ok = step(g, braw0);
        if (ok && g + 1 < ngroups) ok = step(g + 1, braw1);
        if (ok && g + 2 < ngroups) ok = step(g + 2, braw2);
        if (ok && g + 3 < ngroups) ok = step(g + 3, braw3);
    }
    // every MMA the MMA warp issued has completed
    if (ok) ok = ring_wait_gemm(&done, 0, A.status, &s_abort);
    ok = __all_sync(0xffffffffu, ok);  // the tensor-memory loads below are warp-collective
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ok) {
        // warp w reads TMEM lanes 32*(w%4) ..; warps 0-3 take column blocks 0, 32, warps 4-7 blocks 16, 48
        const int q4 = warp & 3;
        for (int c0 = 16 * (warp >> 2); c0 < N; c0 += 32) {
            uint32_t v[16];
            const uint32_t ta = tmem + (uint32_t(q4 * 32) << 16) + uint32_t(c0);
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
                    // lanes of blob tile 4*tile + q4: 0..15 gate, 16..31 up of outputs 16*bt + lane
                    const float up = __shfl_down_sync(0xffffffffu, d, 16);
                    if (lane < 16 && j < M) {
                        // h as fp16, the type the down GEMM's B tile needs (same rounding)
                        const float hv = gelu_tanh(d) * up;
                        const bool in_range = fabsf(hv) <= 65504.f;
                        if (!in_range) s_bad = 1;
                        reinterpret_cast<__half*>(A.h)[s_rows[j].h_off + 16 * (4 * tile + q4) + lane] =
                            __float2half_rn(in_range ? hv : 0.f);
                    }
                } else if (j < M) {
                    atomicAdd(&A.y[size_t(s_rows[j].y_row) * D + 128 * tile + 32 * q4 + lane], s_rows[j].w * d);
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    named_sync(1, kMathThreads);
    if (s_bad && tid == 0) set_status(A.status, MOE_ERR_RANGE);  // an input or h beyond fp16
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
}

cudaError_t gemm_prepare() {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(gemm_smem<0>()));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(gemm_smem<1>()));
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
    const int n_cap = L.row_cap < 1 ? kGemmMaxRows : (L.row_cap > kGemmMaxRows ? kGemmMaxRows : L.row_cap);
    a.b_bytes = ((n_cap + 15) & ~15) * 128;
    if (hook) hook(hook_arg, 0);
    cudaError_t e = launch_kernel(grouped_gemm_kernel<0>, dim3(L.max_tiles_gu), dim3(kGemmWarps * 32),
                                  gemm_smem<0>(a.b_bytes), s, L.pdl, 1, a);
    if (e != cudaSuccess) return e;
    if (hook) hook(hook_arg, 1);
    e = launch_kernel(grouped_gemm_kernel<1>, dim3(L.max_tiles_dn), dim3(kGemmWarps * 32), gemm_smem<1>(a.b_bytes),
                      s, L.pdl, 1, a);
    if (hook) hook(hook_arg, 2);
    return e;
}

// The call's hidden states bf16 -> fp16, the operand type of the tensor-core
// tiles, once per layer call (every expert a token is routed to reads it);
// values beyond the fp16 range become 0 and are reported (MOE_ERR_RANGE).
__global__ void bf16_to_f16_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ out, size_t n8,
                                   int* status) {
    pdl_wait();
    pdl_trigger();
    bool bad = false;
    for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n8; i += size_t(gridDim.x) * blockDim.x) {
        const uint4 q = reinterpret_cast<const uint4*>(x)[i];
        const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
        uint32_t o[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float a = __uint_as_float(w4[t] << 16), b = __uint_as_float(w4[t] & 0xFFFF0000u);
            if (!(fabsf(a) <= 65504.f)) { bad = true; a = 0.f; }
            if (!(fabsf(b) <= 65504.f)) { bad = true; b = 0.f; }
            o[t] = pack_half2(a, b);
        }
        reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    if (bad) set_status(status, MOE_ERR_RANGE);
}

cudaError_t launch_bf16_to_f16(const uint16_t* x, uint16_t* out, size_t n, int* status, bool pdl, cudaStream_t s) {
    const size_t n8 = n / 8;
    const int blocks = int(n8 / 256 + 1 < 592 ? n8 / 256 + 1 : 592);
    return launch_kernel(bf16_to_f16_kernel, dim3(blocks), dim3(256), 0, s, pdl, 1, x, out, n8, status);
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
