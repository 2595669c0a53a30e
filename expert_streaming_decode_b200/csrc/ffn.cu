// ffn.cu -- K3/K4: streamed dequantising GEMV for the expert FFNs, and the
// work-list builder that groups (token, k) pairs by expert slot.
//
// Method: every expert (routed and shared) is a gated FFN with 4-bit affine
// weights in groups of 64 ("TurboFieldfare: motor open source ...", section
// "Estructura de ejecucion para reducir memoria"); routed outputs are weighted
// by the gate and combined with the shared branch (same page, "Proceso de
// generacion de tokens").  Per expert: g = W_g x, u = W_u x,
// h = gelu_tanh(g) * u, y_e = W_d h;  y = y_in + sum_e w_e y_e.
//
// B200 design (decode is HBM-bound: every weight byte is read once):
//   * The blob is a sequence of chunks (32 rows x KS inputs, 18*KS bytes) in
//     exactly the order the kernel consumes them.  A launch's work is the
//     concatenation of all entries' chunks ("units").  The grid is persistent
//     (SMs x resident CTAs) and CTA c owns units [c*U/G, (c+1)*U/G): equal
//     bytes per CTA, no tail wave.
//   * One producer warp streams units into a shared-memory ring with 1-D bulk
//     copies (TMA engine, mbarrier completion, L2 evict-first); consumer warps
//     compute.  Lanes are the chunk's 32 rows, warps split its groups.
//   * 4-bit codes become floats without conversions: one byte permute puts a
//     byte of nibbles into the mantissa of 0.5, giving f = 0.5 + q/256 exactly;
//     A = sum f*x then sum q*x = 256*A - 128*X with X = sum x of the group, so
//     a group contributes s*(256A - 128X) + b*X.  fp32 accumulation.
//   * A tile whose chunks straddle two CTAs is reconciled through partial sums
//     in global scratch and a per-tile counter: the last CTA to finish the tile
//     adds the partials in CTA order and writes the result (deterministic).
//   * K3 finishes each (entry, 16-output tile) with gelu_tanh(g) * u; K4 writes
//     w * (partial dot) per (entry, tile segment) and the last CTA of each
//     32-row output tile sums y_in and every entry in list order.
#include "common.cuh"
#include "decode_wl.cuh"
#include "ffn.cuh"
#include "launch.cuh"

namespace moe {

template <int MODE>
struct GemvCfg;
template <>
struct GemvCfg<0> {  // gate/up: KS = 256, 4 groups per chunk, one per warp
    static constexpr int NW = 4;
    static constexpr int STAGE = 18 * kGuSlice;
    static constexpr int NSTAGES = 8;
};
template <>
struct GemvCfg<1> {  // down: KS <= 704, up to 11 groups per chunk, one per warp
    static constexpr int NW = 11;
    static constexpr int STAGE = 18 * kDownSliceMax;
    static constexpr int NSTAGES = 6;
};

// One-token decode kernels.  Gate/up CTAs take one whole output tile each
// (11 units of 4.6 KB for the 26B-A4B shapes); consumer warps 0-3 read one
// group of every unit, warps 4-7 (when NW = 8) alternate units with them.
template <int MODE>
struct DecodeCfg;
// Gate/up stages hold up to CPS consecutive chunks of one tile (contiguous in
// the blob): one bulk request per stage.  Larger requests raise one CTA's
// share of HBM bandwidth, but the ring's shared memory sets how many of the
// layer's tile CTAs (484 for the 26B-A4B shapes) are resident at once; on
// B200 one-chunk stages (8 x 4.6 KB, five CTAs per SM: every tile in one
// wave) measured faster than 3 x 18 KB (three CTAs per SM).  The two values
// can be set at compile time for tuning.
#ifndef MOE_DECODE_GU_CPS
#define MOE_DECODE_GU_CPS 1
#endif
#ifndef MOE_DECODE_GU_STAGES
#define MOE_DECODE_GU_STAGES 8
#endif
template <>
struct DecodeCfg<0> {
    static constexpr int NW = 4;  // a multiple of 4 (groups per 256-input unit)
    static constexpr int CPS = MOE_DECODE_GU_CPS;  // chunks per stage
    static constexpr int NSTAGES = MOE_DECODE_GU_STAGES;
    static constexpr int STAGE = CPS * 18 * kGuSlice;
    static constexpr int kTilesPerCta = 1;
    static_assert(CPS >= 1 && NSTAGES >= 1, "gate/up ring");
};
#ifndef MOE_DECODE_DN_STAGES
#define MOE_DECODE_DN_STAGES 6
#endif
template <>
struct DecodeCfg<1> {
    static constexpr int NW = 11;
    static constexpr int CPS = 1;
    static constexpr int NSTAGES = MOE_DECODE_DN_STAGES;
    static constexpr int STAGE = 18 * kDownSliceMax;
};

constexpr int kCtaEntries = 24;  // work-list entries a CTA keeps in shared memory
static_assert(kCtaEntries <= 32, "the one-token producer keeps one bit per entry");

struct GemvArgs {
    const WorkList* wl;
    const FfnEntry* entries;
    const FfnRow* rows;
    const uint16_t* x;      // bf16 [T][D]
    float* h;               // activation buffer
    const float* y_in;      // [T][D] or null
    float* y;               // [T][D]
    uint16_t* y_bf16;       // [T][D] or null
    float* partials;        // K3: [2*grid][kMaxRows][32]; K4: [units][kMaxRows][32]
    int* counters;          // K3: per (entry, tile); K4: per output tile
    int D;
    int vstride;            // widest staged input row (D for gate/up, max F for down)
    int* status;
    int list_cap;           // entries (and rows) the work-list buffers hold
    // one-token gate/up: CTAs [0, gs) run the shared expert's tiles, which need
    // nothing the preceding launch writes, without waiting for it
    const uint8_t* shared_blob;
    int FS;
    int h_shared_off;
    int gs;
};

__device__ __forceinline__ int range_start(int c, int U, int G) { return int((long long)c * U / G); }
// The CTA whose range holds unit u (the last CTA whose start is <= u).
__device__ __forceinline__ int cta_of(int u, int U, int G) { return int(((long long)(u + 1) * G + U - 1) / U) - 1; }

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// Bounded wait that gives up at once after any warp of the CTA timed out or
// the producer stopped (the flag is polled while waiting), so a failure costs
// one time-out, not one per stage.
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
    if (*abort_flag) return false;
    unsigned long long t0 = 0;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255) == 255) {
            if (*abort_flag) return false;
            const unsigned long long t = global_ns();
            if (t0 == 0) t0 = t;
            else if (t - t0 > kWaitLimitNs) break;
        }
    }
    set_status(status, MOE_ERR_TIMEOUT);
    *abort_flag = 1;
    return false;
}

// Bounded wait (producer lane) until an entry's blob has landed: *ready ==
// want, written by the stream that copied it (after the copy, with a fence).
// Gives up after kWaitLimitNs, records MOE_ERR_TIMEOUT and stops the CTA.
__device__ __forceinline__ bool ready_wait(const uint32_t* ready, uint32_t want, int* status,
                                           volatile int* abort_flag) {
    unsigned long long t0 = 0;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t v;
        asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(ready) : "memory");
        if (v == want) return true;
        if (*abort_flag) return false;
        if ((i & 15) == 15) {
            const unsigned long long t = global_ns();
            if (t0 == 0) t0 = t;
            else if (t - t0 > kWaitLimitNs) break;
        }
        __nanosleep(64);
    }
    set_status(status, MOE_ERR_TIMEOUT);
    *abort_flag = 1;
    return false;
}

__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {  // u8 x s8
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {  // u8 x u8
    uint32_t d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Per-CTA view of the work list: the entries its unit range touches, staged
// in shared memory (global fallback beyond kCtaEntries).
struct EntryCache {
    const FfnEntry* g;
    const FfnEntry* s;
    int e0, n_staged, n;
    __device__ __forceinline__ const FfnEntry& at(int e) const {
        const int i = e - e0;
        return (i >= 0 && i < n_staged) ? s[i] : g[e];
    }
    template <int MODE>
    __device__ __forceinline__ int base(int e) const {
        return MODE == 0 ? at(e).ubase_gu : at(e).ubase_dn;
    }
    // entry of global unit u, scanning forward from `hint` (units ascend)
    template <int MODE>
    __device__ __forceinline__ int find(int u, int hint) const {
        int e = hint;
        while (e + 1 < n && base<MODE>(e + 1) <= u) ++e;
        return e;
    }
};

// Stages one input row for the integer dot products.  Per group of 64
// inputs: s_x = max|v| / 32767 and v ~= s_x * (256*hi + lo) with hi a signed
// byte and lo an unsigned byte (16-bit fixed point, error <= s_x/2).  The 16
// bytes for 8 inputs k0..k0+7 hold (hi of even k, lo of even k, hi of odd k,
// lo of odd k) as four byte-vectors, in the order the nibble extraction of the
// weights produces (low nibbles = even k, high nibbles = odd k).  X = sum v.
template <int MODE, int NCONS>
__device__ __forceinline__ void stage_row(const void* src, int kin, uint4* xq, float* sx, float* X) {
    const int tasks = kin / 8;
    for (int base = 0; base < tasks; base += NCONS) {
        const int i = base + int(threadIdx.x);
        const bool ok = i < tasks;
        float v[8];
        if (MODE == 0) {
            uint4 q = make_uint4(0, 0, 0, 0);
            if (ok) q = reinterpret_cast<const uint4*>(src)[i];
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[2 * j] = __uint_as_float(w4[j] << 16);
                v[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
            }
        } else {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
            if (ok) {
                a = reinterpret_cast<const float4*>(src)[2 * i];
                b = reinterpret_cast<const float4*>(src)[2 * i + 1];
            }
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
        float amax = 0.f, sum = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            amax = fmaxf(amax, fabsf(v[j]));
            sum += v[j];
        }
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {  // the 8 lanes of one group
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        }
        if (!ok) continue;
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
        xq[i] = make_uint4(hi_e, lo_e, hi_o, lo_o);
        if ((i & 7) == 0) {
            sx[i >> 3] = amax / 32767.f;
            X[i >> 3] = sum;
        }
    }
}

template <int MODE, int RMAX>
__global__ void __launch_bounds__((GemvCfg<MODE>::NW + 1) * 32) stream_gemv_kernel(GemvArgs A) {
    constexpr int NW = GemvCfg<MODE>::NW;
    constexpr int STAGE = GemvCfg<MODE>::STAGE;
    constexpr int kStages = GemvCfg<MODE>::NSTAGES;
    constexpr int NCONS = NW * 32;
    pdl_wait();  // the work list and the inputs come from the preceding launches
    const int D = A.D;
    const int n_entries = A.wl->n_entries;
    const int U = MODE == 0 ? A.wl->units_gu : A.wl->units_dn;
    const int T = A.wl->T;
    const int G = gridDim.x;
    const int c = blockIdx.x;
    const int u_begin = range_start(c, U, G), u_end = range_start(c + 1, U, G);

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * STAGE);
    uint64_t* empty = full + kStages;
    FfnEntry* s_ent = reinterpret_cast<FfnEntry*>(empty + kStages);   // [kCtaEntries]
    float* red = reinterpret_cast<float*>(s_ent + kCtaEntries);         // [NW][RMAX][32]
    const int vstride = A.vstride;
    const int ng_max = vstride / kGroup;
    const int gs = (ng_max + 3) & ~3;                                    // keeps xq 16-byte aligned
    float* sx = red + NW * RMAX * 32;                                    // [RMAX][gs]
    float* Xs = sx + RMAX * gs;                                          // [RMAX][gs]
    uint4* xq = reinterpret_cast<uint4*>(Xs + RMAX * gs);                // [RMAX][vstride/8]
    float* yacc = reinterpret_cast<float*>(xq + RMAX * (vstride / 8));   // [T][32] (MODE 1 finalize)
    __shared__ int s_abort, s_e0, s_n;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NW);
        }
        mbar_fence_init();
        // first entry of the range: binary search on the unit bases
        int lo = 0, hi = n_entries - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((MODE == 0 ? A.entries[mid].ubase_gu : A.entries[mid].ubase_dn) <= u_begin) lo = mid;
            else hi = mid - 1;
        }
        s_e0 = lo;
        s_n = min(kCtaEntries, n_entries - lo);
    }
    __syncthreads();
    pdl_trigger();
    if (u_begin >= u_end) return;
    for (int i = threadIdx.x; i < s_n; i += blockDim.x) s_ent[i] = A.entries[s_e0 + i];
    __syncthreads();
    EntryCache EC{A.entries, s_ent, s_e0, s_n, n_entries};

    if (warp == NW) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            int e = s_e0;
            int issued = 0;
            bool ok = true;
            for (int u = u_begin; u < u_end && ok; ++u, ++issued) {
                e = EC.find<MODE>(u, e);
                const FfnEntry& en = EC.at(e);
                const uint8_t* src;
                uint32_t bytes;
                if (MODE == 0) {
                    src = en.blob + size_t(u - en.ubase_gu) * (18 * kGuSlice);
                    bytes = 18 * kGuSlice;
                } else {
                    const int ks = down_ks(en.F);
                    src = en.blob + gu_section_bytes(D, en.F) + size_t(u - en.ubase_dn) * (18u * ks);
                    bytes = 18u * ks;
                }
                const int st = issued % kStages;
                if (issued >= kStages) ok = ring_wait(&empty[st], ((issued / kStages) - 1) & 1, A.status, &s_abort);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[st], bytes);
                bulk_g2s(ring + size_t(st) * STAGE, src, bytes, &full[st], pol);
            }
            // drain: every issued copy has landed before the CTA may exit
            const int first = issued > kStages ? issued - kStages : 0;
            for (int i = first; i < issued; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1, A.status);
        }
        return;
    }

    // ---------------------------------------------------------- consumers
    float acc[RMAX];
#pragma unroll
    for (int m = 0; m < RMAX; ++m) acc[m] = 0.f;
    int e = -1, nrows = 0, ns = 1, ks = kGuSlice, ubase = 0;
    int seg_start = u_begin;
    for (int u = u_begin; u < u_end; ++u) {
        const int i = u - u_begin;
        const int st = i % kStages;
        const int ne = EC.find<MODE>(u, e < 0 ? s_e0 : e);
        if (ne != e) {
            // new entry: stage its input rows as 16-bit fixed point per group
            e = ne;
            const FfnEntry& en = EC.at(e);
            nrows = en.n_rows;
            if (nrows > RMAX) {  // more rows than this variant stages: keep in bounds, report
                if (threadIdx.x == 0) set_status(A.status, MOE_ERR_RANGE);
                nrows = RMAX;
            }
            ks = MODE == 0 ? kGuSlice : down_ks(en.F);
            ns = MODE == 0 ? D / kGuSlice : en.F / ks;
            ubase = MODE == 0 ? en.ubase_gu : en.ubase_dn;
            const int kin = MODE == 0 ? D : en.F;
            named_sync(1, NCONS);
            for (int m = 0; m < nrows; ++m) {
                const FfnRow r = A.rows[en.row0 + m];
                const void* src = MODE == 0 ? static_cast<const void*>(A.x + size_t(r.x_row) * D)
                                            : static_cast<const void*>(A.h + r.h_off);
                stage_row<MODE, NCONS>(src, kin, xq + m * (vstride / 8), sx + m * gs, Xs + m * gs);
            }
            named_sync(1, NCONS);
        }
        const int ul = u - ubase;
        const int tile = ul / ns, slice = ul - tile * ns;

        // on a time-out the warp skips the compute but keeps every barrier, so
        // no other warp waits on it; the status word carries the error
        const bool have = ring_wait(&full[st], (i / kStages) & 1, A.status, &s_abort);
        const uint8_t* chunk = ring + size_t(st) * STAGE;
        for (int g = warp; have && g < ks / kGroup; g += NW) {
            const uint4 qa = lds128(chunk + ((2 * g) * 32 + lane) * 16);
            const uint4 qb = lds128(chunk + ((2 * g + 1) * 32 + lane) * 16);
            const uint32_t sbw = *reinterpret_cast<const uint32_t*>(chunk + 16 * ks + (g * 32 + lane) * 4);
            const float s = f16_to_f32(uint16_t(sbw & 0xFFFF)), b = f16_to_f32(uint16_t(sbw >> 16));
            const int G64 = (slice * ks) / kGroup + g;      // global group of the input row
            const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
            int shi[RMAX], shi2[RMAX];
            uint32_t slo[RMAX], slo2[RMAX];
#pragma unroll
            for (int m = 0; m < RMAX; ++m) { shi[m] = 0; shi2[m] = 0; slo[m] = 0; slo2[m] = 0; }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t lo = words[j] & 0x0F0F0F0Fu;          // even inputs, one per byte
                const uint32_t hi = (words[j] >> 4) & 0x0F0F0F0Fu;   // odd inputs
#pragma unroll
                for (int m = 0; m < RMAX; ++m) {
                    if (m < nrows) {
                        const uint4 xv = xq[m * (vstride / 8) + G64 * 8 + j];
                        shi[m] = dp4a_us(lo, xv.x, shi[m]);
                        slo[m] = dp4a_uu(lo, xv.y, slo[m]);
                        shi2[m] = dp4a_us(hi, xv.z, shi2[m]);
                        slo2[m] = dp4a_uu(hi, xv.w, slo2[m]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < RMAX; ++m) {
                if (m < nrows) {
                    // sum_k q_k x_k over the group, exact up to x's 16-bit image
                    const int dot = 256 * (shi[m] + shi2[m]) + int(slo[m] + slo2[m]);
                    const float qx = float(dot) * sx[m * gs + G64];
                    acc[m] = fmaf(s, qx, fmaf(b, Xs[m * gs + G64], acc[m]));
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);

        // segment end: next unit is another (entry, tile), or the range ends
        bool seg_end = (u + 1 == u_end);
        if (!seg_end) {
            const int e2 = EC.find<MODE>(u + 1, e);
            seg_end = (e2 != e) || ((ul + 1) / ns != tile);
        }
        if (!seg_end) continue;

        named_sync(1, NCONS);
#pragma unroll
        for (int m = 0; m < RMAX; ++m) red[(warp * RMAX + m) * 32 + lane] = acc[m];
        named_sync(1, NCONS);
#pragma unroll
        for (int m = 0; m < RMAX; ++m) acc[m] = 0.f;
        if (warp == 0) {
            const FfnEntry& en = EC.at(e);
            float tot[RMAX];
#pragma unroll
            for (int m = 0; m < RMAX; ++m) {
                tot[m] = 0.f;
                for (int w = 0; w < NW; ++w) tot[m] += red[(w * RMAX + m) * 32 + lane];
            }
            const int tile_u0 = ubase + tile * ns;  // first unit of (entry, tile)
            if (MODE == 0) {
                const bool whole = (seg_start == tile_u0) && (u + 1 == tile_u0 + ns);
                bool last = whole;
                const int cidx = tile_u0 / ns;  // (entry, tile) counter index
                if (!whole) {
                    const int slot = (seg_start == u_begin) ? 0 : 1;
                    float* P = A.partials + (size_t(2 * c + slot) * kMaxRows) * 32;
#pragma unroll
                    for (int m = 0; m < RMAX; ++m)
                        if (m < nrows) P[m * 32 + lane] = tot[m];
                    __threadfence();
                    __syncwarp();
                    int old = 0;
                    if (lane == 0) old = atomicAdd(&A.counters[cidx], u + 1 - seg_start);
                    old = __shfl_sync(0xffffffffu, old, 0);
                    last = (old + (u + 1 - seg_start) == ns);
                    if (last) {
                        __threadfence();
                        // sum the tile's partials in CTA order
#pragma unroll
                        for (int m = 0; m < RMAX; ++m) tot[m] = 0.f;
                        const int c0 = cta_of(tile_u0, U, G), c1 = cta_of(tile_u0 + ns - 1, U, G);
                        for (int cc = c0; cc <= c1; ++cc) {
                            if (range_start(cc, U, G) >= range_start(cc + 1, U, G)) continue;
                            const int sl = range_start(cc, U, G) >= tile_u0 ? 0 : 1;
                            const float* Q = A.partials + (size_t(2 * cc + sl) * kMaxRows) * 32;
#pragma unroll
                            for (int m = 0; m < RMAX; ++m)
                                if (m < nrows) tot[m] += __ldcg(Q + m * 32 + lane);
                        }
                        if (lane == 0) A.counters[cidx] = 0;
                    }
                }
                if (last) {
                    // lanes 0..15 gate rows, 16..31 up rows of outputs 16*tile + lane
#pragma unroll
                    for (int m = 0; m < RMAX; ++m) {
                        const float up = __shfl_down_sync(0xffffffffu, tot[m], 16);
                        if (m < nrows && lane < 16) {
                            const FfnRow r = A.rows[en.row0 + m];
                            A.h[r.h_off + 16 * tile + lane] = gelu_tanh(tot[m]) * up;
                        }
                    }
                }
            } else {
                float* P = A.partials + (size_t(seg_start) * kMaxRows) * 32;
#pragma unroll
                for (int m = 0; m < RMAX; ++m)
                    if (m < nrows) P[m * 32 + lane] = A.rows[en.row0 + m].w * tot[m];
                __threadfence();
                __syncwarp();
                const int upt = A.wl->units_per_tile_dn;
                int old = 0;
                if (lane == 0) old = atomicAdd(&A.counters[tile], u + 1 - seg_start);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old + (u + 1 - seg_start) == upt) {
                    __threadfence();
                    for (int t = 0; t < T; ++t)
                        yacc[t * 32 + lane] = A.y_in ? A.y_in[size_t(t) * D + 32 * tile + lane] : 0.f;
                    __syncwarp();
                    for (int e2 = 0; e2 < n_entries; ++e2) {
                        const FfnEntry& f = EC.at(e2);
                        const int ks2 = down_ks(f.F), ns2 = f.F / ks2;
                        const int base = f.ubase_dn + tile * ns2;
                        for (int s2 = 0; s2 < ns2; ++s2) {
                            const int us = base + s2;
                            if (s2 != 0 && range_start(cta_of(us, U, G), U, G) != us) continue;  // not a segment start
                            const float* Q = A.partials + (size_t(us) * kMaxRows) * 32;
                            for (int m = 0; m < min(f.n_rows, RMAX); ++m)
                                yacc[A.rows[f.row0 + m].y_row * 32 + lane] += __ldcg(Q + m * 32 + lane);
                        }
                    }
                    __syncwarp();
                    for (int t = 0; t < T; ++t) {
                        const float v = yacc[t * 32 + lane];
                        A.y[size_t(t) * D + 32 * tile + lane] = v;
                        if (A.y_bf16) A.y_bf16[size_t(t) * D + 32 * tile + lane] = f32_to_bf16_rn(v);
                    }
                    if (lane == 0) A.counters[tile] = 0;
                }
            }
        }
        seg_start = u + 1;
    }
}

// ---------------------------------------------------------------------------
// One-token (decode) variant.  Every entry has one row, so each CTA stages its
// inputs once, before its first unit: the token's x (gate/up) or the h rows of
// all entries (down).  Units are entry-major for gate/up (a segment is an
// (entry, 16-output tile)) and tile-major for down (a segment is a 32-row
// output tile across all entries: the CTA sums w_e * dot_e in registers), so a
// segment split across CTAs is reconciled from at most a few per-CTA partials.
// Units map to entries in O(1): shared entries first, then routed ones.
struct DecodeMap {
    int nsh, ush_gu, urt_gu, ns_sh, ns_rt, upt, F, FS, D;
    __device__ __forceinline__ int gu_entry(int u) const {
        const int sh = nsh * ush_gu;
        return u < sh ? u / ush_gu : nsh + (u - sh) / urt_gu;
    }
    __device__ __forceinline__ int gu_base(int e) const {
        return e < nsh ? e * ush_gu : nsh * ush_gu + (e - nsh) * urt_gu;
    }
    // down unit u -> (entry, tile, slice); tiles are 32 output rows
    __device__ __forceinline__ void dn_unit(int u, int& e, int& tile, int& slice) const {
        tile = u / upt;
        const int o = u - tile * upt, sh = nsh * ns_sh;
        if (o < sh) { e = o / ns_sh; slice = o - e * ns_sh; }
        else { const int o2 = o - sh; e = nsh + o2 / ns_rt; slice = o2 - (e - nsh) * ns_rt; }
    }
    __device__ __forceinline__ int width(int e) const { return e < nsh ? FS : F; }
    // first staged 8-input chunk of entry e's h row (down) and of its groups
    __device__ __forceinline__ int stage_chunk0(int e) const {
        return e < nsh ? e * (FS / 8) : nsh * (FS / 8) + (e - nsh) * (F / 8);
    }
};

// One 8-input task of the fixed-point staging (see stage_row).  All 32 lanes
// must call it (shuffles); `ok` marks lanes with a real task.
__device__ __forceinline__ void stage_task(const float (&v)[8], bool ok, int chunk, uint4* xq, float* sx, float* X) {
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
    xq[chunk] = make_uint4(hi_e, lo_e, hi_o, lo_o);
    if ((chunk & 7) == 0) {
        sx[chunk >> 3] = amax / 32767.f;
        X[chunk >> 3] = sum;
    }
}

template <int MODE>
__global__ void __launch_bounds__((DecodeCfg<MODE>::NW + 1) * 32) gemv_decode_kernel(GemvArgs A) {
    constexpr int NW = DecodeCfg<MODE>::NW;
    constexpr int STAGE = DecodeCfg<MODE>::STAGE;
    constexpr int CPS = DecodeCfg<MODE>::CPS;
    constexpr int kStages = DecodeCfg<MODE>::NSTAGES;
    constexpr int NCONS = NW * 32;
    // gate/up: the work list is the previous launch's output, so wait before
    // reading it; the token's hidden state is two or more launches back, so
    // the consumers stage it first.  down: the work list is two launches back
    // (written before the gate/up kernel), so weights stream while gate/up
    // finishes; only the consumers wait, before staging h.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * STAGE);
    uint64_t* empty = full + kStages;
    FfnEntry* s_ent = reinterpret_cast<FfnEntry*>(empty + kStages);     // [kCtaEntries]
    FfnRow* s_row = reinterpret_cast<FfnRow*>(s_ent + kCtaEntries);     // [kCtaEntries]
    float* red = reinterpret_cast<float*>(s_row + kCtaEntries);          // [NW][32]
    const int gs = ((A.vstride / kGroup) + 3) & ~3;
    float* sx = red + NW * 32;                                           // [gs]
    float* Xs = sx + gs;                                                 // [gs]
    uint4* xq = reinterpret_cast<uint4*>(Xs + gs);                       // [vstride / 8]
    __shared__ int s_abort;
    // 16-bit fixed-point image of the inputs, one load round trip per kBatch
    // tasks (8 values each) per thread: MODE 0 the token's x (row 0: these
    // lists carry one token), MODE 1 every entry's h segment
    // task_of maps 0..tasks-1 to the staged task (8 input values) indices;
    // runs of 8 consecutive flat indices must map to one group, in order
    auto stage = [&](int tasks, const DecodeMap& M, auto task_of) {
        constexpr int kBatch = 3;
        for (int base = 0; base < tasks; base += kBatch * NCONS) {
            float v[kBatch][8];
            int tt[kBatch];
#pragma unroll
            for (int r = 0; r < kBatch; ++r) {  // all loads first: one round trip
                const int fi = base + r * NCONS + int(threadIdx.x);
                const int t = fi < tasks ? task_of(fi) : 0;
                tt[r] = t;
                if (fi < tasks) {
                    if (MODE == 0) {
                        const uint4 q = reinterpret_cast<const uint4*>(A.x)[t];
                        const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            v[r][2 * j] = __uint_as_float(w4[j] << 16);
                            v[r][2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
                        }
                    } else {
                        const int shc = M.nsh * (M.FS / 8);
                        const int ee = t < shc ? t / (M.FS / 8) : M.nsh + (t - shc) / (M.F / 8);
                        const float* h = A.h + s_row[ee].h_off + 8 * (t - M.stage_chunk0(ee));
                        const float4 a4 = reinterpret_cast<const float4*>(h)[0];
                        const float4 b4 = reinterpret_cast<const float4*>(h)[1];
                        v[r][0] = a4.x; v[r][1] = a4.y; v[r][2] = a4.z; v[r][3] = a4.w;
                        v[r][4] = b4.x; v[r][5] = b4.y; v[r][6] = b4.z; v[r][7] = b4.w;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[r][j] = 0.f;
                }
            }
#pragma unroll
            for (int r = 0; r < kBatch; ++r) {
                const int fi = base + r * NCONS + int(threadIdx.x);
                stage_task(v[r], fi < tasks, tt[r], xq, sx, Xs);
            }
        }
        named_sync(1, NCONS);
    };
    const int D = A.D;
    const int NSg = D / kGuSlice;
    const int G = gridDim.x, c = blockIdx.x;
    // gate/up CTAs [0, gs): the shared expert's tiles (the list's first entry),
    // known before the wait; the other CTAs wait for the work list
    const bool early = MODE == 0 && c < A.gs;
    if (MODE == 0) {
        if (warp < NW) stage(D / 8, DecodeMap{}, [](int fi) { return fi; });
        if (!early) {
            pdl_wait();
            pdl_trigger();
        }
    }
    WorkList W;
    FfnEntry my_en;
    FfnRow my_row;
    const int n_spec = min(kCtaEntries, A.list_cap);
    if (early) {
        W = WorkList{};
        W.n_entries = 1;
        W.n_shared = 1;
        W.ush_gu = (A.FS / 16) * NSg;
        W.urt_gu = 1;
        W.units_gu = W.ush_gu;
        W.max_rows = 1;
        W.F = 64;
        W.FS = A.FS;
        my_en.blob = A.shared_blob;
        my_en.ready = nullptr;
        my_en.ready_val = 0;
        my_en.F = A.FS;
        my_en.n_rows = 1;
        my_en.row0 = 0;
        my_en.ubase_gu = 0;
        my_en.ubase_dn = 0;
        my_row.x_row = 0;
        my_row.h_off = A.h_shared_off;
        my_row.y_row = 0;
        my_row.w = 1.0f;
    } else {
        // header, entries and rows in one round trip: in a one-token list entry
        // e's row is row e
        W = *A.wl;
        if (int(threadIdx.x) < n_spec) {
            my_en = A.entries[threadIdx.x];
            my_row = A.rows[threadIdx.x];
        }
    }
    const int U = MODE == 0 ? W.units_gu : W.units_dn;
    // unit range: gate/up takes whole output tiles (no cross-CTA reduction),
    // shared-expert tiles on CTAs [0, gs), the rest on [gs, G); down splits
    // its units evenly
    int u_begin, u_end;
    if (MODE == 0) {
        const int t_lo = A.gs > 0 ? (A.FS / 16) : 0;  // first tile of this CTA class
        const int t_hi = early ? t_lo : U / NSg;
        const int c0 = early ? 0 : A.gs, gc = early ? A.gs : G - A.gs;
        const int tb = early ? 0 : t_lo, nt = early ? A.FS / 16 : t_hi - t_lo;
        u_begin = (tb + range_start(c - c0, nt, gc)) * NSg;
        u_end = (tb + range_start(c - c0 + 1, nt, gc)) * NSg;
    } else {
        u_begin = range_start(c, U, G);
        u_end = range_start(c + 1, U, G);
    }
    const DecodeMap M{W.n_shared, W.ush_gu, W.urt_gu, W.ns_sh_dn, W.ns_rt_dn, W.units_per_tile_dn, W.F, W.FS, D};
    const int n_ent = min(W.n_entries, kCtaEntries);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], MODE == 0 ? 4 : NW);  // the warps that read a unit
        }
        mbar_fence_init();
    }
    if (int(threadIdx.x) < n_ent) {
        s_ent[threadIdx.x] = my_en;
        s_row[threadIdx.x] = my_row;
    }
    __syncthreads();
    if (u_begin >= u_end) return;
    if (!early) {
        const int need = MODE == 0 ? D : M.stage_chunk0(W.n_entries) * 8;  // staged input values
        bool bad = W.n_entries > n_spec || W.max_rows > 1 || need > A.vstride;  // not a one-token list
        if (MODE == 0 && A.gs > 0) bad |= W.n_shared != 1 || W.ush_gu != (A.FS / 16) * NSg;
        if (MODE == 0) bad |= (U % NSg) != 0;
        if (bad) {
            if (threadIdx.x == 0) set_status(A.status, MOE_ERR_STATE);
            return;
        }
    }

    if (warp == NW) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            int issued = 0;
            bool ok = true;
            uint32_t landed = 0;  // entries (bit e) whose blob is known to have landed
            for (int u = u_begin, n = 1; u < u_end && ok; u += n, ++issued) {
                const uint8_t* src;
                uint32_t bytes;
                int e;
                if (MODE == 0) {
                    // up to CPS chunks, never past the end of the tile
                    e = M.gu_entry(u);
                    const int ul = u - M.gu_base(e), slice = ul % NSg;
                    n = min(min(CPS - slice % CPS, NSg - slice), u_end - u);
                    src = s_ent[e].blob + size_t(ul) * (18 * kGuSlice);
                    bytes = uint32_t(n) * (18 * kGuSlice);
                } else {
                    int tile, slice;
                    M.dn_unit(u, e, tile, slice);
                    const int F = M.width(e), ks = down_ks(F);
                    src = s_ent[e].blob + gu_section_bytes(D, F) + size_t(tile * (F / ks) + slice) * (18u * ks);
                    bytes = 18u * ks;
                }
                // a miss still being copied in: wait for its ready word first
                // (entries index s_ent, fewer than 32)
                if (!((landed >> e) & 1u)) {
                    if (s_ent[e].ready) ok = ready_wait(s_ent[e].ready, s_ent[e].ready_val, A.status, &s_abort);
                    if (!ok) break;
                    landed |= 1u << e;
                }
                const int st = issued % kStages;
                if (issued >= kStages) ok = ring_wait(&empty[st], ((issued / kStages) - 1) & 1, A.status, &s_abort);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[st], bytes);
                bulk_g2s(ring + size_t(st) * STAGE, src, bytes, &full[st], pol);
            }
            const int first = issued > kStages ? issued - kStages : 0;
            for (int i = first; i < issued; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1, A.status);
        }
        return;
    }

    // ------------------------------------------------ consumers: stage h (down)
    if (MODE == 1) {
        // the input segments this CTA's units read (one slice of one entry's
        // h each), or every entry's h when the range is long
        constexpr int kMaxUnitsStaged = 16;
        __shared__ int s_ub[kMaxUnitsStaged], s_uc[kMaxUnitsStaged + 1];
        const int nu = u_end - u_begin;
        if (threadIdx.x == 0 && nu <= kMaxUnitsStaged) {
            s_uc[0] = 0;
            for (int q = 0; q < nu; ++q) {
                int e, tile, slice;
                M.dn_unit(u_begin + q, e, tile, slice);
                const int ks = down_ks(M.width(e));
                s_ub[q] = M.stage_chunk0(e) + slice * (ks / 8);
                s_uc[q + 1] = s_uc[q] + ks / 8;
            }
        }
        pdl_wait();  // h is the gate/up kernel's output
        pdl_trigger();
        named_sync(1, NCONS);
        if (nu <= kMaxUnitsStaged) {
            stage(s_uc[nu], M, [&](int fi) {
                int q = 0;
                while (fi >= s_uc[q + 1]) ++q;
                return s_ub[q] + (fi - s_uc[q]);
            });
        } else {
            stage(M.stage_chunk0(W.n_entries), M, [](int fi) { return fi; });
        }
    }

    // -------------------------------------------------- consumers: the units
    float acc = 0.f;
    int seg_start = u_begin;
    int q = -1;            // stage sequence number of the current unit
    bool have_q = false;   // whether that stage's copy has landed
    int st_first = 0;      // first slice of the current stage
    for (int u = u_begin; u < u_end; ++u) {
        int e, tile, slice, key_u0, key_len;
        if (MODE == 0) {
            e = M.gu_entry(u);
            const int ul = u - M.gu_base(e);
            tile = ul / NSg;
            slice = ul - tile * NSg;
            key_u0 = M.gu_base(e) + tile * NSg;
            key_len = NSg;
        } else {
            M.dn_unit(u, e, tile, slice);
            key_u0 = tile * M.upt;
            key_len = M.upt;
        }
        const int ks = MODE == 0 ? kGuSlice : down_ks(M.width(e));
        const int g_in0 = MODE == 0 ? slice * (kGuSlice / kGroup) : M.stage_chunk0(e) / 8 + slice * (ks / kGroup);
        const float w = MODE == 0 ? 1.f : s_row[e].w;

        // stages: gate/up, up to CPS chunks of one tile; down, one unit
        const int in_st = MODE == 0 ? slice % CPS : 0;
        const bool stage_start = MODE == 1 || in_st == 0 || u == u_begin;
        const bool stage_end = MODE == 1 || in_st == CPS - 1 || slice == NSg - 1 || u + 1 == u_end;
        if (stage_start) {
            ++q;
            st_first = slice;
            have_q = ring_wait(&full[q % kStages], (q / kStages) & 1, A.status, &s_abort);
        }
        const int st = q % kStages;
        // gate/up: all four warps read every chunk, one group each; down:
        // every warp reads every unit
        const bool mine = true;
        const int gw = MODE == 0 ? (warp & 3) : warp, gstep = MODE == 0 ? 4 : NW;
        const bool have = mine && have_q;
        const uint8_t* chunk = ring + size_t(st) * STAGE + size_t(MODE == 0 ? slice - st_first : 0) * (18 * kGuSlice);
        for (int g = gw; have && g < ks / kGroup; g += gstep) {
            const uint4 qa = lds128(chunk + ((2 * g) * 32 + lane) * 16);
            const uint4 qb = lds128(chunk + ((2 * g + 1) * 32 + lane) * 16);
            const uint32_t sbw = *reinterpret_cast<const uint32_t*>(chunk + 16 * ks + (g * 32 + lane) * 4);
            const float s = f16_to_f32(uint16_t(sbw & 0xFFFF)), b = f16_to_f32(uint16_t(sbw >> 16));
            const int gi = g_in0 + g;  // staged group of the input
            const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
            int shi = 0, shi2 = 0;
            uint32_t slo = 0, slo2 = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t lo = words[j] & 0x0F0F0F0Fu;
                const uint32_t hi = (words[j] >> 4) & 0x0F0F0F0Fu;
                const uint4 xv = xq[gi * 8 + j];
                shi = dp4a_us(lo, xv.x, shi);
                slo = dp4a_uu(lo, xv.y, slo);
                shi2 = dp4a_us(hi, xv.z, shi2);
                slo2 = dp4a_uu(hi, xv.w, slo2);
            }
            const int dot = 256 * (shi + shi2) + int(slo + slo2);
            const float part = fmaf(s, float(dot) * sx[gi], b * Xs[gi]);
            acc = fmaf(w, part, acc);
        }
        __syncwarp();
        if (stage_end && lane == 0) mbar_arrive(&empty[st]);

        const bool seg_end = (u + 1 == u_end) || (u + 1 == key_u0 + key_len);
        if (!seg_end) continue;

        named_sync(1, NCONS);
        red[warp * 32 + lane] = acc;
        named_sync(1, NCONS);
        acc = 0.f;
        if (warp == 0) {
            float tot = 0.f;
            for (int ww = 0; ww < NW; ++ww) tot += red[ww * 32 + lane];
            const bool whole = (seg_start == key_u0) && (u + 1 == key_u0 + key_len);
            bool last = whole;
            const int cidx = MODE == 0 ? key_u0 / NSg : tile;
            if (!whole) {
                const int slot = (seg_start == u_begin) ? 0 : 1;
                A.partials[size_t(2 * c + slot) * 32 + lane] = tot;
                __threadfence();
                __syncwarp();
                int old = 0;
                if (lane == 0) old = atomicAdd(&A.counters[cidx], u + 1 - seg_start);
                old = __shfl_sync(0xffffffffu, old, 0);
                last = (old + (u + 1 - seg_start) == key_len);
                if (last) {
                    __threadfence();
                    // the segment's partials in CTA order (independent loads)
                    tot = 0.f;
                    const int c0 = cta_of(key_u0, U, G), c1 = cta_of(key_u0 + key_len - 1, U, G);
                    for (int cc = c0; cc <= c1; ++cc) {
                        const int rs = range_start(cc, U, G);
                        if (rs >= range_start(cc + 1, U, G)) continue;
                        tot += __ldcg(A.partials + size_t(2 * cc + (rs >= key_u0 ? 0 : 1)) * 32 + lane);
                    }
                    if (lane == 0) A.counters[cidx] = 0;
                }
            }
            if (last) {
                if (MODE == 0) {
                    // lanes 0..15 gate rows, 16..31 up rows of outputs 16*tile + lane
                    const float up = __shfl_down_sync(0xffffffffu, tot, 16);
                    if (lane < 16) A.h[s_row[e].h_off + 16 * tile + lane] = gelu_tanh(tot) * up;
                } else {
                    const int r = 32 * tile + lane;
                    const float yv = (A.y_in ? A.y_in[r] : 0.f) + tot;
                    A.y[r] = yv;
                    if (A.y_bf16) A.y_bf16[r] = f32_to_bf16_rn(yv);
                }
            }
        }
        seg_start = u + 1;
    }
}

// ------------------------------------------------------------ host side
template <int MODE, int RMAX>
static size_t gemv_smem(int vstride, int T) {
    constexpr int NW = GemvCfg<MODE>::NW;
    size_t b = size_t(GemvCfg<MODE>::NSTAGES) * GemvCfg<MODE>::STAGE + 2 * GemvCfg<MODE>::NSTAGES * sizeof(uint64_t);
    b += sizeof(FfnEntry) * kCtaEntries;             // staged work-list entries
    b += size_t(NW) * RMAX * 32 * 4;                 // red
    b += size_t(RMAX) * (((vstride / kGroup) + 3) & ~3) * 4 * 2;  // per-group scale and sum
    b += size_t(RMAX) * vstride * 2;                 // 16-bit fixed-point image of the inputs
    if (MODE == 1) b += size_t(T) * 32 * 4;          // yacc
    return b;
}

// Decode kernel: entries + their rows, red, per-group scale/sum, staged image.
template <int MODE>
static size_t decode_smem(int vstride) {
    constexpr int NW = DecodeCfg<MODE>::NW;
    size_t b = size_t(DecodeCfg<MODE>::NSTAGES) * DecodeCfg<MODE>::STAGE + 2 * DecodeCfg<MODE>::NSTAGES * sizeof(uint64_t);
    b += (sizeof(FfnEntry) + sizeof(FfnRow)) * kCtaEntries;
    b += size_t(NW) * 32 * 4;
    b += size_t(((vstride / kGroup) + 3) & ~3) * 4 * 2;
    b += size_t(vstride) * 2;
    return b;
}

template <typename K>
static cudaError_t shape_of(K kern, int threads, size_t smem, int sms, bool raise_only, GemvShape* out) {
    cudaError_t e;
    if (raise_only) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        if (size_t(fa.maxDynamicSharedSizeBytes) < smem)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    } else {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    }
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    out->grid = sms * per_sm;
    out->smem = smem;
    return cudaSuccess;
}

cudaError_t ffn_prepare(int D, int F, int FS, int K, int T, int sms, GemvShapes* shapes) {
    cudaError_t e;
    const int fmax = F > FS ? F : FS;
    const int vdn = ((fmax + kGroup - 1) / kGroup) * kGroup;
    shapes->vstride_gu = D;
    shapes->vstride_dn = vdn;
    shapes->stage_dn_decode = K * F + FS;
    if ((e = shape_of(gemv_decode_kernel<0>, (DecodeCfg<0>::NW + 1) * 32, decode_smem<0>(D), sms, false,
                      &shapes->gu[0])) != cudaSuccess)
        return e;
    if ((e = shape_of(stream_gemv_kernel<0, kMaxRows>, (GemvCfg<0>::NW + 1) * 32, gemv_smem<0, kMaxRows>(D, T), sms,
                      false, &shapes->gu[1])) != cudaSuccess)
        return e;
    if ((e = shape_of(gemv_decode_kernel<1>, (GemvCfg<1>::NW + 1) * 32, decode_smem<1>(shapes->stage_dn_decode), sms,
                      false, &shapes->dn[0])) != cudaSuccess)
        return e;
    if ((e = shape_of(stream_gemv_kernel<1, kMaxRows>, (GemvCfg<1>::NW + 1) * 32, gemv_smem<1, kMaxRows>(vdn, T), sms,
                      false, &shapes->dn[1])) != cudaSuccess)
        return e;
    return cudaSuccess;
}

cudaError_t ffn_shapes_one_row(int vstride_gu, int stage_dn, int T, int sms, GemvShapes* shapes) {
    (void)T;
    *shapes = GemvShapes{};
    shapes->vstride_gu = vstride_gu;
    shapes->stage_dn_decode = stage_dn;
    cudaError_t e = shape_of(gemv_decode_kernel<0>, (DecodeCfg<0>::NW + 1) * 32, decode_smem<0>(vstride_gu), sms, true,
                             &shapes->gu[0]);
    if (e != cudaSuccess) return e;
    return shape_of(gemv_decode_kernel<1>, (GemvCfg<1>::NW + 1) * 32, decode_smem<1>(stage_dn), sms, true,
                    &shapes->dn[0]);
}

cudaError_t ffn_ensure_one_row_smem(const GemvShapes& shapes) {
    GemvShape tmp;
    const int sms = 1;
    cudaError_t e = shape_of(gemv_decode_kernel<0>, (DecodeCfg<0>::NW + 1) * 32, shapes.gu[0].smem, sms, true, &tmp);
    if (e != cudaSuccess) return e;
    return shape_of(gemv_decode_kernel<1>, (GemvCfg<1>::NW + 1) * 32, shapes.dn[0].smem, sms, true, &tmp);
}

cudaError_t launch_ffn(const GemvLaunch& L, cudaStream_t s, void (*hook)(void*, int), void* hook_arg) {
    GemvArgs a;
    a.wl = L.wl;
    a.entries = L.entries;
    a.rows = L.rows;
    a.x = L.x;
    a.h = L.h;
    a.y_in = L.y_in;
    a.y = L.y;
    a.y_bf16 = L.y_bf16;
    a.D = L.D;
    a.status = L.status;
    a.list_cap = L.list_cap;
    a.shared_blob = L.shared_blob;
    a.FS = L.FS;
    a.h_shared_off = L.h_shared_off;
    a.gs = 0;
    const bool one = L.rmax == 1;
    // K3: gate/up -> h
    a.partials = L.partials_gu;
    a.counters = L.counters_gu;
    a.vstride = L.shapes->vstride_gu;
    const GemvShape& g = L.shapes->gu[one ? 0 : 1];
    int grid_gu = g.grid;
    if (one && L.max_tiles_gu > 0) {
        // whole tiles, kTilesPerCta per CTA: the shared expert's on CTAs
        // [0, gs) (started before the list exists), the rest after them
        constexpr int tpc = DecodeCfg<0>::kTilesPerCta;
        const int sh = L.shared_blob ? L.FS / 16 : 0;
        const int gs = (sh + tpc - 1) / tpc;
        int gr = (L.max_tiles_gu - sh + tpc - 1) / tpc;
        gr = gr < 1 ? 1 : gr;
        grid_gu = gs + gr < g.grid ? gs + gr : g.grid;
        a.gs = gs < grid_gu - 1 ? gs : grid_gu - 1;
    }
    if (hook) hook(hook_arg, 0);
    cudaError_t e;
    if (one)
        e = launch_kernel(gemv_decode_kernel<0>, dim3(grid_gu), dim3((DecodeCfg<0>::NW + 1) * 32), g.smem, s, L.pdl, 1, a);
    else
        e = launch_kernel(stream_gemv_kernel<0, kMaxRows>, dim3(g.grid), dim3((GemvCfg<0>::NW + 1) * 32), g.smem, s,
                          L.pdl, 1, a);
    if (e != cudaSuccess) return e;
    if (hook) hook(hook_arg, 1);
    // K4: down + combine -> y
    a.gs = 0;
    a.partials = L.partials_dn;
    a.counters = L.counters_dn;
    a.vstride = one ? L.shapes->stage_dn_decode : L.shapes->vstride_dn;
    const GemvShape& d = L.shapes->dn[one ? 0 : 1];
    if (one)
        e = launch_kernel(gemv_decode_kernel<1>, dim3(d.grid), dim3((GemvCfg<1>::NW + 1) * 32), d.smem, s, L.pdl, 1, a);
    else
        e = launch_kernel(stream_gemv_kernel<1, kMaxRows>, dim3(d.grid), dim3((GemvCfg<1>::NW + 1) * 32), d.smem, s,
                          L.pdl, 1, a);
    if (hook) hook(hook_arg, 2);
    return e;
}

// ------------------------------------------------------ work-list builder
// One token (GEMV mode): one entry per selection in k order.  Otherwise:
// groups the call's (token, k) pairs by expert slot (ascending slot, pairs in
// ascending index inside a slot), splits each group into entries of at most
// kMaxRows rows (kGemmMaxRows in GEMM mode), puts the shared expert (all
// tokens) first, and computes each entry's first gate/up and down unit.  One
// CTA: counts with shared-memory atomics, prefix sums by block scans, ranks
// by an in-order warp scan over pairs staged in shared memory, entries
// written in parallel.
constexpr int kWlThreads = 256;
constexpr int kWlChunk = 2048;  // pairs staged per round of the ranking scan

// Exclusive scan of v over the CTA (kWlThreads threads); returns the prefix
// of this thread and the total in *total.
__device__ int wl_block_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) warp_tot[warp] = inc;
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < kWlThreads / 32; ++w) {
        if (w < warp) before += warp_tot[w];
        all += warp_tot[w];
    }
    __syncthreads();
    *total = all;
    return before + inc - v;
}

__global__ void __launch_bounds__(kWlThreads) build_worklist_kernel(WorkListArgs a) {
    __shared__ int cnt[1024];
    __shared__ int off[1024];
    __shared__ int ebase[1024];
    __shared__ int run[1024];
    __shared__ int16_t sl_s[kWlChunk];
    __shared__ int warp_tot[kWlThreads / 32];
    __shared__ int s_maxr;
    pdl_wait();
    pdl_trigger();
    if (a.T == 1 && !a.gemm) {
        // one token: one entry per selection, in k order, as the router and
        // plan kernels write it; a slot named twice is streamed twice (each
        // selection carries its own gate weight)
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            int sl = 0;
            float w = 0.f;
            bool take = false;
            if (lane < a.K) {
                take = !a.pair_wave || a.pair_wave[lane] == a.wave;
                sl = a.pair_slot[lane];
                if (sl < 0 || sl >= a.n_slot_range) {
                    if (take) set_status(a.status, MOE_ERR_RANGE);
                    sl = 0;
                }
                w = a.gate_w[lane];
            }
            DecodeWLTarget t;
            t.wl = a.wl;
            t.entries = a.entries;
            t.rows = a.rows;
            t.slot_base = a.slot_base;
            t.slot_stride = a.slot_stride;
            t.shared_blob = a.shared_blob;
            t.F = a.F;
            t.FS = a.FS;
            t.D = a.D;
            t.h_shared_off = a.h_shared_off;
            t.blob_bytes = 0;
            t.ready = nullptr;  // every blob is in place before this list runs
            t.ready_val = 0;
            write_decode_worklist(t, a.K, sl, w, take);
        }
        return;
    }
    const int np = a.T * a.K;
    const int S = a.n_slot_range;
    auto slot_of = [&](int p) -> int {  // -1: not in this wave
        if (a.pair_wave && a.pair_wave[p] != a.wave) return -1;
        const int sl = a.pair_slot[p];
        return (sl < 0 || sl >= S) ? 0 : sl;
    };
    for (int i = threadIdx.x; i < S; i += blockDim.x) { cnt[i] = 0; run[i] = 0; }
    if (threadIdx.x == 0) s_maxr = 0;
    __syncthreads();
    bool bad = false;
    for (int p = threadIdx.x; p < np; p += blockDim.x) {
        if (a.pair_wave && a.pair_wave[p] != a.wave) continue;
        const int sl = a.pair_slot[p];
        if (sl < 0 || sl >= S) bad = true;
        atomicAdd(&cnt[(sl < 0 || sl >= S) ? 0 : sl], 1);
    }
    if (bad) set_status(a.status, MOE_ERR_RANGE);
    __syncthreads();

    const int mr = a.gemm ? kGemmMaxRows : kMaxRows;  // rows per entry
    const int nsh = a.shared_blob ? (a.T + mr - 1) / mr : 0;
    // prefix sums over slots: first row (after the shared rows) and first entry
    // (after the shared entries) of every slot; each thread scans a run of slots
    const int per = (S + kWlThreads - 1) / kWlThreads;
    const int s0 = min(S, int(threadIdx.x) * per), s1 = min(S, s0 + per);
    int rows_mine = 0, ents_mine = 0, maxr_mine = 0;
    for (int sl = s0; sl < s1; ++sl) {
        rows_mine += cnt[sl];
        ents_mine += (cnt[sl] + mr - 1) / mr;
        maxr_mine = max(maxr_mine, min(cnt[sl], mr));
    }
    int rows_tot, ents_tot;
    int ro = wl_block_scan(rows_mine, warp_tot, &rows_tot) + (a.shared_blob ? a.T : 0);
    int eo = wl_block_scan(ents_mine, warp_tot, &ents_tot) + nsh;
    for (int sl = s0; sl < s1; ++sl) {
        off[sl] = ro;
        ebase[sl] = eo;
        ro += cnt[sl];
        eo += (cnt[sl] + mr - 1) / mr;
    }
    if (maxr_mine > 0) atomicMax(&s_maxr, maxr_mine);
    // rows of the shared expert
    for (int t = threadIdx.x; a.shared_blob && t < a.T; t += blockDim.x) {
        FfnRow r;
        r.x_row = t;
        r.h_off = a.h_shared_off + t * a.FS;
        r.y_row = t;
        r.w = 1.0f;
        a.rows[t] = r;
    }
    __syncthreads();

    // routed rows: rank of pair p among the earlier pairs of its slot.  Pairs
    // are staged a chunk at a time; warp 0 walks them 32 at a time in order,
    // lanes holding the same slot rank themselves by lane after the slot's
    // running count.
    for (int base = 0; base < np; base += kWlChunk) {
        const int n = min(kWlChunk, np - base);
        for (int i = threadIdx.x; i < n; i += blockDim.x) sl_s[i] = int16_t(slot_of(base + i));
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            for (int c = 0; c < n; c += 32) {
                const int i = c + lane;
                const int sl = i < n ? int(sl_s[i]) : -1;
                const unsigned same = __match_any_sync(0xffffffffu, sl);
                const int before = __popc(same & ((1u << lane) - 1u));
                const int rank = sl >= 0 ? run[sl] + before : 0;
                __syncwarp();
                if (sl >= 0 && before == 0) run[sl] += __popc(same);  // one lane per slot
                __syncwarp();
                if (sl >= 0) {
                    const int p = base + i;
                    FfnRow r;
                    r.x_row = p / a.K;
                    r.h_off = p * a.F;
                    r.y_row = p / a.K;
                    r.w = a.gate_w[p];
                    a.rows[off[sl] + rank] = r;
                }
            }
        }
        __syncthreads();
    }

    // entries: the shared expert's first, then every slot's in slot order
    const int nsg = a.D / kGuSlice, tiles_dn = a.D / kChunkRows;
    const int ugu_sh = a.gemm ? a.FS / 64 : (a.FS / 16) * nsg;           // units of one shared entry
    const int udn_sh = a.gemm ? a.D / 128 : tiles_dn * (a.FS > 0 ? a.FS / down_ks(a.FS) : 0);
    const int ugu_rt = a.gemm ? a.F / 64 : (a.F / 16) * nsg;             // units of one routed entry
    const int udn_rt = a.gemm ? a.D / 128 : tiles_dn * (a.F / down_ks(a.F));
    for (int j = threadIdx.x; j < nsh; j += blockDim.x) {
        FfnEntry en;
        en.blob = a.shared_blob;
        en.ready = nullptr;
        en.ready_val = 0;
        en.F = a.FS;
        en.row0 = j * mr;
        en.n_rows = min(mr, a.T - j * mr);
        en.ubase_gu = j * ugu_sh;
        en.ubase_dn = j * udn_sh;
        a.entries[j] = en;
    }
    for (int sl = threadIdx.x; sl < S; sl += blockDim.x) {
        for (int j = 0; j * mr < cnt[sl]; ++j) {
            const int e = ebase[sl] + j;
            FfnEntry en;
            en.blob = a.slot_base + size_t(sl) * a.slot_stride;
            en.ready = nullptr;
            en.ready_val = 0;
            en.F = a.F;
            en.row0 = off[sl] + j * mr;
            en.n_rows = min(mr, cnt[sl] - j * mr);
            en.ubase_gu = nsh * ugu_sh + (e - nsh) * ugu_rt;
            en.ubase_dn = nsh * udn_sh + (e - nsh) * udn_rt;
            a.entries[e] = en;
        }
    }
    if (threadIdx.x == 0) {
        const int n_rt = ents_tot;
        WorkList wl;
        wl.n_entries = nsh + n_rt;
        wl.units_gu = nsh * ugu_sh + n_rt * ugu_rt;
        wl.units_dn = nsh * udn_sh + n_rt * udn_rt;
        wl.T = a.T;
        wl.units_per_tile_dn = nsh * (a.FS > 0 ? a.FS / down_ks(a.FS) : 0) + n_rt * (a.F / down_ks(a.F));
        wl.max_rows = max(s_maxr, nsh > 0 ? min(mr, a.T) : 0);
        wl.n_shared = nsh;
        wl.ush_gu = a.FS > 0 ? (a.FS / 16) * nsg : 1;
        wl.urt_gu = (a.F / 16) * nsg;
        wl.ns_sh_dn = a.FS > 0 ? a.FS / down_ks(a.FS) : 1;
        wl.ns_rt_dn = a.F / down_ks(a.F);
        wl.F = a.F;
        wl.FS = a.FS;
        *a.wl = wl;
    }
}

cudaError_t launch_build_worklist(const WorkListArgs& a, bool pdl, cudaStream_t s) {
    return launch_kernel(build_worklist_kernel, dim3(1), dim3(kWlThreads), 0, s, pdl, 1, a);
}

}  // namespace moe
