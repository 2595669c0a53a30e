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
#include "ffn.cuh"

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
    int vstride;            // floats per staged input row (D for gate/up, max F for down)
    int* status;
};

__device__ __forceinline__ int range_start(int c, int U, int G) { return int((long long)c * U / G); }
// The CTA whose range holds unit u (the last CTA whose start is <= u).
__device__ __forceinline__ int cta_of(int u, int U, int G) { return int(((long long)(u + 1) * G + U - 1) / U) - 1; }

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// Bounded wait that gives up at once after any warp of the CTA timed out, so
// a failure costs one time-out, not one per stage.
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity, status)) return true;
    *abort_flag = 1;
    return false;
}

// Entry of global unit u (entries sorted by unit base; small linear scan from a hint).
template <int MODE>
__device__ __forceinline__ int find_entry(const FfnEntry* __restrict__ E, int n, int u, int hint) {
    int e = hint;
    while (e + 1 < n && (MODE == 0 ? E[e + 1].ubase_gu : E[e + 1].ubase_dn) <= u) ++e;
    return e;
}

// One group of 64 inputs for one lane (= one row): 8 words of nibbles from
// the two word-quads qa, qb; accumulates A into a[m] for every token row m.
template <int RMAX>
__device__ __forceinline__ void group_dot(const uint4& qa, const uint4& qb, const float* __restrict__ vin, int vstride,
                                          int k0, int nrows, float (&a0)[RMAX], float (&a1)[RMAX]) {
    const uint32_t words[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t lo = words[j] & 0x0F0F0F0Fu;
        const uint32_t hi = (words[j] >> 4) & 0x0F0F0F0Fu;
        // byte b of lo/hi -> 0.5 + q/256 (nibble in mantissa bits 16..19 of 0.5)
        const float f0 = __uint_as_float(__byte_perm(lo, 0x3F000000u, 0x7044));
        const float f1 = __uint_as_float(__byte_perm(hi, 0x3F000000u, 0x7044));
        const float f2 = __uint_as_float(__byte_perm(lo, 0x3F000000u, 0x7144));
        const float f3 = __uint_as_float(__byte_perm(hi, 0x3F000000u, 0x7144));
        const float f4 = __uint_as_float(__byte_perm(lo, 0x3F000000u, 0x7244));
        const float f5 = __uint_as_float(__byte_perm(hi, 0x3F000000u, 0x7244));
        const float f6 = __uint_as_float(__byte_perm(lo, 0x3F000000u, 0x7344));
        const float f7 = __uint_as_float(__byte_perm(hi, 0x3F000000u, 0x7344));
#pragma unroll
        for (int m = 0; m < RMAX; ++m) {
            if (m < nrows) {
                const float4 xa = *reinterpret_cast<const float4*>(vin + m * vstride + k0 + 8 * j);
                const float4 xb = *reinterpret_cast<const float4*>(vin + m * vstride + k0 + 8 * j + 4);
                a0[m] = fmaf(f0, xa.x, a0[m]);
                a1[m] = fmaf(f1, xa.y, a1[m]);
                a0[m] = fmaf(f2, xa.z, a0[m]);
                a1[m] = fmaf(f3, xa.w, a1[m]);
                a0[m] = fmaf(f4, xb.x, a0[m]);
                a1[m] = fmaf(f5, xb.y, a1[m]);
                a0[m] = fmaf(f6, xb.z, a0[m]);
                a1[m] = fmaf(f7, xb.w, a1[m]);
            }
        }
    }
}

template <int MODE, int RMAX>
__global__ void __launch_bounds__((GemvCfg<MODE>::NW + 1) * 32) stream_gemv_kernel(GemvArgs A) {
    constexpr int NW = GemvCfg<MODE>::NW;
    constexpr int STAGE = GemvCfg<MODE>::STAGE;
    constexpr int kStages = GemvCfg<MODE>::NSTAGES;
    constexpr int NCONS = NW * 32;
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
    float* red = reinterpret_cast<float*>(empty + kStages);      // [NW][RMAX][32]
    const int vstride = A.vstride;                                // max input width per row
    const int xs_stride = ((vstride / kGroup) + 3) & ~3;          // keeps vin 16-byte aligned
    float* xsum = red + NW * RMAX * 32;                           // [RMAX][xs_stride]
    float* vin = xsum + RMAX * xs_stride;                         // [RMAX][vstride]
    float* yacc = vin + RMAX * vstride;                           // [T][32] (MODE 1 finalize)
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NW);
        }
        mbar_fence_init();
    }
    __syncthreads();
    if (u_begin >= u_end) return;

    if (warp == NW) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            int e = find_entry<MODE>(A.entries, n_entries, u_begin, 0);
            int issued = 0;
            bool ok = true;
            for (int u = u_begin; u < u_end && ok; ++u, ++issued) {
                e = find_entry<MODE>(A.entries, n_entries, u, e);
                const FfnEntry& en = A.entries[e];
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
    int e = -1, nrows = 0, ns = 1, ks = kGuSlice;
    int seg_start = u_begin;
    for (int u = u_begin; u < u_end; ++u) {
        const int i = u - u_begin;
        const int st = i % kStages;
        const int ne = find_entry<MODE>(A.entries, n_entries, u, e < 0 ? 0 : e);
        if (ne != e) {
            // new entry: stage its input rows (fp32) and their group sums
            e = ne;
            const FfnEntry& en = A.entries[e];
            nrows = en.n_rows;
            if (nrows > RMAX) {  // more rows than this variant stages: keep in bounds, report
                if (threadIdx.x == 0) set_status(A.status, MOE_ERR_RANGE);
                nrows = RMAX;
            }
            ks = MODE == 0 ? kGuSlice : down_ks(en.F);
            ns = MODE == 0 ? D / kGuSlice : en.F / ks;
            const int kin = MODE == 0 ? D : en.F;
            named_sync(1, NCONS);
            for (int m = 0; m < nrows; ++m) {
                const FfnRow r = A.rows[en.row0 + m];
                if (MODE == 0) {
                    const uint4* src = reinterpret_cast<const uint4*>(A.x + size_t(r.x_row) * D);
                    for (int v = threadIdx.x; v < kin / 8; v += NCONS) {
                        const uint4 q = src[v];
                        const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            vin[m * vstride + 8 * v + 2 * j] = __uint_as_float(w4[j] << 16);
                            vin[m * vstride + 8 * v + 2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
                        }
                    }
                } else {
                    const float4* src = reinterpret_cast<const float4*>(A.h + r.h_off);
                    for (int v = threadIdx.x; v < kin / 4; v += NCONS)
                        *reinterpret_cast<float4*>(vin + m * vstride + 4 * v) = src[v];
                }
            }
            named_sync(1, NCONS);
            for (int gi = threadIdx.x; gi < nrows * (kin / kGroup); gi += NCONS) {
                const int m = gi / (kin / kGroup), g = gi % (kin / kGroup);
                const float* p = vin + m * vstride + g * kGroup;
                float s = 0.f;
#pragma unroll 8
                for (int k = 0; k < kGroup; ++k) s += p[k];
                xsum[m * xs_stride + g] = s;
            }
            named_sync(1, NCONS);
        }
        const FfnEntry& en = A.entries[e];
        const int ul = u - (MODE == 0 ? en.ubase_gu : en.ubase_dn);
        const int tile = ul / ns, slice = ul % ns;

        // on a time-out the warp skips the compute but keeps every barrier, so
        // no other warp waits on it; the status word carries the error
        const bool have = ring_wait(&full[st], (i / kStages) & 1, A.status, &s_abort);
        const uint8_t* chunk = ring + size_t(st) * STAGE;
        for (int g = warp; have && g < ks / kGroup; g += NW) {
            const uint4 qa = lds128(chunk + ((2 * g) * 32 + lane) * 16);
            const uint4 qb = lds128(chunk + ((2 * g + 1) * 32 + lane) * 16);
            const uint32_t sbw = *reinterpret_cast<const uint32_t*>(chunk + 16 * ks + (g * 32 + lane) * 4);
            const float s = f16_to_f32(uint16_t(sbw & 0xFFFF)), b = f16_to_f32(uint16_t(sbw >> 16));
            const int k0 = slice * ks + g * kGroup;
            float a0[RMAX], a1[RMAX];
#pragma unroll
            for (int m = 0; m < RMAX; ++m) { a0[m] = 0.f; a1[m] = 0.f; }
            group_dot<RMAX>(qa, qb, vin, vstride, k0, nrows, a0, a1);
#pragma unroll
            for (int m = 0; m < RMAX; ++m) {
                if (m < nrows) {
                    const float X = xsum[m * xs_stride + k0 / kGroup];
                    const float t = fmaf(256.f, a0[m] + a1[m], -128.f * X);
                    acc[m] = fmaf(s, t, fmaf(b, X, acc[m]));
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);

        // segment end: next unit is another (entry, tile), or the range ends
        bool seg_end = (u + 1 == u_end);
        if (!seg_end) {
            const int e2 = find_entry<MODE>(A.entries, n_entries, u + 1, e);
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
            float tot[RMAX];
#pragma unroll
            for (int m = 0; m < RMAX; ++m) {
                tot[m] = 0.f;
                for (int w = 0; w < NW; ++w) tot[m] += red[(w * RMAX + m) * 32 + lane];
            }
            const int tile_u0 = (MODE == 0 ? en.ubase_gu : en.ubase_dn) + tile * ns;  // first unit of (entry, tile)
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
                        const FfnEntry& f = A.entries[e2];
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

// ------------------------------------------------------------ host side
template <int MODE, int RMAX>
static size_t gemv_smem(int vstride, int T) {
    constexpr int NW = GemvCfg<MODE>::NW;
    size_t b = size_t(GemvCfg<MODE>::NSTAGES) * GemvCfg<MODE>::STAGE + 2 * GemvCfg<MODE>::NSTAGES * sizeof(uint64_t);
    b += size_t(NW) * RMAX * 32 * 4;                 // red
    b += size_t(RMAX) * (((vstride / kGroup) + 3) & ~3) * 4;  // xsum
    b += size_t(RMAX) * vstride * 4;                 // vin
    if (MODE == 1) b += size_t(T) * 32 * 4;          // yacc
    return b;
}

template <int MODE, int RMAX>
static cudaError_t prepare_one(int vstride, int T, int sms, GemvShape* out) {
    const size_t smem = gemv_smem<MODE, RMAX>(vstride, T);
    auto kern = stream_gemv_kernel<MODE, RMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, (GemvCfg<MODE>::NW + 1) * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    out->grid = sms * per_sm;
    out->smem = smem;
    return cudaSuccess;
}

cudaError_t ffn_prepare(int D, int Fmax, int T, int sms, GemvShapes* shapes) {
    cudaError_t e;
    const int vdn = ((Fmax + kGroup - 1) / kGroup) * kGroup;
    shapes->vstride_gu = D;
    shapes->vstride_dn = vdn;
    if ((e = prepare_one<0, 1>(D, T, sms, &shapes->gu[0])) != cudaSuccess) return e;
    if ((e = prepare_one<0, kMaxRows>(D, T, sms, &shapes->gu[1])) != cudaSuccess) return e;
    if ((e = prepare_one<1, 1>(vdn, T, sms, &shapes->dn[0])) != cudaSuccess) return e;
    if ((e = prepare_one<1, kMaxRows>(vdn, T, sms, &shapes->dn[1])) != cudaSuccess) return e;
    return cudaSuccess;
}

template <int MODE>
static cudaError_t raise_smem(size_t smem) {
    auto kern = stream_gemv_kernel<MODE, 1>;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (size_t(fa.maxDynamicSharedSizeBytes) >= smem) return cudaSuccess;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
}

template <int MODE>
static cudaError_t one_row_shape(int vstride, int T, int sms, GemvShape* out) {
    const size_t smem = gemv_smem<MODE, 1>(vstride, T);
    cudaError_t e = raise_smem<MODE>(smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, stream_gemv_kernel<MODE, 1>,
                                                      (GemvCfg<MODE>::NW + 1) * 32, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    out->grid = sms * per_sm;
    out->smem = smem;
    return cudaSuccess;
}

cudaError_t ffn_shapes_one_row(int vstride_gu, int vstride_dn, int T, int sms, GemvShapes* shapes) {
    *shapes = GemvShapes{};
    shapes->vstride_gu = vstride_gu;
    shapes->vstride_dn = vstride_dn;
    cudaError_t e = one_row_shape<0>(vstride_gu, T, sms, &shapes->gu[0]);
    if (e != cudaSuccess) return e;
    return one_row_shape<1>(vstride_dn, T, sms, &shapes->dn[0]);
}

cudaError_t ffn_ensure_one_row_smem(const GemvShapes& shapes) {
    cudaError_t e = raise_smem<0>(shapes.gu[0].smem);
    if (e != cudaSuccess) return e;
    return raise_smem<1>(shapes.dn[0].smem);
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
    const int r = L.rmax == 1 ? 0 : 1;
    // K3: gate/up -> h
    a.partials = L.partials_gu;
    a.counters = L.counters_gu;
    a.vstride = L.shapes->vstride_gu;
    const GemvShape& g = L.shapes->gu[r];
    if (hook) hook(hook_arg, 0);
    if (r == 0)
        stream_gemv_kernel<0, 1><<<g.grid, (GemvCfg<0>::NW + 1) * 32, g.smem, s>>>(a);
    else
        stream_gemv_kernel<0, kMaxRows><<<g.grid, (GemvCfg<0>::NW + 1) * 32, g.smem, s>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (hook) hook(hook_arg, 1);
    // K4: down + combine -> y
    a.partials = L.partials_dn;
    a.counters = L.counters_dn;
    a.vstride = L.shapes->vstride_dn;
    const GemvShape& d = L.shapes->dn[r];
    if (r == 0)
        stream_gemv_kernel<1, 1><<<d.grid, (GemvCfg<1>::NW + 1) * 32, d.smem, s>>>(a);
    else
        stream_gemv_kernel<1, kMaxRows><<<d.grid, (GemvCfg<1>::NW + 1) * 32, d.smem, s>>>(a);
    e = cudaGetLastError();
    if (hook) hook(hook_arg, 2);
    return e;
}

// ------------------------------------------------------ work-list builder
// Groups the call's (token, k) pairs by expert slot (ascending slot, pairs in
// ascending index inside a slot), splits each group into entries of at most
// kMaxRows rows, puts the shared expert (all tokens) first, and computes each
// entry's first gate/up and down unit.
__global__ void __launch_bounds__(256) build_worklist_kernel(WorkListArgs a) {
    __shared__ int cnt[1024];
    __shared__ int off[1025];
    __shared__ int ent_base[1025];
    const int np = a.T * a.K;
    for (int i = threadIdx.x; i < a.n_slot_range; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    bool bad = false;
    for (int p = threadIdx.x; p < np; p += blockDim.x) {
        if (a.pair_wave && a.pair_wave[p] != a.wave) continue;
        int sl = a.pair_slot[p];
        if (sl < 0 || sl >= a.n_slot_range) { bad = true; sl = 0; }
        atomicAdd(&cnt[sl], 1);
    }
    if (bad) set_status(a.status, MOE_ERR_RANGE);
    __syncthreads();
    const int nsh = a.shared_blob ? (a.T + kMaxRows - 1) / kMaxRows : 0;
    if (threadIdx.x == 0) {
        int o = a.shared_blob ? a.T : 0, eb = nsh;
        for (int sl = 0; sl < a.n_slot_range; ++sl) {
            off[sl] = o;
            ent_base[sl] = eb;
            o += cnt[sl];
            eb += (cnt[sl] + kMaxRows - 1) / kMaxRows;
        }
        off[a.n_slot_range] = o;
        ent_base[a.n_slot_range] = eb;
    }
    __syncthreads();
    const int n_ent = ent_base[a.n_slot_range];
    // rows of the shared expert
    for (int t = threadIdx.x; a.shared_blob && t < a.T; t += blockDim.x) {
        FfnRow r;
        r.x_row = t;
        r.h_off = a.h_shared_off + t * a.FS;
        r.y_row = t;
        r.w = 1.0f;
        a.rows[t] = r;
    }
    // routed rows: rank of pair p among the earlier pairs of its slot
    for (int p = threadIdx.x; p < np; p += blockDim.x) {
        if (a.pair_wave && a.pair_wave[p] != a.wave) continue;
        int sl = a.pair_slot[p];
        if (sl < 0 || sl >= a.n_slot_range) sl = 0;
        int rank = 0;
        for (int q = 0; q < p; ++q) {
            if (a.pair_wave && a.pair_wave[q] != a.wave) continue;
            int s2 = a.pair_slot[q];
            if (s2 < 0 || s2 >= a.n_slot_range) s2 = 0;
            rank += (s2 == sl);
        }
        FfnRow r;
        r.x_row = p / a.K;
        r.h_off = p * a.F;
        r.y_row = p / a.K;
        r.w = a.gate_w[p];
        a.rows[off[sl] + rank] = r;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int nsg = a.D / kGuSlice, tiles_dn = a.D / kChunkRows;
        int ugu = 0, udn = 0, maxr = 0, upt = 0;
        int e = 0;
        for (int j = 0; j < nsh; ++j, ++e) {
            FfnEntry en;
            en.blob = a.shared_blob;
            en.F = a.FS;
            en.row0 = j * kMaxRows;
            en.n_rows = min(kMaxRows, a.T - j * kMaxRows);
            en.ubase_gu = ugu;
            en.ubase_dn = udn;
            ugu += (a.FS / 16) * nsg;
            udn += tiles_dn * (a.FS / down_ks(a.FS));
            upt += a.FS / down_ks(a.FS);
            maxr = max(maxr, en.n_rows);
            a.entries[e] = en;
        }
        for (int sl = 0; sl < a.n_slot_range; ++sl) {
            for (int j = 0; j * kMaxRows < cnt[sl]; ++j, ++e) {
                FfnEntry en;
                en.blob = a.slot_base + size_t(sl) * a.slot_stride;
                en.F = a.F;
                en.row0 = off[sl] + j * kMaxRows;
                en.n_rows = min(kMaxRows, cnt[sl] - j * kMaxRows);
                en.ubase_gu = ugu;
                en.ubase_dn = udn;
                ugu += (a.F / 16) * nsg;
                udn += tiles_dn * (a.F / down_ks(a.F));
                upt += a.F / down_ks(a.F);
                maxr = max(maxr, en.n_rows);
                a.entries[e] = en;
            }
        }
        WorkList wl;
        wl.n_entries = n_ent;
        wl.units_gu = ugu;
        wl.units_dn = udn;
        wl.T = a.T;
        wl.units_per_tile_dn = upt;
        wl.max_rows = maxr;
        *a.wl = wl;
    }
}

cudaError_t launch_build_worklist(const WorkListArgs& a, cudaStream_t s) {
    build_worklist_kernel<<<1, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
