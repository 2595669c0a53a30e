// api.cu -- the C ABI of libmoe.so (declared and documented in moe.h): the
// context, argument checking, and the host orchestration of the layer:
// router -> cache plan -> (miss copies on the side stream || shared expert)
// -> routed experts -> combine.
//
// Host I/O design ("TurboFieldfare: motor open source ...", section "Proceso
// de generacion de tokens": the CPU turns the router's ids into a fetch plan
// against the layer's cache, issues the reads of missing experts, and the GPU
// runs the resident shared-expert branch while they are in flight).  Here the
// plan itself is computed on the GPU; the host learns it through a pinned
// mapped mailbox (one poll per layer, bounded), issues one cudaMemcpyAsync per
// missed expert blob from pinned host memory on a side stream, and makes the
// compute stream wait on an event.  The shared expert's kernels are already
// queued before the host polls, so they overlap the copies.
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "common.cuh"
#include "ffn.cuh"
#include "filestore.cuh"
#include "layer.cuh"
#include "plan.cuh"
#include <cstdlib>

namespace moe {
cudaError_t launch_router(const uint16_t* x, const int8_t* wq, const uint16_t* ws, const float* bias, int E, int D,
                          int K, int T, int32_t* ids, float* gate_w, int* status, const DecodeWLTarget& wlt,
                          bool pdl, cudaStream_t s);
size_t router_smem_bytes(int E, int D);
cudaError_t launch_residual_rmsnorm(float* r, const float* y, uint16_t* x_next, int T, int D, bool pdl,
                                    cudaStream_t s);
cudaError_t launch_bf16_to_f32(const uint16_t* x, float* out, size_t n, bool pdl, cudaStream_t s);
}  // namespace moe

using namespace moe;

// cuStreamWriteValue32 (driver API), resolved at run time through the runtime's
// entry-point query so the library links against the runtime only.
typedef int (*StreamWriteValue32)(cudaStream_t stream, unsigned long long addr, unsigned int value,
                                  unsigned int flags);

// Calls of at least this many tokens run the experts as the tcgen05 grouped
// GEMM (tokens grouped per expert); one token runs the streamed GEMV kernels.
// Measured on B200 with the 26B-A4B layer, 30 layers resident: 2 tokens 567
// vs 388 tokens/s, 4 tokens 956 vs 481, 8 tokens 1511 vs 486 (GEMM vs GEMV).
#ifndef MOE_GEMM_MIN_TOKENS
#define MOE_GEMM_MIN_TOKENS 2
#endif

struct moe_ctx {
    moe_dims d;
    int device = 0;
    int sms = 0;
    cudaStream_t side = nullptr;
    cudaEvent_t ev_plan = nullptr, ev_fill = nullptr, ev_wave = nullptr;
    // per-miss completion (optional): after each one-token miss copy the side
    // stream writes the call's sequence number into ready[slot] (a stream
    // memory write, executed by the stream itself, not by a kernel); the
    // routed experts' kernel then waits for it per expert instead of for all
    // copies
    uint32_t* ready = nullptr;                // [n_slots] (device)
    StreamWriteValue32 write_value = nullptr;  // driver entry point, or null: event join
    bool per_miss = false;                    // MOE_PER_MISS=1 (measured slower on B200: off by default)
    bool inject_skip_ready = false;           // MOE_INJECT_SKIP_READY=1: omit the first write of a call
    PlanMailbox* mbox_host = nullptr;
    PlanMailbox* mbox_dev = nullptr;
    uint32_t seq = 0;
    int* status = nullptr;  // device status word
    bool pdl = true;  // programmatic dependent launch between this context's kernels
    // scratch (device); the second work list holds the routed phase of a
    // streamed one-token layer while the first holds its shared phase
    WorkList* wl = nullptr;
    FfnEntry* entries = nullptr;
    FfnRow* rows = nullptr;
    WorkList* wl2 = nullptr;
    FfnEntry* entries2 = nullptr;
    FfnRow* rows2 = nullptr;
    float* h = nullptr;
    int h_shared_off = 0;
    int list_cap = 0;  // entries and rows each work-list buffer holds
    float* partials_gu = nullptr;
    int* counters_gu = nullptr;
    float* partials_dn = nullptr;
    int* counters_dn = nullptr;
    int32_t* ids = nullptr;
    float* gate_w = nullptr;
    int32_t* pair_slot = nullptr;
    int32_t* pair_wave = nullptr;
    uint16_t* x16 = nullptr;  // [max_tokens][D] fp16 copy of a multi-token call's hidden states (GEMM operand)
    GemvShapes shapes{};
    uint64_t launches = 0;
    size_t blob_routed = 0;
    size_t blob_shared = 0;
    FileReader reader;  // file-backed stores: staging buffers and reader threads
    // look-ahead prefetch (moe_prefetch_configure / moe_layer_forward_next)
    int pf_n = 0;                          // HBM blob buffers
    uint8_t* pf_buf = nullptr;             // [pf_n][pf_stride]
    size_t pf_stride = 0;
    int32_t* pf_ids_host = nullptr;        // pinned mapped: the next layer's predicted ids
    int32_t* pf_ids_dev = nullptr;
    float* pf_gw = nullptr;                // device scratch: their gate weights
    cudaStream_t pf_stream = nullptr;
    cudaEvent_t ev_x = nullptr, ev_pred = nullptr;
    // side stream: after the last staging copies; look-ahead stream: after
    // the last moves of staged blobs into their slots
    cudaEvent_t ev_staged = nullptr, ev_moved = nullptr;
    struct Prefetched {
        const int32_t* state;  // the cache the blob was fetched for
        const uint8_t* store;  // and the store it was copied from
        int expert, buf;
    };
    std::vector<Prefetched> pf_table;      // blobs now held by the buffers
    uint64_t pf_issued = 0, pf_used = 0;   // bytes
    // host mirror of each cache's residency (slot of expert e, -1: absent),
    // kept from the plans the host reads; decides what is worth prefetching
    std::unordered_map<const int32_t*, std::vector<int16_t>> mirror;
    // one-token layer kernel (layer.cu): grid, support for the dims, scratch
    int layer_G = 0;
    bool layer_ok = false;
    bool layer_on = true;         // MOE_LAYER_KERNEL=0: never (direct sources then copy)
    bool layer_resident = false;  // MOE_LAYER_KERNEL=1: resident one-token layers too
    bool layer_pdl = true;
    int layer_hvals = 0;
    float* layer_logits = nullptr;
    float* layer_partials = nullptr;  // [6 * G][32]: gate/up (two pools) then down
    unsigned* layer_bar = nullptr;    // [128]
    uint64_t* stats = nullptr;        // [MOE_STATS] device counters
    std::unordered_map<const void*, const uint8_t*> direct_store;  // host store -> device-accessible address
    // instrumentation (moe_ctx_profile)
    struct Rec {
        int kind;
        cudaEvent_t a, b;
    };
    bool prof = false;
    std::vector<cudaEvent_t> pool;
    std::vector<Rec> recs;
    cudaEvent_t open[MOE_PROF_KINDS] = {};
};

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

bool dims_ok(const moe_dims* d) {
    if (!d) return false;
    auto ff_ok = [](int F) { return F > 0 && F % 64 == 0 && (F <= 704 || F % 704 == 0); };
    if (d->d_model <= 0 || d->d_model % 256 || d->d_model > 8192) return false;  // batched GEMV stages 8 input rows in shared memory
    if (d->group != 64) return false;
    if (d->n_experts <= 0 || d->n_experts > 1024 || d->n_experts % 16) return false;  // 16 router CTAs
    if (d->top_k <= 0 || d->top_k > 16 || d->top_k > d->n_experts) return false;
    if (!ff_ok(d->d_ff) || d->d_ff > 3 * 704) return false;
    if (d->d_ff_shared != 0 && (!ff_ok(d->d_ff_shared) || d->d_ff_shared > 3 * 704)) return false;
    if (d->n_slots < d->top_k || d->n_slots > d->n_experts) return false;
    if (d->max_tokens < 1 || d->max_tokens > 1024) return false;
    if (router_smem_bytes(d->n_experts, d->d_model) > (200u << 10)) return false;
    return true;
}

template <typename T>
cudaError_t dalloc(T** p, size_t n) {
    return cudaMalloc(reinterpret_cast<void**>(p), n * sizeof(T) + 16);
}

void free_ctx(moe_ctx* c) {
    if (!c) return;
    if (c->pf_stream) cudaStreamSynchronize(c->pf_stream);
    if (c->side) cudaStreamSynchronize(c->side);
    cudaFree(c->pf_buf);
    cudaFree(c->pf_gw);
    if (c->pf_ids_host) cudaFreeHost(c->pf_ids_host);
    if (c->ev_x) cudaEventDestroy(c->ev_x);
    if (c->ev_pred) cudaEventDestroy(c->ev_pred);
    if (c->ev_staged) cudaEventDestroy(c->ev_staged);
    if (c->ev_moved) cudaEventDestroy(c->ev_moved);
    if (c->pf_stream) cudaStreamDestroy(c->pf_stream);
    for (auto& r : c->recs) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    for (auto e : c->pool) cudaEventDestroy(e);
    cudaFree(c->status);
    cudaFree(c->ready);
    cudaFree(c->layer_logits);
    cudaFree(c->layer_partials);
    cudaFree(c->layer_bar);
    cudaFree(c->stats);
    cudaFree(c->wl);
    cudaFree(c->entries);
    cudaFree(c->rows);
    cudaFree(c->wl2);
    cudaFree(c->entries2);
    cudaFree(c->rows2);
    cudaFree(c->h);
    cudaFree(c->partials_gu);
    cudaFree(c->counters_gu);
    cudaFree(c->partials_dn);
    cudaFree(c->counters_dn);
    cudaFree(c->ids);
    cudaFree(c->gate_w);
    cudaFree(c->pair_slot);
    cudaFree(c->pair_wave);
    cudaFree(c->x16);
    if (c->mbox_host) cudaFreeHost(c->mbox_host);
    if (c->ev_plan) cudaEventDestroy(c->ev_plan);
    if (c->ev_fill) cudaEventDestroy(c->ev_fill);
    if (c->ev_wave) cudaEventDestroy(c->ev_wave);
    if (c->side) cudaStreamDestroy(c->side);
    delete c;
}

// Records an instrumentation event on `s` opening (begin) or closing an
// interval of `kind`; no-op unless profiling is enabled.
void prof_mark(moe_ctx* c, int kind, bool begin, cudaStream_t s) {
    if (!c->prof) return;
    cudaEvent_t ev = nullptr;
    if (!c->pool.empty()) {
        ev = c->pool.back();
        c->pool.pop_back();
    } else if (cudaEventCreate(&ev) != cudaSuccess) {
        c->prof = false;
        return;
    }
    cudaEventRecord(ev, s);
    if (begin) {
        if (c->open[kind]) c->pool.push_back(c->open[kind]);
        c->open[kind] = ev;
    } else if (c->open[kind]) {
        c->recs.push_back({kind, c->open[kind], ev});
        c->open[kind] = nullptr;
    } else {
        c->pool.push_back(ev);
    }
}

struct FfnHookArg {
    moe_ctx* c;
    cudaStream_t s;
};
void ffn_hook(void* p, int where) {
    auto* h = static_cast<FfnHookArg*>(p);
    if (where == 0) prof_mark(h->c, MOE_PROF_GATE_UP, true, h->s);
    if (where == 1) {
        prof_mark(h->c, MOE_PROF_GATE_UP, false, h->s);
        prof_mark(h->c, MOE_PROF_DOWN, true, h->s);
    }
    if (where == 2) prof_mark(h->c, MOE_PROF_DOWN, false, h->s);
}

int max_entries(const moe_dims& d) {
    const int pairs = d.max_tokens * d.top_k;
    return (d.max_tokens + kMaxRows - 1) / kMaxRows + (pairs < 1024 ? pairs : 1024) + (pairs + kMaxRows - 1) / kMaxRows;
}

// K3 (gate/up) and K4 (down + combine) over a work list already on the device.
// shared_blob: the list's first entry is this shared expert and the gate/up
// kernel may start it before the list exists (one-token lists only), or null.
// n_routed_max: most routed entries the list can hold (-1: top_k).
int run_ffn_list(moe_ctx* c, WorkList* wl, FfnEntry* entries, FfnRow* rows, const uint16_t* x, int T,
                 const float* y_in, float* y, uint16_t* y_bf16, cudaStream_t s,
                 const uint8_t* shared_blob = nullptr, int n_routed_max = -1) {
    cudaError_t e;
    GemvLaunch L;
    L.wl = wl;
    L.entries = entries;
    L.rows = rows;
    L.x = x;
    L.h = c->h;
    L.y_in = y_in;
    L.y = y;
    L.y_bf16 = y_bf16;
    L.partials_gu = c->partials_gu;
    L.counters_gu = c->counters_gu;
    L.partials_dn = c->partials_dn;
    L.counters_dn = c->counters_dn;
    L.D = c->d.d_model;
    L.rmax = (T == 1) ? 1 : kMaxRows;
    L.shapes = &c->shapes;
    L.status = c->status;
    L.pdl = c->pdl;
    L.list_cap = c->list_cap;
    if (T == 1)
        L.max_tiles_gu = (shared_blob ? c->d.d_ff_shared / 16 : 0) +
                         (n_routed_max >= 0 ? n_routed_max : c->d.top_k) * (c->d.d_ff / 16);
    if (T == 1 && shared_blob) {
        L.shared_blob = shared_blob;
        L.FS = c->d.d_ff_shared;
        L.h_shared_off = c->h_shared_off;
    }
    FfnHookArg ha{c, s};
    e = launch_ffn(L, s, c->prof ? ffn_hook : nullptr, &ha);
    c->launches += 2;
    return cuda_status(e);
}

// Builds the work list on the device, then K3 and K4.
int run_ffn(moe_ctx* c, const WorkListArgs& wa, const uint16_t* x, int T, const float* y_in, float* y,
            uint16_t* y_bf16, cudaStream_t s) {
    prof_mark(c, MOE_PROF_WORKLIST, true, s);
    cudaError_t e = launch_build_worklist(wa, c->pdl, s);
    prof_mark(c, MOE_PROF_WORKLIST, false, s);
    c->launches += 1;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return run_ffn_list(c, c->wl, c->entries, c->rows, x, T, y_in, y, y_bf16, s);
}

// Batches and prefill chunks: builds a GEMM-mode work list (entries of up to
// kGemmMaxRows rows) and runs the tensor-core grouped GEMM; adds into y, which
// the caller zeroed before the first call of the layer.
// x16: the call's hidden states as fp16 (to_f16 below)
int run_gemm(moe_ctx* c, WorkListArgs wa, const uint16_t* x16, int T, float* y, cudaStream_t s) {
    wa.gemm = 1;
    prof_mark(c, MOE_PROF_WORKLIST, true, s);
    cudaError_t e = launch_build_worklist(wa, c->pdl, s);
    prof_mark(c, MOE_PROF_WORKLIST, false, s);
    c->launches += 1;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const int pairs = T * wa.K;
    const int routed = (pairs < wa.n_slot_range ? pairs : wa.n_slot_range) + (pairs + kGemmMaxRows - 1) / kGemmMaxRows;
    const int shared = wa.shared_blob ? (T + kGemmMaxRows - 1) / kGemmMaxRows : 0;
    GemmLaunch L;
    L.wl = c->wl;
    L.entries = c->entries;
    L.rows = c->rows;
    L.x = x16;
    L.h = c->h;
    L.y = y;
    L.D = c->d.d_model;
    L.max_tiles_gu = (wa.K > 0 ? routed * (c->d.d_ff / 64) : 0) + shared * (c->d.d_ff_shared / 64);
    L.max_tiles_dn = ((wa.K > 0 ? routed : 0) + shared) * (c->d.d_model / 128);
    L.row_cap = T;  // an entry carries one expert's rows: at most one per token
    L.status = c->status;
    L.pdl = c->pdl;
    if (L.max_tiles_gu <= 0 || L.max_tiles_dn <= 0) return MOE_OK;
    FfnHookArg ha{c, s};
    e = launch_gemm(L, s, c->prof ? ffn_hook : nullptr, &ha);
    c->launches += 2;
    return cuda_status(e);
}

// The hidden states of a multi-token call as fp16 (the grouped GEMM's B operand).
int to_f16(moe_ctx* c, const uint16_t* x, int T, cudaStream_t s) {
    c->launches += 1;
    return cuda_status(launch_bf16_to_f16(x, c->x16, size_t(T) * c->d.d_model, c->status, c->pdl, s));
}

DecodeWLTarget decode_target(moe_ctx* c, WorkList* wl, FfnEntry* en, FfnRow* rows, const uint8_t* slot_base,
                             size_t stride, const uint8_t* shared_blob) {
    DecodeWLTarget t;
    t.wl = wl;
    t.entries = en;
    t.rows = rows;
    t.slot_base = slot_base;
    t.slot_stride = stride;
    t.shared_blob = shared_blob;
    t.F = c->d.d_ff;
    t.FS = c->d.d_ff_shared;
    t.D = c->d.d_model;
    t.h_shared_off = c->h_shared_off;
    t.blob_bytes = c->blob_routed;
    t.ready = nullptr;
    t.ready_val = 0;
    return t;
}

WorkListArgs worklist_args(moe_ctx* c, int T, int K, const int32_t* pair_slot, const float* gate_w,
                           const uint8_t* slot_base, size_t stride, int n_slot_range, int F,
                           const uint8_t* shared_blob) {
    WorkListArgs a;
    a.T = T;
    a.K = K;
    a.pair_slot = pair_slot;
    a.pair_wave = nullptr;
    a.wave = 0;
    a.gate_w = gate_w;
    a.slot_base = slot_base;
    a.slot_stride = stride;
    a.n_slot_range = n_slot_range;
    a.F = F;
    a.shared_blob = shared_blob;
    a.FS = c->d.d_ff_shared;
    a.h_shared_off = c->h_shared_off;
    a.D = c->d.d_model;
    a.wl = c->wl;
    a.entries = c->entries;
    a.rows = c->rows;
    a.status = c->status;
    return a;
}

// Waits (bounded) until the plan kernel of call `seq` has published its
// mailbox.  Also watches the plan event so a failed launch is an error, not a
// time-out.
int wait_mailbox(moe_ctx* c, uint32_t seq, int timeout_ms) {
    const auto t0 = std::chrono::steady_clock::now();
    volatile uint32_t* p = &c->mbox_host->seq;
    for (uint64_t it = 0;; ++it) {
        if (*p == seq) {
            std::atomic_thread_fence(std::memory_order_acquire);
            return MOE_OK;
        }
        if ((it & 1023) == 1023) {
            const cudaError_t q = cudaEventQuery(c->ev_plan);
            if (q != cudaSuccess && q != cudaErrorNotReady) return MOE_ERR_CUDA;
            if (q == cudaSuccess && *p != seq) {
                // the kernel finished: its system-scope writes are visible now
                if (*p == seq) return MOE_OK;
                return MOE_ERR_STATE;
            }
            const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0);
            if (ms.count() > timeout_ms) return MOE_ERR_TIMEOUT;
        }
    }
}

void copy_trace(const PlanMailbox* mb, moe_plan_trace* tr, size_t blob, uint64_t h2d) {
    if (!tr) return;
    tr->n_distinct = mb->n_distinct;
    tr->n_waves = mb->n_waves;
    tr->n_misses = mb->n_misses;
    tr->h2d_bytes = h2d;
    const int n = mb->n_distinct < tr->capacity ? mb->n_distinct : tr->capacity;
    for (int i = 0; i < n; ++i) {
        if (tr->expert) tr->expert[i] = mb->expert[i];
        if (tr->slot) tr->slot[i] = mb->slot[i];
        if (tr->hit) tr->hit[i] = mb->hit[i];
        if (tr->victim) tr->victim[i] = mb->victim[i];
        if (tr->wave) tr->wave[i] = mb->wave[i];
    }
    (void)blob;
}

// Issues the copies of wave `w`'s misses on the side stream after `after`
// (an event on the compute stream), then makes `s` wait for them.
int fill_wave(moe_ctx* c, const moe_slot_cache* cache, int w, cudaEvent_t after, cudaStream_t s, uint64_t* bytes,
              uint32_t ready_seq = 0) {
    const PlanMailbox* mb = c->mbox_host;
    const size_t nb = c->blob_routed;
    if (cudaStreamWaitEvent(c->side, after, 0) != cudaSuccess) return MOE_ERR_CUDA;
    prof_mark(c, MOE_PROF_H2D, true, c->side);
    if (cache->source == MOE_SOURCE_FILE) {
        // read each missed blob (whole 4 KB pages, so O_DIRECT descriptors work)
        // into a staging buffer, copy it to its slot as soon as it is read
        const size_t len = (nb + 4095) / 4096 * 4096 <= cache->store_stride ? (nb + 4095) / 4096 * 4096 : nb;
        std::vector<FileRead> reads;
        for (int i = 0; i < mb->n_distinct; ++i) {
            if (mb->wave[i] != w || mb->hit[i]) continue;
            const int e = mb->expert[i], sl = mb->slot[i];
            if (e < 0 || e >= c->d.n_experts || sl < 0 || sl >= c->d.n_slots) return MOE_ERR_RANGE;
            reads.push_back(FileRead{cache->store_fd, cache->store_file_offset + uint64_t(e) * cache->store_stride, len,
                                     nb, cache->slots + size_t(sl) * cache->slot_stride});
        }
        int r = c->reader.ensure((nb + 4095) / 4096 * 4096, c->d.n_slots < 16 ? c->d.n_slots : 16);
        if (r == MOE_OK) r = c->reader.read_and_copy(reads, c->side, 10000, bytes);
        if (r != MOE_OK) return r;
        prof_mark(c, MOE_PROF_H2D, false, c->side);
        if (cudaEventRecord(c->ev_fill, c->side) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaStreamWaitEvent(s, c->ev_fill, 0) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    // Blobs prefetched for this cache are moved from their HBM buffers, the
    // others copied from the host store.  By default the moves run on the
    // look-ahead stream, after the staging copies (event) and the wave's
    // order point, so that the host link starts on the first missed blob at
    // once; the compute stream waits for the moves by event.  With per-miss
    // completion (ready_seq != 0) the staged blobs go first on the side stream
    // and the compute stream waits for them by event: a device-to-device copy
    // may run as a kernel, which must not queue behind routed-expert kernels
    // that wait on these blobs.  The host copies run on the copy engine and are
    // announced one by one.
    const bool move_aside = ready_seq == 0u && c->pf_stream != nullptr;
    bool moving = false;
    bool first_ready = true;
    int n_staged = 0;
    for (int pass = 0; pass < 2; ++pass) {
        for (int i = 0; i < mb->n_distinct; ++i) {
            if (mb->wave[i] != w || mb->hit[i]) continue;
            const int e = mb->expert[i], sl = mb->slot[i];
            if (e < 0 || e >= c->d.n_experts || sl < 0 || sl >= c->d.n_slots) return MOE_ERR_RANGE;
            uint8_t* dst = cache->slots + size_t(sl) * cache->slot_stride;
            int pb = -1;
            for (const auto& f : c->pf_table)
                if (f.state == cache->state && f.store == cache->store && f.expert == e) pb = f.buf;
            if ((pb >= 0) != (pass == 0)) continue;
            if (pb >= 0 && move_aside && !moving) {
                if (cudaStreamWaitEvent(c->pf_stream, after, 0) != cudaSuccess ||
                    cudaStreamWaitEvent(c->pf_stream, c->ev_staged, 0) != cudaSuccess)
                    return MOE_ERR_CUDA;
                moving = true;
            }
            const cudaError_t ce =
                pb >= 0 ? cudaMemcpyAsync(dst, c->pf_buf + size_t(pb) * c->pf_stride, nb, cudaMemcpyDeviceToDevice,
                                          move_aside ? c->pf_stream : c->side)
                        : cudaMemcpyAsync(dst, cache->store + size_t(e) * cache->store_stride, nb,
                                          cudaMemcpyHostToDevice, c->side);
            if (ce != cudaSuccess) return MOE_ERR_CUDA;
            if (ready_seq) {
                // this blob has landed once the stream reaches the write (the
                // default flags fence the copy before it); the fault injection
                // of the tests leaves the call's first write out
                const bool skip = c->inject_skip_ready && first_ready;
                first_ready = false;
                if (!skip &&
                    c->write_value(c->side, reinterpret_cast<unsigned long long>(c->ready + sl), ready_seq, 0) != 0)
                    return MOE_ERR_CUDA;
            }
            if (pb >= 0) {
                c->pf_used += nb;
                ++n_staged;
            }
            *bytes += nb;
        }
        if (pass == 0 && moving) {
            // the list that reads the moved blobs waits for the moves; the next
            // staging copies wait for them too (they may reuse the buffers)
            if (cudaEventRecord(c->ev_moved, c->pf_stream) != cudaSuccess ||
                cudaStreamWaitEvent(s, c->ev_moved, 0) != cudaSuccess)
                return MOE_ERR_CUDA;
        }
        if (pass == 0 && ready_seq && n_staged > 0) {
            if (cudaEventRecord(c->ev_fill, c->side) != cudaSuccess) return MOE_ERR_CUDA;
            if (cudaStreamWaitEvent(s, c->ev_fill, 0) != cudaSuccess) return MOE_ERR_CUDA;
        }
    }
    prof_mark(c, MOE_PROF_H2D, false, c->side);
    if (ready_seq) return MOE_OK;  // the kernels wait per blob
    if (cudaEventRecord(c->ev_fill, c->side) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamWaitEvent(s, c->ev_fill, 0) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

// Residency mirror of a cache, updated from a plan the host has read.
std::vector<int16_t>& mirror_of(moe_ctx* c, const int32_t* state) {
    auto& m = c->mirror[state];
    if (m.empty()) m.assign(size_t(c->d.n_experts), int16_t(-1));
    return m;
}
void mirror_update(moe_ctx* c, const moe_slot_cache* cache) {
    auto& m = mirror_of(c, cache->state);
    const PlanMailbox* mb = c->mbox_host;
    for (int i = 0; i < mb->n_distinct; ++i) {
        if (mb->hit[i]) continue;
        const int e = mb->expert[i], v = mb->victim[i], sl = mb->slot[i];
        if (v >= 0 && v < c->d.n_experts) m[size_t(v)] = -1;
        if (e >= 0 && e < c->d.n_experts) m[size_t(e)] = int16_t(sl);
    }
}

// the cache has a backing store the misses are copied from
bool has_store(const moe_slot_cache* cache) { return cache->store || cache->source == MOE_SOURCE_FILE; }

int check_cache(const moe_ctx* c, const moe_slot_cache* cache) {
    if (!cache || !cache->slots || !cache->state) return MOE_ERR_ARG;
    if (!aligned(cache->slots, 256) || cache->slot_stride % 256 || cache->slot_stride < c->blob_routed) return MOE_ERR_ARG;
    if (!aligned(cache->state, 16)) return MOE_ERR_ARG;
    if (cache->store && cache->store_stride < c->blob_routed) return MOE_ERR_ARG;
    if (cache->policy < MOE_POLICY_LFU || cache->policy > MOE_POLICY_LFU_IN_CACHE) return MOE_ERR_ARG;
    if (cache->source != MOE_SOURCE_HOST && cache->source != MOE_SOURCE_FILE && cache->source != MOE_SOURCE_HOST_DIRECT)
        return MOE_ERR_ARG;
    if (cache->source == MOE_SOURCE_HOST_DIRECT &&
        (!cache->store || !aligned(cache->store, 16) || cache->store_stride % 16))
        return MOE_ERR_ARG;
    if (cache->source == MOE_SOURCE_FILE && (cache->store_fd < 0 || cache->store_stride < c->blob_routed))
        return MOE_ERR_ARG;
    return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_blob_bytes(int d_model, int d_ff) {
    if (d_model <= 0 || d_model % 256 || d_ff <= 0 || d_ff % 64 || (d_ff > 704 && d_ff % 704)) return 0;
    return blob_bytes(d_model, d_ff);
}

size_t moe_cache_state_words(const moe_dims* d) { return d ? size_t(3) * d->n_experts + d->n_slots : 0; }

const char* moe_status_str(int s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "timed out";
        case MOE_ERR_STATE: return "invalid state";
        case MOE_ERR_NAN: return "NaN router logit";
        case MOE_ERR_RANGE: return "index out of range";
        case MOE_ERR_IO: return "expert file read failed";
        default: return "unknown status";
    }
}

int moe_ctx_create(const moe_dims* dims, int device, moe_ctx** out) {
    if (!out) return MOE_ERR_ARG;
    *out = nullptr;
    if (!dims_ok(dims)) return MOE_ERR_ARG;
    if (cudaSetDevice(device) != cudaSuccess) return MOE_ERR_CUDA;
    moe_ctx* c = new (std::nothrow) moe_ctx();
    if (!c) return MOE_ERR_CUDA;
    c->d = *dims;
    c->device = device;
    c->blob_routed = blob_bytes(dims->d_model, dims->d_ff);
    c->blob_shared = dims->d_ff_shared > 0 ? blob_bytes(dims->d_model, dims->d_ff_shared) : 0;
    const moe_dims& d = c->d;
    bool ok = cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, device) == cudaSuccess;
    ok = ok && cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&c->ev_plan, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&c->ev_fill, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&c->ev_wave, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaHostAlloc(reinterpret_cast<void**>(&c->mbox_host), sizeof(PlanMailbox), cudaHostAllocMapped) == cudaSuccess;
    ok = ok && cudaHostGetDevicePointer(reinterpret_cast<void**>(&c->mbox_dev), c->mbox_host, 0) == cudaSuccess;
    if (ok) std::memset(c->mbox_host, 0, sizeof(PlanMailbox));
    const int T = d.max_tokens, pairs = T * d.top_k;
    const int fmax = d.d_ff > d.d_ff_shared ? d.d_ff : d.d_ff_shared;
    ok = ok && ffn_prepare(d.d_model, d.d_ff, d.d_ff_shared, d.top_k, T, c->sms, &c->shapes) == cudaSuccess;
    ok = ok && gemm_prepare() == cudaSuccess;
    const int ment = max_entries(d);
    const size_t h_floats = size_t(pairs) * d.d_ff + size_t(T) * d.d_ff_shared;
    c->h_shared_off = pairs * d.d_ff;
    int grid_gu = c->shapes.gu[0].grid > c->shapes.gu[1].grid ? c->shapes.gu[0].grid : c->shapes.gu[1].grid;
    const size_t tiles_gu = size_t(ment) * (fmax / 16);
    const int ns_dn_max = fmax / down_ks(fmax);
    const size_t units_dn = size_t(ment) * (d.d_model / kChunkRows) * ns_dn_max;
    ok = ok && dalloc(&c->status, 1) == cudaSuccess;
    c->list_cap = ment < T + pairs ? ment : T + pairs;
    ok = ok && dalloc(&c->wl, 1) == cudaSuccess;
    ok = ok && dalloc(&c->entries, ment) == cudaSuccess;
    ok = ok && dalloc(&c->rows, size_t(T) + pairs) == cudaSuccess;
    ok = ok && dalloc(&c->wl2, 1) == cudaSuccess;
    ok = ok && dalloc(&c->entries2, ment) == cudaSuccess;
    ok = ok && dalloc(&c->rows2, size_t(T) + pairs) == cudaSuccess;
    if (const char* v = std::getenv("MOE_NO_PDL")) c->pdl = !(v[0] == '1');
    ok = ok && dalloc(&c->h, h_floats) == cudaSuccess;
    ok = ok && dalloc(&c->partials_gu, size_t(2) * grid_gu * kMaxRows * 32) == cudaSuccess;
    ok = ok && dalloc(&c->counters_gu, tiles_gu) == cudaSuccess;
    ok = ok && dalloc(&c->partials_dn, units_dn * kMaxRows * 32) == cudaSuccess;
    ok = ok && dalloc(&c->counters_dn, size_t(d.d_model / kChunkRows)) == cudaSuccess;
    ok = ok && dalloc(&c->ids, pairs) == cudaSuccess;
    ok = ok && dalloc(&c->gate_w, pairs) == cudaSuccess;
    ok = ok && dalloc(&c->pair_slot, pairs) == cudaSuccess;
    ok = ok && dalloc(&c->pair_wave, pairs) == cudaSuccess;
    ok = ok && dalloc(&c->x16, size_t(T) * d.d_model) == cudaSuccess;
    ok = ok && layer_grid(device, &c->layer_G) == cudaSuccess;
    if (ok) {
        c->layer_ok = layer_supported(d.d_model, d.n_experts, d.top_k, d.d_ff, d.d_ff_shared, d.n_slots, c->layer_G);
        c->layer_hvals = layer_hvals(d.d_model, d.top_k, d.d_ff, d.d_ff_shared, c->layer_G);
        if (const char* v = std::getenv("MOE_LAYER_KERNEL")) {
            c->layer_on = v[0] != '0';
            c->layer_resident = v[0] == '1';
        }
    }
    ok = ok && dalloc(&c->layer_logits, size_t(d.n_experts)) == cudaSuccess;
    ok = ok && dalloc(&c->layer_partials, size_t(6) * c->layer_G * 32) == cudaSuccess;
    ok = ok && dalloc(&c->layer_bar, 128) == cudaSuccess;
    ok = ok && dalloc(&c->stats, MOE_STATS) == cudaSuccess;
    ok = ok && dalloc(&c->ready, size_t(d.n_slots)) == cudaSuccess;
    ok = ok && cudaMemset(c->ready, 0, size_t(d.n_slots) * sizeof(uint32_t)) == cudaSuccess;
    if (ok) {
        // the stream memory write; without it the routed experts wait for all
        // of a call's copies through an event, as multi-token calls do
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuStreamWriteValue32", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess && fn)
            c->write_value = reinterpret_cast<StreamWriteValue32>(fn);
        cudaGetLastError();
        if (const char* v = std::getenv("MOE_PER_MISS")) c->per_miss = v[0] == '1';
        if (const char* v = std::getenv("MOE_INJECT_SKIP_READY")) c->inject_skip_ready = v[0] == '1';
    }
    ok = ok && cudaMemset(c->layer_bar, 0, 128 * sizeof(unsigned)) == cudaSuccess;
    ok = ok && cudaMemset(c->stats, 0, MOE_STATS * sizeof(uint64_t)) == cudaSuccess;
    ok = ok && cudaMemset(c->status, 0, sizeof(int)) == cudaSuccess;
    ok = ok && cudaMemset(c->counters_gu, 0, tiles_gu * sizeof(int)) == cudaSuccess;
    ok = ok && cudaMemset(c->counters_dn, 0, size_t(d.d_model / kChunkRows) * sizeof(int)) == cudaSuccess;
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        free_ctx(c);
        return MOE_ERR_CUDA;
    }
    *out = c;
    return MOE_OK;
}

int moe_ctx_destroy(moe_ctx* c) {
    if (!c) return MOE_OK;
    cudaSetDevice(c->device);
    const auto t0 = std::chrono::steady_clock::now();
    while (cudaStreamQuery(c->side) == cudaErrorNotReady &&
           std::chrono::steady_clock::now() - t0 < std::chrono::seconds(10)) {
    }
    free_ctx(c);
    return MOE_OK;
}

uint64_t moe_ctx_launches(const moe_ctx* c) { return c ? c->launches : 0; }

int moe_gemm_min_tokens(void) { return MOE_GEMM_MIN_TOKENS; }

int moe_ctx_profile(moe_ctx* c, int enable) {
    if (!c) return MOE_ERR_ARG;
    c->prof = enable != 0;
    return MOE_OK;
}

int moe_ctx_profile_read(moe_ctx* c, double* total_ms, uint64_t* count) {
    if (!c || !total_ms || !count) return MOE_ERR_ARG;
    for (int k = 0; k < MOE_PROF_KINDS; ++k) {
        total_ms[k] = 0.0;
        count[k] = 0;
    }
    int rc = MOE_OK;
    for (auto& r : c->recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            rc = MOE_ERR_CUDA;
        total_ms[r.kind] += ms;
        count[r.kind] += 1;
        c->pool.push_back(r.a);
        c->pool.push_back(r.b);
    }
    c->recs.clear();
    return rc;
}

int moe_ctx_sync(moe_ctx* c, cudaStream_t s, int timeout_ms) {
    if (!c) return MOE_ERR_ARG;
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t a = cudaStreamQuery(s), b = cudaStreamQuery(c->side);
        if ((a != cudaSuccess && a != cudaErrorNotReady) || (b != cudaSuccess && b != cudaErrorNotReady))
            return MOE_ERR_CUDA;
        if (a == cudaSuccess && b == cudaSuccess) break;
        const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0);
        if (ms.count() > timeout_ms) return MOE_ERR_TIMEOUT;
    }
    int st = 0;
    if (cudaMemcpy(&st, c->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (st != 0 && cudaMemset(c->status, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
    return st;
}

int moe_router_topk(moe_ctx* c, const uint16_t* x, const int8_t* wq, const uint16_t* ws, const float* bias, int T,
                    int32_t* ids, float* gate_w, cudaStream_t s) {
    if (!c || !x || !wq || !ws || !ids || !gate_w) return MOE_ERR_ARG;
    if (T < 1 || T > c->d.max_tokens) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(wq, 16) || !aligned(ws, 4) || !aligned(ids, 4) || !aligned(gate_w, 4))
        return MOE_ERR_ARG;
    prof_mark(c, MOE_PROF_ROUTER, true, s);
    const cudaError_t e = launch_router(x, wq, ws, bias, c->d.n_experts, c->d.d_model, c->d.top_k, T, ids, gate_w,
                                        c->status, DecodeWLTarget{}, c->pdl, s);
    prof_mark(c, MOE_PROF_ROUTER, false, s);
    c->launches += 1;
    return cuda_status(e);
}

int moe_cache_reset(moe_ctx* c, moe_slot_cache* cache, cudaStream_t s) {
    if (!c || !cache || !cache->state) return MOE_ERR_ARG;
    mirror_of(c, cache->state).assign(size_t(c->d.n_experts), int16_t(-1));
    // staged look-ahead blobs fetched for this cache no longer match its state
    for (size_t i = 0; i < c->pf_table.size();)
        if (c->pf_table[i].state == cache->state) c->pf_table.erase(c->pf_table.begin() + long(i));
        else ++i;
    c->launches += 1;
    return cuda_status(launch_cache_reset(cache->state, c->d.n_experts, c->d.n_slots, c->pdl, s));
}

// Plans the call; when the host needs the plan (store or trace) waits for the
// mailbox.  *waves receives the wave count (0 when not waited for).
static int plan_call(moe_ctx* c, moe_slot_cache* cache, const int32_t* ids, int T, uint32_t step, int32_t* pair_slot,
                     bool need_host, int* waves, cudaStream_t s) {
    const uint32_t seq = ++c->seq;
    prof_mark(c, MOE_PROF_PLAN, true, s);
    cudaError_t e = launch_plan(ids, T * c->d.top_k, c->d.n_experts, c->d.n_slots, cache->policy, cache->decay_period,
                                cache->state, step, pair_slot,
                                c->pair_wave, need_host ? c->mbox_dev : nullptr, seq, c->status, nullptr,
                                DecodeWLTarget{}, DecodeWLTarget{}, c->stats, c->blob_routed, c->pdl, s);
    prof_mark(c, MOE_PROF_PLAN, false, s);
    c->launches += 1;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaEventRecord(c->ev_plan, s) != cudaSuccess) return MOE_ERR_CUDA;
    *waves = 0;
    if (!need_host) return MOE_OK;
    const int r = wait_mailbox(c, seq, 10000);
    if (r != MOE_OK) return r;
    *waves = c->mbox_host->n_waves;
    return MOE_OK;
}

int moe_cache_plan(moe_ctx* c, moe_slot_cache* cache, const int32_t* ids, int T, uint32_t step, int32_t* pair_slot,
                   moe_plan_trace* trace, cudaStream_t s) {
    if (!c || !ids || !pair_slot) return MOE_ERR_ARG;
    if (T < 1 || T > c->d.max_tokens) return MOE_ERR_ARG;
    int r = check_cache(c, cache);
    if (r != MOE_OK) return r;
    const bool need_host = has_store(cache) || trace;
    int waves = 0;
    r = plan_call(c, cache, ids, T, step, pair_slot, need_host, &waves, s);
    if (r != MOE_OK) return r;
    uint64_t bytes = 0;
    if (need_host) mirror_update(c, cache);
    if (has_store(cache) && waves == 1) {
        r = fill_wave(c, cache, 0, c->ev_plan, s, &bytes);
        if (r != MOE_OK) return r;
    }
    if (need_host) copy_trace(c->mbox_host, trace, c->blob_routed, bytes);
    return MOE_OK;
}

int moe_expert_ffn(moe_ctx* c, const uint16_t* x, int T, int top_k, const int32_t* pair_slot, const float* gate_w,
                   const uint8_t* slot_base, size_t slot_stride, int n_slot_range, int d_ff, const float* y_in,
                   float* y, uint16_t* y_bf16, cudaStream_t s) {
    if (!c || !x || !pair_slot || !gate_w || !slot_base || !y) return MOE_ERR_ARG;
    if (T < 1 || T > 32 || T > c->d.max_tokens || top_k < 1 || top_k > c->d.top_k) return MOE_ERR_ARG;
    if (n_slot_range < 1 || n_slot_range > 1024) return MOE_ERR_ARG;
    if (d_ff <= 0 || (d_ff != c->d.d_ff && d_ff != c->d.d_ff_shared)) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(slot_base, 256) || slot_stride % 256 || !aligned(y, 16)) return MOE_ERR_ARG;
    if (y_in && !aligned(y_in, 16)) return MOE_ERR_ARG;
    if (slot_stride < blob_bytes(c->d.d_model, d_ff) && n_slot_range > 1) return MOE_ERR_ARG;
    WorkListArgs wa = worklist_args(c, T, top_k, pair_slot, gate_w, slot_base, slot_stride, n_slot_range, d_ff, nullptr);
    if (d_ff != c->d.d_ff) {
        // the shared-width expert through the routed interface: its rows live
        // in the shared part of the activation buffer
        if (T * top_k * d_ff > c->h_shared_off + T * c->d.d_ff_shared) return MOE_ERR_ARG;
    }
    return run_ffn(c, wa, x, T, y_in, y, y_bf16, s);
}

}  // extern "C"

// Device-accessible address of a pinned host store (the kernels read missed
// experts from it directly); null when the memory is not pinned and mapped.
static const uint8_t* direct_store(moe_ctx* c, const uint8_t* store) {
    auto it = c->direct_store.find(store);
    if (it != c->direct_store.end()) return it->second;
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, store) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (pa.type != cudaMemoryTypeHost || !pa.devicePointer) return nullptr;
    const uint8_t* dp = static_cast<const uint8_t*>(pa.devicePointer);
    c->direct_store[store] = dp;
    return dp;
}

// One token through the whole layer in one launch (layer.cu): experts
// resident (cache == null) or served from the slot cache with misses read
// straight from the pinned host store by the kernel.
static int run_layer_kernel(moe_ctx* c, const moe_layer_weights* W, moe_slot_cache* cache, const uint16_t* x,
                            uint32_t step, const float* bias, float* y, uint16_t* y_bf16, int32_t* ids, float* gate_w,
                            moe_plan_trace* trace, cudaStream_t s) {
    if (!aligned(W->router_q, 16) || !aligned(W->router_s, 4)) return MOE_ERR_ARG;
    LayerArgs a{};
    a.x = x;
    a.wq = W->router_q;
    a.ws = W->router_s;
    a.bias = bias;
    a.shared_blob = W->shared_blob;
    if (!cache) {
        a.experts = W->experts;
        a.expert_stride = W->expert_stride;
    } else {
        a.slots = cache->slots;
        a.slot_stride = cache->slot_stride;
        a.state = cache->state;
        a.store = direct_store(c, cache->store);
        if (!a.store) return MOE_ERR_ARG;
        a.store_stride = cache->store_stride;
        a.policy = cache->policy;
        a.decay_period = cache->decay_period;
    }
    a.step = step;
    a.D = c->d.d_model;
    a.E = c->d.n_experts;
    a.K = c->d.top_k;
    a.F = c->d.d_ff;
    a.FS = W->shared_blob ? c->d.d_ff_shared : 0;
    a.S = c->d.n_slots;
    a.blob_bytes = c->blob_routed;
    a.hvals = c->layer_hvals;
    a.y = y;
    a.y_bf16 = y_bf16;
    a.ids = ids;
    a.gate_w = gate_w;
    a.mailbox = (cache && trace) ? c->mbox_dev : nullptr;
    a.seq = ++c->seq;
    a.stats = cache ? c->stats : nullptr;
    a.logits = c->layer_logits;
    a.h = c->h;
    a.partials_gu = c->layer_partials;
    a.partials_dn = c->layer_partials + size_t(4) * c->layer_G * 32;
    a.counters_gu = c->counters_gu;
    a.counters_dn = c->counters_dn;
    a.bar = c->layer_bar;
    a.status = c->status;
    prof_mark(c, MOE_PROF_LAYER, true, s);
    cudaError_t e = launch_layer(a, c->layer_G, c->pdl && c->layer_pdl, s);
    if (e != cudaSuccess && c->pdl && c->layer_pdl) {
        // a cooperative launch the driver will not chain programmatically
        cudaGetLastError();
        c->layer_pdl = false;
        e = launch_layer(a, c->layer_G, false, s);
    }
    prof_mark(c, MOE_PROF_LAYER, false, s);
    c->launches += 1;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // the mailbox wait watches this event to tell a failed kernel from a slow one
    if (cudaEventRecord(c->ev_plan, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cache && trace) {
        const int r = wait_mailbox(c, a.seq, 10000);
        if (r != MOE_OK) return r;
        mirror_update(c, cache);
        copy_trace(c->mbox_host, trace, c->blob_routed, uint64_t(c->mbox_host->n_misses) * c->blob_routed);
    }
    return MOE_OK;
}

// the layer; `next` (or null) asks for a look-ahead prefetch of the next layer
static int layer_forward(moe_ctx* c, const moe_layer_weights* W, moe_slot_cache* cache, const uint16_t* x, int T,
                         uint32_t step, const float* bias, float* y, uint16_t* y_bf16, int32_t* ids, float* gate_w,
                         moe_plan_trace* trace, const moe_next_layer* next, cudaStream_t s) {
    if (!c || !W || !W->router_q || !W->router_s || !x || !y) return MOE_ERR_ARG;
    if (T < 1 || T > c->d.max_tokens) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(y, 16)) return MOE_ERR_ARG;
    if (W->shared_blob && (!aligned(W->shared_blob, 256) || c->d.d_ff_shared == 0)) return MOE_ERR_ARG;
    if (!cache && (!W->experts || !aligned(W->experts, 256) || W->expert_stride % 256 ||
                   W->expert_stride < c->blob_routed))
        return MOE_ERR_ARG;
    if (cache) {
        const int r = check_cache(c, cache);
        if (r != MOE_OK) return r;
    }
    int32_t* id = ids ? ids : c->ids;
    float* gw = gate_w ? gate_w : c->gate_w;
    const int K = c->d.top_k;
    int r;
    // look-ahead: the next layer's router on this layer's input, on its own
    // stream, while this layer runs (one token, host stores, buffers configured)
    const bool prefetch = next && T == 1 && c->pf_n > 0 && next->W && next->W->router_q && next->W->router_s &&
                          next->cache && next->cache->source == MOE_SOURCE_HOST && next->cache->store;
    // the layer after next, staged for only when next has nothing to stage
    const moe_next_layer* after = prefetch && next->after && next->after->W && next->after->W->router_q &&
                                          next->after->W->router_s && next->after->cache &&
                                          next->after->cache->source == MOE_SOURCE_HOST && next->after->cache->store &&
                                          next->after->cache->state != next->cache->state
                                      ? next->after
                                      : nullptr;
    // the one-launch layer kernel: always for direct-fill caches (the kernel
    // reads the misses), for resident experts when asked (MOE_LAYER_KERNEL=1;
    // the separate router / GEMV kernels are faster there today)
    if (T == 1 && c->layer_ok && c->layer_on && !prefetch &&
        ((cache && cache->source == MOE_SOURCE_HOST_DIRECT) || (!cache && c->layer_resident)))
        return run_layer_kernel(c, W, cache, x, step, bias, y, y_bf16, id, gw, trace, s);
    if (T == 1 && !cache) {
        // one token, resident: the router writes the work list itself
        const DecodeWLTarget t = decode_target(c, c->wl, c->entries, c->rows, W->experts, W->expert_stride,
                                               W->shared_blob);
        prof_mark(c, MOE_PROF_ROUTER, true, s);
        const cudaError_t e = launch_router(x, W->router_q, W->router_s, bias, c->d.n_experts, c->d.d_model, K, 1,
                                            id, gw, c->status, t, c->pdl, s);
        prof_mark(c, MOE_PROF_ROUTER, false, s);
        c->launches += 1;
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        return run_ffn_list(c, c->wl, c->entries, c->rows, x, 1, nullptr, y, y_bf16, s, W->shared_blob);
    }
    if (prefetch) {
        if (cudaEventRecord(c->ev_x, s) != cudaSuccess || cudaStreamWaitEvent(c->pf_stream, c->ev_x, 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        cudaError_t pe = launch_router(x, next->W->router_q, next->W->router_s, next->bias, c->d.n_experts,
                                       c->d.d_model, K, 1, c->pf_ids_dev, c->pf_gw, c->status, DecodeWLTarget{},
                                       false, c->pf_stream);
        c->launches += 1;
        if (pe == cudaSuccess && after) {
            pe = launch_router(x, after->W->router_q, after->W->router_s, after->bias, c->d.n_experts, c->d.d_model,
                               K, 1, c->pf_ids_dev + K, c->pf_gw + K, c->status, DecodeWLTarget{}, false,
                               c->pf_stream);
            c->launches += 1;
        }
        if (pe != cudaSuccess || cudaEventRecord(c->ev_pred, c->pf_stream) != cudaSuccess) return MOE_ERR_CUDA;
    }
    r = moe_router_topk(c, x, W->router_q, W->router_s, bias, T, id, gw, s);
    if (r != MOE_OK) return r;
    const bool gemm = T >= MOE_GEMM_MIN_TOKENS;  // tensor-core grouped GEMM
    if (!cache) {
        // resident: expert e's blob is W->experts + e * stride, one pass
        WorkListArgs wa = worklist_args(c, T, K, id, gw, W->experts, W->expert_stride, c->d.n_experts, c->d.d_ff,
                                        W->shared_blob);
        if (!gemm) return run_ffn(c, wa, x, T, nullptr, y, y_bf16, s);
        if (cudaMemsetAsync(y, 0, sizeof(float) * size_t(T) * c->d.d_model, s) != cudaSuccess) return MOE_ERR_CUDA;
        r = to_f16(c, x, T, s);
        if (r == MOE_OK) r = run_gemm(c, wa, c->x16, T, y, s);
        if (r != MOE_OK) return r;
        if (y_bf16) {
            c->launches += 1;
            return cuda_status(launch_f32_to_bf16(y, y_bf16, size_t(T) * c->d.d_model, c->pdl, s));
        }
        return MOE_OK;
    }
    // streaming: plan, then the shared expert (queued before the host waits,
    // so it runs during the copies), then the routed experts wave by wave
    const uint32_t seq = ++c->seq;
    // one token: the plan kernel also writes both work lists
    const bool one = (T == 1);
    // list A: shared expert + hits (no copy needed); list B: misses
    const DecodeWLTarget t_sh = one ? decode_target(c, c->wl, c->entries, c->rows, cache->slots, cache->slot_stride,
                                                    W->shared_blob)
                                    : DecodeWLTarget{};
    DecodeWLTarget t_rt = one ? decode_target(c, c->wl2, c->entries2, c->rows2, cache->slots, cache->slot_stride,
                                              nullptr)
                              : DecodeWLTarget{};
    // one token from host memory, when enabled: list B waits per missed blob.
    // Measured on B200 (30 layers, 16 slots): the stream memory write after
    // each copy leaves the link idle for a few microseconds, more than the
    // overlap gains (143.7 vs 152.4 tokens/s), so the default joins all of a
    // call's copies with one event before list B
    const bool per_miss = one && c->per_miss && c->write_value && cache->source == MOE_SOURCE_HOST && cache->store &&
                          seq != 0u;
    if (per_miss) {
        t_rt.ready = c->ready;
        t_rt.ready_val = seq;
    }
    prof_mark(c, MOE_PROF_PLAN, true, s);
    cudaError_t e = launch_plan(id, T * K, c->d.n_experts, c->d.n_slots, cache->policy, cache->decay_period,
                                cache->state, step, c->pair_slot,
                                c->pair_wave, c->mbox_dev, seq, c->status, gw, t_sh, t_rt, c->stats, c->blob_routed,
                                c->pdl, s);
    prof_mark(c, MOE_PROF_PLAN, false, s);
    c->launches += 1;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaEventRecord(c->ev_plan, s) != cudaSuccess) return MOE_ERR_CUDA;
    bool have_y = false;
    if (one) {
        // list A runs now, during the copies; without a shared expert it may be
        // empty, so y starts from zero and both lists accumulate into it
        if (!W->shared_blob && cudaMemsetAsync(y, 0, sizeof(float) * c->d.d_model, s) != cudaSuccess)
            return MOE_ERR_CUDA;
        r = run_ffn_list(c, c->wl, c->entries, c->rows, x, 1, W->shared_blob ? nullptr : y, y, y_bf16, s,
                         W->shared_blob);
        if (r != MOE_OK) return r;
        have_y = true;
    } else if (gemm) {
        // prefill chunk: every contribution is added into y
        if (cudaMemsetAsync(y, 0, sizeof(float) * size_t(T) * c->d.d_model, s) != cudaSuccess) return MOE_ERR_CUDA;
        r = to_f16(c, x, T, s);
        if (r != MOE_OK) return r;
        if (W->shared_blob) {
            WorkListArgs wa = worklist_args(c, T, 0, c->pair_slot, gw, cache->slots, cache->slot_stride, c->d.n_slots,
                                            c->d.d_ff, W->shared_blob);
            r = run_gemm(c, wa, c->x16, T, y, s);
            if (r != MOE_OK) return r;
        }
        have_y = true;
    } else if (W->shared_blob) {
        {
            WorkListArgs wa = worklist_args(c, T, 0, c->pair_slot, gw, cache->slots, cache->slot_stride, c->d.n_slots,
                                            c->d.d_ff, W->shared_blob);
            r = run_ffn(c, wa, x, T, nullptr, y, nullptr, s);
        }
        if (r != MOE_OK) return r;
        have_y = true;
    }
    r = wait_mailbox(c, seq, 10000);
    if (r != MOE_OK) return r;
    mirror_update(c, cache);
    const int waves = c->mbox_host->n_waves;
    uint64_t bytes = 0;
    for (int w = 0; w < waves; ++w) {
        if (one && c->mbox_host->n_misses == 0) break;  // everything hit: list A was the whole layer
        if (has_store(cache)) {
            // wave w's victims may be slots wave w-1 still reads: copy after it
            cudaEvent_t after = c->ev_plan;
            if (w > 0) {
                if (cudaEventRecord(c->ev_wave, s) != cudaSuccess) return MOE_ERR_CUDA;
                after = c->ev_wave;
            }
            r = fill_wave(c, cache, w, after, s, &bytes, per_miss ? seq : 0u);
            if (r != MOE_OK) return r;
        }
        if (one) {
            // list B holds exactly the misses the mailbox reported
            r = run_ffn_list(c, c->wl2, c->entries2, c->rows2, x, 1, have_y ? y : nullptr, y, y_bf16, s, nullptr,
                             c->mbox_host->n_misses);
        } else if (gemm) {
            WorkListArgs wa = worklist_args(c, T, K, c->pair_slot, gw, cache->slots, cache->slot_stride,
                                            c->d.n_slots, c->d.d_ff, nullptr);
            wa.pair_wave = c->pair_wave;
            wa.wave = w;
            r = run_gemm(c, wa, c->x16, T, y, s);
        } else {
            WorkListArgs wa = worklist_args(c, T, K, c->pair_slot, gw, cache->slots, cache->slot_stride,
                                            c->d.n_slots, c->d.d_ff, nullptr);
            wa.pair_wave = c->pair_wave;
            wa.wave = w;
            r = run_ffn(c, wa, x, T, have_y ? y : nullptr, y, (w + 1 == waves) ? y_bf16 : nullptr, s);
        }
        if (r != MOE_OK) return r;
        have_y = true;
    }
    if (gemm && y_bf16) {
        c->launches += 1;
        if (launch_f32_to_bf16(y, y_bf16, size_t(T) * c->d.d_model, c->pdl, s) != cudaSuccess) return MOE_ERR_CUDA;
    }
    // this layer has run: the blobs staged for its cache were used or are
    // stale (also when this call stages nothing, e.g. the last layer)
    for (size_t i = 0; i < c->pf_table.size();)
        if (c->pf_table[i].state == cache->state) c->pf_table.erase(c->pf_table.begin() + long(i));
        else ++i;
    if (prefetch) {
        // The next layer's predicted experts its cache does not hold, in logit
        // order, after this layer's own copies on the side stream.  Blobs
        // staged for this layer are used or stale now, and blobs for layers
        // other than the next two are not wanted; blobs staged earlier for the
        // next layer (as its "after") stay.  When nothing of the next layer is
        // worth staging, a free buffer takes the top predicted miss of the
        // layer after it.
        if (cudaEventSynchronize(c->ev_pred) != cudaSuccess) return MOE_ERR_CUDA;
        const int32_t* keep_a = next->cache->state;
        const int32_t* keep_b = after ? after->cache->state : nullptr;
        for (size_t i = 0; i < c->pf_table.size();)
            if (c->pf_table[i].state != keep_a && (!keep_b || c->pf_table[i].state != keep_b))
                c->pf_table.erase(c->pf_table.begin() + long(i));
            else
                ++i;
        auto staged = [&](const int32_t* state, int e) {
            for (const auto& f : c->pf_table)
                if (f.state == state && f.expert == e) return true;
            return false;
        };
        auto free_buf = [&]() {
            for (int b = 0; b < c->pf_n; ++b) {
                bool used = false;
                for (const auto& f : c->pf_table) used = used || f.buf == b;
                if (!used) return b;
            }
            return -1;
        };
        bool waited = false;  // the side stream waits for the moves once, before the first staging copy
        // stage up to `limit` predicted misses of layer L (ids at pred); returns
        // how many of its predicted misses are missing from its cache and the buffers
        auto stage = [&](const moe_next_layer* L, const int32_t* pred, int limit, int* n_stage) -> int {
            const auto& m = mirror_of(c, L->cache->state);
            int wanted = 0;
            for (int k = 0; k < K; ++k) {
                const int e = pred[k];
                if (e < 0 || e >= c->d.n_experts || m[size_t(e)] >= 0 || staged(L->cache->state, e)) continue;
                ++wanted;
                const int b = *n_stage < limit ? free_buf() : -1;
                if (b < 0) continue;
                // a buffer freed by this call may still be read by its move
                if (!waited && cudaStreamWaitEvent(c->side, c->ev_moved, 0) != cudaSuccess) return -1;
                waited = true;
                if (cudaMemcpyAsync(c->pf_buf + size_t(b) * c->pf_stride, L->cache->store + size_t(e) * L->cache->store_stride,
                                    c->blob_routed, cudaMemcpyHostToDevice, c->side) != cudaSuccess)
                    return -1;
                c->pf_table.push_back({L->cache->state, L->cache->store, e, b});
                c->pf_issued += c->blob_routed;
                ++*n_stage;
            }
            return wanted;
        };
        int n_stage = 0;
        const int wanted = stage(next, c->pf_ids_host, c->pf_n, &n_stage);
        if (wanted < 0) return MOE_ERR_CUDA;
        if (wanted == 0 && after) {
            int n2 = 0;
            if (stage(after, c->pf_ids_host + K, 1, &n2) < 0) return MOE_ERR_CUDA;
        }
        // the moves of staged blobs wait for this point of the side stream
        if (waited && cudaEventRecord(c->ev_staged, c->side) != cudaSuccess) return MOE_ERR_CUDA;
    }
    copy_trace(c->mbox_host, trace, c->blob_routed, bytes);
    return MOE_OK;
}

extern "C" {

int moe_layer_forward(moe_ctx* c, const moe_layer_weights* W, moe_slot_cache* cache, const uint16_t* x, int T,
                      uint32_t step, const float* bias, float* y, uint16_t* y_bf16, int32_t* ids, float* gate_w,
                      moe_plan_trace* trace, cudaStream_t s) {
    return layer_forward(c, W, cache, x, T, step, bias, y, y_bf16, ids, gate_w, trace, nullptr, s);
}

int moe_layer_forward_next(moe_ctx* c, const moe_layer_weights* W, moe_slot_cache* cache, const uint16_t* x, int T,
                           uint32_t step, const float* bias, float* y, uint16_t* y_bf16, int32_t* ids, float* gate_w,
                           moe_plan_trace* trace, const moe_next_layer* next, cudaStream_t s) {
    if (next && next->cache) {
        const int r = check_cache(c, next->cache);
        if (r != MOE_OK) return r;
    }
    return layer_forward(c, W, cache, x, T, step, bias, y, y_bf16, ids, gate_w, trace, next, s);
}

int moe_prefetch_configure(moe_ctx* c, int n_buffers) {
    if (!c || n_buffers < 0 || n_buffers > 16) return MOE_ERR_ARG;
    // drop the old buffers once nothing queued can still use them
    if ((c->side && cudaStreamSynchronize(c->side) != cudaSuccess) ||
        (c->pf_stream && cudaStreamSynchronize(c->pf_stream) != cudaSuccess))
        return MOE_ERR_CUDA;
    cudaFree(c->pf_buf);
    c->pf_buf = nullptr;
    c->pf_table.clear();
    c->pf_n = 0;
    if (n_buffers == 0) return MOE_OK;
    bool ok = true;
    if (!c->pf_stream) {
        ok = ok && cudaStreamCreateWithFlags(&c->pf_stream, cudaStreamNonBlocking) == cudaSuccess;
        ok = ok && cudaEventCreateWithFlags(&c->ev_x, cudaEventDisableTiming) == cudaSuccess;
        ok = ok && cudaEventCreateWithFlags(&c->ev_pred, cudaEventDisableTiming) == cudaSuccess;
        ok = ok && cudaEventCreateWithFlags(&c->ev_staged, cudaEventDisableTiming) == cudaSuccess;
        ok = ok && cudaEventCreateWithFlags(&c->ev_moved, cudaEventDisableTiming) == cudaSuccess;
        // the predicted ids of the next layer, then of the layer after it
        ok = ok && cudaHostAlloc(reinterpret_cast<void**>(&c->pf_ids_host), sizeof(int32_t) * size_t(2 * c->d.top_k),
                                 cudaHostAllocMapped) == cudaSuccess;
        ok = ok && cudaHostGetDevicePointer(reinterpret_cast<void**>(&c->pf_ids_dev), c->pf_ids_host, 0) == cudaSuccess;
        ok = ok && dalloc(&c->pf_gw, size_t(2 * c->d.top_k)) == cudaSuccess;
    }
    c->pf_stride = (c->blob_routed + 255) / 256 * 256;
    ok = ok && cudaMalloc(reinterpret_cast<void**>(&c->pf_buf), c->pf_stride * size_t(n_buffers)) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    c->pf_n = n_buffers;
    return MOE_OK;
}

int moe_prefetch_stats(const moe_ctx* c, uint64_t* issued_bytes, uint64_t* used_bytes) {
    if (!c) return MOE_ERR_ARG;
    if (issued_bytes) *issued_bytes = c->pf_issued;
    if (used_bytes) *used_bytes = c->pf_used;
    return MOE_OK;
}

int moe_ctx_stats(moe_ctx* c, cudaStream_t s, uint64_t* out) {
    if (!c || !out) return MOE_ERR_ARG;
    if (cudaMemcpyAsync(out, c->stats, MOE_STATS * sizeof(uint64_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_ctx_stats_reset(moe_ctx* c, cudaStream_t s) {
    if (!c) return MOE_ERR_ARG;
    return cuda_status(cudaMemsetAsync(c->stats, 0, MOE_STATS * sizeof(uint64_t), s));
}

int moe_residual_rmsnorm(moe_ctx* c, float* r, const float* y, uint16_t* x_next, int T, cudaStream_t s) {
    if (!c || !r || !y || !x_next || T < 1) return MOE_ERR_ARG;
    if (!aligned(r, 16) || !aligned(y, 16) || !aligned(x_next, 8)) return MOE_ERR_ARG;
    c->launches += 1;
    prof_mark(c, MOE_PROF_HARNESS, true, s);
    const cudaError_t e = launch_residual_rmsnorm(r, y, x_next, T, c->d.d_model, c->pdl, s);
    prof_mark(c, MOE_PROF_HARNESS, false, s);
    return cuda_status(e);
}

int moe_bf16_to_f32(moe_ctx* c, const uint16_t* x, float* out, size_t n, cudaStream_t s) {
    if (!c || !x || !out) return MOE_ERR_ARG;
    c->launches += 1;
    return cuda_status(launch_bf16_to_f32(x, out, n, c->pdl, s));
}

}  // extern "C"
