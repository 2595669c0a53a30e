/*
 * moe.h -- C ABI of libmoe.so: a routed Mixture-of-Experts layer whose 4-bit
 * experts are served from a small per-layer LFU slot cache in GPU memory and
 * streamed in from pinned host memory on a miss.  NVIDIA B200 (sm_100a).
 *
 * The method (sources: five web pages about the TurboFieldfare runtime for
 * Gemma 4 26B-A4B; cited by page title and section):
 *   - "TurboFieldfare: motor open source para ejecutar Gemma 4 26B con 2 GB de
 *     RAM en cualquier Mac serie M", section "Proceso de generacion de tokens":
 *     per layer the router's top-8 expert ids are checked against a 16-slot
 *     LFU cache of that layer, misses are read in with bounded parallelism,
 *     the resident shared-expert branch runs while the reads are in flight,
 *     then shared and routed outputs are combined; prompts are prefilled in
 *     chunks of up to 128 tokens so one fetched expert serves several rows.
 *     Section "Estructura de ejecucion para reducir memoria": experts (shared
 *     and routed) are 4-bit MLX-affine with groups of 64, the router 8-bit.
 *   - "El milagro de la IA de 2GB en Apple Silicon", sections "Por que la
 *     mayor parte de tu modelo de IA es peso muerto" (128 experts, the 8 most
 *     relevant per token), "Mas inteligente que tu RAM" (30 layers, each an LFU
 *     cache of 16 of its 128 experts; a miss replaces the least frequently used
 *     resident expert) and "El arma secreta de Apple" (experts are stored in
 *     the exact 4-bit layout the kernel consumes).
 *   - "Gemma 4 26B en ~2 GB de RAM: el runtime en Swift que streamea los
 *     experts desde el SSD", section "Por que funciona: el A4B del nombre"
 *     (the per-token loop: router on the GPU, fetch plan on the CPU, bounded
 *     parallel reads of missing experts, combine on the GPU).
 *
 * Conventions for every call:
 *   - Every pointer is caller-owned.  "dev" = device memory of the context's
 *     device, "host" = host memory, "pinned" = page-locked host memory
 *     (cudaHostAlloc / torch pin_memory).  The library never frees caller
 *     memory and keeps no pointer after a call returns, except for the work
 *     it has enqueued on the given stream (which reads/writes the buffers
 *     until that work completes).
 *   - Calls are asynchronous on the given cudaStream_t unless stated.  They
 *     return a status code (MOE_OK or a negative MOE_ERR_*); nothing throws.
 *     Argument errors are detected before anything is enqueued.  Errors found
 *     by kernels (NaN router logits, out-of-range slot, a bounded wait that
 *     gave up) are recorded in the context's status word and reported by the
 *     next moe_ctx_sync(); the kernels keep every access in bounds.
 *   - A context is not thread-safe: one host thread drives it at a time.
 *   - Device buffers must be 16-byte aligned; expert blobs 256-byte aligned.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
#define MOE_OK            0
#define MOE_ERR_ARG      -1  /* bad argument: null/misaligned pointer, size out of range */
#define MOE_ERR_CUDA     -2  /* a CUDA runtime call failed (launch, copy, allocation) */
#define MOE_ERR_TIMEOUT  -3  /* a bounded wait (host mailbox or device barrier) gave up */
#define MOE_ERR_STATE    -4  /* call not valid in the context's current state */
#define MOE_ERR_NAN      -5  /* a router logit was NaN: no top-k order exists */
#define MOE_ERR_RANGE    -6  /* an expert id or slot index out of range reached a kernel */
#define MOE_ERR_IO       -7  /* reading an expert from a file-backed store failed or came up short */

/* ------------------------------------------------------------------ shapes
 * Gemma 4 26B-A4B MoE layer: d_model 2816, 128 experts, top-8, expert FFN
 * width 704, shared-expert FFN width 2112, quantisation group 64, 16 slots.
 * Supported: d_model % 256 == 0 and d_model <= 8192; d_ff and d_ff_shared
 * multiples of 64 that are <= 704 or multiples of 704 (at most 2112); group ==
 * 64; top_k <= 16; n_experts % 16 == 0 and n_experts <= 1024; top_k <= n_slots
 * <= n_experts; 1 <= max_tokens <= 1024.  moe_ctx_create returns MOE_ERR_ARG
 * for anything else. */
typedef struct moe_dims {
    int d_model;      /* D */
    int n_experts;    /* E */
    int top_k;        /* K */
    int d_ff;         /* F, routed experts */
    int d_ff_shared;  /* FS, shared expert (0: no shared expert) */
    int group;        /* G, must be 64 */
    int n_slots;      /* S, LFU slots per layer */
    int max_tokens;   /* largest T any call on this context will pass */
} moe_dims;

/* ---------------------------------------------------------- expert blob
 * One expert = one contiguous blob in the kernel-ready layout, identical in
 * the pinned store, in a cache slot and in the resident array, so a miss is
 * one plain copy.  Matrices gate W_g [F x D], up W_u [F x D], down W_d [D x F];
 * w[n][k] = s[n][k/64] * q[n][k] + b[n][k/64], q a 4-bit code 0..15, s and b
 * IEEE binary16.  The blob is two sections of "chunks"; a chunk holds 32 rows
 * x KS inputs in 18*KS bytes:
 *   q part  (KS/32 word-quads) x (32 rows) x 16 bytes; in a row's 16 bytes,
 *           input 32*wq + 8*w + j sits in byte 4*w + j/2, low nibble for
 *           even j, high nibble for odd j;
 *   sb part (KS/64 groups) x (32 rows) x (binary16 s, binary16 b).
 *   section 0 (gate/up): F/16 tiles x D/256 slices, KS = 256, tile-major;
 *             tile t rows 0..15 = gate rows 16t.., rows 16..31 = up rows 16t..
 *   section 1 (down):    D/32 tiles x F/KS slices, KS = F if F <= 704 else
 *             704, tile-major; tile t rows = down rows 32t..32t+31.
 * Size: 3,345,408 bytes for D=2816, F=704; 10,036,224 for F=2112. */
size_t moe_blob_bytes(int d_model, int d_ff);

/* ------------------------------------------------------------- context */
typedef struct moe_ctx moe_ctx;

/* Creates a context on `device`: a side stream for miss copies, events, a
 * pinned mapped mailbox (plan results the host needs to issue the copies), a
 * device status word, and device scratch sized for dims->max_tokens
 * (intermediate activations, per-tile partial sums, work lists).  The scratch
 * is owned by the context and freed by moe_ctx_destroy.  Makes `device`
 * current on the calling thread.  Returns MOE_ERR_ARG for unsupported dims,
 * MOE_ERR_CUDA if an allocation fails (nothing is leaked). */
int moe_ctx_create(const moe_dims *dims, int device, moe_ctx **out);

/* Waits (bounded, 10 s) for the context's own streams, frees everything it
 * owns.  Safe on NULL. */
int moe_ctx_destroy(moe_ctx *ctx);

/* Waits for `stream` and the context's side stream, at most timeout_ms
 * milliseconds (MOE_ERR_TIMEOUT after that; the work is left running), then
 * returns and clears the device status word: MOE_OK or the first error a
 * kernel recorded (MOE_ERR_NAN, MOE_ERR_RANGE, MOE_ERR_TIMEOUT), or
 * MOE_ERR_CUDA if a CUDA call reported an error.  Synchronous. */
int moe_ctx_sync(moe_ctx *ctx, cudaStream_t stream, int timeout_ms);

/* Human-readable name of a status code (static string). */
const char *moe_status_str(int status);

/* Number of device kernels the context has launched so far (all entry
 * points, all streams).  Host counter; used to report launch counts. */
uint64_t moe_ctx_launches(const moe_ctx *ctx);

/* Smallest token count T for which moe_layer_forward runs the experts as the
 * tcgen05 grouped GEMM (tokens grouped per expert, fp16 dequantised weight
 * tiles); one-token calls run the streamed GEMV kernels.  Host only. */
int moe_gemm_min_tokens(void);

/* --------------------------------------------------------------- router
 * Router + top-K + gate weights for T tokens ("El milagro ...", "Por que la
 * mayor parte ...": the layer's small router keeps the K most relevant of the
 * E experts per token; "TurboFieldfare ...", "Estructura ...": 8-bit router).
 *   x       dev bf16 bits [T][D]          hidden states
 *   wq      dev int8 [E][D]               router weights, symmetric int8
 *   ws      dev binary16 bits [E][D/64]   per-group scales
 *   bias    dev fp32 [E] or NULL          added to each logit
 *   ids     dev int32 [T][K]  out         expert ids, logit descending, ties
 *                                         to the lower id
 *   gate_w  dev fp32 [T][K]   out         softmax over the K chosen logits
 * logit_e = (fp32 FMA chain over groups g ascending of s[e][g] * S_g) + bias_e,
 * S_g = fp32 FMA chain over k ascending in group g of q[e][k] * x[k]; every
 * step is one correctly rounded fp32 FMA, so ids are reproducible bit for bit.
 * 1 <= T <= max_tokens.  NaN logits: ids are filled with 0..K-1 (valid
 * indices) and MOE_ERR_NAN is recorded for moe_ctx_sync.  One launch. */
int moe_router_topk(moe_ctx *ctx, const uint16_t *x, const int8_t *wq, const uint16_t *ws,
                    const float *bias, int T, int32_t *ids, float *gate_w, cudaStream_t stream);

/* ---------------------------------------------------------- slot cache
 * The cache of one layer ("El milagro ...", "Mas inteligente que tu RAM").
 *   slots         dev: n_slots blobs, slot s at slots + s*slot_stride
 *   slot_stride   bytes, multiple of 256, >= moe_blob_bytes(D, F)
 *   state         dev int32 [moe_cache_state_words(dims)]: the layer's LFU
 *                 state, zero-initialised by moe_cache_reset; save/restore by
 *                 copying it (and the slots)
 *   store         pinned host: n_experts blobs of this layer, expert e at
 *                 store + e*store_stride; NULL = no backing store (the plan
 *                 is computed but nothing is copied: slots must be filled
 *                 by the caller)
 *   store_stride  bytes, >= moe_blob_bytes(D, F)
 *   policy        replacement rule (MOE_POLICY_*; 0 = LFU, the pages' rule)
 *   decay_period  MOE_POLICY_LFU_DECAY: counts are halved at the start of
 *                 every call whose step is a positive multiple of it (0: never)
 *   source        MOE_SOURCE_HOST (the pinned `store` above, misses copied
 *                 by the copy engine after the host has read the plan),
 *                 MOE_SOURCE_HOST_DIRECT (the same pinned `store`, 16-byte
 *                 aligned with store_stride % 16 == 0, but for one-token
 *                 calls the layer kernel reads each missed expert straight
 *                 from it over the bus and writes it into its slot as it
 *                 computes with it: no host round trip; calls of two or more
 *                 tokens copy as MOE_SOURCE_HOST does), or
 *                 MOE_SOURCE_FILE: expert e is read from file descriptor
 *                 store_fd at byte store_file_offset + e*store_stride with
 *                 positional reads, several in flight, into pinned staging
 *                 buffers of the context, then copied to its slot ("Gemma 4
 *                 26B en ~2 GB de RAM ...", "Por que pread y no mmap").  For a
 *                 descriptor opened with O_DIRECT, store_stride and
 *                 store_file_offset must be multiples of 4096.  The caller
 *                 owns the descriptor; a read that fails or comes up short is
 *                 MOE_ERR_IO.
 * A zero-initialised struct's new fields select LFU, no decay, host store. */
typedef struct moe_slot_cache {
    uint8_t *slots;
    size_t slot_stride;
    int32_t *state;
    const uint8_t *store;
    size_t store_stride;
    int32_t policy;
    uint32_t decay_period;
    int32_t source;
    int32_t store_fd;
    uint64_t store_file_offset;
} moe_slot_cache;

#define MOE_SOURCE_HOST 0
#define MOE_SOURCE_FILE 1
#define MOE_SOURCE_HOST_DIRECT 2

/* Replacement rules of the slot cache ("El milagro ...", "Mas inteligente
 * que tu RAM": a miss replaces the least frequently used resident expert;
 * "Gemma 4 26B en ~2 GB de RAM ...", "La parte que se gana la confianza":
 * other cache policies were measured against it).  All share the waves,
 * the pinning of the current wave's experts and the empty-slot rule:
 *   LFU          victim = smallest (count, last_use, id); count = selections
 *                so far, kept across evictions
 *   LRU          victim = smallest (last_use, id)
 *   LFU_DECAY    LFU with counts halved (integer shift) at the start of every
 *                call whose step is a positive multiple of decay_period
 *   LFU_IN_CACHE LFU whose count of an expert restarts at 0 when evicted */
#define MOE_POLICY_LFU          0
#define MOE_POLICY_LRU          1
#define MOE_POLICY_LFU_DECAY    2
#define MOE_POLICY_LFU_IN_CACHE 3

/* int32 words of LFU state per layer: count[E], last_use[E], slot_of[E],
 * expert_in[S]. */
size_t moe_cache_state_words(const moe_dims *dims);

/* Cold start: counts and last-use 0, nothing resident, all slots empty.
 * Also drops any look-ahead blob staged for this cache (moe_layer_forward_next).
 * Enqueued on `stream`. */
int moe_cache_reset(moe_ctx *ctx, moe_slot_cache *cache, cudaStream_t stream);

/* Per-call plan result, copied to host memory when requested.  The caller
 * provides arrays of capacity >= min(T*K, n_experts) entries; one entry per
 * distinct expert of the call, ascending id. */
typedef struct moe_plan_trace {
    int32_t capacity;      /* in: length of the arrays below */
    int32_t n_distinct;    /* out */
    int32_t n_waves;       /* out */
    int32_t n_misses;      /* out */
    uint64_t h2d_bytes;    /* out: bytes copied from the store for this call */
    int32_t *expert;       /* out: expert id */
    int32_t *slot;         /* out: slot it occupies during its wave */
    int32_t *hit;          /* out: 1 resident, 0 miss */
    int32_t *victim;       /* out: evicted expert, or -1 */
    int32_t *wave;         /* out: wave index */
} moe_plan_trace;

/* LFU cache plan for T tokens' top-K ids ("TurboFieldfare ...", "Proceso de
 * generacion de tokens"; "El milagro ...", "Mas inteligente que tu RAM"):
 * counts the selections, marks hits, picks a slot for each miss (lowest empty
 * slot first, else evicts the resident expert with the smallest (count,
 * last_use, id) that the current wave does not use), records last_use =
 * step+1, and writes pair_slot[T][K] (dev int32, out).  Distinct experts are
 * planned in ascending id, in waves of at most n_slots.
 * When cache->store != NULL or trace != NULL the call is synchronous with
 * respect to the plan: it waits (bounded, MOE_ERR_TIMEOUT) until the plan
 * kernel has published the plan through the pinned mailbox, then, for a
 * single-wave plan, enqueues one cudaMemcpyAsync per miss (store -> slot) on
 * the context's side stream after all work already on `stream`, and makes
 * `stream` wait for those copies.  A plan with several waves copies nothing
 * (the fills must be interleaved with compute; moe_layer_forward does that).
 * cache == NULL is not allowed here. */
int moe_cache_plan(moe_ctx *ctx, moe_slot_cache *cache, const int32_t *ids, int T,
                   uint32_t step, int32_t *pair_slot, moe_plan_trace *trace,
                   cudaStream_t stream);

/* ---------------------------------------------------------- expert FFNs
 * Routed experts + combine for T tokens ("TurboFieldfare ...", "Proceso de
 * generacion de tokens": routed outputs are combined with the shared branch):
 *   y[t] = (y_in ? y_in[t] : 0) + sum_{k<top_k} gate_w[t][k] * FFN_{slot[t][k]}(x[t])
 *   FFN(x) = W_d (gelu_tanh(W_g x) * (W_u x)), fp32 accumulation
 *   x          dev bf16 bits [T][D]
 *   pair_slot  dev int32 [T][top_k], 0 <= slot < n_slot_range
 *   gate_w     dev fp32 [T][top_k]
 *   slot_base  dev: expert blob of slot s at slot_base + s*slot_stride
 *   d_ff       FFN width of the referenced experts (F, or FS for the shared
 *              expert passed as top_k = 1, pair_slot 0, gate_w 1)
 *   y_in       dev fp32 [T][D] or NULL; y dev fp32 [T][D] out (may equal y_in)
 *   y_bf16     dev bf16 bits [T][D] out, or NULL
 * 1 <= T <= 32 (dequantising GEMV kernels; moe_layer_forward runs batches on
 * the grouped tensor-core path instead).  With T = 1 a slot may appear more
 * than once in pair_slot (each selection is computed with its own weight).
 * Slot indices outside [0, n_slot_range) are clamped and MOE_ERR_RANGE is
 * recorded.  Uses context scratch; calls on one context must not overlap. */
int moe_expert_ffn(moe_ctx *ctx, const uint16_t *x, int T, int top_k, const int32_t *pair_slot,
                   const float *gate_w, const uint8_t *slot_base, size_t slot_stride,
                   int n_slot_range, int d_ff, const float *y_in, float *y, uint16_t *y_bf16,
                   cudaStream_t stream);

/* Routed experts + combine for ONE token without any device allocation, for
 * callers that may not allocate: code running inside another program's memory
 * budget (an engine that gives each plugin a fixed workspace and owns every
 * device allocation), or code on a latency-critical path where cudaMalloc and
 * cudaFree can synchronise the device.  Such callers cannot create a moe_ctx,
 * whose scratch is allocated; this entry point needs none.  (The pages have
 * no counterpart: their runtime is a single process that owns its memory.)
 * Computes, for T = 1,
 *   y = (y_in ? y_in : 0) + sum_{k<top_k} gate_w[k] * FFN_{pair_slot[k]}(x)
 * with the same kernels and arguments as moe_expert_ffn (x dev bf16 [d_model],
 * pair_slot dev int32 [top_k], gate_w dev fp32 [top_k], slot_base/slot_stride/
 * n_slot_range as there, y_in/y dev fp32 [d_model], y_bf16 dev bf16 or NULL).
 * Limits of the fixed scratch: d_model <= 2816 (multiple of 256), d_ff <= 2112,
 * top_k <= 8; larger sizes return MOE_ERR_ARG before any CUDA call.  A slot
 * may appear more than once in pair_slot: each selection is computed with its
 * own gate weight (the blob is streamed once per selection).
 * Scratch: a 4 MiB file-scope device array inside libmoe.so, present on every
 * GPU that loads the library until the process exits.  The FIRST call on each
 * device sets up that device (looks up the array's device address and the
 * kernels' launch shapes, with the device current).  Every call shares the
 * array and it keeps the last call's contents: calls whose work overlaps on
 * the GPU race, so issue them on one stream (or order them).  Errors: MOE_ERR_ARG (sizes, pointers),
 * MOE_ERR_CUDA (a launch or the set-up failed), MOE_ERR_STATE (the GPU has
 * more SMs than the scratch covers).  Slot indices out of range are clamped;
 * there is no status word to read back. */
int moe_expert_ffn_noalloc(int d_model, int d_ff, int top_k, const uint16_t *x, const int32_t *pair_slot,
                           const float *gate_w, const uint8_t *slot_base, size_t slot_stride,
                           int n_slot_range, const float *y_in, float *y, uint16_t *y_bf16,
                           cudaStream_t stream);

/* ----------------------------------------------------------- whole layer
 * Resident weights of one layer. */
typedef struct moe_layer_weights {
    const int8_t *router_q;        /* dev int8 [E][D] */
    const uint16_t *router_s;      /* dev binary16 [E][D/64] */
    const uint8_t *shared_blob;    /* dev blob of width d_ff_shared, or NULL */
    const uint8_t *experts;        /* dev: all E expert blobs (resident mode), or NULL */
    size_t expert_stride;          /* bytes between resident blobs */
} moe_layer_weights;

/* One MoE layer for T tokens ("Gemma 4 26B en ~2 GB de RAM ...", "Por que
 * funciona": the per-token loop; "TurboFieldfare ...", "Proceso de generacion
 * de tokens"): router -> top-K -> (cache plan -> miss copies on the side
 * stream, overlapped with the shared expert) -> routed experts -> combine
 *   y[t] = shared(x[t]) + sum_k gate_w[t][k] * expert_{ids[t][k]}(x[t]).
 * cache == NULL: resident mode, expert e read from W->experts + e*stride.
 * cache != NULL: experts are served from cache->slots; misses are copied from
 * cache->store (host-synchronous on the plan, see moe_cache_plan).
 * T = 1 with a MOE_SOURCE_HOST_DIRECT cache runs the whole layer as one
 * cooperative kernel (router, top-K, plan, shared and routed expert GEMVs,
 * combine; all CTAs resident, two bounded grid-wide barriers; the plan reaches
 * the host only when a trace is requested); so does T = 1 with resident
 * experts when the environment sets MOE_LAYER_KERNEL=1 (MOE_LAYER_KERNEL=0
 * never uses it).  Other one-token calls run the router, plan and dequantising
 * GEMV kernels; with a MOE_SOURCE_HOST cache the routed experts' kernels wait
 * for all of the call's copies through one event, or, when the environment
 * sets MOE_PER_MISS=1 at context creation, start at once and wait per expert
 * for a completion word written after that expert's copy (bounded:
 * MOE_ERR_TIMEOUT);
 * T >= moe_gemm_min_tokens() (a batched decode step or a prefill chunk) groups
 * the tokens by expert and runs the tcgen05 tensor-core grouped GEMM, one wave
 * of at most n_slots experts at a time.
 *   x dev bf16 [T][D]; bias dev fp32 [E] or NULL; y dev fp32 [T][D] out;
 *   y_bf16 dev bf16 [T][D] out or NULL; ids/gate_w dev [T][K] out or NULL;
 *   trace host, or NULL. */
int moe_layer_forward(moe_ctx *ctx, const moe_layer_weights *W, moe_slot_cache *cache,
                      const uint16_t *x, int T, uint32_t step, const float *bias,
                      float *y, uint16_t *y_bf16, int32_t *ids, float *gate_w,
                      moe_plan_trace *trace, cudaStream_t stream);

/* ------------------------------------------------- look-ahead prefetch
 * Opt-in; off unless moe_prefetch_configure gave buffers.  The pages disagree
 * on whether expert loads can be started a layer early: one says the router
 * gives a layer of warning ("Gemma 4 26B en ~2 GB de RAM ...", section "Por
 * que pread y no mmap"); the discussion threads consider speculative expert
 * prefetch hard, because a layer's routing depends on the previous layers'
 * output, and note that reading mispredicted experts costs the bandwidth the
 * real misses need ("Show HN: Motor de codigo abierto ...", section
 * "Direcciones futuras e ideas de investigacion"; "TurboFieldfare: motor open
 * source ...", section "Comentarios de Hacker News").  This path makes the trade measurable:
 * while layer l runs on x, layer l+1's router is evaluated on the same x on a
 * separate stream; after layer l's own miss copies, up to n_buffers of its
 * predicted experts that layer l+1's cache does not hold (as far as the host
 * has seen from the plans it read) are copied from layer l+1's host store into
 * HBM staging buffers.  When layer l+1 runs, a miss whose blob is staged is
 * filled by a device-to-device copy instead of a host copy, issued on the
 * look-ahead stream so that the host copies of its other misses start at once
 * (the layer's routed experts wait for both by event).  The cache plan,
 * the trace and the outputs are exactly those of moe_layer_forward; only
 * where a missed blob is copied from changes.
 *
 * A staged blob is a copy of the host store taken when it was prefetched: the
 * store must not be rewritten while buffers are configured, or the caller must
 * drop the staged blobs first (moe_prefetch_configure, or moe_cache_reset of
 * the cache they were fetched for).
 *
 * Sets the number of HBM staging buffers (0..16; 0 turns prefetch off and
 * frees them), one expert blob each, and drops every staged blob.  Waits for
 * the context's copy streams.
 * MOE_ERR_ARG (count out of range), MOE_ERR_CUDA (allocation failed). */
int moe_prefetch_configure(moe_ctx *ctx, int n_buffers);

/* Bytes copied into the staging buffers so far, and the part of them later
 * used to fill a miss; issued - used is the bandwidth spent on wrong guesses. */
int moe_prefetch_stats(const moe_ctx *ctx, uint64_t *issued_bytes, uint64_t *used_bytes);

/* The layer after the one being run: its weights, its cache (which must have
 * a host store, source MOE_SOURCE_HOST) and its router bias (or NULL). */
typedef struct moe_next_layer {
    const moe_layer_weights *W;
    moe_slot_cache *cache;
    const float *bias;
    /* the layer after this one, or NULL: when none of this layer's predicted
     * experts is missing from its cache (nothing to stage for it), a free
     * buffer stages the top predicted miss of `after` instead (its router is
     * also evaluated on the current input); after->after is ignored */
    const struct moe_next_layer *after;
} moe_next_layer;

/* moe_layer_forward, plus the look-ahead prefetch of `next` when T = 1, buffers
 * are configured and next->cache has a host store; otherwise (next NULL or any
 * of these missing) exactly moe_layer_forward.  The staged blobs are matched to
 * a later miss by (cache state, store, expert); a blob is kept until the
 * layer it was staged for has run (or its cache is reset), and blobs for any
 * layer other than next and next->after are dropped.  The host waits for the prediction router
 * (issued before this layer's own router) after queueing this layer's copies.
 * Errors: those of moe_layer_forward, and next->cache is checked as any cache. */
int moe_layer_forward_next(moe_ctx *ctx, const moe_layer_weights *W, moe_slot_cache *cache,
                           const uint16_t *x, int T, uint32_t step, const float *bias,
                           float *y, uint16_t *y_bf16, int32_t *ids, float *gate_w,
                           moe_plan_trace *trace, const moe_next_layer *next, cudaStream_t stream);

/* ------------------------------------------------------ decode attention
 * The other per-token kernel of the layer loop ("TurboFieldfare: motor open
 * source ...", section "Proceso de generacion de tokens": decode attention is an
 * exact split-K/V method over an fp16 KV cache held as a bounded ring for the
 * sliding-window layers and as linear storage for the full-attention layers;
 * "Gemma 4 26B en ~2 GB de RAM ...", section "Por que funciona: el A4B del
 * nombre", the same cache).  For one token:
 *   o[h] = sum_p softmax_p(scale * q[h] . k[g][slot(p)]) v[g][slot(p)],
 *   g = h / (n_heads_q / n_heads_kv) (consecutive query heads share a KV head),
 * over the cache's newest min(n_tokens, capacity) positions, position p held in
 * slot p mod capacity (a ring; a linear cache has capacity >= n_tokens, so the
 * attended slots are 0 .. n_tokens-1).  Since attention does not depend on the
 * order of the positions, the call attends to slots 0 .. min(n_tokens,
 * capacity)-1.  The slots are split into parts across CTAs; each part keeps
 * its maximum, exponential sum and unnormalised value sum, and the parts are
 * merged exactly (by rescaling), in a fixed order, so results are
 * reproducible bit for bit.
 *   q        dev bf16 [n_heads_q][head_dim]
 *   k_cache  dev binary16 [n_heads_kv][capacity][head_dim]; v_cache likewise
 *   o        dev fp32 [n_heads_q][head_dim] out
 *   scale    the score scale (e.g. 1/sqrt(head_dim)), finite and > 0
 *   workspace dev, >= moe_attn_workspace_bytes(n_heads_q, head_dim) bytes,
 *            ZEROED by the caller before its first use; each call leaves it
 *            ready for the next one.  Calls sharing a workspace must not overlap
 *            on the GPU (issue them on one stream).
 * Supported: head_dim in {64, 128, 256, 512}; n_heads_q / n_heads_kv in
 * {1, 2, 4, 8} with (head_dim / 32) * group <= 32; n_heads_kv <= 64; every
 * pointer 16-byte aligned.  One launch, no host synchronisation, capturable in a
 * CUDA graph.  Errors: MOE_ERR_ARG (sizes, n_tokens < 1, pointers, alignment,
 * workspace too small), MOE_ERR_CUDA (launch failed). */
int moe_attn_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                    int n_heads_q, int n_heads_kv, int head_dim, int capacity, int n_tokens,
                    float scale, float *o, void *workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/* Workspace bytes moe_attn_decode needs for these sizes (a per-KV-head ticket
 * and each part's partial results); 0 for sizes below 1.  Host-only. */
size_t moe_attn_workspace_bytes(int n_heads_q, int head_dim);

/* ------------------------------------------------------ instrumentation */
#define MOE_PROF_ROUTER    0   /* moe_router_topk kernel */
#define MOE_PROF_PLAN      1   /* cache-plan kernel */
#define MOE_PROF_WORKLIST  2   /* work-list builder kernel */
#define MOE_PROF_GATE_UP   3   /* expert gate/up GEMV kernel */
#define MOE_PROF_DOWN      4   /* expert down GEMV + combine kernel */
#define MOE_PROF_HARNESS   5   /* harness kernels (residual/RMS, bf16 widening) */
#define MOE_PROF_H2D       6   /* one batch of miss copies on the side stream */
#define MOE_PROF_LAYER     7   /* one-token layer kernel (the whole layer) */
#define MOE_PROF_KINDS     8

/* Kernel timing for benchmarks.  While enabled, the context records a pair of
 * CUDA events on the launching stream around every kernel it launches (and
 * around each batch of miss copies on its side stream), tagged by the kinds
 * above.  Disabled by default (no events recorded).  Host-only. */
int moe_ctx_profile(moe_ctx *ctx, int enable);

/* Synchronises on every recorded event and writes, per kind (arrays of
 * MOE_PROF_KINDS entries, host memory), the summed elapsed milliseconds and
 * the number of intervals since the previous read; then clears the records.
 * MOE_ERR_CUDA if an event could not be read. */
int moe_ctx_profile_read(moe_ctx *ctx, double *total_ms, uint64_t *count);

/* Cache counters kept on the device by the plan kernel and the one-token
 * layer kernel, for every call with a slot cache: calls, hits and misses
 * (distinct experts), bytes of missed experts, experts also chosen at the
 * previous step of that cache (last_use == step) and at one of the two
 * previous steps, and distinct experts planned (the denominator of the two
 * repeat counts).  Reading them needs no host round trip per call. */
#define MOE_STAT_CALLS        0
#define MOE_STAT_HITS         1
#define MOE_STAT_MISSES       2
#define MOE_STAT_MISS_BYTES   3
#define MOE_STAT_REPEAT_PREV  4
#define MOE_STAT_REPEAT_PREV2 5
#define MOE_STAT_PLANNED      6
#define MOE_STATS             8

/* Copies the counters (MOE_STATS words) into out (host) after the work
 * already on `stream`; waits for it.  MOE_ERR_CUDA on a failed copy. */
int moe_ctx_stats(moe_ctx *ctx, cudaStream_t stream, uint64_t *out);

/* Zeroes the counters, enqueued on `stream`. */
int moe_ctx_stats_reset(moe_ctx *ctx, cudaStream_t stream);

/* ------------------------------------------------------ harness helpers
 * Not part of the method: the residual/RMS step a test or benchmark puts
 * between layers so that layer l+1's routing depends on layer l's output.
 *   r[t] += y[t] (fp32, in place);  x_next[t] = bf16(r[t] / rms(r[t])),
 *   rms = sqrt(mean(r^2) + 1e-6).   r dev fp32 [T][D], y dev fp32 [T][D],
 *   x_next dev bf16 [T][D]; r and y 16-byte aligned, x_next 8-byte aligned
 *   (MOE_ERR_ARG otherwise).  One launch. */
int moe_residual_rmsnorm(moe_ctx *ctx, float *r, const float *y, uint16_t *x_next, int T,
                         cudaStream_t stream);

/* bf16 -> fp32 widening copy (harness: initialises the residual stream). */
int moe_bf16_to_f32(moe_ctx *ctx, const uint16_t *x, float *out, size_t n, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
