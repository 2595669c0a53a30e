// noalloc.cu -- moe_expert_ffn_noalloc: the routed-expert FFN + combine for
// one token, for callers that are not allowed to allocate device memory.
//
// Who needs this: code that runs inside another program's memory budget (a
// serving engine or inference runtime that hands each plugin a fixed workspace and
// owns every device allocation itself), and code on a latency-critical path,
// where cudaMalloc/cudaFree may synchronise the whole device and take an
// unbounded time.  Such callers cannot create a moe_ctx (it allocates its
// scratch), so this entry point keeps its scratch in one file-scope device
// array instead and allocates nothing, ever.
//
// The scratch (kNoAllocScratchBytes, 4 MiB) lives in a `static __device__`
// array: every GPU that loads the library holds it until the process exits.
// Its name is only a host-side stand-in; the device address is obtained once
// per device with cudaGetSymbolAddress (with that device current) on the
// first call made on it.  All calls share the array and it keeps the last
// call's contents, so calls whose kernels overlap on the GPU race; the parts
// that must start at zero are cleared on the caller's stream every call.
#include <mutex>

#include "common.cuh"
#include "ffn.cuh"

namespace moe {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;

// The scratch itself: file scope, one copy per device, held until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kNoAllocMaxD = 2816;   // largest d_model
constexpr int kNoAllocMaxF = 2112;   // largest d_ff
constexpr int kNoAllocMaxK = 8;      // largest top_k
constexpr int kMaxDevices = 64;

struct Layout {
    size_t status, wl, entries, rows, h, partials_gu, counters_gu, partials_dn, counters_dn, total;
};

struct DeviceState {
    bool ready = false;
    unsigned char* base = nullptr;  // device address of g_noalloc_scratch
    GemvShapes shapes{};
    Layout lay{};
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

size_t up256(size_t b) { return (b + 255) / 256 * 256; }

// Offsets of every scratch region for the largest supported shapes and the
// device's persistent grid; total must fit the array.
Layout make_layout(const GemvShapes& sh) {
    Layout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += up256(bytes); return at; };
    const int max_entries = kNoAllocMaxK;  // one token: at most top_k distinct slots
    const int tiles_dn = kNoAllocMaxD / kChunkRows;
    const int ns_dn = kNoAllocMaxF / down_ks(kNoAllocMaxF);
    L.status = take(sizeof(int));
    L.wl = take(sizeof(WorkList));
    L.entries = take(sizeof(FfnEntry) * max_entries);
    L.rows = take(sizeof(FfnRow) * (kNoAllocMaxK + 1));
    L.h = take(sizeof(float) * size_t(kNoAllocMaxK) * kNoAllocMaxF);
    L.partials_gu = take(sizeof(float) * size_t(2) * sh.gu[0].grid * kMaxRows * 32);
    L.counters_gu = take(sizeof(int) * size_t(max_entries) * (kNoAllocMaxF / 16));
    L.partials_dn = take(sizeof(float) * size_t(max_entries) * tiles_dn * ns_dn * kMaxRows * 32);
    L.counters_dn = take(sizeof(int) * size_t(tiles_dn));
    L.total = o;
    return L;
}

// First call on a device: device address of the scratch array and the launch
// shapes.  Runs under the mutex with the caller's device current.
int setup_device(int dev, DeviceState* st) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return MOE_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
    GemvShapes sh;
    if (ffn_shapes_one_row(kNoAllocMaxD, kNoAllocMaxK * kNoAllocMaxF, 1, sms, &sh) != cudaSuccess) return MOE_ERR_CUDA;
    const Layout L = make_layout(sh);
    if (L.total > kNoAllocScratchBytes) return MOE_ERR_STATE;  // a GPU with more SMs than the array covers
    st->base = static_cast<unsigned char*>(p);
    st->shapes = sh;
    st->lay = L;
    st->ready = true;
    return MOE_OK;
}

bool aligned(const void* q, size_t a) { return (reinterpret_cast<uintptr_t>(q) % a) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_expert_ffn_noalloc(int d_model, int d_ff, int top_k, const uint16_t* x,
                                      const int32_t* pair_slot, const float* gate_w, const uint8_t* slot_base,
                                      size_t slot_stride, int n_slot_range, const float* y_in, float* y,
                                      uint16_t* y_bf16, cudaStream_t stream) {
    // sizes beyond what the fixed scratch holds are rejected before any CUDA call
    if (d_model <= 0 || d_model % 256 || d_model > kNoAllocMaxD) return MOE_ERR_ARG;
    if (d_ff <= 0 || d_ff % 64 || d_ff > kNoAllocMaxF || (d_ff > 704 && d_ff % 704)) return MOE_ERR_ARG;
    if (top_k < 1 || top_k > kNoAllocMaxK) return MOE_ERR_ARG;
    if (n_slot_range < 1 || n_slot_range > 1024) return MOE_ERR_ARG;
    if (!x || !pair_slot || !gate_w || !slot_base || !y) return MOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(slot_base, 256) || slot_stride % 256 || !aligned(y, 16)) return MOE_ERR_ARG;
    if (y_in && !aligned(y_in, 16)) return MOE_ERR_ARG;
    if (n_slot_range > 1 && slot_stride < blob_bytes(d_model, d_ff)) return MOE_ERR_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_STATE;
    DeviceState* st = &g_dev[dev];
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!st->ready) {
            const int r = setup_device(dev, st);
            if (r != MOE_OK) return r;
        }
    }
    if (ffn_ensure_one_row_smem(st->shapes) != cudaSuccess) return MOE_ERR_CUDA;
    unsigned char* b = st->base;
    const Layout& L = st->lay;
    int* status = reinterpret_cast<int*>(b + L.status);
    int* counters_gu = reinterpret_cast<int*>(b + L.counters_gu);
    int* counters_dn = reinterpret_cast<int*>(b + L.counters_dn);
    // tile counters and the status word start every call at zero
    if (cudaMemsetAsync(status, 0, sizeof(int), stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(counters_gu, 0, sizeof(int) * size_t(kNoAllocMaxK) * (kNoAllocMaxF / 16), stream) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaMemsetAsync(counters_dn, 0, sizeof(int) * size_t(kNoAllocMaxD / kChunkRows), stream) != cudaSuccess)
        return MOE_ERR_CUDA;

    WorkListArgs wa;
    wa.T = 1;
    wa.K = top_k;
    wa.pair_slot = pair_slot;
    wa.pair_wave = nullptr;
    wa.wave = 0;
    wa.gate_w = gate_w;
    wa.slot_base = slot_base;
    wa.slot_stride = slot_stride;
    wa.n_slot_range = n_slot_range;
    wa.F = d_ff;
    wa.shared_blob = nullptr;
    wa.FS = 0;
    wa.h_shared_off = 0;
    wa.D = d_model;
    wa.wl = reinterpret_cast<WorkList*>(b + L.wl);
    wa.entries = reinterpret_cast<FfnEntry*>(b + L.entries);
    wa.rows = reinterpret_cast<FfnRow*>(b + L.rows);
    wa.status = status;
    if (launch_build_worklist(wa, true, stream) != cudaSuccess) return MOE_ERR_CUDA;

    GemvLaunch G;
    G.wl = wa.wl;
    G.entries = wa.entries;
    G.rows = wa.rows;
    G.x = x;
    G.h = reinterpret_cast<float*>(b + L.h);
    G.y_in = y_in;
    G.y = y;
    G.y_bf16 = y_bf16;
    G.partials_gu = reinterpret_cast<float*>(b + L.partials_gu);
    G.counters_gu = counters_gu;
    G.partials_dn = reinterpret_cast<float*>(b + L.partials_dn);
    G.counters_dn = counters_dn;
    G.D = d_model;
    G.rmax = 1;
    G.list_cap = kNoAllocMaxK;  // entries capacity (rows hold one more)
    G.max_tiles_gu = top_k * (d_ff / 16);
    G.shapes = &st->shapes;
    G.status = status;
    return launch_ffn(G, stream, nullptr, nullptr) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
