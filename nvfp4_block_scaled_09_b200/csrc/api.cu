// api.cu -- host side of the C ABI: device registry, status word, launch
// accounting, status strings and the whole-layer orchestration.
#include <atomic>
#include <mutex>

#include "common.cuh"

// One status word per device context; kernels latch error bits into it.
__device__ uint32_t g_nvfp4_device_status;
// Work counters of the grouped GEMM's dynamic schedule: launches draw the slots in turn (two words each,
// left at zero by the launch's last CTA), so GEMMs in flight on different streams use different slots.
constexpr int kSchedSlots = 64;
__device__ uint32_t g_nvfp4_sched[2 * kSchedSlots];

namespace nvfp4 {

static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint64_t> g_timeout_ns{1000000000ull};
static std::atomic<uint32_t> g_debug_flags{0};

struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    int smem_optin = 0;
    uint32_t* status = nullptr;
    uint32_t* sched = nullptr;
    std::atomic<uint32_t> sched_next{0};
};

constexpr int kMaxDevices = 64;
static DeviceInfo g_devices[kMaxDevices];
static std::mutex g_mutex;

static DeviceInfo* device_info() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& di = g_devices[d];
    if (!di.ready) {
        if (cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return nullptr;
        if (cudaDeviceGetAttribute(&di.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess)
            return nullptr;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_nvfp4_device_status) != cudaSuccess) return nullptr;
        di.status = static_cast<uint32_t*>(p);
        if (cudaGetSymbolAddress(&p, g_nvfp4_sched) != cudaSuccess) return nullptr;
        di.sched = static_cast<uint32_t*>(p);
        di.ready = true;
    }
    return &di;
}

uint32_t* status_word_ptr() {
    DeviceInfo* di = device_info();
    return di ? di->status : nullptr;
}
uint32_t* sched_counter_slot() {
    DeviceInfo* di = device_info();
    if (!di) return nullptr;
    return di->sched + 2 * (di->sched_next.fetch_add(1u) % kSchedSlots);
}
uint64_t wait_timeout_ns() { return g_timeout_ns.load(); }
uint32_t debug_flags() { return g_debug_flags.load(); }
void count_launch(int n) { g_launches.fetch_add((uint64_t)n); }
int device_sm_count() {
    DeviceInfo* di = device_info();
    return di ? di->sm_count : 1;
}
int device_smem_optin() {
    DeviceInfo* di = device_info();
    return di ? di->smem_optin : -1;
}
nvfp4_status check_launch() { return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

static inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace nvfp4

using namespace nvfp4;

extern "C" const char* nvfp4_status_string(nvfp4_status s) {
    switch (s) {
        case NVFP4_OK: return "NVFP4_OK";
        case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
        case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED";
        case NVFP4_ERR_UNSUPPORTED_SHAPE: return "NVFP4_ERR_UNSUPPORTED_SHAPE";
        case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE";
        case NVFP4_ERR_SMEM_BUDGET: return "NVFP4_ERR_SMEM_BUDGET";
        case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
        case NVFP4_ERR_DEVICE_TIMEOUT: return "NVFP4_ERR_DEVICE_TIMEOUT";
        case NVFP4_ERR_DEVICE_INPUT: return "NVFP4_ERR_DEVICE_INPUT";
    }
    return "NVFP4_ERR_UNKNOWN";
}

extern "C" void nvfp4_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns == 0 ? 1 : ns); }
extern "C" uint64_t nvfp4_get_wait_timeout_ns(void) { return g_timeout_ns.load(); }
extern "C" void nvfp4_debug_set_flags(uint32_t flags) { g_debug_flags.store(flags & kCtlStallProducer); }
extern "C" uint64_t nvfp4_launch_count(void) { return g_launches.load(); }

extern "C" nvfp4_status nvfp4_get_device_status(nvfp4_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NVFP4_ERR_CUDA;
    DeviceInfo* di = device_info();
    if (!di) return NVFP4_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, di->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
    const uint32_t zero = 0;
    if (cudaMemcpy(di->status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (v & kStatusTimeout) return NVFP4_ERR_DEVICE_TIMEOUT;
    if (v & kStatusBadInput) return NVFP4_ERR_DEVICE_INPUT;
    return NVFP4_OK;
}

extern "C" nvfp4_status moe_layer_workspace_layout(int32_t T, int32_t k, int32_t E, int64_t H, int64_t I,
                                                   nvfp4_layer_workspace* L) {
    if (!L || T <= 0 || k <= 0 || E <= 0 || H <= 0 || I <= 0) return NVFP4_ERR_INVALID_ARG;
    const size_t A = 256;
    const size_t R = (size_t)T * (size_t)k;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes, A);
        return at;
    };
    L->q_x = take((size_t)T * H / 2);
    L->sf_x = take((size_t)T * H / 16);
    L->g_x = take(sizeof(float));
    L->q_perm = take(R * H / 2);
    L->sf_perm = take(R * ((size_t)H + 255) / 256 * 16);   // K-stage slabs (the last one zero-padded)
    L->offsets = take(sizeof(int32_t) * ((size_t)E + 1));
    L->perm_src = take(sizeof(int32_t) * R);
    L->inv_perm = take(sizeof(int32_t) * R);
    L->h = take(R * I * 2);
    L->q_h = take(R * I / 2);
    L->sf_h = take(R * ((size_t)I + 255) / 256 * 16);
    L->g_h = take(sizeof(float));
    L->amax_h = take(sizeof(uint32_t));
    L->fin_counters = take(moe_finalize_counters_size(T, H));
    L->y = take(R * H * 2);
    size_t scratch = moe_permute_workspace_size(T, k, E);
    const size_t qx = nvfp4_quantize_workspace_size(T, H), qh = nvfp4_quantize_workspace_size((int64_t)R, I);
    if (qx > scratch) scratch = qx;
    if (qh > scratch) scratch = qh;
    if (scratch < 1024) scratch = 1024;   // the fused quantize-permute's amax partials (up to 148 words)
    L->scratch = take(scratch);
    L->topk_ids = take(sizeof(int32_t) * (size_t)T * (size_t)k);
    L->topk_w = take(sizeof(float) * (size_t)T * (size_t)k);
    L->total = o;
    return NVFP4_OK;
}

extern "C" size_t moe_layer_workspace_size(int32_t T, int32_t k, int32_t E, int64_t H, int64_t I) {
    nvfp4_layer_workspace L;
    if (moe_layer_workspace_layout(T, k, E, H, I, &L) != NVFP4_OK) return 0;
    return L.total;
}

// L2 prefetch hints of the layer: while the latency-bound kernel before a GEMM runs (the front before gate/up,
// quantize(h) before down), it pulls the start of that GEMM's packed weights into L2 -- the first experts' tiles,
// which the GEMM's schedule takes first. Only for decode-sized batches (under 32 rows per expert: the narrow-tile
// GEMMs that stream their weights at HBM rate). Measured on B200, decode layer (moe_layer_nvfp4 back to back,
// same box): 0.824 -> 0.816 ms with 96 + 48 MB (32 + 16 MB: 0.820, 64 + 32 MB: 0.817, 112 MB no better); the
// Zipf layer (32 rows per expert) did not gain.
constexpr size_t kLayerPrefetchGateUp = (size_t)96 << 20;
constexpr size_t kLayerPrefetchDown = (size_t)48 << 20;
extern "C" void moe_layer_l2_prefetch_bytes(int32_t T, int32_t k, int32_t E, int64_t H, int64_t I, size_t* gate_up,
                                            size_t* down) {
    const int64_t R = (int64_t)T * k;
    const bool streams = T > 0 && k > 0 && E > 0 && H > 0 && I > 0 && R < 32 * (int64_t)E;
    const size_t w13 = streams ? (size_t)E * (size_t)(2 * I) * (size_t)(H / 2 + H / 16) : 0;
    const size_t w2 = streams ? (size_t)E * (size_t)H * (size_t)(I / 2 + I / 16) : 0;
    if (gate_up) *gate_up = w13 < kLayerPrefetchGateUp ? w13 : kLayerPrefetchGateUp;
    if (down) *down = w2 < kLayerPrefetchDown ? w2 : kLayerPrefetchDown;
}

// The layer; with `logits` non-null the router first writes the routing into the workspace.
// permute.cu: nvfp4_quantize + moe_permute with caller-given token-order buffers and scratch
namespace nvfp4 {
nvfp4_status quantize_permute(const uint16_t* x, int32_t T, int64_t H, const int32_t* topk_ids, int32_t k, int32_t E,
                              uint8_t* q_perm, uint8_t* sf_perm, nvfp4_sf_layout layout, float* g_x,
                              int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm, uint8_t* q_x,
                              uint8_t* sf_x, void* scratch, size_t scratch_bytes, cudaStream_t s,
                              const void* l2_next, size_t l2_next_bytes);
}  // namespace nvfp4

static nvfp4_status layer(const uint16_t* x, const float* logits, const int32_t* topk_ids, const float* topk_w,
                          int32_t T, int32_t k, int32_t E, int64_t H, int64_t I, const uint8_t* w13_packed,
                          const float* w13_gscale, const uint8_t* w2_packed, const float* w2_gscale, uint16_t* out,
                          void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    if (!x || !w13_packed || !w13_gscale || !w2_packed || !w2_gscale || !out) return NVFP4_ERR_INVALID_ARG;
    if (logits == nullptr && (!topk_ids || !topk_w)) return NVFP4_ERR_INVALID_ARG;
    nvfp4_layer_workspace L;
    nvfp4_status st = moe_layer_workspace_layout(T, k, E, H, I, &L);
    if (st != NVFP4_OK) return st;
    if (!ws || ws_bytes < L.total) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_MISALIGNED;
    if ((st = nvfp4_can_implement(2 * I, H, E, NVFP4_EPI_SWIGLU)) != NVFP4_OK) return st;
    if ((st = nvfp4_can_implement(H, I, E, NVFP4_EPI_NONE)) != NVFP4_OK) return st;
    if (logits != nullptr) {
        if (E > 1024 || k > 32 || k > E) return NVFP4_ERR_UNSUPPORTED_SHAPE;
        if ((uintptr_t)logits & 3u) return NVFP4_ERR_MISALIGNED;
    }
    uint8_t* b = static_cast<uint8_t*>(ws);
    const int64_t R = (int64_t)T * k;
    uint8_t* q_x = b + L.q_x;
    uint8_t* sf_x = b + L.sf_x;
    float* g_x = reinterpret_cast<float*>(b + L.g_x);
    uint8_t* q_perm = b + L.q_perm;
    uint8_t* sf_perm = b + L.sf_perm;
    int32_t* off = reinterpret_cast<int32_t*>(b + L.offsets);
    int32_t* perm_src = reinterpret_cast<int32_t*>(b + L.perm_src);
    int32_t* inv_perm = reinterpret_cast<int32_t*>(b + L.inv_perm);
    uint16_t* h = reinterpret_cast<uint16_t*>(b + L.h);
    uint8_t* q_h = b + L.q_h;
    uint8_t* sf_h = b + L.sf_h;
    float* g_h = reinterpret_cast<float*>(b + L.g_h);
    uint32_t* amax_h = reinterpret_cast<uint32_t*>(b + L.amax_h);
    uint16_t* y = reinterpret_cast<uint16_t*>(b + L.y);
    void* scratch = b + L.scratch;
    const size_t scratch_bytes = L.topk_ids - L.scratch;

    // the gate/up GEMM raises amax_h; it starts from 0, and so do the fused combine's counters right after it
    // (one memset before the first kernel, so that every kernel boundary after it keeps its programmatic
    // launch)
    if (cudaMemsetAsync(amax_h, 0, L.fin_counters + moe_finalize_counters_size(T, H) - L.amax_h,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (logits != nullptr) {
        int32_t* ids_ws = reinterpret_cast<int32_t*>(b + L.topk_ids);
        float* w_ws = reinterpret_cast<float*>(b + L.topk_w);
        if ((st = moe_route_topk(logits, T, E, k, ids_ws, w_ws, stream))) return st;
        topk_ids = ids_ws;
        topk_w = w_ws;
    }
    // the latency-bound kernel before each GEMM pulls the start of its weights into L2 (decode-sized batches)
    size_t pf13 = 0, pf2 = 0;
    moe_layer_l2_prefetch_bytes(T, k, E, H, I, &pf13, &pf2);
    // x quantised straight into expert order (small batches never write its codes in token order)
    if ((st = quantize_permute(x, T, H, topk_ids, k, E, q_perm, sf_perm, NVFP4_SF_KSTAGE, g_x, off, perm_src,
                               inv_perm, q_x, sf_x, scratch, scratch_bytes, reinterpret_cast<cudaStream_t>(stream),
                               w13_packed, pf13)))
        return st;
    if ((st = moe_grouped_gemm_nvfp4_amax(q_perm, sf_perm, g_x, w13_packed, w13_gscale, off, E, R, 2 * I, H,
                                          NVFP4_EPI_SWIGLU, h, amax_h, stream)))
        return st;
    if ((st = nvfp4_quantize_from_amax_prefetch(h, R, I, amax_h, q_h, sf_h, g_h, NVFP4_SF_KSTAGE, w2_packed, pf2,
                                                stream)))
        return st;
    // the down GEMM, then the combine as its own kernel: measured on B200 faster than the down GEMM with
    // the combine fused into its epilogue (moe_grouped_gemm_nvfp4_finalize gives the same bits) on the
    // decode, Zipf and prefill layers
    if ((st = moe_grouped_gemm_nvfp4(q_h, sf_h, g_h, w2_packed, w2_gscale, off, E, R, H, I, NVFP4_EPI_NONE, y,
                                     stream)))
        return st;
    return moe_unpermute_combine(y, inv_perm, topk_w, T, k, H, out, stream);
}

extern "C" nvfp4_status moe_layer_nvfp4(const uint16_t* x, const int32_t* topk_ids, const float* topk_w, int32_t T,
                                        int32_t k, int32_t E, int64_t H, int64_t I, const uint8_t* w13_packed,
                                        const float* w13_gscale, const uint8_t* w2_packed, const float* w2_gscale,
                                        uint16_t* out, void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    if (!topk_ids || !topk_w) return NVFP4_ERR_INVALID_ARG;
    return layer(x, nullptr, topk_ids, topk_w, T, k, E, H, I, w13_packed, w13_gscale, w2_packed, w2_gscale, out, ws,
                 ws_bytes, stream);
}

extern "C" nvfp4_status moe_layer_nvfp4_from_logits(const uint16_t* x, const float* logits, int32_t T, int32_t k,
                                                    int32_t E, int64_t H, int64_t I, const uint8_t* w13_packed,
                                                    const float* w13_gscale, const uint8_t* w2_packed,
                                                    const float* w2_gscale, uint16_t* out, void* ws, size_t ws_bytes,
                                                    nvfp4_stream_t stream) {
    if (!logits) return NVFP4_ERR_INVALID_ARG;
    return layer(x, logits, nullptr, nullptr, T, k, E, H, I, w13_packed, w13_gscale, w2_packed, w2_gscale, out, ws,
                 ws_bytes, stream);
}
