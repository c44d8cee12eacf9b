// C ABI of the fused MoE FFN layer (declared in include/mmoe.h): handle,
// workspace, weight loading and the stream-ordered forward pass.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "mmoe.h"
#include "mmoe_internal.cuh"

using namespace mmoe;

namespace {

thread_local std::string g_err;

mmoe_status fail(mmoe_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
mmoe_status fail(mmoe_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

mmoe_status cuda_fail(cudaError_t e, const char* what) {
    return fail(e == cudaErrorMemoryAllocation ? MMOE_ERR_OOM : MMOE_ERR_CUDA, "%s: %s (%s)", what,
                cudaGetErrorString(e), cudaGetErrorName(e));
}

#define MMOE_CUDA(call, what)                          \
    do {                                               \
        cudaError_t e_ = (call);                       \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

// Makes the handle's device current for the scope and restores the caller's.
struct DeviceGuard {
    int prev = -1;
    bool ok = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

// mmoe_forward_host splits a batch of T tokens into n = min(kHostChunksMax,
// T / kHostChunkMinTokens) chunks (boundaries on multiples of 128 tokens; for
// n >= 3 the first and last chunks are a third of the others), so that the
// copies of one chunk overlap the layer on another.  Every token's output
// depends on that token alone, so the split leaves y unchanged.
constexpr int kHostChunksMax = 4;
constexpr int64_t kHostChunkMinTokens = 8192;

// Chunk boundaries of a T-token host-buffer forward: bound[0] = 0 < ... <
// bound[n] = T (T > 0), chunk weights 1, 3, ..., 3, 1 for n >= 3.  Returns n.
int host_chunk_bounds(int64_t T, int64_t (&bound)[kHostChunksMax + 1]) {
    const int nch = (int)std::max<int64_t>(1, std::min<int64_t>(kHostChunksMax, T / kHostChunkMinTokens));
    const int64_t wsum = nch < 3 ? nch : 3 * nch - 4;
    int64_t wacc = 0;
    bound[0] = 0;
    for (int i = 0; i < nch; ++i) {
        wacc += (nch < 3 || i == 0 || i == nch - 1) ? 1 : 3;
        bound[i + 1] = i == nch - 1 ? T : (T * wacc / wsum) / 128 * 128;
    }
    return nch;
}

}  // namespace

struct mmoe_handle {
    mmoe_config cfg;
    int device = 0;
    int hmax = 0;
    int64_t max_tokens = 0;
    bool loaded = false;
    int64_t last_T = -1;
    // weights (interchange layout)
    float* w_router = nullptr;
    float* router_bias = nullptr;
    uint16_t* w_router_split = nullptr;  // tensor-core router pieces (when d_model % 64 == 0)
    uint8_t* w_gate_up = nullptr;
    float* s_gate_up = nullptr;
    uint8_t* w_down = nullptr;
    float* s_down = nullptr;
    size_t n_gu_bytes = 0, n_gu_scales = 0, n_d_bytes = 0, n_d_scales = 0;
    // workspace
    int8_t* xq = nullptr;
    float* sx = nullptr;
    float* logits = nullptr;
    int32_t* idx = nullptr;
    float* gate = nullptr;
    int32_t* chunk_cnt = nullptr;
    int32_t* chunk_base = nullptr;
    int32_t* offsets = nullptr;
    int32_t* counts = nullptr;
    int32_t* tiles = nullptr;
    int32_t* tile_count = nullptr;
    int32_t* row_src = nullptr;
    float* row_gate = nullptr;
    int32_t* slot_row = nullptr;
    float* act = nullptr;
    int8_t* hq = nullptr;
    float* sh = nullptr;
    float* obuf = nullptr;
    uint16_t* x_stage = nullptr;
    float* y_stage = nullptr;
    // mmoe_forward_host: copy streams and the events that order chunks against the compute stream
    cudaStream_t s_h2d = nullptr, s_d2h = nullptr;
    cudaEvent_t ev_start = nullptr, ev_done = nullptr;
    cudaEvent_t ev_in[kHostChunksMax] = {}, ev_out[kHostChunksMax] = {};
    // tensor-core path: kind (kTcF16, kTcI8 or kTcNone), pre-tiled weights, f16 codes, tensor maps of the
    // activation / SwiGLU codes, error flag and the limit of the bounded waits
    int tc_kind = kTcNone;
    uint8_t* w_gate_up_t = nullptr;
    float* s_gate_up_t = nullptr;
    uint8_t* w_down_t = nullptr;
    float* s_down_t = nullptr;
    uint16_t* w_gate_up_f16 = nullptr;
    uint16_t* w_down_f16 = nullptr;
    uint16_t* xq16 = nullptr;
    uint16_t* hq16 = nullptr;
    long long wait_limit = kDefaultWaitLimit;
    bool stall_next = false;   // the next prefill forward injects a stall (mmoe_debug_set_wait_limit)
    bool fuse_requant = false; // kind::f16: the gate/up GEMM requantises the SwiGLU output itself (clusters)
    alignas(64) unsigned char tmap_xq[128] = {};
    alignas(64) unsigned char tmap_hq[128] = {};
    int* err_host = nullptr;   // mapped pinned host memory; kernels write its device alias
    int* err_host_dev = nullptr;
    int* err_dev = nullptr;    // device memory copy read by every CTA
    // decode path: weights in the decode layout, row absmax, group list
    bool use_dec = false;
    bool last_dec = false;
    int dec_max_T = 0;
    int dec_cluster = 0;
    uint8_t* w_gate_up_d = nullptr;
    uint8_t* w_down_d = nullptr;
    int32_t* dec_groups = nullptr;
    int32_t* dec_ngroups = nullptr;
    // fused one-launch decode: synchronisation words (kept zero between launches), router partials,
    // per-unit SwiGLU absmax
    bool use_dec_fused = false;
    DecFusedShape dec_shape = {};
    uint32_t* dec_sync = nullptr;  // the one-launch decode's per-token contribution counters
    float* dec_obuf = nullptr;     // its expert-output rows
    // per-stage timing (mmoe_profile_*)
    struct ProfRec {
        int stage, launches;
        cudaEvent_t a, b;
    };
    bool prof_on = false;
    std::vector<ProfRec> prof;
    std::vector<cudaEvent_t> ev_pool;
    int32_t prof_launches[MMOE_PROF_STAGES] = {};
    double prof_ms[MMOE_PROF_STAGES] = {};
};

namespace {

// Allocation-failure injection (mmoe_debug_fail_alloc): the number of device
// allocations this thread may still make before one fails; -1: never.
thread_local int64_t g_fail_alloc_after = -1;

template <class T>
cudaError_t dalloc(T** p, size_t count) {
    *p = nullptr;
    if (g_fail_alloc_after == 0) {
        g_fail_alloc_after = -1;
        return cudaErrorMemoryAllocation;
    }
    if (g_fail_alloc_after > 0) --g_fail_alloc_after;
    if (count == 0) count = 1;
    return cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T));
}

void free_all(mmoe_handle* h) {
    void* ptrs[] = {h->w_router, h->router_bias, h->w_router_split, h->w_gate_up, h->s_gate_up, h->w_down, h->s_down,
                    h->xq, h->sx, h->logits, h->idx, h->gate, h->chunk_cnt, h->chunk_base, h->offsets,
                    h->counts, h->tiles, h->tile_count, h->row_src, h->row_gate, h->slot_row, h->act, h->hq,
                    h->sh, h->obuf, h->x_stage, h->y_stage, h->w_gate_up_t, h->s_gate_up_t, h->w_down_t,
                    h->s_down_t, h->err_dev, h->w_gate_up_d, h->w_down_d, h->dec_groups,
                    h->dec_ngroups, h->w_gate_up_f16, h->w_down_f16, h->xq16, h->hq16, h->dec_sync,
                    h->dec_obuf};
    for (void* p : ptrs)
        if (p) cudaFree(p);
    if (h->err_host) cudaFreeHost(h->err_host);
    for (cudaStream_t st : {h->s_h2d, h->s_d2h})
        if (st) cudaStreamDestroy(st);
    for (cudaEvent_t ev : {h->ev_start, h->ev_done})
        if (ev) cudaEventDestroy(ev);
    for (int i = 0; i < kHostChunksMax; ++i) {
        if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
        if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
    }
}

mmoe_status check_config(const mmoe_config* c) {
    if (!c) return fail(MMOE_ERR_INVALID_ARG, "config is NULL");
    if (c->d_model < 64 || c->d_model > 8192 || c->d_model % kGroup)
        return fail(MMOE_ERR_INVALID_ARG, "d_model=%d: must be a multiple of 32 in [64, 8192]", c->d_model);
    if (c->n_experts < 1 || c->n_experts > kMaxExperts)
        return fail(MMOE_ERR_INVALID_ARG, "n_experts=%d: must be in [1, %d]", c->n_experts, kMaxExperts);
    if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > kMaxTopK)
        return fail(MMOE_ERR_INVALID_ARG, "top_k=%d: must be in [1, min(n_experts, %d)]", c->top_k, kMaxTopK);
    if (c->expert_hidden < 32 || c->expert_hidden > 4096 || c->expert_hidden % kGroup)
        return fail(MMOE_ERR_INVALID_ARG, "expert_hidden=%d: must be a multiple of 32 in [32, 4096]",
                    c->expert_hidden);
    if (c->shared_hidden < 32 || c->shared_hidden > 4096 || c->shared_hidden % kGroup)
        return fail(MMOE_ERR_INVALID_ARG, "shared_hidden=%d: must be a multiple of 32 in [32, 4096]",
                    c->shared_hidden);
    if (c->group_size != kGroup) return fail(MMOE_ERR_INVALID_ARG, "group_size=%d: must be 32", c->group_size);
    if (c->max_tokens < 1 || c->max_tokens > (1 << 20))
        return fail(MMOE_ERR_INVALID_ARG, "max_tokens=%d: must be in [1, 2^20]", c->max_tokens);
    if (c->gating != MMOE_GATE_SOFTMAX && c->gating != MMOE_GATE_SIGMOID_TOPK_NORM &&
        c->gating != MMOE_GATE_SIGMOID_TOPK_NORM_SEL_BIAS)
        return fail(MMOE_ERR_INVALID_ARG, "gating=%d: unknown", c->gating);
    if (c->has_router_bias != 0 && c->has_router_bias != 1)
        return fail(MMOE_ERR_INVALID_ARG, "has_router_bias=%d: must be 0 or 1", c->has_router_bias);
    if (c->flags & ~(MMOE_FLAG_DETERMINISTIC | MMOE_FLAG_CUDA_CORES | MMOE_FLAG_NO_DECODE | MMOE_FLAG_ATOMIC_COMBINE |
                     MMOE_FLAG_TC_INT8 | MMOE_FLAG_NO_FUSED_DECODE | MMOE_FLAG_FUSED_REQUANT))
        return fail(MMOE_ERR_INVALID_ARG, "flags=0x%x: unknown bits", c->flags);
    return MMOE_OK;
}

Plan make_plan(const mmoe_handle* h, const uint16_t* x, int64_t T, float* y) {
    const mmoe_config& c = h->cfg;
    Plan p{};
    p.d = c.d_model;
    p.h = c.expert_hidden;
    p.hs = c.shared_hidden;
    p.hmax = h->hmax;
    p.E = c.n_experts;
    p.k = c.top_k;
    p.gating = c.gating;
    p.T = T;
    p.Tk = T * c.top_k;
    p.R = T * (c.top_k + 1);
    p.deterministic = (c.flags & MMOE_FLAG_DETERMINISTIC) != 0;
    p.w_router = h->w_router;
    p.router_bias = c.has_router_bias ? h->router_bias : nullptr;
    p.w_router_split = h->w_router_split;
    p.w_gate_up = h->w_gate_up;
    p.s_gate_up = h->s_gate_up;
    p.w_down = h->w_down;
    p.s_down = h->s_down;
    p.x = x;
    p.y = y;
    p.xq = h->xq;
    p.sx = h->sx;
    p.logits = h->logits;
    p.idx = h->idx;
    p.gate = h->gate;
    p.chunk_cnt = h->chunk_cnt;
    p.chunk_base = h->chunk_base;
    p.offsets = h->offsets;
    p.counts = h->counts;
    p.tiles = h->tiles;
    p.tile_count = h->tile_count;
    p.row_src = h->row_src;
    p.row_gate = h->row_gate;
    p.slot_row = h->slot_row;
    p.act = h->act;
    p.hq = h->hq;
    p.sh = h->sh;
    p.obuf = h->obuf;
    p.tc_kind = h->tc_kind;
    p.tile_rows = p.tc_kind != kTcNone ? kTcTileRows : kTileRows;
    p.max_tiles = max_tiles_for(T, c.top_k, c.n_experts, p.tile_rows);
    p.nchunks = (int)((p.Tk + kChunk - 1) / kChunk);
    p.w_gate_up_t = h->w_gate_up_t;
    p.s_gate_up_t = h->s_gate_up_t;
    p.w_down_t = h->w_down_t;
    p.s_down_t = h->s_down_t;
    p.w_gate_up_f16 = h->w_gate_up_f16;
    p.w_down_f16 = h->w_down_f16;
    p.xq16 = h->xq16;
    p.hq16 = h->hq16;
    p.wait_limit = h->wait_limit;
    p.fuse_requant = h->fuse_requant;
    p.tmap_xq = h->tmap_xq;
    p.tmap_hq = h->tmap_hq;
    p.err = h->err_dev;
    p.err_host = h->err_host_dev;
    p.w_gate_up_d = h->w_gate_up_d;
    p.w_down_d = h->w_down_d;
    p.dec_groups = h->dec_groups;
    p.dec_ngroups = h->dec_ngroups;
    return p;
}

cudaError_t run_gate_up(const Plan& p, cudaStream_t s, int32_t* dump, int64_t r0, int64_t nr) {
    switch (p.tc_kind) {
        case kTcF16: return launch_gate_up_f16(p, s, dump, r0, nr);
        case kTcI8: return launch_gate_up_tc(p, s, dump, r0, nr);
        default: return launch_gate_up(p, s, dump, r0, nr);
    }
}

cudaError_t run_down(const Plan& p, cudaStream_t s, int32_t* dump, int64_t r0, int64_t nr) {
    switch (p.tc_kind) {
        case kTcF16: return launch_down_f16(p, s, dump, r0, nr);
        case kTcI8: return launch_down_tc(p, s, dump, r0, nr);
        default: return launch_down(p, s, dump, r0, nr);
    }
}

// The one-launch decode's counters: per-token contribution counters, then the two counters of a chain
// of layers.
size_t dec_sync_words() { return dec_fused_counter_words() + dec_chain_counter_words(); }

// A bounded device-side wait of an earlier call gave up: report it once and
// clear both copies of the flag (the device copy in stream order).
mmoe_status check_device_flag(mmoe_handle* h, cudaStream_t s) {
    if (!h->err_host) return MMOE_OK;
    const int v = *reinterpret_cast<volatile int*>(h->err_host);
    if (v == 0) return MMOE_OK;
    *reinterpret_cast<volatile int*>(h->err_host) = 0;
    cudaMemsetAsync(h->err_dev, 0, sizeof(int), s);
    // a one-launch decode that gave up may have left contribution counters set
    if (h->dec_sync) cudaMemsetAsync(h->dec_sync, 0, dec_sync_words() * sizeof(uint32_t), s);
    return fail(MMOE_ERR_TIMEOUT, "a tensor-core kernel gave up waiting (site %d); its results were not written", v);
}

cudaEvent_t take_event(mmoe_handle* h) {
    if (!h->ev_pool.empty()) {
        cudaEvent_t e = h->ev_pool.back();
        h->ev_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Runs one stage's launches, bracketed by an event pair when profiling is on.
template <class F>
cudaError_t run_stage(mmoe_handle* h, int stage, int launches, cudaStream_t s, F&& f) {
    if (!h->prof_on) return f();
    cudaEvent_t a = take_event(h), b = take_event(h);
    if (!a || !b) return cudaErrorMemoryAllocation;
    cudaError_t e = cudaEventRecord(a, s);
    if (e == cudaSuccess) e = f();
    if (e == cudaSuccess) e = cudaEventRecord(b, s);
    if (e != cudaSuccess) {
        h->ev_pool.push_back(a);
        h->ev_pool.push_back(b);
        return e;
    }
    h->prof.push_back({stage, launches, a, b});
    return cudaSuccess;
}

// Scratch of mmoe_forward_static_scratch: one array per device, alive for the
// whole process.  Host code must not use its name as a device address; it
// reaches the kernels only through the address cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_static_scratch[MMOE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once per device).
mmoe_status static_scratch_address(int dev, unsigned char** out) {
    if (dev < 0 || dev >= kMaxDevices) return fail(MMOE_ERR_INVALID_ARG, "device %d: unsupported index", dev);
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_addr[dev]) {
        void* a = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&a, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
        g_static_addr[dev] = a;
    }
    *out = static_cast<unsigned char*>(g_static_addr[dev]);
    return MMOE_OK;
}

// Lays the forward's intermediate buffers out in [base, base + cap); returns
// the bytes needed (more than cap means the call does not fit).
size_t carve_static_plan(Plan& p, unsigned char* base, size_t cap) {
    size_t off = 0;
    auto take = [&](size_t bytes) -> void* {
        off = (off + 255) & ~size_t(255);
        void* q = off + bytes <= cap ? static_cast<void*>(base + off) : nullptr;
        off += bytes;
        return q;
    };
    const size_t R = (size_t)p.R, T = (size_t)p.T, d = (size_t)p.d, k = (size_t)p.k, E = (size_t)p.E;
    p.xq = static_cast<int8_t*>(take(R * d));
    p.sx = static_cast<float*>(take(T * 4));
    p.logits = static_cast<float*>(take(T * E * 4));
    p.idx = static_cast<int32_t*>(take(T * k * 4));
    p.gate = static_cast<float*>(take(T * k * 4));
    p.chunk_cnt = static_cast<int32_t*>(take((size_t)p.nchunks * kMaxExperts * 4));
    p.chunk_base = static_cast<int32_t*>(take((size_t)p.nchunks * kMaxExperts * 4));
    p.offsets = static_cast<int32_t*>(take((E + 2) * 4));
    p.counts = static_cast<int32_t*>(take((E + 1) * 4));
    p.tiles = static_cast<int32_t*>(take((size_t)p.max_tiles * 4));
    p.tile_count = static_cast<int32_t*>(take(4));
    p.row_src = static_cast<int32_t*>(take(R * 4));
    p.row_gate = static_cast<float*>(take(R * 4));
    p.slot_row = static_cast<int32_t*>(take(T * k * 4));
    p.act = static_cast<float*>(take(R * (size_t)p.hmax * 8));
    p.hq = static_cast<int8_t*>(take(R * (size_t)p.hmax));
    p.sh = static_cast<float*>(take(R * 4));
    p.obuf = p.deterministic ? static_cast<float*>(take(R * d * 4)) : nullptr;
    return off;
}

}  // namespace

extern "C" {

const char* mmoe_last_error(void) { return g_err.c_str(); }

mmoe_status mmoe_create(const mmoe_config* cfg, int device, mmoe_handle** out) {
    if (!out) return fail(MMOE_ERR_INVALID_ARG, "out is NULL");
    mmoe_status st = check_config(cfg);
    if (st != MMOE_OK) return st;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev)
        return fail(MMOE_ERR_INVALID_ARG, "device %d: not a CUDA device (found %d)", device, ndev);
    DeviceGuard dg(device);
    if (!dg.ok) return fail(MMOE_ERR_CUDA, "cudaSetDevice(%d) failed", device);

    mmoe_handle* h = new (std::nothrow) mmoe_handle();
    if (!h) return fail(MMOE_ERR_OOM, "host allocation of the handle failed");
    h->cfg = *cfg;
    h->device = device;
    h->hmax = cfg->expert_hidden > cfg->shared_hidden ? cfg->expert_hidden : cfg->shared_hidden;
    h->max_tokens = cfg->max_tokens;

    const int64_t d = cfg->d_model, hh = cfg->expert_hidden, hs = cfg->shared_hidden, E = cfg->n_experts;
    const int64_t k = cfg->top_k, Tm = cfg->max_tokens, R = Tm * (k + 1);
    h->n_gu_bytes = (size_t)(E * 2 * hh + 2 * hs) * (d / 2);
    h->n_gu_scales = (size_t)(E * 2 * hh + 2 * hs) * (d / kGroup);
    h->n_d_bytes = (size_t)(E * hh + hs) * d / 2;
    h->n_d_scales = (size_t)(E * hh + hs) * d / kGroup;
    const int64_t nchunks = (Tm * k + kChunk - 1) / kChunk;

    // which kernels serve this handle: the decode path for few tokens, and for prefill the kind::f16
    // tensor-core GEMMs (default), the kind::i8 ones (MMOE_FLAG_TC_INT8, or shapes only they take) or
    // the CUDA-core ones
    h->use_dec = !(cfg->flags & (MMOE_FLAG_CUDA_CORES | MMOE_FLAG_NO_DECODE)) && dec_supported((int)d, (int)hh, (int)hs);
    if (h->use_dec) {
        h->dec_max_T = dec_max_tokens((int)d, h->hmax);
        h->dec_cluster = dec_router_cluster((int)d, (int)E);
        if (h->dec_max_T <= 0 || h->dec_cluster == 0) h->use_dec = false;
    }
    if (!(cfg->flags & MMOE_FLAG_CUDA_CORES)) {
        const bool f16ok = f16tc_supported((int)d, (int)hh, (int)hs) && router_mma_supported((int)d, (int)E);
        const bool i8ok = tc_supported((int)d, (int)hh, (int)hs);
        if ((cfg->flags & MMOE_FLAG_TC_INT8) && i8ok) h->tc_kind = kTcI8;
        else if (f16ok) h->tc_kind = kTcF16;
        else if (i8ok) h->tc_kind = kTcI8;
    }
    // rows of the INT8 code buffers: every row when a prefill kernel set reads them, else only the
    // decode path's
    const int64_t Rd = h->use_dec ? (Tm < h->dec_max_T ? Tm : h->dec_max_T) * (k + 1) : 1;
    const int64_t R8 = h->tc_kind == kTcF16 ? Rd : R;
    // with MMOE_FLAG_FUSED_REQUANT the SwiGLU requantisation runs inside the kind::f16 gate/up GEMM when
    // one cluster of CTAs can hold all hidden-feature blocks of a token tile (at most 8 blocks of 128)
    // and the device fits such clusters; the FP32 SwiGLU buffer then serves only the decode rows
    if (h->tc_kind == kTcF16 && (cfg->flags & MMOE_FLAG_FUSED_REQUANT)) {
        const int fb = h->hmax / 128;
        h->fuse_requant = fb >= 1 && fb <= 8 && f16tc_fused_clusters(fb) > 0;
    }
    const int64_t Ract = h->fuse_requant ? Rd : R;

    cudaError_t e = cudaSuccess;
#define ALLOC(ptr, n) \
    if (e == cudaSuccess) e = dalloc(&h->ptr, (size_t)(n))
    ALLOC(w_router, d * E);
    ALLOC(router_bias, E);
    if (router_mma_supported((int)d, (int)E)) ALLOC(w_router_split, router_split_bytes((int)d) / 2);
    ALLOC(w_gate_up, h->n_gu_bytes);
    ALLOC(s_gate_up, h->n_gu_scales);
    ALLOC(w_down, h->n_d_bytes);
    ALLOC(s_down, h->n_d_scales);
    ALLOC(xq, R8 * d);
    ALLOC(sx, Tm);
    ALLOC(logits, Tm * E);
    ALLOC(idx, Tm * k);
    ALLOC(gate, Tm * k);
    ALLOC(chunk_cnt, nchunks * kMaxExperts);
    ALLOC(chunk_base, nchunks * kMaxExperts);
    ALLOC(offsets, E + 2);
    ALLOC(counts, E + 1);
    ALLOC(tiles, max_tiles_for(Tm, (int)k, (int)E));
    ALLOC(tile_count, 1);
    ALLOC(row_src, R);
    ALLOC(row_gate, R);
    ALLOC(slot_row, Tm * k);
    ALLOC(act, Ract * 2 * h->hmax);  // (gate, up) pairs
    ALLOC(hq, R8 * h->hmax);
    ALLOC(sh, R);
    if (h->use_dec) {
        ALLOC(w_gate_up_d, h->n_gu_bytes + h->n_gu_scales * 4);
        ALLOC(w_down_d, h->n_d_bytes + h->n_d_scales * 4);
        ALLOC(dec_groups, E + 1);
        ALLOC(dec_ngroups, 1);
        if (!(cfg->flags & MMOE_FLAG_NO_FUSED_DECODE)) {
            h->dec_shape = dec_fused_shape((int)d, (int)cfg->expert_hidden, (int)cfg->shared_hidden, (int)E);
            h->use_dec_fused = h->dec_shape.clusters8 > 0;
        }
        if (h->use_dec_fused) {
            ALLOC(dec_sync, dec_sync_words());
            ALLOC(dec_obuf, dec_fused_obuf_floats((int)d));
            if (e == cudaSuccess) e = cudaMemset(h->dec_sync, 0, dec_sync_words() * sizeof(uint32_t));
        }
    }
    if (e == cudaSuccess) {
        // the fixed-order combine (deterministic mode) needs the per-row outputs
        const bool det = (cfg->flags & MMOE_FLAG_DETERMINISTIC) != 0;
        if (det) ALLOC(obuf, R * d);
    }
    if (h->tc_kind != kTcNone || h->use_dec) {
        ALLOC(err_dev, 1);
        if (e == cudaSuccess) e = cudaMemset(h->err_dev, 0, sizeof(int));
        if (e == cudaSuccess) e = cudaHostAlloc(reinterpret_cast<void**>(&h->err_host), sizeof(int), cudaHostAllocMapped);
        if (e == cudaSuccess) {
            *h->err_host = 0;
            e = cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->err_host_dev), h->err_host, 0);
        }
    }
    if (h->tc_kind == kTcF16) {
        ALLOC(w_gate_up_f16, f16tc_image_elems((int)d, (int)hh, (int)hs, (int)E, true));
        ALLOC(s_gate_up_t, h->n_gu_scales);
        ALLOC(w_down_f16, f16tc_image_elems((int)d, (int)hh, (int)hs, (int)E, false));
        ALLOC(s_down_t, h->n_d_scales);
        ALLOC(xq16, R * d);
        ALLOC(hq16, R * h->hmax);
        if (e == cudaSuccess) e = make_tensor_map(h->tmap_xq, h->xq16, (uint64_t)d, (uint64_t)R, (uint64_t)d * 2, 2);
        if (e == cudaSuccess)
            e = make_tensor_map(h->tmap_hq, h->hq16, (uint64_t)h->hmax, (uint64_t)R, (uint64_t)h->hmax * 2, 2);
    } else if (h->tc_kind == kTcI8) {
        ALLOC(w_gate_up_t, 2 * h->n_gu_bytes);  // INT8 stage images: twice the packed INT4 bytes
        ALLOC(s_gate_up_t, h->n_gu_scales);
        ALLOC(w_down_t, 2 * h->n_d_bytes);
        ALLOC(s_down_t, h->n_d_scales);
        if (e == cudaSuccess) e = make_tensor_map(h->tmap_xq, h->xq, (uint64_t)d, (uint64_t)R, (uint64_t)d, 1);
        if (e == cudaSuccess)
            e = make_tensor_map(h->tmap_hq, h->hq, (uint64_t)h->hmax, (uint64_t)R, (uint64_t)h->hmax, 1);
    }
#undef ALLOC
    if (e != cudaSuccess) {
        free_all(h);
        delete h;
        return cuda_fail(e, "workspace allocation");
    }
    *out = h;
    return MMOE_OK;
}

mmoe_status mmoe_load_quantized_weights(mmoe_handle* h, const mmoe_weights* w, void* stream) {
    if (!h || !w) return fail(MMOE_ERR_INVALID_ARG, "handle or weights is NULL");
    if (!w->w_router || !w->w_gate_up || !w->s_gate_up || !w->w_down || !w->s_down)
        return fail(MMOE_ERR_INVALID_ARG, "a weight pointer is NULL");
    if (h->cfg.has_router_bias && !w->router_bias)
        return fail(MMOE_ERR_INVALID_ARG, "the config has a router bias but router_bias is NULL");
    if (w->on_device != 0 && w->on_device != 1) return fail(MMOE_ERR_INVALID_ARG, "on_device must be 0 or 1");
    DeviceGuard dg(h->device);
    // a load that fails part way leaves a mix of old and new weights: unloaded until one succeeds
    h->loaded = false;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaMemcpyKind kind = w->on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    const size_t d = h->cfg.d_model, E = h->cfg.n_experts;
    MMOE_CUDA(cudaMemcpyAsync(h->w_router, w->w_router, d * E * sizeof(float), kind, s), "copy w_router");
    if (h->cfg.has_router_bias)
        MMOE_CUDA(cudaMemcpyAsync(h->router_bias, w->router_bias, E * sizeof(float), kind, s), "copy router_bias");
    if (h->w_router_split)
        MMOE_CUDA(launch_split_router(h->w_router, (int)d, (int)E, h->w_router_split, s), "router split launch");
    MMOE_CUDA(cudaMemcpyAsync(h->w_gate_up, w->w_gate_up, h->n_gu_bytes, kind, s), "copy w_gate_up");
    MMOE_CUDA(cudaMemcpyAsync(h->s_gate_up, w->s_gate_up, h->n_gu_scales * sizeof(float), kind, s), "copy s_gate_up");
    MMOE_CUDA(cudaMemcpyAsync(h->w_down, w->w_down, h->n_d_bytes, kind, s), "copy w_down");
    MMOE_CUDA(cudaMemcpyAsync(h->s_down, w->s_down, h->n_d_scales * sizeof(float), kind, s), "copy s_down");
    if (h->tc_kind == kTcF16)
        MMOE_CUDA(launch_retile_f16(h->w_gate_up, h->s_gate_up, h->w_down, h->s_down, h->w_gate_up_f16,
                                    h->s_gate_up_t, h->w_down_f16, h->s_down_t, h->cfg.d_model, h->cfg.expert_hidden,
                                    h->cfg.shared_hidden, h->cfg.n_experts, s),
                  "weight re-tiling launch");
    if (h->tc_kind == kTcI8)
        MMOE_CUDA(launch_retile(h->w_gate_up, h->s_gate_up, h->w_down, h->s_down, h->w_gate_up_t, h->s_gate_up_t,
                                h->w_down_t, h->s_down_t, h->cfg.d_model, h->cfg.expert_hidden, h->cfg.shared_hidden,
                                h->cfg.n_experts, s),
                  "weight re-tiling launch");
    if (h->use_dec)
        MMOE_CUDA(launch_retile_dec(h->w_gate_up, h->s_gate_up, h->w_down, h->s_down, h->w_gate_up_d, h->w_down_d,
                                    h->cfg.d_model, h->cfg.expert_hidden, h->cfg.shared_hidden, h->cfg.n_experts, s),
                  "decode-layout re-tiling launch");
    h->loaded = true;
    return MMOE_OK;
}

mmoe_status mmoe_forward(mmoe_handle* h, const uint16_t* x, int64_t T, float* y, void* stream,
                         int32_t* topk_idx, float* topk_gate, int32_t* expert_counts) {
    if (!h) return fail(MMOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0 || T > h->max_tokens)
        return fail(MMOE_ERR_INVALID_ARG, "T=%lld: must be in [0, max_tokens=%lld]", (long long)T,
                    (long long)h->max_tokens);
    if (!h->loaded) return fail(MMOE_ERR_NOT_LOADED, "forward before mmoe_load_quantized_weights");
    if (T == 0) return MMOE_OK;
    if (!x || !y) return fail(MMOE_ERR_INVALID_ARG, "x or y is NULL");
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15)
        return fail(MMOE_ERR_INVALID_ARG, "x and y must be 16-byte aligned");
    DeviceGuard dg(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    mmoe_status fst = check_device_flag(h, s);
    if (fst != MMOE_OK) return fst;
    const bool dec = h->use_dec && T <= h->dec_max_T;
    Plan p = make_plan(h, x, T, y);
    if (dec) {
        // the decode kernels work on the INT8 code buffers
        p.xq16 = nullptr;
        p.hq16 = nullptr;
    }
    // fixed-order combine only in deterministic mode: by default the expert GEMMs add into y with atomics
    // (measured on B200 with the kind::f16 GEMMs, T = 32768: down 1.59 ms against 1.55 + 0.26 ms of row
    // outputs and the fixed-order combine)
    p.deterministic = (h->cfg.flags & MMOE_FLAG_DETERMINISTIC) != 0;
    const bool fused = dec && h->use_dec_fused && T <= dec_fused_max_tokens();
    if (fused) {
        // the whole layer in one launch (routing, gate/up, down, the fixed-order combine into y); it also
        // writes the caller's copies of the routing
        MMOE_CUDA(run_stage(h, MMOE_PROF_DECODE_FUSED, 1, s,
                            [&] {
                                return launch_decode_fused(p, h->dec_shape, h->dec_sync, h->dec_obuf,
                                                           h->dec_sync + dec_fused_counter_words(), topk_idx,
                                                           topk_gate, expert_counts, s);
                            }),
                  "one-launch decode");
    } else if (dec) {
        // decode path: router + permutation, gate/up (also clears y), requantisation, down
        MMOE_CUDA(run_stage(h, MMOE_PROF_ROUTER, 1, s, [&] { return launch_router_dec(p, h->dec_cluster, s); }),
                  "decode router launch");
        MMOE_CUDA(run_stage(h, MMOE_PROF_GATE_UP, 1, s, [&] { return launch_gate_up_dec(p, s, nullptr, 0, 0); }),
                  "decode gate/up launch");
        MMOE_CUDA(run_stage(h, MMOE_PROF_REQUANT, 1, s, [&] { return launch_requant(p, s); }),
                  "decode requant launch");
        MMOE_CUDA(run_stage(h, MMOE_PROF_DOWN, 1, s, [&] { return launch_down_dec(p, s, nullptr, 0, 0); }),
                  "decode down launch");
    }
    // y is accumulated with atomics: cleared first (the tensor-core router clears its tokens' rows itself)
    if (!dec && !p.deterministic && !p.w_router_split)
        MMOE_CUDA(run_stage(h, MMOE_PROF_ZERO_Y, 0, s,
                            [&] { return cudaMemsetAsync(y, 0, (size_t)T * p.d * sizeof(float), s); }),
                  "zero y");
    if (!dec) {
        MMOE_CUDA(run_stage(h, MMOE_PROF_ROUTER, 1, s, [&] { return launch_router_quant(p, s); }),
                  "router/quantiser launch");
        MMOE_CUDA(run_stage(h, MMOE_PROF_PERMUTE, 4, s, [&] { return launch_permute(p, s); }), "permute launch");
        p.debug_stall = h->stall_next && p.tc_kind == kTcF16 ? 1 : 0;
        h->stall_next = false;
        MMOE_CUDA(run_stage(h, MMOE_PROF_GATE_UP, 1, s, [&] { return run_gate_up(p, s, nullptr, 0, 0); }),
                  "gate/up launch");
        p.debug_stall = 0;
        if (!p.fuse_requant)
            MMOE_CUDA(run_stage(h, MMOE_PROF_REQUANT, 1, s, [&] { return launch_requant(p, s); }), "requant launch");
        MMOE_CUDA(run_stage(h, MMOE_PROF_DOWN, 1, s, [&] { return run_down(p, s, nullptr, 0, 0); }), "down launch");
    }
    if (p.deterministic && !fused)
        MMOE_CUDA(run_stage(h, MMOE_PROF_COMBINE, 1, s, [&] { return launch_combine(p, s); }), "combine launch");
    if (topk_idx && !fused)
        MMOE_CUDA(cudaMemcpyAsync(topk_idx, h->idx, (size_t)p.Tk * sizeof(int32_t), cudaMemcpyDeviceToDevice, s),
                  "copy topk_idx");
    if (topk_gate && !fused)
        MMOE_CUDA(cudaMemcpyAsync(topk_gate, h->gate, (size_t)p.Tk * sizeof(float), cudaMemcpyDeviceToDevice, s),
                  "copy topk_gate");
    if (expert_counts && !fused)
        MMOE_CUDA(cudaMemcpyAsync(expert_counts, h->counts, (size_t)(p.E + 1) * sizeof(int32_t),
                                  cudaMemcpyDeviceToDevice, s),
                  "copy expert_counts");
    h->last_T = T;
    h->last_dec = dec;
    return MMOE_OK;
}

mmoe_status mmoe_forward_chain(mmoe_handle* const* layers, int32_t n_layers, const uint16_t* x, int64_t T,
                               float* const* y_layers, void* stream) {
    if (!layers || !y_layers) return fail(MMOE_ERR_INVALID_ARG, "layers or y_layers is NULL");
    if (n_layers < 1 || n_layers > MMOE_MAX_CHAIN_LAYERS)
        return fail(MMOE_ERR_INVALID_ARG, "n_layers=%d: must be in [1, %d]", n_layers, MMOE_MAX_CHAIN_LAYERS);
    for (int l = 0; l < n_layers; ++l)
        for (int m = 0; m < l; ++m)
            if (y_layers[l] && y_layers[l] == y_layers[m])
                return fail(MMOE_ERR_INVALID_ARG, "y_layers[%d] and y_layers[%d] are the same buffer", m, l);
    mmoe_handle* h0 = layers[0];
    if (!h0) return fail(MMOE_ERR_INVALID_ARG, "layer 0's handle is NULL");
    const mmoe_config& c0 = h0->cfg;
    for (int l = 0; l < n_layers; ++l) {
        const mmoe_handle* h = layers[l];
        if (!h) return fail(MMOE_ERR_INVALID_ARG, "layer %d's handle is NULL", l);
        const mmoe_config& c = h->cfg;
        if (c.d_model != c0.d_model || c.n_experts != c0.n_experts || c.top_k != c0.top_k ||
            c.expert_hidden != c0.expert_hidden || c.shared_hidden != c0.shared_hidden || c.gating != c0.gating ||
            h->device != h0->device)
            return fail(MMOE_ERR_INVALID_ARG, "layer %d: shapes, gating or device differ from layer 0's", l);
        if (T < 0 || T > h->max_tokens)
            return fail(MMOE_ERR_INVALID_ARG, "T=%lld: must be in [0, max_tokens=%lld] of layer %d", (long long)T,
                        (long long)h->max_tokens, l);
        if (!h->loaded) return fail(MMOE_ERR_NOT_LOADED, "layer %d: forward before mmoe_load_quantized_weights", l);
        if (!y_layers[l] || (reinterpret_cast<uintptr_t>(y_layers[l]) & 15))
            return fail(MMOE_ERR_INVALID_ARG, "y_layers[%d] is NULL or not 16-byte aligned", l);
    }
    if (T == 0) return MMOE_OK;
    if (!x || (reinterpret_cast<uintptr_t>(x) & 15)) return fail(MMOE_ERR_INVALID_ARG, "x is NULL or misaligned");
    {
        // no two outputs, and no output and the input, may overlap (each layer's y is cleared and added
        // into, and x is read while they are written)
        const uintptr_t ylen = (uintptr_t)T * (uintptr_t)c0.d_model * sizeof(float);
        const uintptr_t x0 = reinterpret_cast<uintptr_t>(x), x1 = x0 + (uintptr_t)T * c0.d_model * sizeof(uint16_t);
        for (int l = 0; l < n_layers; ++l) {
            const uintptr_t a0 = reinterpret_cast<uintptr_t>(y_layers[l]), a1 = a0 + ylen;
            if (a0 < x1 && x0 < a1) return fail(MMOE_ERR_INVALID_ARG, "y_layers[%d] overlaps x", l);
            for (int m = 0; m < l; ++m) {
                const uintptr_t b0 = reinterpret_cast<uintptr_t>(y_layers[m]), b1 = b0 + ylen;
                if (a0 < b1 && b0 < a1) return fail(MMOE_ERR_INVALID_ARG, "y_layers[%d] and y_layers[%d] overlap", m, l);
            }
        }
    }
    DeviceGuard dg(h0->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t d = c0.d_model;
    const bool one_launch = h0->use_dec && h0->use_dec_fused && T <= h0->dec_max_T && T <= dec_fused_max_tokens();
    if (one_launch) {
        mmoe_status fst = check_device_flag(h0, s);
        if (fst != MMOE_OK) return fst;
        Plan p = make_plan(h0, x, T, y_layers[0]);
        p.xq16 = nullptr;
        p.hq16 = nullptr;
        DecChainLayer L[MMOE_MAX_CHAIN_LAYERS];
        for (int l = 0; l < n_layers; ++l)
            // (a handle without a router bias in its config has the buffer, but nothing was loaded into it)
            L[l] = DecChainLayer{layers[l]->w_router,
                                 layers[l]->cfg.has_router_bias ? layers[l]->router_bias : nullptr,
                                 layers[l]->w_gate_up_d,
                                 layers[l]->w_down_d,
                                 y_layers[l],
                                 nullptr,
                                 nullptr,
                                 nullptr};
        MMOE_CUDA(run_stage(h0, MMOE_PROF_DECODE_FUSED, 1, s,
                            [&] {
                                return launch_decode_chain(p, h0->dec_shape, h0->dec_sync, h0->dec_obuf,
                                                           h0->dec_sync + dec_fused_counter_words(), L, n_layers, s);
                            }),
                  "one-launch decode of a chain of layers");
        h0->last_T = T;
        h0->last_dec = true;
        return MMOE_OK;
    }
    // one forward per layer; the next layer's input is the BF16 rounding of this one's y
    const uint16_t* xin = x;
    for (int l = 0; l < n_layers; ++l) {
        const mmoe_status st = mmoe_forward(layers[l], xin, T, y_layers[l], stream, nullptr, nullptr, nullptr);
        if (st != MMOE_OK) return st;
        if (l + 1 < n_layers) {
            mmoe_handle* hn = layers[l + 1];
            if (!hn->x_stage) MMOE_CUDA(dalloc(&hn->x_stage, (size_t)hn->max_tokens * d), "staging allocation");
            MMOE_CUDA(launch_f32_to_bf16(y_layers[l], hn->x_stage, T * d, s), "BF16 rounding of y");
            xin = hn->x_stage;
        }
    }
    return MMOE_OK;
}

namespace {

// The copy streams and events of mmoe_forward_host, created all or nothing.
mmoe_status ensure_host_copy_state(mmoe_handle* h) {
    if (h->s_h2d) return MMOE_OK;
    cudaStream_t a = nullptr, b = nullptr;
    cudaEvent_t ev[2 + 2 * kHostChunksMax] = {};
    cudaError_t e = cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking);
    for (cudaEvent_t& x : ev)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
    if (e != cudaSuccess) {
        if (a) cudaStreamDestroy(a);
        if (b) cudaStreamDestroy(b);
        for (cudaEvent_t x : ev)
            if (x) cudaEventDestroy(x);
        return cuda_fail(e, "copy streams and events");
    }
    h->s_h2d = a;
    h->s_d2h = b;
    h->ev_start = ev[0];
    h->ev_done = ev[1];
    for (int i = 0; i < kHostChunksMax; ++i) {
        h->ev_in[i] = ev[2 + i];
        h->ev_out[i] = ev[2 + kHostChunksMax + i];
    }
    return MMOE_OK;
}

}  // namespace

mmoe_status mmoe_forward_host(mmoe_handle* h, const uint16_t* x_host, int64_t T, float* y_host, void* stream) {
    if (!h) return fail(MMOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0 || T > h->max_tokens)
        return fail(MMOE_ERR_INVALID_ARG, "T=%lld: must be in [0, max_tokens=%lld]", (long long)T,
                    (long long)h->max_tokens);
    if (!h->loaded) return fail(MMOE_ERR_NOT_LOADED, "forward before mmoe_load_quantized_weights");
    if (T == 0) return MMOE_OK;
    if (!x_host || !y_host) return fail(MMOE_ERR_INVALID_ARG, "x or y is NULL");
    DeviceGuard dg(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t d = h->cfg.d_model;
    if (!h->x_stage) MMOE_CUDA(dalloc(&h->x_stage, (size_t)h->max_tokens * d), "staging allocation");
    if (!h->y_stage) MMOE_CUDA(dalloc(&h->y_stage, (size_t)h->max_tokens * d), "staging allocation");
    const mmoe_status cs = ensure_host_copy_state(h);
    if (cs != MMOE_OK) return cs;
    // short first and last chunks shorten the copy-in before the first forward and the copy-out
    // after the last one
    int64_t bound[kHostChunksMax + 1];
    const int nch = host_chunk_bounds(T, bound);
    // The first failure is kept and ends the enqueueing, but the copy streams are always joined
    // and waited for, so that no copy touches x_host or y_host after this call returns.
    cudaError_t ce = cudaSuccess;
    const char* what = "";
    auto ok = [&](cudaError_t e, const char* w) {
        if (ce == cudaSuccess && e != cudaSuccess) {
            ce = e;
            what = w;
        }
        return ce == cudaSuccess;
    };
    // copies start after the caller's earlier work on `stream`
    bool go = ok(cudaEventRecord(h->ev_start, s), "event record") &&
              ok(cudaStreamWaitEvent(h->s_h2d, h->ev_start, 0), "stream wait") &&
              ok(cudaStreamWaitEvent(h->s_d2h, h->ev_start, 0), "stream wait");
    for (int i = 0; go && i < nch; ++i) {
        const int64_t t0 = bound[i], Ti = bound[i + 1] - bound[i];
        go = ok(cudaMemcpyAsync(h->x_stage + t0 * d, x_host + t0 * d, (size_t)Ti * d * sizeof(uint16_t),
                                cudaMemcpyHostToDevice, h->s_h2d),
                "copy x to the device") &&
             ok(cudaEventRecord(h->ev_in[i], h->s_h2d), "event record");
    }
    mmoe_status st = MMOE_OK;
    for (int i = 0; go && i < nch; ++i) {
        const int64_t t0 = bound[i], Ti = bound[i + 1] - bound[i];
        if (!ok(cudaStreamWaitEvent(s, h->ev_in[i], 0), "stream wait")) break;
        st = mmoe_forward(h, h->x_stage + t0 * d, Ti, h->y_stage + t0 * d, stream, nullptr, nullptr, nullptr);
        if (st != MMOE_OK) break;
        go = ok(cudaEventRecord(h->ev_out[i], s), "event record") &&
             ok(cudaStreamWaitEvent(h->s_d2h, h->ev_out[i], 0), "stream wait") &&
             ok(cudaMemcpyAsync(y_host + t0 * d, h->y_stage + t0 * d, (size_t)Ti * d * sizeof(float),
                                cudaMemcpyDeviceToHost, h->s_d2h),
                "copy y to the host");
    }
    // `stream` is left ordered after both copy streams, whatever happened above
    cudaError_t j1 = cudaEventRecord(h->ev_done, h->s_h2d);
    if (j1 == cudaSuccess) j1 = cudaStreamWaitEvent(s, h->ev_done, 0);
    cudaError_t j2 = cudaEventRecord(h->ev_done, h->s_d2h);
    if (j2 == cudaSuccess) j2 = cudaStreamWaitEvent(s, h->ev_done, 0);
    const cudaError_t w1 = cudaStreamSynchronize(h->s_h2d);
    const cudaError_t w2 = cudaStreamSynchronize(h->s_d2h);
    const cudaError_t w3 = cudaStreamSynchronize(s);
    if (st != MMOE_OK) return st;
    ok(j1, "stream order");
    ok(j2, "stream order");
    ok(w1, "stream synchronize");
    ok(w2, "stream synchronize");
    ok(w3, "stream synchronize");
    if (ce != cudaSuccess) return cuda_fail(ce, what);
    return MMOE_OK;
}

mmoe_status mmoe_debug_host_chunks(int64_t T, int64_t* bounds, int32_t cap, int32_t* n) {
    if (T < 0) return fail(MMOE_ERR_INVALID_ARG, "T=%lld: must be >= 0", (long long)T);
    if (!bounds || !n) return fail(MMOE_ERR_INVALID_ARG, "bounds or n is NULL");
    int64_t b[kHostChunksMax + 1];
    const int nch = host_chunk_bounds(T, b);
    if (cap < nch + 1) return fail(MMOE_ERR_INVALID_ARG, "cap=%d: %d boundaries needed", (int)cap, nch + 1);
    for (int i = 0; i <= nch; ++i) bounds[i] = b[i];
    *n = nch;
    return MMOE_OK;
}

mmoe_status mmoe_destroy(mmoe_handle* h) {
    if (!h) return MMOE_OK;
    DeviceGuard dg(h->device);
    cudaError_t e = cudaDeviceSynchronize();
    const int flag = h->err_host ? *reinterpret_cast<volatile int*>(h->err_host) : 0;
    for (auto& r : h->prof) {
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    for (cudaEvent_t ev : h->ev_pool) cudaEventDestroy(ev);
    free_all(h);
    delete h;
    if (e != cudaSuccess) return cuda_fail(e, "synchronize before destroy");
    if (flag) return fail(MMOE_ERR_TIMEOUT, "a tensor-core kernel gave up waiting (site %d)", flag);
    return MMOE_OK;
}

mmoe_status mmoe_quantize_int4(const float* w, int64_t rows, int64_t K, uint8_t* packed, float* scales,
                               void* stream) {
    if (rows < 0 || K <= 0 || K % kGroup)
        return fail(MMOE_ERR_INVALID_ARG, "rows=%lld K=%lld: rows >= 0 and K a positive multiple of 32",
                    (long long)rows, (long long)K);
    if (rows == 0) return MMOE_OK;
    if (!w || !packed || !scales) return fail(MMOE_ERR_INVALID_ARG, "a pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(packed)) & 15)
        return fail(MMOE_ERR_INVALID_ARG, "w and packed must be 16-byte aligned");
    MMOE_CUDA(launch_quantize_int4(w, rows, K, packed, scales, reinterpret_cast<cudaStream_t>(stream)),
              "quantize launch");
    return MMOE_OK;
}

mmoe_status mmoe_debug_copy_stage(mmoe_handle* h, int32_t stage, void* dst, size_t bytes, void* stream) {
    if (!h || !dst) return fail(MMOE_ERR_INVALID_ARG, "handle or dst is NULL");
    if (h->last_T < 0) return fail(MMOE_ERR_INVALID_ARG, "no forward has run on this handle");
    const int64_t T = h->last_T, k = h->cfg.top_k, E = h->cfg.n_experts, d = h->cfg.d_model;
    const int64_t R = T * (k + 1);
    const void* src = nullptr;
    size_t have = 0;
    switch (stage) {
        case MMOE_STAGE_XQ: src = h->xq + T * k * d; have = (size_t)(T * d); break;
        case MMOE_STAGE_SX: src = h->sx; have = (size_t)T * 4; break;
        case MMOE_STAGE_OFFSETS: src = h->offsets; have = (size_t)(E + 2) * 4; break;
        case MMOE_STAGE_ROW_SRC: src = h->row_src; have = (size_t)R * 4; break;
        case MMOE_STAGE_SLOT_ROW: src = h->slot_row; have = (size_t)(T * k) * 4; break;
        case MMOE_STAGE_HQ: src = h->hq; have = (size_t)(R * h->hmax); break;
        case MMOE_STAGE_SH: src = h->sh; have = (size_t)R * 4; break;
        case MMOE_STAGE_LOGITS: src = h->logits; have = (size_t)(T * E) * 4; break;
        default: return fail(MMOE_ERR_INVALID_ARG, "stage %d: unknown", stage);
    }
    if (bytes > have) return fail(MMOE_ERR_INVALID_ARG, "stage %d holds %zu bytes, asked for %zu", stage, have, bytes);
    DeviceGuard dg(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!h->last_dec && h->tc_kind == kTcF16 && (stage == MMOE_STAGE_XQ || stage == MMOE_STAGE_HQ)) {
        // the kind::f16 path keeps these codes as f16: converted to INT8 on the way out
        const uint16_t* src16 = stage == MMOE_STAGE_XQ ? h->xq16 + T * k * d : h->hq16;
        MMOE_CUDA(launch_codes_f16_to_i8(src16, static_cast<int8_t*>(dst), (int64_t)bytes, s), "code conversion");
        return MMOE_OK;
    }
    MMOE_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s), "copy stage");
    return MMOE_OK;
}

mmoe_status mmoe_debug_partials(mmoe_handle* h, int32_t which, int64_t row0, int64_t nrows, int32_t* dst,
                                void* stream) {
    if (!h || !dst) return fail(MMOE_ERR_INVALID_ARG, "handle or dst is NULL");
    if (!h->loaded) return fail(MMOE_ERR_NOT_LOADED, "no weights loaded");
    if (h->last_T <= 0) return fail(MMOE_ERR_INVALID_ARG, "no forward with T > 0 has run on this handle");
    const int64_t R = h->last_T * (h->cfg.top_k + 1);
    if (which != 0 && which != 1) return fail(MMOE_ERR_INVALID_ARG, "which=%d: must be 0 or 1", which);
    if (row0 < 0 || nrows < 0 || row0 + nrows > R)
        return fail(MMOE_ERR_INVALID_ARG, "rows [%lld, %lld) outside [0, %lld)", (long long)row0,
                    (long long)(row0 + nrows), (long long)R);
    DeviceGuard dg(h->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const Plan p = make_plan(h, nullptr, h->last_T, nullptr);
    if (h->last_dec) {
        Plan pd = p;
        pd.xq16 = nullptr;
        pd.hq16 = nullptr;
        if (which == 0) MMOE_CUDA(launch_gate_up_dec(pd, s, dst, row0, nrows), "gate/up dump launch");
        else MMOE_CUDA(launch_down_dec(pd, s, dst, row0, nrows), "down dump launch");
    } else {
        if (which == 0) MMOE_CUDA(run_gate_up(p, s, dst, row0, nrows), "gate/up dump launch");
        else MMOE_CUDA(run_down(p, s, dst, row0, nrows), "down dump launch");
    }
    return MMOE_OK;
}

mmoe_status mmoe_debug_fail_alloc(int64_t after) {
    if (after < -1) return fail(MMOE_ERR_INVALID_ARG, "after=%lld: must be >= -1", (long long)after);
    g_fail_alloc_after = after;
    return MMOE_OK;
}

mmoe_status mmoe_debug_set_wait_limit(mmoe_handle* h, int64_t clocks, int32_t stall_next) {
    if (!h) return fail(MMOE_ERR_INVALID_ARG, "handle is NULL");
    if (clocks < 0) return fail(MMOE_ERR_INVALID_ARG, "clocks=%lld: must be >= 0", (long long)clocks);
    if (stall_next != 0 && stall_next != 1) return fail(MMOE_ERR_INVALID_ARG, "stall_next=%d: must be 0 or 1", stall_next);
    if (stall_next && h->tc_kind != kTcF16)
        return fail(MMOE_ERR_UNIMPLEMENTED, "an injected stall needs the kind::f16 tensor-core GEMMs on this handle");
    h->wait_limit = clocks == 0 ? kDefaultWaitLimit : clocks;
    h->stall_next = stall_next != 0;
    return MMOE_OK;
}

mmoe_status mmoe_profile_enable(mmoe_handle* h, int32_t enable) {
    if (!h) return fail(MMOE_ERR_INVALID_ARG, "handle is NULL");
    DeviceGuard dg(h->device);
    if (enable) {
        for (auto& r : h->prof) {
            h->ev_pool.push_back(r.a);
            h->ev_pool.push_back(r.b);
        }
        h->prof.clear();
        for (int i = 0; i < MMOE_PROF_STAGES; ++i) {
            h->prof_launches[i] = 0;
            h->prof_ms[i] = 0.0;
        }
    }
    h->prof_on = enable != 0;
    return MMOE_OK;
}

mmoe_status mmoe_profile_read(mmoe_handle* h, int32_t* launches, double* total_ms, int32_t n) {
    if (!h || !launches || !total_ms || n < 1) return fail(MMOE_ERR_INVALID_ARG, "bad arguments");
    DeviceGuard dg(h->device);
    for (auto& r : h->prof) {
        MMOE_CUDA(cudaEventSynchronize(r.b), "profile event wait");
        float ms = 0.0f;
        MMOE_CUDA(cudaEventElapsedTime(&ms, r.a, r.b), "profile elapsed time");
        h->prof_launches[r.stage] += r.launches;
        h->prof_ms[r.stage] += ms;
        h->ev_pool.push_back(r.a);
        h->ev_pool.push_back(r.b);
    }
    h->prof.clear();
    for (int i = 0; i < n; ++i) {
        launches[i] = i < MMOE_PROF_STAGES ? h->prof_launches[i] : 0;
        total_ms[i] = i < MMOE_PROF_STAGES ? h->prof_ms[i] : 0.0;
    }
    return MMOE_OK;
}

mmoe_status mmoe_forward_static_scratch(const mmoe_config* cfg, const mmoe_weights* w, const uint16_t* x,
                                        int64_t T, float* y, void* stream) {
    mmoe_status st = check_config(cfg);
    if (st != MMOE_OK) return st;
    if (!w || !w->w_router || !w->w_gate_up || !w->s_gate_up || !w->w_down || !w->s_down)
        return fail(MMOE_ERR_INVALID_ARG, "weights or a weight pointer is NULL");
    if (w->on_device != 1) return fail(MMOE_ERR_INVALID_ARG, "weights must be device pointers (on_device = 1)");
    if (cfg->has_router_bias && !w->router_bias)
        return fail(MMOE_ERR_INVALID_ARG, "the config has a router bias but router_bias is NULL");
    // the weights are read in place by kernels that load the packed codes 16 bytes and the FP32
    // arrays 4 bytes at a time
    if ((reinterpret_cast<uintptr_t>(w->w_gate_up) | reinterpret_cast<uintptr_t>(w->w_down)) & 15)
        return fail(MMOE_ERR_INVALID_ARG, "w_gate_up and w_down must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(w->w_router) | reinterpret_cast<uintptr_t>(w->router_bias) |
         reinterpret_cast<uintptr_t>(w->s_gate_up) | reinterpret_cast<uintptr_t>(w->s_down)) & 3)
        return fail(MMOE_ERR_INVALID_ARG, "w_router, router_bias, s_gate_up and s_down must be 4-byte aligned");
    if (T < 0 || T > (1 << 20)) return fail(MMOE_ERR_INVALID_ARG, "T=%lld: must be in [0, 2^20]", (long long)T);
    if (T == 0) return MMOE_OK;
    if (!x || !y) return fail(MMOE_ERR_INVALID_ARG, "x or y is NULL");
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 15)
        return fail(MMOE_ERR_INVALID_ARG, "x and y must be 16-byte aligned");

    Plan p{};
    p.d = cfg->d_model;
    p.h = cfg->expert_hidden;
    p.hs = cfg->shared_hidden;
    p.hmax = p.h > p.hs ? p.h : p.hs;
    p.E = cfg->n_experts;
    p.k = cfg->top_k;
    p.gating = cfg->gating;
    p.T = T;
    p.Tk = T * p.k;
    p.R = T * (p.k + 1);
    // fixed-order combine unless atomics were asked for (this entry point keeps y bit-reproducible by
    // default, unlike mmoe_forward)
    p.deterministic = (cfg->flags & MMOE_FLAG_DETERMINISTIC) || !(cfg->flags & MMOE_FLAG_ATOMIC_COMBINE);
    p.w_router = w->w_router;
    p.router_bias = cfg->has_router_bias ? w->router_bias : nullptr;
    p.w_gate_up = w->w_gate_up;
    p.s_gate_up = w->s_gate_up;
    p.w_down = w->w_down;
    p.s_down = w->s_down;
    p.x = x;
    p.y = y;
    p.tc_kind = kTcNone;
    p.tile_rows = kTileRows;
    p.max_tiles = max_tiles_for(T, p.k, p.E, p.tile_rows);
    p.nchunks = (int)((p.Tk + kChunk - 1) / kChunk);

    // size check first (no device needed), then the one-time address lookup
    Plan probe = p;
    const size_t need = carve_static_plan(probe, nullptr, 0);
    if (need > MMOE_STATIC_SCRATCH_BYTES)
        return fail(MMOE_ERR_INVALID_ARG,
                    "T=%lld needs %zu bytes of scratch; the static scratch array holds %u bytes "
                    "(use fewer tokens per call)",
                    (long long)T, need, (unsigned)MMOE_STATIC_SCRATCH_BYTES);
    int dev = 0;
    MMOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    unsigned char* base = nullptr;
    st = static_scratch_address(dev, &base);
    if (st != MMOE_OK) return st;
    carve_static_plan(p, base, MMOE_STATIC_SCRATCH_BYTES);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!p.deterministic) MMOE_CUDA(cudaMemsetAsync(y, 0, (size_t)T * p.d * sizeof(float), s), "zero y");
    MMOE_CUDA(launch_router_quant(p, s), "router/quantiser launch");
    MMOE_CUDA(launch_permute(p, s), "permute launch");
    MMOE_CUDA(launch_gate_up(p, s, nullptr, 0, 0), "gate/up launch");
    MMOE_CUDA(launch_requant(p, s), "requant launch");
    MMOE_CUDA(launch_down(p, s, nullptr, 0, 0), "down launch");
    if (p.deterministic) MMOE_CUDA(launch_combine(p, s), "combine launch");
    return MMOE_OK;
}

}  // extern "C"
