/*
 * mmoe.h -- C ABI of the fused MoE feed-forward layer for B200 (sm_100a).
 *
 * The layer is Eq. (*) of "MobileMoE: Scaling On-Device Mixture of Experts"
 * (paper-archivist reading, section "MoE preliminaries and three design
 * factors"):
 *
 *     y = sum_{i in Top-k} router_i(x) * FFN_i(x) + FFN^(s)(x)
 *
 * 60 fine-grained routed SwiGLU experts, top-4, one always-on shared expert
 * ("Finding 3" and the final architecture paragraph), an FP32 router
 * ("MoE training stability techniques"), symmetric group-32 INT4 weights with
 * FP32 scales (Eq. (6), section "QAT") and INT8 activations quantised per
 * token on the fly (same section).  The pages run the whole FFN as one fused
 * operator call (section "custom MoE kernel", principle 2); mmoe_forward is
 * that call.
 *
 * Conventions for every function below:
 *   - Every function returns an mmoe_status; no exception or signal crosses
 *     the ABI.  On failure, mmoe_last_error() returns a thread-local message
 *     that stays valid until the next call on the same thread.
 *   - "device" pointers are CUDA global-memory addresses on the handle's
 *     device; "host" pointers are ordinary process memory (pinned memory
 *     makes the copies asynchronous, pageable memory is accepted too).
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *     default stream.  Work is enqueued on it in order; no function except
 *     mmoe_forward_host, mmoe_create, mmoe_destroy and mmoe_profile_read
 *     waits for the GPU.
 *   - A handle is not thread-safe: one forward at a time per handle.
 *   - Arguments are checked before anything is launched; a rejected call
 *     leaves the handle and every buffer untouched.
 */
#ifndef MMOE_H
#define MMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mmoe_handle mmoe_handle; /* opaque */

typedef enum {
    MMOE_OK = 0,
    MMOE_ERR_INVALID_ARG = 1,   /* bad pointer, size, shape or enum value */
    MMOE_ERR_NOT_LOADED = 2,    /* forward before mmoe_load_quantized_weights */
    MMOE_ERR_OOM = 3,           /* a device or host allocation failed */
    MMOE_ERR_CUDA = 4,          /* a CUDA runtime call failed (message has the CUDA error) */
    MMOE_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up; the context stays usable */
    MMOE_ERR_UNIMPLEMENTED = 6  /* a valid request this build does not serve */
} mmoe_status;

/* Router gating.  Selection is the top-k of the FP32 biased logits for
 * gating 0 and 1 (the lower expert index first among equal logits; the two
 * select the same experts and differ in the gates), and of the biased
 * sigmoid scores for gating 2. */
typedef enum {
    /* p = softmax over all experts, gate_j = p[idx_j], no renormalisation
     * (the gating the layer benchmark fixes) */
    MMOE_GATE_SOFTMAX = 0,
    /* p_e = sigmoid(l_e), gate_j = p[idx_j] / sum_j' p[idx_j'] ("sigmoid
     * gating with per-token top-k normalisation", section "MoE training
     * stability techniques") */
    MMOE_GATE_SIGMOID_TOPK_NORM = 1,
    /* as MMOE_GATE_SIGMOID_TOPK_NORM, with the router bias (has_router_bias)
     * used the way the auxiliary-loss-free load balancing uses it ("MoE
     * training stability techniques": a per-expert bias adjusted from the
     * load imbalance, with no extra loss): p_e = sigmoid(l_e) with l_e WITHOUT
     * the bias, idx = top-k of the FP32 sums p_e + b_e (lower index first
     * among equal sums), gate_j = p[idx_j] / sum_j' p[idx_j'].  The bias moves
     * the selection only and never enters a gate; the logits reported by
     * MMOE_STAGE_LOGITS exclude it. */
    MMOE_GATE_SIGMOID_TOPK_NORM_SEL_BIAS = 2
} mmoe_gating;

/* mmoe_config.flags */
#define MMOE_FLAG_DETERMINISTIC 1u /* combine in a fixed order, y = FFN_s + g_0 FFN_0 + ... + g_{k-1} FFN_{k-1},
                                      on every path, so that y is bit-reproducible (by default the
                                      prefill and decode expert GEMMs add into y with FP32 atomics, in
                                      whatever order they arrive); needs an extra
                                      [max_tokens*(k+1), d_model] FP32 workspace */
#define MMOE_FLAG_CUDA_CORES 2u    /* run the expert GEMMs on CUDA cores (dp4a) even where the tensor-core
                                      kernels apply (those need d_model and both hidden sizes to be
                                      multiples of 128); same results, slower */
#define MMOE_FLAG_ATOMIC_COMBINE 8u /* atomics into y: the default of mmoe_forward (accepted, changes
                                      nothing there); for mmoe_forward_static_scratch, whose default is
                                      the fixed-order combine, it selects the atomics (ignored with
                                      MMOE_FLAG_DETERMINISTIC) */
#define MMOE_FLAG_NO_DECODE 4u     /* never take the decode path: by default a forward with few tokens
                                      (T <= 64 where d_model and both hidden sizes are multiples of 64)
                                      runs the weight-streaming decode kernels; same results */
#define MMOE_FLAG_NO_FUSED_DECODE 32u /* a forward of at most 8 tokens on the decode path runs the layer as
                                      one launch of thread-block clusters by default (each cluster routes
                                      the tokens itself and computes whole experts; y is cleared and
                                      added with atomics, or in the fixed order of Eq. (*) with
                                      MMOE_FLAG_DETERMINISTIC); this flag keeps the four launches of the
                                      larger decode batches; the same routing and codes, y within
                                      FP32 rounding of the router's summation order */
#define MMOE_FLAG_FUSED_REQUANT 64u /* the prefill gate/up GEMM (default tensor-core kind) requantises its
                                      SwiGLU output itself: the CTAs that hold the hidden-feature blocks of
                                      a token tile form a cluster and exchange the per-token maxima through
                                      distributed shared memory, so no FP32 SwiGLU buffer and no separate
                                      requantisation pass exist (needs max hidden size <= 1024); same
                                      results.  Off by default: measured on B200 it is slower than the
                                      separate pass (c4: 6.9 ms against 2.5 ms of gate/up GEMM
                                      and 0.36 ms of SwiGLU and requantisation) */
#define MMOE_FLAG_TC_INT8 16u      /* prefill expert GEMMs on the INT8 tensor-core kind (tcgen05 kind::i8,
                                      S32 group partials) instead of the default f16 kind (exact integer
                                      group partials in FP32 accumulators, which the promotion reads
                                      without a conversion; d_model a multiple of 256 and both hidden
                                      sizes multiples of 128); same results, slower */

typedef struct {
    int32_t d_model;        /* multiple of 32, 64 <= d_model <= 8192 */
    int32_t n_experts;      /* routed experts, 1..64 (60 in MobileMoE) */
    int32_t top_k;          /* 1..min(n_experts, 8) (4 in MobileMoE); with n_experts = top_k every expert runs */
    int32_t expert_hidden;  /* routed expert hidden size h, multiple of 32, 32..4096 */
    int32_t shared_hidden;  /* shared expert hidden size, multiple of 32, 32..4096 */
    int32_t group_size;     /* must be 32 (Eq. (6) group size) */
    int32_t max_tokens;     /* largest T a forward may pass, 1..2^20; sizes the workspace */
    int32_t gating;         /* mmoe_gating */
    int32_t has_router_bias;/* 0 or 1: a per-expert FP32 bias, added to the logits before gating
                               (gating 0, 1) or to the sigmoid scores for the selection only (2) */
    uint32_t flags;         /* MMOE_FLAG_* */
} mmoe_config;

/* Quantised weights in the interchange layout (row-major, packed INT4 with
 * the element of even K index in the low nibble, sign in two's complement,
 * one FP32 scale per 32 consecutive K elements of a row, as Eq. (6)).
 * Expert index n_experts is the shared expert; its blocks follow the routed
 * ones at the same per-expert stride (so expert g starts at g times the
 * routed expert's block size) and hold shared_hidden rows/columns.
 *
 *   w_router    FP32 [d_model, n_experts]
 *   router_bias FP32 [n_experts], or NULL when has_router_bias = 0
 *   w_gate_up   uint8 expert g at byte g*2h*d/2: [2*hid, d/2]; rows 0..hid-1 are
 *               the gate projection, rows hid..2hid-1 the up projection
 *   s_gate_up   FP32  expert g at g*2h*d/32:     [2*hid, d/32]
 *   w_down      uint8 expert g at byte g*d*h/2:  [d, hid/2]
 *   s_down      FP32  expert g at g*d*h/32:      [d, hid/32]
 * (h = expert_hidden, hid = h for routed experts and shared_hidden for the
 * shared one, d = d_model). */
typedef struct {
    const float* w_router;
    const float* router_bias;
    const uint8_t* w_gate_up;
    const float* s_gate_up;
    const uint8_t* w_down;
    const float* s_down;
    int32_t on_device; /* 1: all pointers are device pointers; 0: host pointers */
} mmoe_weights;

/* Creates a handle on CUDA device `device` and allocates its workspace (sized
 * by max_tokens) and weight buffers.  The handle owns that memory until
 * mmoe_destroy.  *out is set only on success.
 * Errors: INVALID_ARG (cfg out of range, bad device), OOM, CUDA. */
mmoe_status mmoe_create(const mmoe_config* cfg, int device, mmoe_handle** out);

/* Copies the weights into the handle's buffers and re-tiles them into the
 * kernels' layouts (stream-ordered, asynchronous).  The caller keeps
 * ownership of `w` and may free or reuse it once the stream has reached this
 * point.  May be called again to replace the weights.  A call that fails
 * after its argument checks leaves the handle unloaded: forwards return
 * NOT_LOADED until a load succeeds.
 * Errors: INVALID_ARG (NULL pointer, bias presence not matching the config), CUDA. */
mmoe_status mmoe_load_quantized_weights(mmoe_handle* h, const mmoe_weights* w, void* stream);

/* The layer, Eq. (*): y[T, d_model] (FP32, device) from x[T, d_model]
 * (BF16 bit patterns, device).  Optional device outputs, each may be NULL:
 *   topk_idx      int32 [T, top_k]  selected experts, by descending logit
 *   topk_gate     FP32  [T, top_k]  their gates
 *   expert_counts int32 [n_experts + 1] tokens per routed expert, then T for
 *                 the shared expert (the expert-utilisation histogram)
 * T = 0 is a no-op.  x and y must be 16-byte aligned and must not overlap;
 * y is fully overwritten.
 * Paths: T <= 64 runs the decode kernels (weight streaming; T <= 8 as one
 * launch, see MMOE_FLAG_NO_FUSED_DECODE) unless the config sets
 * MMOE_FLAG_NO_DECODE or the shapes do not allow them; larger T runs the
 * prefill kernels (grouped tensor-core GEMMs).  The paths sum the router's
 * FP32 products in different orders, so a token whose k-th and (k+1)-th
 * logits lie within that rounding may be routed differently; otherwise they
 * have the same routing, integer partials and SwiGLU codes, and y is the same
 * up to FP32 rounding of its summation order (atomics by default; bit for
 * bit repeatable with MMOE_FLAG_DETERMINISTIC).
 * Errors: INVALID_ARG (T < 0, T > max_tokens, NULL or misaligned x or y),
 * NOT_LOADED, TIMEOUT (a bounded wait of an earlier call gave up), CUDA. */
mmoe_status mmoe_forward(mmoe_handle* h, const uint16_t* x_bf16, int64_t T, float* y, void* stream,
                         int32_t* topk_idx, float* topk_gate, int32_t* expert_counts);

/* The same layer with HOST buffers: x (host, BF16 bits [T, d_model]) in,
 * y (host, FP32 [T, d_model]) out; returns when y is written.  A batch of
 * T >= 16384 tokens runs as n = min(4, T / 8192) chunks (for n >= 3 the first
 * and last are a third the size of the others): chunk i's
 * x is copied on an internal stream, mmoe_forward runs on `stream` after that
 * copy, and its y is copied back on a second internal stream, so copies and
 * the layer overlap.  Each token's output depends on that token alone, so y
 * equals that of one unsplit forward.  Pinned host memory makes the copies
 * asynchronous; pageable memory works but overlaps less.  `stream` is ordered
 * after both internal streams on return.  The inspection functions below then
 * describe the last chunk.  Errors: as mmoe_forward. */
mmoe_status mmoe_forward_host(mmoe_handle* h, const uint16_t* x_bf16_host, int64_t T, float* y_host,
                              void* stream);

/* Layers one after another on the same tokens, as in a decoder stack: layer 0
 * reads x (BF16, device, [T, d_model]); layer l + 1 reads layer l's y rounded
 * to BF16 (round to nearest even); y_layers[l] (device, FP32 [T, d_model], each
 * 16-byte aligned) receives layer l's y.  layers[l] is the handle of layer l
 * (host array of n_layers handles; y_layers likewise a host array of device
 * pointers).  Every handle must be loaded, on the same device and created with
 * the same d_model, n_experts, top_k, expert_hidden, shared_hidden and gating.
 * When layer 0's handle runs the one-launch decode and T <= 8, the whole stack
 * is ONE launch: its clusters move from layer to layer, each layer's router
 * starting once every contribution to the previous layer's y is in (a bounded
 * wait on a counter in global memory: TIMEOUT on the next call if it gave up),
 * with the next layer's router weights fetched and the shared expert's weights
 * requested before the layer's input is there.  Layer 0's flags decide the
 * combine (atomics, or the fixed order with MMOE_FLAG_DETERMINISTIC).  That
 * launch uses layer 0's workspace; the inspection functions of the other
 * handles are not updated.  Otherwise each layer is one mmoe_forward on its own
 * handle, with the BF16 rounding of y in between.  Either way each layer's y
 * equals that of mmoe_forward on the rounded input, within FP32 rounding of the
 * router's and the combine's summation orders (bit for bit in deterministic
 * mode on the same kernels).
 * The y_layers must not overlap one another or x.
 * Errors: INVALID_ARG (n_layers outside [1, MMOE_MAX_CHAIN_LAYERS], NULL or
 * mismatched handles, T outside [0, max_tokens] of any handle, NULL,
 * misaligned or overlapping pointers), NOT_LOADED, TIMEOUT, OOM, CUDA. */
#define MMOE_MAX_CHAIN_LAYERS 32
mmoe_status mmoe_forward_chain(mmoe_handle* const* layers, int32_t n_layers, const uint16_t* x_bf16, int64_t T,
                               float* const* y_layers, void* stream);

/* Waits for the handle's pending work, frees everything it owns and the
 * handle itself.  NULL is accepted (no-op). */
mmoe_status mmoe_destroy(mmoe_handle* h);

/* Thread-local text of the last error on this thread ("" if none). */
const char* mmoe_last_error(void);

/* Eq. (6) (section "QAT") on the device: W[rows, K] FP32 (device) ->
 * packed INT4 [rows, K/2] (device, interchange layout) and scales
 * FP32 [rows, K/32] (device): s = 2 max|W_g| / 15 (IEEE division),
 * q = clamp(round-half-even(W / s), -8, 7); an all-zero group gets s = 0.
 * Errors: INVALID_ARG (NULL pointer, rows < 0, K not a multiple of 32), CUDA. */
mmoe_status mmoe_quantize_int4(const float* w, int64_t rows, int64_t K, uint8_t* packed, float* scales,
                               void* stream);

/* ---- inspection of the last forward (tests and profiling) ----------------
 * Copies an internal buffer of the handle, as left by the last mmoe_forward,
 * into `dst` (device, `bytes` long; stream-ordered).  R = T*(top_k+1) rows:
 * rows of the routed experts in expert order, each expert's rows in
 * ascending (token, slot), then the T shared-expert rows in token order.
 *   MMOE_STAGE_XQ       int8  [T, d_model]  activation codes
 *   MMOE_STAGE_SX       FP32  [T]           activation scales
 *   MMOE_STAGE_OFFSETS  int32 [n_experts+2] first row of each group, then R
 *   MMOE_STAGE_ROW_SRC  int32 [R]           token of each row
 *   MMOE_STAGE_SLOT_ROW int32 [T, top_k]    row of each (token, slot)
 *   MMOE_STAGE_HQ       int8  [R, hmax]     SwiGLU output codes (hmax = max hidden)
 *   MMOE_STAGE_SH       FP32  [R]           SwiGLU output scales
 *   MMOE_STAGE_LOGITS   FP32  [T, n_experts] router logits (biased for gating 0 and 1)
 * Errors: INVALID_ARG (unknown stage, bytes larger than the stage), CUDA. */
typedef enum {
    MMOE_STAGE_XQ = 0,
    MMOE_STAGE_SX = 1,
    MMOE_STAGE_OFFSETS = 2,
    MMOE_STAGE_ROW_SRC = 3,
    MMOE_STAGE_SLOT_ROW = 4,
    MMOE_STAGE_HQ = 5,
    MMOE_STAGE_SH = 6,
    MMOE_STAGE_LOGITS = 7
} mmoe_stage;

mmoe_status mmoe_debug_copy_stage(mmoe_handle* h, int32_t stage, void* dst, size_t bytes, void* stream);

/* Re-runs the expert GEMMs of the last forward with their INT32 group
 * partials written out (the exact per-group INT8 x INT4 sums the tensor
 * cores accumulate), for rows [row0, row0 + nrows) of the permuted order:
 *   which = 0: gate/up partials  int32 [nrows, 2*hmax, d_model/32] (gate rows, then up rows)
 *   which = 1: down partials     int32 [nrows, d_model, hmax/32]
 * `dst` is device memory.  Errors: INVALID_ARG, NOT_LOADED, CUDA. */
mmoe_status mmoe_debug_partials(mmoe_handle* h, int32_t which, int64_t row0, int64_t nrows, int32_t* dst,
                                void* stream);

/* The chunks mmoe_forward_host splits a T-token batch into (host only, no
 * device call): writes n + 1 boundaries 0 = bounds[0] < ... < bounds[n] = T
 * (for T > 0; T = 0 gives n = 1, bounds {0, 0}) to the host array `bounds`
 * of `cap` entries and n to `*n`.  Errors: INVALID_ARG (T < 0, NULL pointer,
 * cap < n + 1). */
mmoe_status mmoe_debug_host_chunks(int64_t T, int64_t* bounds, int32_t cap, int32_t* n);

/* Allocation-failure injection (tests): after `after` more device
 * allocations by the library on the calling thread, the next one fails as if
 * the device were out of memory (mmoe_create, the staging buffers of
 * mmoe_forward_host); after = 0 fails the very next one, -1 turns the
 * injection off.  It fires once, then turns itself off.  The failing call
 * returns MMOE_ERR_OOM and frees whatever it had allocated.
 * Errors: INVALID_ARG (after < -1). */
mmoe_status mmoe_debug_fail_alloc(int64_t after);

/* Failure detection without a GPU fault.  Sets how long (in SM clock
 * cycles) a bounded device-side wait of the prefill tensor-core GEMMs
 * (default kind) lasts before it gives up; clocks = 0 restores the default
 * (4e9 cycles, about 2 s).  With stall_next = 1 the next forward that takes
 * the prefill path makes one of those waits wait for a barrier that nothing
 * signals, as a hung producer would: the wait runs out after `clocks`, the
 * GEMM drains its copies in flight and exits without writing its outputs, and
 * the following mmoe_forward (or mmoe_destroy) on the handle returns
 * MMOE_ERR_TIMEOUT; later forwards run normally.  A caller has no reason to
 * call this outside tests.
 * Errors: INVALID_ARG (NULL handle, clocks < 0, stall_next not 0 or 1),
 * UNIMPLEMENTED (stall_next = 1 on a handle without the default tensor-core
 * GEMMs). */
mmoe_status mmoe_debug_set_wait_limit(mmoe_handle* h, int64_t clocks, int32_t stall_next);

/* ---- per-stage timing ------------------------------------------------------
 * While profiling is enabled, every forward records a CUDA event pair on its
 * own stream around each stage's kernels.  mmoe_profile_read waits for those
 * events and returns, per stage, the number of kernel launches and their
 * summed device time in milliseconds, accumulated since the last enable.
 * Stages (index into the arrays):
 *   MMOE_PROF_ZERO_Y    clearing y before the atomic combine (a memset, not a kernel)
 *   MMOE_PROF_ROUTER    activation quantiser + FP32 router + top-k
 *   MMOE_PROF_PERMUTE   histogram, scan, stable scatter, row gather
 *   MMOE_PROF_GATE_UP   grouped gate/up GEMM with SwiGLU
 *   MMOE_PROF_REQUANT   per-row requantisation of the SwiGLU output
 *   MMOE_PROF_DOWN      grouped down GEMM with the gate-weighted combine
 *   MMOE_PROF_COMBINE   deterministic combine
 *   MMOE_PROF_DECODE_FUSED  the one-launch decode of up to 8 tokens (all of the above)
 * Errors: INVALID_ARG (n < 1, NULL arrays), CUDA. */
enum {
    MMOE_PROF_ZERO_Y = 0,
    MMOE_PROF_ROUTER = 1,
    MMOE_PROF_PERMUTE = 2,
    MMOE_PROF_GATE_UP = 3,
    MMOE_PROF_REQUANT = 4,
    MMOE_PROF_DOWN = 5,
    MMOE_PROF_COMBINE = 6,
    MMOE_PROF_DECODE_FUSED = 7,
    MMOE_PROF_STAGES = 8
};

mmoe_status mmoe_profile_enable(mmoe_handle* h, int32_t enable);
mmoe_status mmoe_profile_read(mmoe_handle* h, int32_t* launches, double* total_ms, int32_t n);

/* ---- forward without any allocation --------------------------------------
 * The paper has no counterpart to this entry point; it serves callers that
 * must not allocate device memory on their own: a host framework that owns
 * all of the GPU's memory through its own pool and hands an operator only the
 * buffers it passes, or a serving loop that may not block on (or fail in)
 * cudaMalloc once it runs.  mmoe_create allocates its workspace and weight
 * copies, so those callers cannot use a handle.
 *
 * This call runs the same layer as mmoe_forward on weights the caller keeps
 * on the device in the interchange layout (mmoe_weights, on_device = 1,
 * read in place: nothing is copied or re-tiled), with x and y as in
 * mmoe_forward.  All intermediate data lives in one array that the library
 * declares at file scope in device memory, MMOE_STATIC_SCRATCH_BYTES long;
 * every GPU that loads the library holds that array until the process exits.
 *   - Kernels: the CUDA-core expert GEMMs (no re-tiled weight copies exist in
 *     this mode).  The expert outputs are added in the fixed order of
 *     mmoe_forward's prefill path (y bit-reproducible from run to run) unless
 *     cfg->flags has MMOE_FLAG_ATOMIC_COMBINE, which adds them with atomics
 *     and needs less scratch.
 *   - Alignment: x, y, w_gate_up and w_down 16-byte aligned; w_router,
 *     router_bias, s_gate_up and s_down 4-byte aligned (they are read in
 *     place with vector loads).
 *   - Size limit: T <= 2^20, and the scratch a call needs grows with T,
 *     d_model, the hidden sizes and top_k: about
 *     T*(top_k+1)*(d_model + 9*max_hidden) bytes, plus T*(top_k+1)*d_model*4
 *     for the fixed-order combine.  A call that needs more than the array
 *     holds is rejected with MMOE_ERR_INVALID_ARG before anything is
 *     launched.  cfg->max_tokens is not used.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current; make that
 *     first call before any stream capture.
 *   - Sharing: every call on a device uses the same array and leaves its
 *     contents behind.  Each kernel writes every scratch word it later reads,
 *     so nothing needs clearing between calls (also when T changes from one
 *     call to the next), but calls whose work overlaps on the GPU (different
 *     streams, or different host threads) race on the array and corrupt each
 *     other's results: order them on one stream.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 * Errors: INVALID_ARG (bad config, NULL, host or misaligned weight pointers,
 * T < 0 or T > 2^20, NULL or misaligned x or y, the scratch limit), CUDA. */
#define MMOE_STATIC_SCRATCH_BYTES (8u * 1024u * 1024u)

mmoe_status mmoe_forward_static_scratch(const mmoe_config* cfg, const mmoe_weights* w, const uint16_t* x_bf16,
                                        int64_t T, float* y, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MMOE_H */
