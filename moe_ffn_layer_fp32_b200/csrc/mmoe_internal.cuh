// Internal declarations shared by the kernels and the C-ABI of the fused MoE
// FFN layer (MobileMoE, Eq. (*)).  Not part of the public interface.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "mmoe.h"

namespace mmoe {

constexpr int kGroup = 32;          // Eq. (6) group size along K
constexpr int kMaxExperts = 64;     // routed experts supported by the router kernel
constexpr int kMaxTopK = 8;
constexpr int kChunk = 1024;        // routing slots per permutation block
constexpr int kTileRows = 32;       // rows (token slots) per CUDA-core expert-GEMM tile
constexpr int kTcTileRows = 128;    // rows per tensor-core expert-GEMM tile
constexpr int kTcNone = 0, kTcF16 = 1, kTcI8 = 2;  // Plan::tc_kind
constexpr long long kDefaultWaitLimit = 4000000000ll;  // about 2 s of SM clock

// Everything a forward pass needs, as plain device pointers.
struct Plan {
    // shapes
    int d, h, hs, hmax, E, k, gating;
    int64_t T, R, Tk;       // tokens, rows (T*(k+1)), routed rows (T*k)
    bool deterministic;
    // weights (interchange layout)
    const float* w_router;
    const float* router_bias;
    const uint16_t* w_router_split;  // W_r as three BF16 pieces (tensor-core router), or null
    const uint8_t* w_gate_up;
    const float* s_gate_up;
    const uint8_t* w_down;
    const float* s_down;
    // activations and routing
    const uint16_t* x;      // [T, d] bf16
    float* y;               // [T, d]
    int8_t* xq;             // [R, d]: routed rows (expert order), then the shared rows = x codes
    float* sx;              // [T]
    float* logits;          // [T, E]
    int32_t* idx;           // [T, k]
    float* gate;            // [T, k]
    int32_t* chunk_cnt;     // [nchunks, kMaxExperts]
    int32_t* chunk_base;    // [nchunks, kMaxExperts]
    int32_t* offsets;       // [E + 2]
    int32_t* counts;        // [E + 1]
    int32_t* tiles;         // [max_tiles]: group << 24 | tile index within the group
    int32_t* tile_count;    // [1]
    int32_t* row_src;       // [R]
    float* row_gate;        // [R]
    int32_t* slot_row;      // [T, k]
    float* act;             // [R, hmax] pairs (gv, uv): gate and up times the row's activation scale
    int8_t* hq;             // [R, hmax]
    float* sh;              // [R]
    float* obuf;            // [R, d] expert outputs (deterministic combine only)
    int64_t max_tiles;
    int nchunks;
    int tile_rows;          // kTileRows (CUDA-core GEMMs) or kTcTileRows (tensor-core GEMMs)
    // tensor-core path: kTcNone (CUDA-core GEMMs), kTcF16 (kind::f16, exact integer partials, the
    // default) or kTcI8 (kind::i8, S32 partials)
    int tc_kind;
    const uint8_t* w_gate_up_t;   // kTcI8: INT8 stage images
    const float* s_gate_up_t;     // pre-tiled group scales (both tensor-core kinds)
    const uint8_t* w_down_t;
    const float* s_down_t;
    const uint16_t* w_gate_up_f16;  // kTcF16: f16 stage images
    const uint16_t* w_down_f16;
    uint16_t* xq16;               // kTcF16: [R, d] activation codes as f16 (replaces xq on that path)
    uint16_t* hq16;               // kTcF16: [R, hmax] SwiGLU codes as f16 (replaces hq on that path)
    const void* tmap_xq;          // host pointers to CUtensorMap of the activation and SwiGLU codes
    const void* tmap_hq;
    long long wait_limit;         // SM clocks a bounded wait of the kind::f16 GEMMs lasts before giving up
    int debug_stall;              // 1: the kind::f16 gate/up GEMM injects a stall (failure-detection tests)
    bool fuse_requant;            // kind::f16: the gate/up GEMM writes the SwiGLU codes itself (clusters)
    int* err;                     // device flag: a bounded wait gave up (later CTAs exit at once)
    int* err_host;                // device alias of the host-mapped copy of that flag
    // decode path (k_decode.cu)
    const uint8_t* w_gate_up_d;   // weights + scales in the decode layout
    const uint8_t* w_down_d;
    int32_t* dec_groups;          // [E + 1] groups with at least one row: the shared one first, then routed ascending
    int32_t* dec_ngroups;         // [1]
};

// Upper bound on the number of tile_rows-row tiles over all groups.
inline int64_t max_tiles_for(int64_t T, int k, int E, int tile_rows = kTileRows) {
    return (T * k + tile_rows - 1) / tile_rows + E + (T + tile_rows - 1) / tile_rows + 1;
}

// launchers (each returns the launch error, if any)
cudaError_t launch_router_quant(const Plan& p, cudaStream_t s);
bool router_mma_supported(int d, int E);
size_t router_split_bytes(int d);
cudaError_t launch_split_router(const float* w, int d, int E, uint16_t* out, cudaStream_t s);
cudaError_t launch_router_mma(const Plan& p, cudaStream_t s);
cudaError_t launch_permute(const Plan& p, cudaStream_t s);
cudaError_t launch_gate_up(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_requant(const Plan& p, cudaStream_t s);
cudaError_t launch_down(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_combine(const Plan& p, cudaStream_t s);
// dst[i] = BF16 bits of src[i] rounded to nearest even (n elements)
cudaError_t launch_f32_to_bf16(const float* src, uint16_t* dst, int64_t n, cudaStream_t s);
// tensor-core path, kind::f16 (k_expert_f16.cu)
bool f16tc_supported(int d, int h, int hs);
int f16tc_fused_clusters(int c);  // clusters of c CTAs of the fused gate/up GEMM the device holds at once
size_t f16tc_image_elems(int d, int h, int hs, int E, bool gate_up);
cudaError_t launch_gate_up_f16(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_down_f16(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_retile_f16(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn,
                              uint16_t* gu_t, float* sgu_t, uint16_t* dn_t, float* sdn_t, int d, int h, int hs, int E,
                              cudaStream_t s);
// f16 codes (integers in [-127, 127]) -> INT8 codes, for the inspection entry point
cudaError_t launch_codes_f16_to_i8(const uint16_t* src, int8_t* dst, int64_t n, cudaStream_t s);
// tensor-core path, kind::i8 (k_expert_tc.cu)
bool tc_supported(int d, int h, int hs);
cudaError_t launch_gate_up_tc(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_down_tc(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_retile(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn, uint8_t* gu_t,
                          float* sgu_t, uint8_t* dn_t, float* sdn_t, int d, int h, int hs, int E, cudaStream_t s);
// decode path (k_decode.cu): T <= dec_max_tokens, expert GEMVs on mma.sync
bool dec_supported(int d, int h, int hs);
int dec_max_tokens(int d, int hmax);
int dec_router_cluster(int d, int E);
cudaError_t launch_router_dec(const Plan& p, int cluster, cudaStream_t s);
// the one-launch decode of up to dec_fused_max_tokens() tokens: clusters of 8 or 16 CTAs (how many
// of each the device holds at once for a shape; 0 where that size does not fit), per-token
// contribution counters (zero before the first launch; every launch leaves them zero) and a small
// row buffer of expert outputs
struct DecFusedShape {
    int clusters8, clusters16;
};
int dec_fused_max_tokens();
DecFusedShape dec_fused_shape(int d, int h, int hs, int E);
size_t dec_fused_counter_words();
size_t dec_fused_obuf_floats(int d);
// One layer as one launch; `chain`: dec_chain_counter_words() words as for launch_decode_chain.
cudaError_t launch_decode_fused(const Plan& p, const DecFusedShape& shape, uint32_t* cnt, float* obuf,
                                uint32_t* chain, int32_t* out_idx, float* out_gate, int32_t* out_counts,
                                cudaStream_t s);
// Layers run back to back by one launch of the same kernel: layer l + 1 reads layer l's y rounded to
// BF16.  All layers share p's shapes, gating and workspace; each brings its own weights (decode layout)
// and output.  `chain`: dec_chain_counter_words() words, zero before the first launch (every launch
// leaves them zero).
constexpr int kDecChainMax = 32;
struct DecChainLayer {
    const float* w_router;
    const float* router_bias;
    const uint8_t* w_gate_up_d;
    const uint8_t* w_down_d;
    float* y;
    int32_t* out_idx;
    float* out_gate;
    int32_t* out_counts;
};
size_t dec_chain_counter_words();
cudaError_t launch_decode_chain(const Plan& p, const DecFusedShape& shape, uint32_t* cnt, float* obuf,
                                uint32_t* chain, const DecChainLayer* layers, int nl, cudaStream_t s);
cudaError_t launch_gate_up_dec(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_down_dec(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_retile_dec(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn,
                              uint8_t* gu_d, uint8_t* dn_d, int d, int h, int hs, int E, cudaStream_t s);
size_t tensor_map_bytes();
// 2-D tensor map of a row-major [rows, inner] matrix of 1- or 2-byte elements, 128-byte swizzle,
// boxes of 128 bytes x 128 rows
cudaError_t make_tensor_map(void* map, void* base, uint64_t inner_elems, uint64_t rows, uint64_t row_stride_bytes,
                            int elem_bytes);
cudaError_t launch_quantize_int4(const float* w, int64_t rows, int64_t K, uint8_t* packed, float* scales,
                                 cudaStream_t s);

// W_r as three BF16 pieces (hi + mid + lo = the FP32 weight), in K chunks of 64:
// per chunk three pieces of [64 experts][72] BF16 (64 K values + 8 of padding
// that keep the mma.sync fragment loads free of shared-memory bank conflicts).
constexpr int kRouterKChunk = 64;
constexpr int kRouterRow = 72;
constexpr int kRouterPieceBytes = 64 * kRouterRow * 2;          // 9216
constexpr int kRouterChunkBytes = 3 * kRouterPieceBytes;        // 27648

// --- device helpers -------------------------------------------------------
// D = A * B (C = 0), m16n8k16, BF16 inputs, FP32 result
__device__ __forceinline__ void mma_bf16_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// D += A * B, m16n8k16, BF16 inputs, FP32 accumulators
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16-wide K step of the router for an m16 x n8 tile: the partial of the step
// (lo, mid, hi pieces on the tensor cores; they only ever sum 48 exact products)
// added to the running logits with round-to-nearest FP32 additions.  `wr` points
// at expert row n*8 + gid, column kk + 2*t4 of the hi piece of the chunk.
__device__ __forceinline__ void router_kstep(float (&acc)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             const uint16_t* wr) {
    float part[4];
    mma_bf16_first(part, a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(wr + kRouterPieceBytes),
                   *reinterpret_cast<const uint32_t*>(wr + kRouterPieceBytes + 8));
    mma_bf16(part, a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(wr + kRouterPieceBytes / 2),
             *reinterpret_cast<const uint32_t*>(wr + kRouterPieceBytes / 2 + 8));
    mma_bf16(part, a0, a1, a2, a3, *reinterpret_cast<const uint32_t*>(wr), *reinterpret_cast<const uint32_t*>(wr + 8));
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = __fadd_rn(acc[i], part[i]);
}

__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// f16 bit pattern of an integer code in [-2048, 2048] (exact)
__device__ __forceinline__ uint32_t code_f16(int q) { return (uint32_t)__half_as_ushort(__int2half_rn(q)); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// SwiGLU of one feature from its gate and up values already scaled by the token's activation scale:
// silu(gv) * uv, silu(v) = v / (1 + exp(-v)), each step an IEEE FP32 operation.  The gate/up GEMMs
// store (gv, uv) pairs; the requantisation pass applies this.
__device__ __forceinline__ float swiglu_pair(float gv, float uv) {
    return __fmul_rn(__fdiv_rn(gv, __fadd_rn(1.0f, expf(-gv))), uv);
}

// Symmetric INT8 code of v with scale s (s = absmax / 127): IEEE division,
// round half to even, clamp to [-127, 127]; s = 0 gives 0.
__device__ __forceinline__ int quant_i8(float v, float s) {
    if (!(s > 0.0f)) return 0;
    int q = __float2int_rn(__fdiv_rn(v, s));
    return max(-127, min(127, q));
}

// Order-preserving unsigned image of an FP32 selection key: key_order(a) > key_order(b) exactly when
// a > b, equal keys (-0 and +0 among them) have equal images, and every key, -inf included, maps above
// 0, the mark of an expert that does not exist or is already selected.
__device__ __forceinline__ uint32_t key_order(float key) {
    const uint32_t b = __float_as_uint(__fadd_rn(key, 0.0f));
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One round of the top-k selection over a warp: the expert with the largest key, the lower index among
// equal keys; u0, u1 are the key_order images of experts lane and lane + 32 (0: not a candidate).
__device__ __forceinline__ int warp_argmax_key(uint32_t u0, uint32_t u1) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, max(u0, u1));
    const unsigned b0 = __ballot_sync(0xffffffffu, u0 == m), b1 = __ballot_sync(0xffffffffu, u1 == m);
    return b0 ? __ffs(b0) - 1 : 31 + __ffs(b1);
}

// The FP32 value of a key_order image (+0 for both zeros).
__device__ __forceinline__ float key_value(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// The gating probabilities of experts lane and lane + 32 and their selection keys (the logit, or for
// gating 2 the sigmoid score plus the bias; -inf where the expert does not exist).
__device__ __forceinline__ void gate_probs_keys(const Plan& p, const float* bias, float l0, float l1, int lane,
                                                float& p0, float& p1, float& k0, float& k1) {
    const int E = p.E;
    const bool v0 = lane < E, v1 = lane + 32 < E;
    if (p.gating == MMOE_GATE_SOFTMAX) {
        const float mx = key_value(__reduce_max_sync(0xffffffffu, key_order(fmaxf(l0, l1))));
        const float e0 = v0 ? expf(__fsub_rn(l0, mx)) : 0.0f;
        const float e1 = v1 ? expf(__fsub_rn(l1, mx)) : 0.0f;
        const float sum = warp_sum(__fadd_rn(e0, e1));
        p0 = __fdiv_rn(e0, sum);
        p1 = __fdiv_rn(e1, sum);
    } else {
        p0 = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-l0)));
        p1 = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-l1)));
    }
    k0 = l0;
    k1 = l1;
    if (p.gating == MMOE_GATE_SIGMOID_TOPK_NORM_SEL_BIAS) {
        k0 = v0 ? (bias ? __fadd_rn(p0, bias[lane]) : p0) : -INFINITY;
        k1 = v1 ? (bias ? __fadd_rn(p1, bias[lane + 32]) : p1) : -INFINITY;
    }
}

// Gating and top-k of token t by one warp.  Lane l holds the logits of
// experts l and l + 32 (-inf where the expert does not exist); the router bias
// is already in them for gating 0 and 1 and not for gating 2 (where `bias` is
// added to the score).  Softmax over all experts (or per-expert sigmoid), then
// k rounds of a warp arg-max on (key descending, index ascending), the key
// being the logit, or for gating 2 the sigmoid score plus the bias (which then
// moves the selection but enters no gate); writes logits (if kept), idx and
// gate (idx and gate may be shared memory).
__device__ __forceinline__ void gate_topk_warp(const Plan& p, const float* bias, int64_t t, float l0, float l1,
                                               int lane, int32_t* idx, float* gate, float* logits) {
    const int E = p.E, k = p.k;
    const bool v0 = lane < E, v1 = lane + 32 < E;
    if (logits) {
        if (v0) logits[t * E + lane] = l0;
        if (v1) logits[t * E + lane + 32] = l1;
    }
    if (p.gating == MMOE_GATE_SOFTMAX) {
        // the keys are the logits: the first round's maximum is the softmax's, and the sum of the
        // exponentials (needed only for the k selected gates) runs alongside the remaining rounds
        uint32_t u0 = v0 ? key_order(l0) : 0u, u1 = v1 ? key_order(l1) : 0u;
        uint32_t m = __reduce_max_sync(0xffffffffu, max(u0, u1));
        const float mx = key_value(m);
        const float e0 = v0 ? expf(__fsub_rn(l0, mx)) : 0.0f;
        const float e1 = v1 ? expf(__fsub_rn(l1, mx)) : 0.0f;
        const float sum = warp_sum(__fadd_rn(e0, e1));
        int my = 0;
        float ge = 0.0f;
        for (int j = 0; j < k; ++j) {
            if (j > 0) m = __reduce_max_sync(0xffffffffu, max(u0, u1));
            const unsigned b0 = __ballot_sync(0xffffffffu, u0 == m), b1 = __ballot_sync(0xffffffffu, u1 == m);
            const int bi = b0 ? __ffs(b0) - 1 : 31 + __ffs(b1);
            if (bi == lane) u0 = 0u;
            if (bi == lane + 32) u1 = 0u;
            const float ev = __shfl_sync(0xffffffffu, (bi < 32) ? e0 : e1, bi & 31);
            if (lane == j) {
                my = bi;
                ge = ev;
            }
        }
        if (lane < k) {
            idx[t * k + lane] = my;
            gate[t * k + lane] = __fdiv_rn(ge, sum);
        }
        return;
    }
    float p0, p1, k0, k1;
    gate_probs_keys(p, bias, l0, l1, lane, p0, p1, k0, k1);
    uint32_t u0 = v0 ? key_order(k0) : 0u, u1 = v1 ? key_order(k1) : 0u;
    int my = 0;
    float g = 0.0f, gsum = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int bi = warp_argmax_key(u0, u1);
        if (bi == lane) u0 = 0u;
        if (bi == lane + 32) u1 = 0u;
        const float pv = __shfl_sync(0xffffffffu, (bi < 32) ? p0 : p1, bi & 31);
        if (lane == j) { my = bi; g = pv; }
        gsum = __fadd_rn(gsum, pv);
    }
    if (lane < k) {
        if (p.gating != MMOE_GATE_SOFTMAX) g = __fdiv_rn(g, gsum);
        idx[t * k + lane] = my;
        gate[t * k + lane] = g;
    }
}

__device__ __forceinline__ void gate_topk_warp(const Plan& p, int64_t t, float l0, float l1, int lane) {
    gate_topk_warp(p, p.router_bias, t, l0, l1, lane, p.idx, p.gate, p.logits);
}

// The router bias enters the logit for gating 0 and 1 (and only the selection key for gating 2).
__device__ __forceinline__ float biased_logit(const Plan& p, const float* bias, float l, int e) {
    return (bias && p.gating != MMOE_GATE_SIGMOID_TOPK_NORM_SEL_BIAS) ? __fadd_rn(l, bias[e]) : l;
}
__device__ __forceinline__ float biased_logit(const Plan& p, float l, int e) {
    return biased_logit(p, p.router_bias, l, e);
}

}  // namespace mmoe
