// Internal declarations shared by the kernels and the C-ABI of the fused MoE
// FFN layer (MobileMoE, Eq. (*)).  Not part of the public interface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mmoe.h"

namespace mmoe {

constexpr int kGroup = 32;          // Eq. (6) group size along K
constexpr int kMaxExperts = 64;     // routed experts supported by the router kernel
constexpr int kMaxTopK = 8;
constexpr int kChunk = 1024;        // routing slots per permutation block
constexpr int kTileRows = 32;       // rows (token slots) per CUDA-core expert-GEMM tile
constexpr int kTcTileRows = 128;    // rows per tensor-core expert-GEMM tile

// Everything a forward pass needs, as plain device pointers.
struct Plan {
    // shapes
    int d, h, hs, hmax, E, k, gating;
    int64_t T, R, Tk;       // tokens, rows (T*(k+1)), routed rows (T*k)
    bool deterministic;
    // weights (interchange layout)
    const float* w_router;
    const float* router_bias;
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
    float* act;             // [R, hmax] SwiGLU output before requantisation
    int8_t* hq;             // [R, hmax]
    float* sh;              // [R]
    float* obuf;            // [R, d] expert outputs (deterministic combine only)
    int64_t max_tiles;
    int nchunks;
    int tile_rows;          // kTileRows (CUDA-core GEMMs) or kTcTileRows (tensor-core GEMMs)
    // tensor-core path
    bool use_tc;
    const uint8_t* w_gate_up_t;   // pre-tiled weights (tensor-core layout)
    const float* s_gate_up_t;
    const uint8_t* w_down_t;
    const float* s_down_t;
    const void* tmap_xq;          // host pointers to CUtensorMap of xq and hq (128B-swizzled 128 x 128 boxes)
    const void* tmap_hq;
    int* err;                     // device flag: a bounded wait gave up (later CTAs exit at once)
    int* err_host;                // device alias of the host-mapped copy of that flag
};

// Upper bound on the number of tile_rows-row tiles over all groups.
inline int64_t max_tiles_for(int64_t T, int k, int E, int tile_rows = kTileRows) {
    return (T * k + tile_rows - 1) / tile_rows + E + (T + tile_rows - 1) / tile_rows + 1;
}

// launchers (each returns the launch error, if any)
cudaError_t launch_router_quant(const Plan& p, cudaStream_t s);
cudaError_t launch_permute(const Plan& p, cudaStream_t s);
cudaError_t launch_gate_up(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_requant(const Plan& p, cudaStream_t s);
cudaError_t launch_down(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_combine(const Plan& p, cudaStream_t s);
// tensor-core path (k_expert_tc.cu)
bool tc_supported(int d, int h, int hs);
cudaError_t launch_gate_up_tc(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_down_tc(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows);
cudaError_t launch_retile(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn, uint8_t* gu_t,
                          float* sgu_t, uint8_t* dn_t, float* sdn_t, int d, int h, int hs, int E, cudaStream_t s);
size_t tensor_map_bytes();
cudaError_t make_tensor_map(void* map, void* base, uint64_t inner_bytes, uint64_t rows, uint64_t row_stride);
cudaError_t launch_quantize_int4(const float* w, int64_t rows, int64_t K, uint8_t* packed, float* scales,
                                 cudaStream_t s);

// --- device helpers -------------------------------------------------------
__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

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

// Symmetric INT8 code of v with scale s (s = absmax / 127): IEEE division,
// round half to even, clamp to [-127, 127]; s = 0 gives 0.
__device__ __forceinline__ int quant_i8(float v, float s) {
    if (!(s > 0.0f)) return 0;
    int q = __float2int_rn(__fdiv_rn(v, s));
    return max(-127, min(127, q));
}

}  // namespace mmoe
