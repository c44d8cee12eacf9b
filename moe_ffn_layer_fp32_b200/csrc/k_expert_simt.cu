// Grouped expert GEMMs on CUDA cores (dp4a), the SwiGLU requantisation and
// the deterministic combine.
//
// MobileMoE pages (paper-archivist reading): each expert is a SwiGLU FFN
// ("base architecture"), run per expert on its contiguous token slice with
// the gate and up projections in one GEMM, then SwiGLU, the down projection
// and a weighted scatter back to token order (section "custom MoE kernel");
// weights are symmetric group-32 INT4 with FP32 scales (Eq. (6)) and
// activations INT8 (section "QAT").
//
// Every group of 32 K elements gives an exact INT32 partial P_j (INT8 x INT4);
// it is promoted as acc = fma(float(P_j), s_j, acc) for j ascending, then
// multiplied by the row's activation scale.
#include <cuda_bf16.h>

#include "mmoe_internal.cuh"

namespace mmoe {
namespace {

constexpr int kThreads = 256;
constexpr int kBF = 64;        // output features per block
constexpr int kKChunk = 2048;  // K elements staged in shared memory at a time

// Sign-extends the 8 nibbles of w: the 4 nibbles at even positions (bytes'
// low halves) go to *lo, the odd ones to *hi, one signed byte each.
__device__ __forceinline__ void unpack_int4(uint32_t w, int& lo, int& hi) {
    const uint32_t l = w & 0x0f0f0f0fu, h = (w >> 4) & 0x0f0f0f0fu;
    lo = (int)(l | ((l & 0x08080808u) * 0x1eu));
    hi = (int)(h | ((h & 0x08080808u) * 0x1eu));
}

// Stages rows [0, 32) of an INT8 matrix slice (columns [c0, c0 + kc)) into
// shared memory with every 8-byte chunk split into its even and odd bytes,
// matching the nibble order of unpack_int4.  Rows >= nr are zero.
__device__ __forceinline__ void stage_rows(uint32_t* xs, const int8_t* src, int64_t ld, int nr, int c0, int kc) {
    const int cpr = kc / 8;
    for (int i = threadIdx.x; i < kTileRows * cpr; i += kThreads) {
        const int r = i / cpr, c = i % cpr;
        uint2 v = make_uint2(0, 0);
        if (r < nr) v = *reinterpret_cast<const uint2*>(src + r * ld + c0 + c * 8);
        xs[r * (kc / 4) + 2 * c] = __byte_perm(v.x, v.y, 0x6420);
        xs[r * (kc / 4) + 2 * c + 1] = __byte_perm(v.x, v.y, 0x7531);
    }
}

// acc[r] += float(P_j(row r)) * s for one group (32 K elements) of one weight row
__device__ __forceinline__ void group_dot8(const uint32_t* xs, int kcw, int row0, int jw, const uint4 w, float s,
                                           float (&acc)[8], int32_t (&praw)[8]) {
    int lo[4], hi[4];
    unpack_int4(w.x, lo[0], hi[0]);
    unpack_int4(w.y, lo[1], hi[1]);
    unpack_int4(w.z, lo[2], hi[2]);
    unpack_int4(w.w, lo[3], hi[3]);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const uint32_t* xr = xs + (row0 + r) * kcw + jw;
        const uint4 a = *reinterpret_cast<const uint4*>(xr);
        const uint4 b = *reinterpret_cast<const uint4*>(xr + 4);
        int P = 0;
        P = __dp4a((int)a.x, lo[0], P);
        P = __dp4a((int)a.y, hi[0], P);
        P = __dp4a((int)a.z, lo[1], P);
        P = __dp4a((int)a.w, hi[1], P);
        P = __dp4a((int)b.x, lo[2], P);
        P = __dp4a((int)b.y, hi[2], P);
        P = __dp4a((int)b.z, lo[3], P);
        P = __dp4a((int)b.w, hi[3], P);
        praw[r] = P;
        acc[r] = fmaf((float)P, s, acc[r]);
    }
}

struct TileInfo {
    int g, hid, nr;
    int64_t row0;  // first global row of the tile
};

__device__ __forceinline__ bool decode_tile(const Plan& p, TileInfo& ti) {
    if ((int)blockIdx.x >= *p.tile_count) return false;
    const int code = p.tiles[blockIdx.x];
    ti.g = code >> 24;
    const int t = code & 0xffffff;
    ti.hid = ti.g < p.E ? p.h : p.hs;
    const int cnt = p.offsets[ti.g + 1] - p.offsets[ti.g];
    ti.row0 = (int64_t)p.offsets[ti.g] + (int64_t)t * kTileRows;
    ti.nr = min(kTileRows, cnt - t * kTileRows);
    return true;
}

// gate/up GEMM + SwiGLU: act[row, n] = silu(g) * u
__global__ void __launch_bounds__(kThreads) gate_up_simt_kernel(Plan p, int32_t* dump, int64_t drow0, int64_t dnrows)
{
    extern __shared__ __align__(16) uint32_t xs[];
    TileInfo ti;
    if (!decode_tile(p, ti)) return;
    const int n0 = blockIdx.y * kBF;
    if (n0 >= ti.hid) return;
    const int d = p.d, ng = d / kGroup;
    const int tid = threadIdx.x, f = tid & (kBF - 1), tq = tid / kBF;
    const int n = n0 + f;
    const bool active = n < ti.hid;
    const uint8_t* wexp = p.w_gate_up + (int64_t)ti.g * 2 * p.h * (d / 2);
    const float* sexp = p.s_gate_up + (int64_t)ti.g * 2 * p.h * ng;
    const uint4* wg = reinterpret_cast<const uint4*>(wexp + (int64_t)(active ? n : 0) * (d / 2));
    const uint4* wu = reinterpret_cast<const uint4*>(wexp + (int64_t)(ti.hid + (active ? n : 0)) * (d / 2));
    const float* sg = sexp + (int64_t)(active ? n : 0) * ng;
    const float* su = sexp + (int64_t)(ti.hid + (active ? n : 0)) * ng;
    float ag[8], au[8];
    int32_t pg[8], pu[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) ag[r] = au[r] = 0.0f;
    for (int c0 = 0; c0 < d; c0 += kKChunk) {
        const int kc = min(kKChunk, d - c0);
        __syncthreads();
        stage_rows(xs, p.xq + ti.row0 * d, d, ti.nr, c0, kc);
        __syncthreads();
        if (active) {
            for (int jl = 0; jl < kc / kGroup; ++jl) {
                const int j = c0 / kGroup + jl;
                group_dot8(xs, kc / 4, tq * 8, jl * 8, wg[j], sg[j], ag, pg);
                group_dot8(xs, kc / 4, tq * 8, jl * 8, wu[j], su[j], au, pu);
                if (dump) {
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const int64_t grow = ti.row0 + tq * 8 + r;
                        if (tq * 8 + r < ti.nr && grow >= drow0 && grow < drow0 + dnrows) {
                            int32_t* base = dump + (grow - drow0) * 2 * p.hmax * ng;
                            base[(int64_t)n * ng + j] = pg[r];
                            base[(int64_t)(p.hmax + n) * ng + j] = pu[r];
                        }
                    }
                }
            }
        }
    }
    if (!active) return;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        if (tq * 8 + r >= ti.nr) continue;
        const int64_t grow = ti.row0 + tq * 8 + r;
        const float sxr = p.sx[p.row_src[grow]];
        reinterpret_cast<float2*>(p.act)[grow * p.hmax + n] = make_float2(__fmul_rn(ag[r], sxr), __fmul_rn(au[r], sxr));
    }
}

// per-row SwiGLU and requantisation: a = silu(gv) * uv from the gate/up pairs, s_h = absmax / 127, the
// codes; one warp per row, its SwiGLU values kept in shared memory between the two passes
__global__ void __launch_bounds__(kThreads) requant_kernel(Plan p)
{
    extern __shared__ __align__(16) float arow[];  // [warps][hmax]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + warp;
    if (row >= p.R) return;
    const int hid = row >= p.Tk ? p.hs : p.h;
    float* a = arow + (size_t)warp * p.hmax;
    // 32 bytes per lane: rows start on 8 * hmax bytes and hid is a multiple of 32
    const float4* pr = reinterpret_cast<const float4*>(p.act + row * 2 * p.hmax);
    float m = 0.0f;
#pragma unroll 2
    for (int i = lane; i < hid / 4; i += 32) {
        const float4 v0 = pr[2 * i], v1 = pr[2 * i + 1];
        const float4 s4 = make_float4(swiglu_pair(v0.x, v0.y), swiglu_pair(v0.z, v0.w), swiglu_pair(v1.x, v1.y),
                                      swiglu_pair(v1.z, v1.w));
        reinterpret_cast<float4*>(a)[i] = s4;
        m = fmaxf(m, fmaxf(fmaxf(fabsf(s4.x), fabsf(s4.y)), fmaxf(fabsf(s4.z), fabsf(s4.w))));
    }
    m = warp_max(m);
    const float s = __fdiv_rn(m, 127.0f);
    const float4* a4 = reinterpret_cast<const float4*>(a);
    if (p.hq16) {
        // f16 codes for the kind::f16 down GEMM
        uint2* q = reinterpret_cast<uint2*>(p.hq16 + row * p.hmax);
#pragma unroll 4
        for (int i = lane; i < hid / 4; i += 32) {
            const float4 v = a4[i];
            q[i] = make_uint2(code_f16(quant_i8(v.x, s)) | (code_f16(quant_i8(v.y, s)) << 16),
                              code_f16(quant_i8(v.z, s)) | (code_f16(quant_i8(v.w, s)) << 16));
        }
    } else {
        uint32_t* q = reinterpret_cast<uint32_t*>(p.hq + row * p.hmax);
#pragma unroll 4
        for (int i = lane; i < hid / 4; i += 32) {
            const float4 v = a4[i];
            q[i] = (uint32_t)(quant_i8(v.x, s) & 0xff) | (uint32_t)(quant_i8(v.y, s) & 0xff) << 8 |
                   (uint32_t)(quant_i8(v.z, s) & 0xff) << 16 | (uint32_t)(quant_i8(v.w, s) & 0xff) << 24;
        }
    }
    if (lane == 0) p.sh[row] = s;
}

// down GEMM; the epilogue scatters gate * o into y (atomic) or stores o (deterministic)
__global__ void __launch_bounds__(kThreads) down_simt_kernel(Plan p, int32_t* dump, int64_t drow0, int64_t dnrows)
{
    extern __shared__ __align__(16) uint32_t xs[];
    TileInfo ti;
    if (!decode_tile(p, ti)) return;
    const int d = p.d;
    const int m0 = blockIdx.y * kBF;
    const int tid = threadIdx.x, f = tid & (kBF - 1), tq = tid / kBF;
    const int m = m0 + f;
    const bool active = m < d;
    const int hid = ti.hid, ng = hid / kGroup;
    const uint8_t* wexp = p.w_down + (int64_t)ti.g * d * (p.h / 2);
    const float* sexp = p.s_down + (int64_t)ti.g * d * (p.h / kGroup);
    const uint4* wr = reinterpret_cast<const uint4*>(wexp + (int64_t)(active ? m : 0) * (hid / 2));
    const float* sr = sexp + (int64_t)(active ? m : 0) * ng;
    float acc[8];
    int32_t praw[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = 0.0f;
    for (int c0 = 0; c0 < hid; c0 += kKChunk) {
        const int kc = min(kKChunk, hid - c0);
        __syncthreads();
        stage_rows(xs, p.hq + ti.row0 * p.hmax, p.hmax, ti.nr, c0, kc);
        __syncthreads();
        if (active) {
            for (int jl = 0; jl < kc / kGroup; ++jl) {
                const int j = c0 / kGroup + jl;
                group_dot8(xs, kc / 4, tq * 8, jl * 8, wr[j], sr[j], acc, praw);
                if (dump) {
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const int64_t grow = ti.row0 + tq * 8 + r;
                        if (tq * 8 + r < ti.nr && grow >= drow0 && grow < drow0 + dnrows)
                            dump[((grow - drow0) * d + m) * (p.hmax / kGroup) + j] = praw[r];
                    }
                }
            }
        }
    }
    if (!active || dump) return;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        if (tq * 8 + r >= ti.nr) continue;
        const int64_t grow = ti.row0 + tq * 8 + r;
        const float o = __fmul_rn(acc[r], p.sh[grow]);
        if (p.deterministic) {
            p.obuf[grow * d + m] = o;
        } else {
            atomicAdd(p.y + (int64_t)p.row_src[grow] * d + m, __fmul_rn(p.row_gate[grow], o));
        }
    }
}

// y[t] = o(shared row of t) + sum_j gate[t, j] * o(row of slot j), in that order
// (4 consecutive outputs per thread; d_model is a multiple of 32 and the rows 16-byte aligned)
__global__ void __launch_bounds__(kThreads) combine_kernel(Plan p)
{
    const int64_t i4 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i4 >= p.T * p.d / 4) return;
    const int64_t t = i4 * 4 / p.d;
    const int m = (int)(i4 * 4 % p.d);
    float4 y = *reinterpret_cast<const float4*>(p.obuf + (p.Tk + t) * p.d + m);
    for (int j = 0; j < p.k; ++j) {
        const int64_t r = p.slot_row[t * p.k + j];
        const float g = p.gate[t * p.k + j];
        const float4 o = *reinterpret_cast<const float4*>(p.obuf + r * p.d + m);
        y.x = __fadd_rn(y.x, __fmul_rn(g, o.x));
        y.y = __fadd_rn(y.y, __fmul_rn(g, o.y));
        y.z = __fadd_rn(y.z, __fmul_rn(g, o.z));
        y.w = __fadd_rn(y.w, __fmul_rn(g, o.w));
    }
    *reinterpret_cast<float4*>(p.y + i4 * 4) = y;
}

__global__ void f32_to_bf16_kernel(const float* src, uint16_t* dst, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) dst[i] = __bfloat16_as_ushort(__float2bfloat16_rn(src[i]));
}

}  // namespace

cudaError_t launch_f32_to_bf16(const float* src, uint16_t* dst, int64_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    f32_to_bf16_kernel<<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, s>>>(src, dst, n);
    return cudaGetLastError();
}

cudaError_t launch_gate_up(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    if (p.T == 0) return cudaSuccess;
    const size_t smem = (size_t)kTileRows * min(p.d, kKChunk);
    cudaError_t e = cudaFuncSetAttribute(gate_up_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)p.max_tiles, (unsigned)((p.hmax + kBF - 1) / kBF));
    gate_up_simt_kernel<<<grid, kThreads, smem, s>>>(p, dump, row0, nrows);
    return cudaGetLastError();
}

cudaError_t launch_requant(const Plan& p, cudaStream_t s) {
    if (p.T == 0) return cudaSuccess;
    const int64_t blocks = (p.R + kThreads / 32 - 1) / (kThreads / 32);
    const size_t smem = (size_t)(kThreads / 32) * p.hmax * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(requant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    requant_kernel<<<(unsigned)blocks, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_down(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    if (p.T == 0) return cudaSuccess;
    const size_t smem = (size_t)kTileRows * min(p.hmax, kKChunk);
    cudaError_t e = cudaFuncSetAttribute(down_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)p.max_tiles, (unsigned)((p.d + kBF - 1) / kBF));
    down_simt_kernel<<<grid, kThreads, smem, s>>>(p, dump, row0, nrows);
    return cudaGetLastError();
}

cudaError_t launch_combine(const Plan& p, cudaStream_t s) {
    if (p.T == 0) return cudaSuccess;
    const int64_t n = p.T * p.d / 4;
    combine_kernel<<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace mmoe
