// K1 + K2: per-token INT8 activation quantisation and the FP32 router with
// softmax / sigmoid gating and top-k, in one pass over x.
//
// MobileMoE pages (paper-archivist reading): Eq. (*) selects the top-k experts
// by router score; "MoE training stability techniques" keeps every router
// computation in FP32 (and names sigmoid gating with per-token top-k
// normalisation); section "QAT" quantises activations to INT8 on the fly.
// The benchmark recipe fixes s_x = absmax / 127 and softmax over all experts
// without renormalisation; among equal logits the lower expert index wins.
#include "mmoe_internal.cuh"

namespace mmoe {
namespace {

constexpr int kThreads = 256;

// One block handles TB tokens: their BF16 rows are staged in shared memory
// once and serve both the quantiser and the router.  Router work split: 64
// expert lanes x 4 quarters of the K range; the 4 quarter sums are added in
// a fixed order, so the logits do not depend on scheduling.
template <int TB>
__global__ void __launch_bounds__(kThreads)
router_quant_kernel(Plan p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int d = p.d, E = p.E;
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem);              // [TB][d]
    float* part = reinterpret_cast<float*>(xs + (size_t)TB * d);   // [4][TB][64]
    float* lg = part + 4 * TB * 64;                                // [TB][64]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t t0 = (int64_t)blockIdx.x * TB;
    const int nt = (int)((p.T - t0) < TB ? (p.T - t0) : TB);

    // stage x rows (16-byte vectors; d is a multiple of 32 so rows are 64-byte aligned)
    {
        const uint4* src = reinterpret_cast<const uint4*>(p.x + t0 * d);
        uint4* dst = reinterpret_cast<uint4*>(xs);
        const int nvec = nt * d / 8;
        for (int i = tid; i < nvec; i += kThreads) dst[i] = src[i];
        for (int i = nvec + tid; i < TB * d / 8; i += kThreads) dst[i] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();

    // K1: activation codes of the shared-expert rows (rows Tk + t of xq)
    for (int tt = warp; tt < nt; tt += kThreads / 32) {
        const uint16_t* row = xs + (size_t)tt * d;
        float m = 0.0f;
        for (int i = lane; i < d; i += 32) m = fmaxf(m, fabsf(bf16_to_f32(row[i])));
        m = warp_max(m);
        const float s = __fdiv_rn(m, 127.0f);
        const int64_t t = t0 + tt;
        if (p.xq16) {
            uint16_t* q = p.xq16 + (p.Tk + t) * d;
            for (int i = lane; i < d; i += 32) q[i] = (uint16_t)code_f16(quant_i8(bf16_to_f32(row[i]), s));
        } else {
            int8_t* q = p.xq + (p.Tk + t) * d;
            for (int i = lane * 4; i < d; i += 128) {
                uint32_t w = 0;
#pragma unroll
                for (int u = 0; u < 4; ++u) w |= (uint32_t)(quant_i8(bf16_to_f32(row[i + u]), s) & 0xff) << (8 * u);
                *reinterpret_cast<uint32_t*>(q + i) = w;
            }
        }
        if (lane == 0) {
            p.sx[t] = s;
            p.row_src[p.Tk + t] = (int32_t)t;
            p.row_gate[p.Tk + t] = 1.0f;
        }
    }

    // K2: logits, FP32 products accumulated in FP32 over a quarter of K each
    {
        const int e = tid & 63, kq = tid >> 6;
        const int kc = d / 4;  // multiple of 8
        float acc[TB];
#pragma unroll
        for (int t = 0; t < TB; ++t) acc[t] = 0.0f;
        if (e < E) {
            for (int kk = kq * kc; kk < (kq + 1) * kc; kk += 8) {
                float w[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) w[u] = __ldg(p.w_router + (size_t)(kk + u) * E + e);
#pragma unroll
                for (int t = 0; t < TB; ++t) {
                    const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)t * d + kk);
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        acc[t] = fmaf(__uint_as_float(xw[u] << 16), w[2 * u], acc[t]);
                        acc[t] = fmaf(__uint_as_float(xw[u] & 0xffff0000u), w[2 * u + 1], acc[t]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TB; ++t) part[(kq * TB + t) * 64 + e] = acc[t];
    }
    __syncthreads();
    for (int i = tid; i < TB * 64; i += kThreads) {
        const int t = i / 64, e = i % 64;
        if (e < E) {
            float l = __fadd_rn(__fadd_rn(__fadd_rn(part[(0 * TB + t) * 64 + e], part[(1 * TB + t) * 64 + e]),
                                          part[(2 * TB + t) * 64 + e]),
                                part[(3 * TB + t) * 64 + e]);
            lg[i] = biased_logit(p, l, e);
        }
    }
    __syncthreads();

    // gating and top-k: one warp per token, lanes hold experts lane and lane + 32
    for (int tt = warp; tt < nt; tt += kThreads / 32) {
        const int64_t t = t0 + tt;
        const float l0 = lane < E ? lg[tt * 64 + lane] : -INFINITY;
        const float l1 = lane + 32 < E ? lg[tt * 64 + lane + 32] : -INFINITY;
        gate_topk_warp(p, t, l0, l1, lane);
    }
}

template <int TB>
cudaError_t launch_tb(const Plan& p, cudaStream_t s) {
    const size_t smem = (size_t)TB * p.d * 2 + (size_t)5 * TB * 64 * 4;
    cudaError_t e = cudaFuncSetAttribute(router_quant_kernel<TB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (p.T + TB - 1) / TB;
    router_quant_kernel<TB><<<(unsigned)blocks, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_quant(const Plan& p, cudaStream_t s) {
    if (p.T == 0) return cudaSuccess;
    if (p.w_router_split) return launch_router_mma(p, s);
    // token tile: as many rows as fit in about 160 KB of shared memory
    if ((size_t)32 * p.d * 2 <= 160 * 1024) return launch_tb<32>(p, s);
    if ((size_t)16 * p.d * 2 <= 160 * 1024) return launch_tb<16>(p, s);
    return launch_tb<8>(p, s);
}

}  // namespace mmoe

// ---------------------------------------------------------------------------
// K1 + K2 for prefill on the tensor cores.
//
// W_r (FP32) is held as three BF16 pieces w = hi + mid + lo, exact for every
// normal FP32 value (each piece carries 8 significant bits of the remainder
// left by the pieces before it, with round-to-nearest), so with BF16 x every
// product x * piece is exact in FP32 and the logit is an FP32 sum of the
// exact products x_k * w_k, accumulated by the tensor cores.
//
// Split layout: K chunks of 64; per chunk three pieces of [64 experts][72]
// BF16 (64 K values + 8 of padding, which keeps the fragment loads free of
// shared-memory bank conflicts); experts >= E are zero.
namespace mmoe {
namespace rmma {

// Tokens per CTA: TOK in {16, 32, 64, 128}, one 16-row MMA tile per warp for the first TOK / 16 warps; the
// gating, top-k and codes of the CTA's tokens are spread over all 8 warps.  Small batches take small TOK,
// so that their CTAs cover the SMs (each CTA reads the whole split W_r from L2).
constexpr int kThreads = 256;
constexpr int kKC = kRouterKChunk;        // K per chunk
constexpr int kRow = kRouterRow;          // padded BF16 row of a chunk
constexpr int kWPieceBytes = kRouterPieceBytes;
constexpr int kWChunkBytes = kRouterChunkBytes;
constexpr int kStages = 2;
constexpr int kLgRow = 65;                // padded logits row
template <int TOK>
struct Tiling {
    static constexpr int kXChunkBytes = TOK * kRow * 2;
    // the logits and scales (TOK x 65 + TOK floats) alias the stages
    static constexpr size_t kSmem = (size_t)kStages * (kXChunkBytes + kWChunkBytes);
    static_assert((size_t)TOK * (kLgRow + 1) * 4 <= kSmem, "logits fit in the stages");
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float bf16_abs(uint32_t bits16) { return fabsf(__uint_as_float(bits16 << 16)); }

// round-to-nearest-even FP32 -> BF16 bits (finite inputs)
__device__ __forceinline__ uint32_t bf16_rn_bits(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
}

// stage K chunk c of x (rows t0 .. t0 + TOK - 1, zero beyond T) and of the split weights
template <int TOK>
__device__ __forceinline__ void load_chunk(const Plan& p, int64_t t0, int nt, int c, uint8_t* xs, uint8_t* ws,
                                           int tid) {
    const int d = p.d;
    for (int i = tid; i < TOK * (kKC / 8); i += kThreads) {
        const int r = i >> 3, v = i & 7;
        uint8_t* dst = xs + r * (kRow * 2) + v * 16;
        if (r < nt) cp_async16(dst, p.x + (t0 + r) * d + c * kKC + v * 8);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.w_router_split) + (size_t)c * kWChunkBytes;
    for (int i = tid; i < kWChunkBytes / 16; i += kThreads) cp_async16(ws + i * 16, src + i * 16);
}

template <int TOK>
__global__ void __launch_bounds__(kThreads, 2) router_mma_kernel(Plan p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int kXChunkBytes = Tiling<TOK>::kXChunkBytes;
    const int d = p.d, E = p.E;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t4 = lane & 3;
    const bool mma_warp = warp * 16 < TOK;
    const int64_t t0 = (int64_t)blockIdx.x * TOK;
    const int nt = (int)((p.T - t0) < TOK ? (p.T - t0) : TOK);
    auto xs = [&](int c) { return smem + (c % kStages) * (kXChunkBytes + kWChunkBytes); };
    auto ws = [&](int c) { return smem + (c % kStages) * (kXChunkBytes + kWChunkBytes) + kXChunkBytes; };
    if (!p.deterministic && p.y) {
        // the expert GEMMs add into y with atomics: this CTA's rows start at zero
        float4* y4 = reinterpret_cast<float4*>(p.y + t0 * d);
        for (int i = tid; i < nt * d / 4; i += kThreads) y4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    const int nchunks = d / kKC;
    float acc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
    float amax_lo = 0.0f, amax_hi = 0.0f;  // |x| max of rows g and g + 8 of this warp, over this lane's elements

    load_chunk<TOK>(p, t0, nt, 0, xs(0), ws(0), tid);
    cp_async_commit();
    for (int c = 0; c < nchunks; ++c) {
        if (c + 1 < nchunks) load_chunk<TOK>(p, t0, nt, c + 1, xs(c + 1), ws(c + 1), tid);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (!mma_warp) {
            __syncthreads();
            continue;
        }
        const uint16_t* xa = reinterpret_cast<const uint16_t*>(xs(c)) + (warp * 16 + g) * kRow + 2 * t4;
        const uint16_t* wb = reinterpret_cast<const uint16_t*>(ws(c)) + g * kRow + 2 * t4;
#pragma unroll
        for (int kk = 0; kk < kKC; kk += 16) {
            const uint32_t a0 = *reinterpret_cast<const uint32_t*>(xa + kk);
            const uint32_t a1 = *reinterpret_cast<const uint32_t*>(xa + 8 * kRow + kk);
            const uint32_t a2 = *reinterpret_cast<const uint32_t*>(xa + kk + 8);
            const uint32_t a3 = *reinterpret_cast<const uint32_t*>(xa + 8 * kRow + kk + 8);
            amax_lo = fmaxf(amax_lo, fmaxf(fmaxf(bf16_abs(a0 & 0xffffu), bf16_abs(a0 >> 16)),
                                           fmaxf(bf16_abs(a2 & 0xffffu), bf16_abs(a2 >> 16))));
            amax_hi = fmaxf(amax_hi, fmaxf(fmaxf(bf16_abs(a1 & 0xffffu), bf16_abs(a1 >> 16)),
                                           fmaxf(bf16_abs(a3 & 0xffffu), bf16_abs(a3 >> 16))));
            // the 16-wide K step's partial (lo, mid, hi pieces) on the tensor cores, then one
            // round-to-nearest FP32 addition into the running logit: the tensor cores only
            // ever sum 48 exact products, so their internal rounding stays far below FP32's
            // over the whole K range
#pragma unroll
            for (int n = 0; n < 8; ++n) router_kstep(acc[n], a0, a1, a2, a3, wb + n * 8 * kRow + kk);
        }
        __syncthreads();  // the stage is refilled by the next iteration
    }
    cp_async_wait<0>();

    // logits into shared memory (aliasing the stages): D fragment rows g / g + 8, columns 2 t4, 2 t4 + 1
    float* lg = reinterpret_cast<float*>(smem);
    float* sxs = lg + TOK * kLgRow;
    if (mma_warp) {
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int col = n * 8 + 2 * t4;
            lg[(warp * 16 + g) * kLgRow + col] = acc[n][0];
            lg[(warp * 16 + g) * kLgRow + col + 1] = acc[n][1];
            lg[(warp * 16 + g + 8) * kLgRow + col] = acc[n][2];
            lg[(warp * 16 + g + 8) * kLgRow + col + 1] = acc[n][3];
        }
        amax_lo = fmaxf(amax_lo, __shfl_xor_sync(0xffffffffu, amax_lo, 1));
        amax_lo = fmaxf(amax_lo, __shfl_xor_sync(0xffffffffu, amax_lo, 2));
        amax_hi = fmaxf(amax_hi, __shfl_xor_sync(0xffffffffu, amax_hi, 1));
        amax_hi = fmaxf(amax_hi, __shfl_xor_sync(0xffffffffu, amax_hi, 2));
        if (t4 == 0) {
            sxs[warp * 16 + g] = __fdiv_rn(amax_lo, 127.0f);
            sxs[warp * 16 + g + 8] = __fdiv_rn(amax_hi, 127.0f);
        }
    }
    __syncthreads();

    // gating and top-k, one warp per token; then the codes of the token's row (rows Tk + t of xq)
    for (int tt = warp; tt < nt; tt += kThreads / 32) {
        const int64_t t = t0 + tt;
        float l0 = -INFINITY, l1 = -INFINITY;
        if (lane < E) l0 = biased_logit(p, lg[tt * kLgRow + lane], lane);
        if (lane + 32 < E) l1 = biased_logit(p, lg[tt * kLgRow + lane + 32], lane + 32);
        gate_topk_warp(p, t, l0, l1, lane);
        const float s = sxs[tt];
        const uint4* xr = reinterpret_cast<const uint4*>(p.x + t * d);
        if (p.xq16) {
            // f16 codes for the kind::f16 expert GEMMs
            uint4* q = reinterpret_cast<uint4*>(p.xq16 + (p.Tk + t) * d);
            for (int i = lane; i < d / 8; i += 32) {
                const uint4 v = xr[i];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    o[u] = code_f16(quant_i8(bf16_to_f32(w[u] & 0xffffu), s)) |
                           (code_f16(quant_i8(bf16_to_f32(w[u] >> 16), s)) << 16);
                q[i] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        } else {
            uint2* q = reinterpret_cast<uint2*>(p.xq + (p.Tk + t) * d);
            for (int i = lane; i < d / 8; i += 32) {
                const uint4 v = xr[i];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[2] = {0u, 0u};
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t bits = (w[u >> 1] >> (16 * (u & 1))) & 0xffffu;
                    o[u >> 2] |= (uint32_t)(quant_i8(bf16_to_f32(bits), s) & 0xff) << (8 * (u & 3));
                }
                q[i] = make_uint2(o[0], o[1]);
            }
        }
        if (lane == 0) {
            p.sx[t] = s;
            p.row_src[p.Tk + t] = (int32_t)t;
            p.row_gate[p.Tk + t] = 1.0f;
        }
    }
}

// W_r [d, E] FP32 -> the split layout above (one thread per (chunk, expert row, k))
__global__ void split_router_kernel(const float* w, int d, int E, uint16_t* out) {
    const int64_t n = (int64_t)(d / kKC) * 64 * kKC;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int kk = (int)(i % kKC), e = (int)((i / kKC) % 64), c = (int)(i / (64 * kKC));
        const float v = e < E ? w[(int64_t)(c * kKC + kk) * E + e] : 0.0f;
        const uint32_t hi = bf16_rn_bits(v);
        const float r1 = __fsub_rn(v, __uint_as_float(hi << 16));
        const uint32_t mid = bf16_rn_bits(r1);
        const float r2 = __fsub_rn(r1, __uint_as_float(mid << 16));
        const uint32_t lo = bf16_rn_bits(r2);
        uint16_t* base = out + (size_t)c * (kWChunkBytes / 2) + e * kRow + kk;
        base[0] = (uint16_t)hi;
        base[kWPieceBytes / 2] = (uint16_t)mid;
        base[2 * (kWPieceBytes / 2)] = (uint16_t)lo;
    }
    // padding columns stay as the caller cleared them
}

}  // namespace rmma

bool router_mma_supported(int d, int E) { return d % rmma::kKC == 0 && E <= 64; }

size_t router_split_bytes(int d) { return (size_t)(d / rmma::kKC) * rmma::kWChunkBytes; }

cudaError_t launch_split_router(const float* w, int d, int E, uint16_t* out, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(out, 0, router_split_bytes(d), s);
    if (e != cudaSuccess) return e;
    rmma::split_router_kernel<<<256, 256, 0, s>>>(w, d, E, out);
    return cudaGetLastError();
}

namespace rmma {
template <int TOK>
cudaError_t launch_tok(const Plan& p, cudaStream_t s) {
    constexpr size_t smem = Tiling<TOK>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(router_mma_kernel<TOK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (p.T + TOK - 1) / TOK;
    router_mma_kernel<TOK><<<(unsigned)blocks, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}
}  // namespace rmma

cudaError_t launch_router_mma(const Plan& p, cudaStream_t s) {
    if (p.T == 0) return cudaSuccess;
    // the largest tile that still gives every SM a CTA (16 tokens at the least).  Measured on B200 (router
    // stage, us): T = 2048: 111 with 128-token tiles, 38.6 with 16; T = 8192 (d 1536): 152 with 128, 75.7
    // with 32, 105 with 16 (two CTAs per SM: every CTA reads the whole split W_r from L2); T = 32768: 276
    // with 128, 286 with 64.
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = sms;
    if (p.T >= 128 * want) return rmma::launch_tok<128>(p, s);
    if (p.T >= 64 * want) return rmma::launch_tok<64>(p, s);
    if (p.T >= 32 * want) return rmma::launch_tok<32>(p, s);
    return rmma::launch_tok<16>(p, s);
}

}  // namespace mmoe
