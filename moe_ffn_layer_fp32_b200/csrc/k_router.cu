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
        int8_t* q = p.xq + (p.Tk + t) * d;
        for (int i = lane * 4; i < d; i += 128) {
            uint32_t w = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) w |= (uint32_t)(quant_i8(bf16_to_f32(row[i + u]), s) & 0xff) << (8 * u);
            *reinterpret_cast<uint32_t*>(q + i) = w;
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
            if (p.router_bias) l = __fadd_rn(l, p.router_bias[e]);
            lg[i] = l;
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
    // token tile: as many rows as fit in about 160 KB of shared memory
    if ((size_t)32 * p.d * 2 <= 160 * 1024) return launch_tb<32>(p, s);
    if ((size_t)16 * p.d * 2 <= 160 * 1024) return launch_tb<16>(p, s);
    return launch_tb<8>(p, s);
}

}  // namespace mmoe
