// Eq. (6) of the MobileMoE pages (paper-archivist reading, section "QAT"):
// symmetric INT4 weights in groups of 32 along K with one FP32 scale per
// group, s = 2 max|W_g| / (2^4 - 1), q = clamp(round(W / s), -8, 7).
// Round half to even, IEEE divisions; an all-zero group gets s = 0, q = 0.
#include "mmoe_internal.cuh"

namespace mmoe {
namespace {

__global__ void __launch_bounds__(256)
quantize_int4_kernel(const float* __restrict__ w, int64_t ngroups, uint8_t* __restrict__ packed,
                     float* __restrict__ scales)
{
    const int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gi >= ngroups) return;
    const float4* src = reinterpret_cast<const float4*>(w + gi * kGroup);
    float v[kGroup];
#pragma unroll
    for (int i = 0; i < kGroup / 4; ++i) {
        const float4 f = src[i];
        v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kGroup; ++i) m = fmaxf(m, fabsf(v[i]));
    const float s = __fdiv_rn(__fmul_rn(2.0f, m), 15.0f);
    uint32_t out[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < kGroup; ++i) {
        int q = 0;
        if (s > 0.0f) q = max(-8, min(7, __float2int_rn(__fdiv_rn(v[i], s))));
        out[i / 8] |= (uint32_t)(q & 15) << (4 * (i % 8));
    }
    reinterpret_cast<uint4*>(packed)[gi] = make_uint4(out[0], out[1], out[2], out[3]);
    scales[gi] = s;
}

}  // namespace

cudaError_t launch_quantize_int4(const float* w, int64_t rows, int64_t K, uint8_t* packed, float* scales,
                                 cudaStream_t s) {
    const int64_t ng = rows * (K / kGroup);
    if (ng == 0) return cudaSuccess;
    quantize_int4_kernel<<<(unsigned)((ng + 255) / 256), 256, 0, s>>>(w, ng, packed, scales);
    return cudaGetLastError();
}

}  // namespace mmoe
