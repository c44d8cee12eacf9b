// Micro-benchmark: how fast can one SM run the grouped INT4 x INT8 contraction
// of the expert FFNs when every 32-wide K group must leave the tensor core as
// an exact integer partial and be promoted into an FP32 accumulator with its
// own weight scale (acc = fma(P_j, s_j, acc), in group order)?
//
// Not part of the library: the build compiles only the .cu files one level up.
// Build and run (one GPU, about ten seconds):
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o /tmp/promotion_ceiling \
//        moe_ffn_layer_fp32_b200/csrc/ubench/promotion_ceiling.cu -lcuda && /tmp/promotion_ceiling
//
// Two tensor-core kinds are compared:
//   kind::i8  : one MMA (K = 32) per group into an S32 accumulator; promotion converts S32 to FP32
//               (integer add of a magic constant, packed FP32 subtract) then a packed FMA.
//   kind::f16 : two MMAs (K = 16 each) per group with F16 operands holding the integer codes and
//               activations; the F32 accumulator holds the exact integer sum (|sum| < 2^15 < 2^24),
//               so promotion is a packed FMA only.
// Modes: 1 = MMAs only (the tensor-core ceiling), 4 = MMA + commit/arrive handoff + tcgen05.ld
// with no arithmetic, 0 = the whole loop (handoff + ld + promotion).
// The operands stay resident in shared memory: this measures the SM, not HBM.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "../sm100_tc.cuh"

using namespace mmoe;
using async::mbar_arrive;
using async::mbar_init;
using async::mbar_try_wait;
using async::su32;

namespace {

constexpr int kBN = 128;             // N of one group's MMA (the kernel's tile width)
constexpr int kBufs = 512 / kBN;     // TMEM buffers, one group each
constexpr int kW = 8;                // promotion warps
constexpr int kColGroups = kW / 4;   // warps that share a lane quarter split its columns
constexpr int kCols = kBN / kColGroups;

constexpr long long kSpinLimit = 2000000000ll;  // clocks; a wait that runs out sets the error flag

// SM clock, ordered with the memory operations and barriers around it
__device__ __forceinline__ long long clk() {
    long long t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t)::"memory");
    return t;
}

struct Shm {
    uint64_t accf[4];  // MMA -> promotion: group in buffer b is in TMEM
    uint64_t acce[4];  // promotion -> MMA: buffer b has been read
    uint64_t done;
    uint32_t tmem;
    int abort_;
};

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clk();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*(volatile int*)abort_flag) return false;
        if (clk() - t0 > kSpinLimit) {
            atomicExch(abort_flag, 1);
            return false;
        }
    }
}

template <int KIND>
__device__ __forceinline__ void promote2(float& a0, float& a1, uint32_t v0, uint32_t v1, float s) {
    float2 acc = make_float2(a0, a1), sc = make_float2(s, s), p;
    if (KIND == 0) {
        // exact S32 -> F32 for |v| < 2^22: add 1.5 * 2^23 as an integer, subtract it as a float
        const float2 minus_magic = make_float2(-12582912.0f, -12582912.0f);
        p = make_float2(__uint_as_float(v0 + 0x4B400000u), __uint_as_float(v1 + 0x4B400000u));
        p = __fadd2_rn(p, minus_magic);
    } else {
        p = make_float2(__uint_as_float(v0), __uint_as_float(v1));
    }
    acc = __ffma2_rn(p, sc, acc);
    a0 = acc.x;
    a1 = acc.y;
}

template <int KIND>
__device__ __forceinline__ void issue_group(uint32_t d, uint64_t ad, uint64_t bd, int k) {
    if (KIND == 0) {
        tc5::mma_i8<tc5::idesc_i8(kBN)>(d, ad + 2 * k, bd + 2 * k, 0);
    } else {
        tc5::mma_f16<tc5::idesc_f16(kBN)>(d, ad + 4 * (k & 1), bd + 4 * (k & 1), 0);
        tc5::mma_f16<tc5::idesc_f16(kBN)>(d, ad + 4 * (k & 1) + 2, bd + 4 * (k & 1) + 2, 1);
    }
}

// Warp 1 issues the MMAs; warps 2..2+kW-1 promote.  Every CTA runs `ngroups` groups.
template <int KIND, int MODE>
__global__ void __launch_bounds__(64 + kW * 32, 1) ceiling_kernel(int ngroups, float* out, long long* cyc, int* err) {
    extern __shared__ __align__(1024) uint8_t raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
    uint8_t* A = base;           // 128 rows x 128 bytes
    uint8_t* B = base + 16384;   // kBN rows x 128 bytes
    Shm* sm = (Shm*)(B + kBN * 128);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // small integer operands (the MMA rate does not depend on the values)
    for (int i = tid; i < (16384 + kBN * 128) / 2; i += blockDim.x) {
        const uint32_t hsh = (uint32_t)i * 2654435761u ^ (blockIdx.x * 40503u);
        uint16_t* p = (uint16_t*)base;
        if (KIND == 0) {
            const int8_t a = (int8_t)((hsh >> 3) % 255 - 127), b = (int8_t)((hsh >> 13) % 16 - 8);
            p[i] = (uint16_t)((uint8_t)a | ((uint16_t)(uint8_t)(i < 8192 ? b : a) << 8));
        } else {
            const int v = i < 8192 ? (int)((hsh >> 7) % 16) - 8 : (int)((hsh >> 5) % 255) - 127;
            p[i] = __half_as_ushort(__int2half_rn(v));
        }
    }
    if (tid == 0) {
        for (int b = 0; b < 4; ++b) {
            mbar_init(&sm->accf[b], 1);
            mbar_init(&sm->acce[b], kW);
        }
        mbar_init(&sm->done, 1);
        sm->abort_ = 0;
        async::fence_barrier_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 1) {
        tc5::tmem_alloc(&sm->tmem, 512);
        tc5::before_sync();
    }
    __syncthreads();
    tc5::after_sync();
    const uint32_t tmem = sm->tmem;
    const long long t0 = clk();
    float res = 0.0f;
    if (warp == 1) {
        if (lane == 0) {
            const uint64_t ad = tc5::smem_desc_sw128(A), bd = tc5::smem_desc_sw128(B);
            for (int g = 0; g < ngroups; ++g) {
                const int b = g % kBufs;
                if (MODE != 1) {
                    if (g >= kBufs && !wait_bounded(&sm->acce[b], ((g / kBufs) - 1) & 1, &sm->abort_)) break;
                    tc5::after_sync();
                }
                issue_group<KIND>(tmem + b * kBN, ad, bd, g & 3);
                if (MODE != 1) tc5::commit(&sm->accf[b]);
            }
            tc5::commit(&sm->done);
            wait_bounded(&sm->done, 0, &sm->abort_);
        }
        __syncwarp();  // the warp is whole again before the CTA barrier below (its lanes wait for lane 0)
    } else if (warp >= 2 && MODE != 1) {
        const int pw = warp - 2, q = warp & 3, cgi = pw >> 2;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cgi * kCols);
        float acc[kCols];
#pragma unroll
        for (int c = 0; c < kCols; ++c) acc[c] = 0.0f;
        float s = 1.0f + lane * 1e-3f;
        uint32_t xr = 0;
        for (int g = 0; g < ngroups; ++g) {
            const int b = g % kBufs;
            bool ok = true;
            if (lane == 0) ok = wait_bounded(&sm->accf[b], (g / kBufs) & 1, &sm->abort_);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            tc5::after_sync();
#pragma unroll
            for (int c0 = 0; c0 < kCols; c0 += 32) {
                uint32_t v[32];
                tc5::tmem_ld32(tl + b * kBN + c0, v);
                tc5::tmem_wait_ld(v);
                if (c0 + 32 >= kCols) {
                    tc5::before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm->acce[b]);
                }
                if (MODE == 0) {
#pragma unroll
                    for (int c = 0; c < 32; c += 2) promote2<KIND>(acc[c0 + c], acc[c0 + c + 1], v[c], v[c + 1], s);
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) xr ^= v[c];
                }
            }
            s = s * 1.0000001f;
        }
#pragma unroll
        for (int c = 0; c < kCols; ++c) res += acc[c];
        res += __uint_as_float(xr & 0x3fffffffu);
    }
    __syncthreads();
    const long long t1 = clk();
    if (tid == 0) {
        cyc[blockIdx.x] = t1 - t0;
        if (sm->abort_) atomicExch(err, 1);
    }
    if (warp >= 2) out[blockIdx.x * blockDim.x + tid] = res;
    if (warp == 1) {
        tc5::after_sync();
        tc5::tmem_dealloc(tmem, 512);
    }
}

// Exactness: one CTA computes D[128 x kBN] = A[128 x 64] * B[kBN x 64]^T (4 f16 MMAs of K = 16, or
// 2 i8 MMAs of K = 32) from operands given in the 128-byte-swizzled K-major image.
template <int KIND>
__global__ void exact_kernel(const uint8_t* img, uint32_t* dout, int* err) {
    extern __shared__ __align__(1024) uint8_t raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
    Shm* sm = (Shm*)(base + 16384 + kBN * 128);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < (16384 + kBN * 128) / 16; i += blockDim.x) ((uint4*)base)[i] = ((const uint4*)img)[i];
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (tid == 0) {
        mbar_init(&sm->done, 1);
        sm->abort_ = 0;
        async::fence_barrier_init();
    }
    if (warp == 0) {
        tc5::tmem_alloc(&sm->tmem, 512);
        tc5::before_sync();
    }
    __syncthreads();
    tc5::after_sync();
    const uint32_t tmem = sm->tmem;
    if (tid == 0) {
        const uint64_t ad = tc5::smem_desc_sw128(base), bd = tc5::smem_desc_sw128(base + 16384);
        if (KIND == 0) {
            for (int k = 0; k < 2; ++k) tc5::mma_i8<tc5::idesc_i8(kBN)>(tmem, ad + 2 * k, bd + 2 * k, k);
        } else {
            for (int k = 0; k < 4; ++k) tc5::mma_f16<tc5::idesc_f16(kBN)>(tmem, ad + 2 * k, bd + 2 * k, k);
        }
        tc5::commit(&sm->done);
    }
    __syncwarp();
    if (lane == 0 && !wait_bounded(&sm->done, 0, &sm->abort_)) atomicExch(err, 1);
    __syncwarp();
    tc5::after_sync();
    for (int c0 = 0; c0 < kBN; c0 += 16) {
        uint32_t v[16];
        tc5::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
        tc5::tmem_wait_ld(v);
        for (int c = 0; c < 16; ++c) dout[(warp * 32 + lane) * kBN + c0 + c] = v[c];
    }
    tc5::before_sync();
    __syncthreads();
    if (warp == 0) {
        tc5::after_sync();
        tc5::tmem_dealloc(tmem, 512);
    }
}

int smem_bytes() { return 1024 + 16384 + kBN * 128 + 256; }
// The timed kernel asks for more shared memory than it uses so that one CTA (and one 512-column
// TMEM allocation) is resident per SM.
int smem_one_per_sm() { return 120 * 1024; }

// pattern 0: random codes in [-8, 7] and activations in [-127, 127]; pattern 1: the extremes
template <int KIND>
bool check_exact(int pattern) {
    std::vector<int> A(128 * 64), B(kBN * 64);
    uint32_t st = 12345u + pattern;
    auto rnd = [&]() { st = st * 1664525u + 1013904223u; return st >> 8; };
    for (int i = 0; i < 128 * 64; ++i) A[i] = pattern == 0 ? (int)(rnd() % 16) - 8 : ((i / 64) % 2 ? 7 : -8);
    for (int i = 0; i < kBN * 64; ++i)
        B[i] = pattern == 0 ? (int)(rnd() % 255) - 127 : ((i / 64) % 3 == 0 ? 127 : ((i / 64) % 3 == 1 ? -127 : 0));
    std::vector<uint8_t> img(16384 + kBN * 128, 0);
    auto put = [&](uint8_t* b, int r, int k, int v) {
        const int kb = k * (KIND == 0 ? 1 : 2);
        uint8_t* p = b + r * 128 + (((kb / 16) ^ (r & 7)) * 16) + kb % 16;
        if (KIND == 0) {
            *p = (uint8_t)(int8_t)v;
        } else {
            const __half h = __float2half((float)v);
            memcpy(p, &h, 2);
        }
    };
    for (int r = 0; r < 128; ++r)
        for (int k = 0; k < 64; ++k) put(img.data(), r, k, A[r * 64 + k]);
    for (int n = 0; n < kBN; ++n)
        for (int k = 0; k < 64; ++k) put(img.data() + 16384, n, k, B[n * 64 + k]);
    uint8_t* dimg;
    uint32_t* dd;
    int* derr;
    cudaMalloc(&dimg, img.size());
    cudaMalloc(&dd, 128 * kBN * 4);
    cudaMalloc(&derr, 4);
    cudaMemset(derr, 0, 4);
    cudaMemcpy(dimg, img.data(), img.size(), cudaMemcpyHostToDevice);
    cudaFuncSetAttribute(exact_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes());
    exact_kernel<KIND><<<1, 128, smem_bytes()>>>(dimg, dd, derr);
    const cudaError_t e = cudaDeviceSynchronize();
    std::vector<uint32_t> D(128 * kBN);
    int herr = 0;
    cudaMemcpy(D.data(), dd, D.size() * 4, cudaMemcpyDeviceToHost);
    cudaMemcpy(&herr, derr, 4, cudaMemcpyDeviceToHost);
    long long bad = 0, maxabs = 0;
    for (int m = 0; m < 128; ++m)
        for (int n = 0; n < kBN; ++n) {
            long long ref = 0;
            for (int k = 0; k < 64; ++k) ref += (long long)A[m * 64 + k] * B[n * 64 + k];
            maxabs = std::max(maxabs, ref < 0 ? -ref : ref);
            long long got;
            if (KIND == 0) {
                got = (int32_t)D[m * kBN + n];
            } else {
                float f;
                memcpy(&f, &D[m * kBN + n], 4);
                got = (long long)f;
                if ((float)got != f) got = 1ll << 40;
            }
            bad += got != ref;
        }
    printf("exact  kind=%s pattern=%d: %s, %lld mismatches of %d (max |sum| %lld)\n", KIND == 0 ? "i8 " : "f16",
           pattern, e == cudaSuccess && !herr ? "ran" : "FAILED", bad, 128 * kBN, maxabs);
    cudaFree(dimg);
    cudaFree(dd);
    cudaFree(derr);
    return e == cudaSuccess && !herr && bad == 0;
}

template <int KIND, int MODE>
bool run(int nsm, int ngroups, float* out, long long* cyc, int* err) {
    auto k = ceiling_kernel<KIND, MODE>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_one_per_sm());
    cudaMemset(err, 0, 4);
    cudaMemset(cyc, 0, nsm * sizeof(long long));
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    float ms = 0.0f;
    if (e == cudaSuccess) {
        k<<<nsm, 64 + kW * 32, smem_one_per_sm()>>>(ngroups / 8, out, cyc, err);  // warm-up
        cudaEventRecord(e0);
        k<<<nsm, 64 + kW * 32, smem_one_per_sm()>>>(ngroups, out, cyc, err);
        cudaEventRecord(e1);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e == cudaSuccess) cudaEventElapsedTime(&ms, e0, e1);
    if (e != cudaSuccess) printf("launch: %s\n", cudaGetErrorString(e));
    int clock_khz = 0;
    cudaDeviceGetAttribute(&clock_khz, cudaDevAttrClockRate, 0);
    int herr = 0;
    cudaMemcpy(&herr, err, 4, cudaMemcpyDeviceToHost);
    // one group = 128 x kBN x 32 multiply-adds; the nominal dense rates per SM and clock are
    // 8192 (i8) and 4096 (f16) multiply-adds.  Clocks per group from the event time at the device's
    // maximum SM clock.
    const double macs = 128.0 * kBN * 32.0, clk_per_group = (double)ms * clock_khz / ngroups;
    static const char* kModes[] = {"handoff+ld+promotion", "MMA only", "", "", "handoff+ld, no math"};
    printf("%-4s %-22s %s %.3f ms, clk/group %6.1f = %5.1f%% of the nominal i8 rate, %5.1f%% of the nominal f16 "
           "rate\n",
           KIND == 0 ? "i8" : "f16", kModes[MODE], e == cudaSuccess && !herr ? "ok " : "ERR", ms, clk_per_group,
           100.0 * (macs / 8192.0) / clk_per_group, 100.0 * (macs / 4096.0) / clk_per_group);
    return e == cudaSuccess && !herr;
}

}  // namespace

int main(int argc, char** argv) {
    int nsm = 148;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, 0);
    const int ng = argc > 1 ? atoi(argv[1]) : 16384;
    float* out;
    long long* cyc;
    int* err;
    cudaMalloc(&out, (size_t)nsm * 1024 * sizeof(float));
    cudaMalloc(&cyc, nsm * sizeof(long long));
    cudaMalloc(&err, 4);
    bool ok = check_exact<0>(0) && check_exact<0>(1) && check_exact<1>(0) && check_exact<1>(1);
    ok = ok && run<0, 1>(nsm, ng, out, cyc, err) && run<1, 1>(nsm, ng, out, cyc, err);
    ok = ok && run<0, 4>(nsm, ng, out, cyc, err) && run<1, 4>(nsm, ng, out, cyc, err);
    ok = ok && run<0, 0>(nsm, ng, out, cyc, err) && run<1, 0>(nsm, ng, out, cyc, err);
    return ok ? 0 : 1;
}
