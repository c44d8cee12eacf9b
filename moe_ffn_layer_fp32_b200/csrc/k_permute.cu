// K3: expert histogram, exclusive scan and stable token permutation.
//
// MobileMoE pages (paper-archivist reading, section "custom MoE kernel",
// principle 1): tokens are reordered by their assigned expert id with a
// counting sort, so that each expert's tokens are contiguous and every expert
// processes its slice as one batched matmul.  Dispatch is dropless (section
// "SFT" and the counting sort keep every token).
//
// Row order: routed rows grouped by expert, each expert's rows in ascending
// (token, slot) order; then the T rows of the shared expert in token order.
#include <algorithm>

#include "mmoe_internal.cuh"

namespace mmoe {
namespace {

constexpr int kThreads = 256;

// per-chunk expert counts
__global__ void __launch_bounds__(kThreads) count_kernel(Plan p)
{
    __shared__ int c[kMaxExperts];
    for (int i = threadIdx.x; i < kMaxExperts; i += kThreads) c[i] = 0;
    __syncthreads();
    const int64_t S = p.Tk;
    const int64_t s0 = (int64_t)blockIdx.x * kChunk;
    for (int i = threadIdx.x; i < kChunk; i += kThreads) {
        const int64_t s = s0 + i;
        if (s < S) atomicAdd(&c[p.idx[s]], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kMaxExperts; i += kThreads) p.chunk_cnt[(int64_t)blockIdx.x * kMaxExperts + i] = c[i];
}

// totals, group offsets, per-chunk bases and the GEMM tile table (one block)
__global__ void __launch_bounds__(kThreads) scan_kernel(Plan p)
{
    __shared__ int tot[kMaxExperts + 1];
    __shared__ int off[kMaxExperts + 2];
    __shared__ int tstart[kMaxExperts + 2];
    const int E = p.E;
    const int tid = threadIdx.x;
    if (tid < E) {
        // running count of expert tid before each chunk; counts read 16 at a time (read-only path)
        int acc = 0;
        for (int c0 = 0; c0 < p.nchunks; c0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                v[u] = c0 + u < p.nchunks ? __ldg(p.chunk_cnt + (int64_t)(c0 + u) * kMaxExperts + tid) : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (c0 + u < p.nchunks) p.chunk_base[(int64_t)(c0 + u) * kMaxExperts + tid] = acc;
                acc += v[u];
            }
        }
        tot[tid] = acc;
    }
    __syncthreads();
    if (tid == 0) {
        int o = 0, ts = 0;
        for (int e = 0; e < E; ++e) {
            off[e] = o;
            tstart[e] = ts;
            o += tot[e];
            ts += (tot[e] + p.tile_rows - 1) / p.tile_rows;
        }
        tot[E] = (int)p.T;
        off[E] = o;             // = T*k
        off[E + 1] = o + (int)p.T;
        tstart[E] = ts;
        ts += (int)((p.T + p.tile_rows - 1) / p.tile_rows);
        tstart[E + 1] = ts;
        *p.tile_count = ts;
    }
    __syncthreads();
    for (int e = tid; e < E + 2; e += kThreads) p.offsets[e] = off[e];
    for (int e = tid; e <= E; e += kThreads) p.counts[e] = tot[e];
    // tile table: entry i -> (group, tile index within the group)
    const int ntiles = tstart[E + 1];
    for (int i = tid; i < ntiles; i += kThreads) {
        int lo = 0, hi = E;  // the last g with tstart[g] <= i
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tstart[mid] <= i) lo = mid;
            else hi = mid - 1;
        }
        p.tiles[i] = (lo << 24) | (i - tstart[lo]);
    }
}

// stable scatter: rank of every slot among same-expert slots of lower index
__global__ void __launch_bounds__(kThreads) scatter_kernel(Plan p)
{
    __shared__ int base[kMaxExperts];
    __shared__ int wcnt[kThreads / 32][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t S = p.Tk;
    const int64_t c = blockIdx.x;
    for (int i = tid; i < kMaxExperts; i += kThreads)
        base[i] = i < p.E ? p.chunk_base[c * kMaxExperts + i] + p.offsets[i] : 0;
    for (int round = 0; round < kChunk / kThreads; ++round) {
        for (int i = tid; i < (kThreads / 32) * kMaxExperts; i += kThreads) (&wcnt[0][0])[i] = 0;
        __syncthreads();
        const int64_t s = c * kChunk + round * kThreads + tid;
        const bool valid = s < S;
        const int e = valid ? p.idx[s] : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & ((1u << lane) - 1u));
        if (valid && rank == 0) wcnt[warp][e] = __popc(same);
        __syncthreads();
        if (valid) {
            int pre = 0;
            for (int w = 0; w < warp; ++w) pre += wcnt[w][e];
            const int r = base[e] + pre + rank;
            p.row_src[r] = (int32_t)(s / p.k);
            p.row_gate[r] = p.gate[s];
            p.slot_row[s] = r;
        }
        __syncthreads();
        if (tid < kMaxExperts) {
            int sum = 0;
            for (int w = 0; w < kThreads / 32; ++w) sum += wcnt[w][tid];
            base[tid] += sum;
        }
        __syncthreads();
    }
}

// gather the activation codes of every routed row from its token's row
__global__ void __launch_bounds__(kThreads) gather_rows_kernel(Plan p)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (row >= p.Tk) return;
    const int64_t t = p.row_src[row];
    if (p.xq16) {
        const uint4* src = reinterpret_cast<const uint4*>(p.xq16 + (p.Tk + t) * p.d);
        uint4* dst = reinterpret_cast<uint4*>(p.xq16 + row * p.d);
        for (int i = lane; i < p.d / 8; i += 32) dst[i] = src[i];
    } else {
        const uint4* src = reinterpret_cast<const uint4*>(p.xq + (p.Tk + t) * p.d);
        uint4* dst = reinterpret_cast<uint4*>(p.xq + row * p.d);
        for (int i = lane; i < p.d / 16; i += 32) dst[i] = src[i];
    }
}

// f16 codes -> INT8 codes (both exact integers in [-127, 127])
__global__ void codes_f16_to_i8_kernel(const uint16_t* __restrict__ src, int8_t* __restrict__ dst, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = (int8_t)__half2int_rn(__ushort_as_half(src[i]));
}

}  // namespace

cudaError_t launch_codes_f16_to_i8(const uint16_t* src, int8_t* dst, int64_t n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4096);
    codes_f16_to_i8_kernel<<<(unsigned)blocks, 256, 0, s>>>(src, dst, n);
    return cudaGetLastError();
}

cudaError_t launch_permute(const Plan& p, cudaStream_t s) {
    if (p.T == 0) return cudaSuccess;
    count_kernel<<<p.nchunks, kThreads, 0, s>>>(p);
    scan_kernel<<<1, kThreads, 0, s>>>(p);
    scatter_kernel<<<p.nchunks, kThreads, 0, s>>>(p);
    const int64_t blocks = (p.Tk + kThreads / 32 - 1) / (kThreads / 32);
    gather_rows_kernel<<<(unsigned)blocks, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace mmoe
