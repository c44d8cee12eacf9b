// K7: the decode path (T <= 64 tokens), the same mathematics as K1-K6 with
// the work laid out for streaming weights rather than for reusing them.
//
// MobileMoE pages (paper-archivist reading): decode is bound by memory
// bandwidth (section "on-device inference", the roofline discussion), so every
// byte of a selected expert is read once and nothing of an unselected one is
// read.  Eq. (*) and Eq. (6) fix what is computed: the INT32 partial of each
// 32-element group, scaled by its FP32 weight scale and summed over groups in
// ascending order, then the per-token activation scale, SwiGLU, the per-row
// requantisation, the down projection and the gate-weighted combine.
//
// Four launches (up to 8 tokens: the one-launch decode further below):
//  1. router_decode_kernel: one cluster of `cs` CTAs splits the K range of the
//     FP32 router for all tokens; partial logits and partial absmax meet in
//     distributed shared memory, each CTA quantises its slice of x, the owner
//     CTA of a token runs softmax / top-k, and rank 0 builds the expert
//     permutation (counts, offsets, stable scatter).
//  2. expert_decode_kernel<gate/up>: one warp per 16 weight rows (8 gate + 8
//     up rows of one output column block) of one selected group.  The warp
//     streams its rows with bulk copies into a private ring, unpacks INT4 to
//     INT8 in registers and multiplies with mma.sync m16n8k32 (weights as the
//     16-row A operand, up to 8 tokens as B).  The accumulator starts at
//     the bit pattern of 1.5 * 2^19, so the float with the result's bits
//     minus 1.5 * 2^19 is the group partial exactly (weights enter as 16 x
//     their code).  SwiGLU in registers, the row absmax by atomicMax.
//  3. requant_kernel (the prefill path's): h_q and s_h of every row, once.
//  4. expert_decode_kernel<down>: stages its group's h_q rows in the prologue,
//     then the same streaming GEMV; the epilogue adds gate * o into y (or
//     stores o for the fixed-order combine).
#include <cuda_bf16.h>

#include <algorithm>

#include "mmoe_internal.cuh"
#include "sm100_async.cuh"

namespace mmoe {
namespace dec {
namespace {

using async::bulk_load;
using async::clk;
using async::fence_barrier_init;
using async::mbar_expect_tx;
using async::mbar_init;
using async::mbar_try_wait;
using async::su32;

// decode weight layout: per group, per block of 16 weight rows, per pair of
// K groups: 32 lanes x 16 bytes of packed codes, then 8 x 16 bytes of scales
constexpr int kJP = 640;
constexpr int kStageJP = 4;                     // K-group pairs per bulk copy
constexpr int kStageBytes = kStageJP * kJP;     // 2560
constexpr int kRingMax = 4;                     // bulk copies in flight per warp (at most)
constexpr int kMaxWarps = 8;
constexpr int kMaxChunks = 8;                   // T <= 64 = 8 B operands of 8 tokens
constexpr int kPassRows = 16;                   // rows of a group per pass (2 B operands)
constexpr int kHeadBytes = 512;                 // mbarriers (256) + row scales (64 floats)
constexpr int kMaxT = kMaxChunks * 8;
constexpr uint32_t kAccBias = 0x49400000u;      // bits of 786432.0f = 1.5 * 2^19 (ulp 1/16)
constexpr float kAccBiasF = 786432.0f;
constexpr long long kTimeoutClk = 4000000000ll; // about 2 s of SM clock
constexpr int kSmemLimit = 232448;

constexpr int kRThreads = 256;
constexpr int kRTok = 64;                       // tokens of the decode path (one router cluster)
constexpr int kRHeadBytes = (kRTok * 64 + 2 * kRTok) * 4 + 16;  // partial logits, absmax, s_x, mbarrier

// router shared memory: head | x slice [kRTok][ks + 8] BF16 | W_r pieces of the slice (ks / 64 chunks)
__host__ __device__ constexpr size_t router_smem(int d, int cs) {
    return (size_t)kRHeadBytes + (size_t)kRTok * (d / cs + 8) * 2 + (size_t)(d / cs / kRouterKChunk) * kRouterChunkBytes;
}

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// the same shared variable in CTA `rank` of the cluster (read after a cluster barrier)
__device__ __forceinline__ float ld_peer(const float* p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(su32(p)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

// v[c] = the variable in CTA c, c < cs <= 16: all loads issued before any is used
__device__ __forceinline__ void ld_peers(float (&v)[16], const float* p, int cs) {
#pragma unroll
    for (int c = 0; c < 16; ++c) v[c] = c < cs ? ld_peer(p, (uint32_t)c) : 0.0f;
}

// sum over the cluster in rank order
__device__ __forceinline__ float cluster_sum(const float* p, int cs) {
    float v[16];
    ld_peers(v, p, cs);
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < 16; ++c)
        if (c < cs) s = __fadd_rn(s, v[c]);
    return s;
}

// D = A * B + C on the tensor cores (m16n8k32, INT8 x INT8 -> INT32), C = kAccBias
__device__ __forceinline__ void mma_bias(int32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    const int32_t c = (int32_t)kAccBias;
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %11, %12, %13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c), "r"(c), "r"(c), "r"(c));
}

// (a0, a1) = fma((P0, P1), s, (a0, a1)) with P the partials held in v0, v1
// (float(bits) - 1.5 * 2^19 is exact); paired FP32 instructions, each half an
// ordinary IEEE operation.
__device__ __forceinline__ void promote2(float& a0, float& a1, int32_t v0, int32_t v1, float s) {
    asm("{\n\t.reg .b64 t, acc, sc, mg;\n\t"
        "mov.b64 t, {%2, %3};\n\t"
        "mov.b64 acc, {%0, %1};\n\t"
        "mov.b64 mg, {%5, %5};\n\t"
        "mov.b64 sc, {%4, %4};\n\t"
        "sub.rn.f32x2 t, t, mg;\n\t"
        "fma.rn.f32x2 acc, t, sc, acc;\n\t"
        "mov.b64 {%0, %1}, acc;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "r"(v0), "r"(v1), "f"(s), "f"(kAccBiasF));
}

// programmatic dependent launch: let the next launch of the stream start its
// prologue / wait until the previous launch has completed and its writes are visible
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ int32_t partial_of(int32_t v) { return (v - (int32_t)kAccBias) >> 4; }

__device__ __forceinline__ void set_error(const Plan& p, int where) {
    if (p.err) *reinterpret_cast<volatile int*>(p.err) = where;
    if (p.err_host) *reinterpret_cast<volatile int*>(p.err_host) = where;
    __threadfence_system();
}

// bounded wait for the phase of `parity`; false after about 2 s.  The first test is inline (the phase
// has usually completed), the polling loop is not.
__device__ __noinline__ bool wait_bounded_poll(uint64_t* bar, uint32_t parity) {
    const long long t0 = clk();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clk() - t0 > kTimeoutClk) return false;
    }
}
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || wait_bounded_poll(bar, parity);
}

__device__ __forceinline__ uint32_t pack_codes(float a, float b, float c, float d, float s) {
    return (uint32_t)(quant_i8(a, s) & 0xff) | ((uint32_t)(quant_i8(b, s) & 0xff) << 8) |
           ((uint32_t)(quant_i8(c, s) & 0xff) << 16) | ((uint32_t)(quant_i8(d, s) & 0xff) << 24);
}

// ------------------------------------------------------------------ router
__device__ __forceinline__ void prefetch_l2(const void* ptr, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

constexpr int64_t kDownPrefetchLimit = 32ll << 20;

// Asks L2 for `bytes` bytes at `ptr` in 32 KB pieces (bytes a multiple of 16); one thread.
__device__ void prefetch_range(const uint8_t* ptr, int64_t bytes) {
    for (int64_t o = 0; o < bytes; o += 32768) prefetch_l2(ptr + o, (uint32_t)(bytes - o < 32768 ? bytes - o : 32768));
}

// The permutation of the routing slots, by one block of kRThreads threads:
// per-expert counts, offsets, the list of groups with rows, and a stable
// scatter (rows of an expert in ascending slot order).
__device__ void permute_block(const Plan& p) {
    __shared__ int cnt[kMaxExperts];
    __shared__ int base[kMaxExperts];
    __shared__ int wcnt[kRThreads / 32][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = p.E, k = p.k;
    const int S = (int)p.Tk;
    for (int i = tid; i < kMaxExperts; i += kRThreads) cnt[i] = 0;
    __syncthreads();
    for (int s = tid; s < S; s += kRThreads) atomicAdd(&cnt[__ldcg(p.idx + s)], 1);
    __syncthreads();
    if (warp == 0) {
        // exclusive scan of the counts (experts lane and lane + 32) and the list of groups with
        // rows: the shared one first, then the routed ones in ascending order
        const int c0 = lane < E ? cnt[lane] : 0, c1 = lane + 32 < E ? cnt[lane + 32] : 0;
        int s0 = c0, s1 = c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u0 = __shfl_up_sync(0xffffffffu, s0, o), u1 = __shfl_up_sync(0xffffffffu, s1, o);
            if (lane >= o) { s0 += u0; s1 += u1; }
        }
        const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
        s1 += tot0;
        const int tot = __shfl_sync(0xffffffffu, s1, 31);
        const unsigned b0 = __ballot_sync(0xffffffffu, c0 > 0), b1 = __ballot_sync(0xffffffffu, c1 > 0);
        const unsigned lt = (1u << lane) - 1u;
        if (lane < E) {
            base[lane] = s0 - c0;
            p.offsets[lane] = s0 - c0;
            p.counts[lane] = c0;
            if (c0) p.dec_groups[1 + __popc(b0 & lt)] = lane;
        }
        if (lane + 32 < E) {
            base[lane + 32] = s1 - c1;
            p.offsets[lane + 32] = s1 - c1;
            p.counts[lane + 32] = c1;
            if (c1) p.dec_groups[1 + __popc(b0) + __popc(b1 & lt)] = lane + 32;
        }
        const int nrouted = __popc(b0) + __popc(b1);
        if (lane == 0) {
            p.dec_groups[0] = E;
            *p.dec_ngroups = 1 + nrouted;
            p.offsets[E] = tot;
            p.offsets[E + 1] = tot + (int)p.T;
            p.counts[E] = (int)p.T;
        }
    }
    __syncthreads();
    for (int s0 = 0; s0 < S; s0 += kRThreads) {
        for (int i = tid; i < (kRThreads / 32) * kMaxExperts; i += kRThreads) (&wcnt[0][0])[i] = 0;
        __syncthreads();
        const int s = s0 + tid;
        const bool valid = s < S;
        const int e = valid ? __ldcg(p.idx + s) : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & ((1u << lane) - 1u));
        if (valid && rank == 0) wcnt[warp][e] = __popc(same);
        __syncthreads();
        if (valid) {
            int pre = 0;
            for (int w = 0; w < warp; ++w) pre += wcnt[w][e];
            const int r = base[e] + pre + rank;
            p.row_src[r] = s / k;
            p.row_gate[r] = __ldcg(p.gate + s);
            p.slot_row[s] = r;
        }
        __syncthreads();
        if (tid < E) {
            int sum = 0;
            for (int w = 0; w < kRThreads / 32; ++w) sum += wcnt[w][tid];
            base[tid] += sum;
        }
        __syncthreads();
    }
}

// One cluster of `cs` CTAs handles all T <= 64 tokens; CTA `rank` the K rows
// [rank ks, (rank + 1) ks) of W_r and x (ks a multiple of 64).  Its partial
// logits come from the tensor cores (W_r as exact BF16 pieces, each 16-wide K
// step added in FP32).  After the first cluster barrier every CTA knows the
// activation scales (max over the cluster) and quantises its slice; the owner
// CTA of token t (t mod cs) adds the partial logits in rank order and runs
// gating and top-k; after the second barrier rank 0 builds the permutation (the
// barrier's release / acquire orders the owners' writes of idx and gate) and
// asks L2 for the selected experts' weights.
__global__ void __launch_bounds__(kRThreads) router_decode_kernel(Plan p, int cs)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int d = p.d, E = p.E;
    const int ks = d / cs;
    const int xrow = ks + 8;  // padded BF16 row of the x slice
    float* part = reinterpret_cast<float*>(smem);             // [kRTok][64] partial logits
    float* pmax = part + kRTok * 64;                          // [kRTok] partial absmax
    float* sxs = pmax + kRTok;                                // [kRTok] s_x
    uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + kRHeadBytes - 16);
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + kRHeadBytes);  // [kRTok][xrow]
    uint8_t* ws = reinterpret_cast<uint8_t*>(xs + kRTok * xrow);      // ks / 64 chunks of W_r pieces
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, t4 = lane & 3;
    const int rank = (int)cluster_rank();
    const int nt = (int)p.T;
    const int k0 = rank * ks;
    const int mtiles = (nt + 15) >> 4;
    pdl_trigger();

    if (warp == 0) {
        const uint32_t wbytes = (uint32_t)(ks / kRouterKChunk) * kRouterChunkBytes, xbytes = (uint32_t)ks * 2;
        if (lane == 0) {
            mbar_init(wbar, 1);
            fence_barrier_init();
            mbar_expect_tx(wbar, wbytes + xbytes * nt);
            bulk_load(ws, reinterpret_cast<const uint8_t*>(p.w_router_split) + (size_t)(k0 / kRouterKChunk) * kRouterChunkBytes,
                      wbytes, wbar);
        }
        __syncwarp();
        // the token rows' slices: one copy each, issued by all lanes
        for (int t = lane; t < nt; t += 32) bulk_load(xs + t * xrow, p.x + (int64_t)t * d + k0, xbytes, wbar);
    }
    // rows of the last m16 tile beyond T are zero (disjoint from the copies)
    for (int i = nt * (xrow / 8) + tid; i < mtiles * 16 * (xrow / 8); i += kRThreads)
        reinterpret_cast<uint4*>(xs)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    const bool have = wait_bounded(wbar, 0);
    if (!have && tid == 0) set_error(p, 8);

    // partial logits: work item (m16 tile of tokens, pair of n8 tiles of experts)
    for (int it = warp; it < mtiles * 4; it += kRThreads / 32) {
        const int m = it >> 2, np = it & 3;
        float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
        if (have) {
            const uint16_t* xa = xs + (m * 16 + gid) * xrow + 2 * t4;
            for (int kk = 0; kk < ks; kk += 16) {
                const uint32_t a0 = *reinterpret_cast<const uint32_t*>(xa + kk);
                const uint32_t a1 = *reinterpret_cast<const uint32_t*>(xa + 8 * xrow + kk);
                const uint32_t a2 = *reinterpret_cast<const uint32_t*>(xa + kk + 8);
                const uint32_t a3 = *reinterpret_cast<const uint32_t*>(xa + 8 * xrow + kk + 8);
                const uint16_t* wb = reinterpret_cast<const uint16_t*>(ws + (kk / kRouterKChunk) * kRouterChunkBytes) +
                                     gid * kRouterRow + 2 * t4 + (kk % kRouterKChunk);
#pragma unroll
                for (int j = 0; j < 2; ++j) router_kstep(acc[j], a0, a1, a2, a3, wb + (2 * np + j) * 8 * kRouterRow);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int col = (2 * np + j) * 8 + 2 * t4;
            part[(m * 16 + gid) * 64 + col] = acc[j][0];
            part[(m * 16 + gid) * 64 + col + 1] = acc[j][1];
            part[(m * 16 + gid + 8) * 64 + col] = acc[j][2];
            part[(m * 16 + gid + 8) * 64 + col + 1] = acc[j][3];
        }
    }
    // partial absmax of each token over the slice (integer maximum of the BF16 magnitude bits, exact)
    for (int t = warp; t < nt; t += kRThreads / 32) {
        const uint2* xr = reinterpret_cast<const uint2*>(xs + t * xrow);
        uint32_t m2 = 0u;
        for (int i = lane; i < ks / 4; i += 32) {
            const uint2 v = xr[i];
            m2 = __vmaxu2(m2, __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu));
        }
        const uint32_t mb = __reduce_max_sync(0xffffffffu, max(m2 & 0xffffu, m2 >> 16));
        if (lane == 0) pmax[t] = bf16_to_f32(mb);
    }
    cluster_sync();
    for (int t = tid; t < nt; t += kRThreads) {
        float v[16];
        ld_peers(v, &pmax[t], cs);
        float m = 0.0f;
#pragma unroll
        for (int c = 0; c < 16; ++c) m = fmaxf(m, v[c]);
        sxs[t] = __fdiv_rn(m, 127.0f);
    }
    __syncthreads();
    // K1 on this CTA's slice: codes of the shared-expert rows (rows Tk + t of xq)
    for (int i = tid; i < nt * (ks / 4); i += kRThreads) {
        const int t = i / (ks / 4), v = i % (ks / 4);
        const uint16_t* xr = xs + t * xrow + v * 4;
        *reinterpret_cast<uint32_t*>(p.xq + (p.Tk + t) * d + k0 + v * 4) =
            pack_codes(bf16_to_f32(xr[0]), bf16_to_f32(xr[1]), bf16_to_f32(xr[2]), bf16_to_f32(xr[3]), sxs[t]);
    }
    // logits (slices added in rank order), gating and top-k of the tokens this CTA owns
    for (int t = rank + warp * cs; t < nt; t += (kRThreads / 32) * cs) {
        const float s0 = cluster_sum(&part[t * 64 + lane], cs);
        const float s1 = cluster_sum(&part[t * 64 + lane + 32], cs);
        float l0 = -INFINITY, l1 = -INFINITY;
        if (lane < E) l0 = biased_logit(p, s0, lane);
        if (lane + 32 < E) l1 = biased_logit(p, s1, lane + 32);
        gate_topk_warp(p, t, l0, l1, lane);
        if (lane == 0) {
            p.sx[t] = sxs[t];
            p.row_src[p.Tk + t] = t;
            p.row_gate[p.Tk + t] = 1.0f;
        }
    }
    cluster_sync();  // idx / gate of every token written; no CTA leaves while a peer may read its smem
    if (rank == 0) permute_block(p);
}

// ------------------------------------------------------------------ experts
// One warp's weight stream: `npass` passes over blocks `pstride` bytes apart
// (0: the same block again), each of nst stages.  Stage sc of the stream (from
// 0) is stage sc % nst of pass sc / nst and lands in ring slot (base + sc) %
// nring, so slot and phase carry over from stream to stream when `base` is the
// warp's running stage count.  A pass consumes stages sc0 .. sc0 + nst - 1 and
// refills the ring with stages below ntot.  NR: the ring size where it is fixed
// at compile time (0: nring_rt).
template <int NR>
struct WarpStream {
    const uint8_t* src;   // the warp's first 16-row block in the decode layout
    uint8_t* ring;
    uint64_t* bars;
    int64_t pstride;
    int NJ, nst, sc0, nring_rt, ntot, base;
    __device__ __forceinline__ int nring() const { return NR ? NR : nring_rt; }
    __device__ __forceinline__ int slot(int sc) const { return (base + sc) % nring(); }
    __device__ __forceinline__ uint32_t parity(int sc) const { return (uint32_t)(((base + sc) / nring()) & 1); }
    __device__ __forceinline__ void issue(int sc) const {
        const int st = sc % nst;
        const int jp = NJ - st * kStageJP;
        const uint32_t bytes = (uint32_t)((jp < kStageJP ? jp : kStageJP) * kJP);
        mbar_expect_tx(&bars[slot(sc)], bytes);
        bulk_load(ring + slot(sc) * kStageBytes, src + (int64_t)(sc / nst) * pstride + (int64_t)st * kStageBytes, bytes,
                  &bars[slot(sc)]);
    }
};

// The K loop of one warp over one pass of up to 8 * NCH rows: the accumulators
// of its 16 weight rows (A rows 0-7 in alo, 8-15 in ahi) for every row column.
// Returns false if a bounded wait gave up (the copies in flight have landed).
template <bool GU, bool DUMP, int NCH, int NR>
__device__ __forceinline__ bool warp_gemv(const Plan& p, const WarpStream<NR>& S, const uint8_t* codes, int cs, int lane,
                                          int rb, int64_t rrow0, int prows, int32_t* dump, int64_t drow0,
                                          int64_t dnrows, float (&alo)[NCH][2], float (&ahi)[NCH][2])
{
    const int gid = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int c = 0; c < NCH; ++c) alo[c][0] = alo[c][1] = ahi[c][0] = ahi[c][1] = 0.0f;
    const int ng = p.d / kGroup, ngh = p.hmax / kGroup;
    const uint8_t* bbase = codes + (size_t)gid * cs + t4 * 8;
    for (int st = 0; st < S.nst; ++st) {
        const int sc = S.sc0 + st;
        if (!wait_bounded(&S.bars[S.slot(sc)], S.parity(sc))) {
            if (lane == 0) set_error(p, 7);
            // let the copies in flight land before the CTA's shared memory goes away
            const int issued = sc + S.nring() < S.ntot ? sc + S.nring() : S.ntot;
            for (int s = sc; s < issued; ++s) wait_bounded(&S.bars[S.slot(s)], S.parity(s));
            return false;
        }
        const uint8_t* sb = S.ring + S.slot(sc) * kStageBytes;
        const int njs = S.NJ - st * kStageJP < kStageJP ? S.NJ - st * kStageJP : kStageJP;
        auto stage_q = [&](int q) {
            const uint4 wv = *reinterpret_cast<const uint4*>(sb + q * kJP + lane * 16);
            const float4 sv = *reinterpret_cast<const float4*>(sb + q * kJP + 512 + gid * 16);
            const int jp = st * kStageJP + q;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const uint32_t w0 = jj ? wv.z : wv.x, w1 = jj ? wv.w : wv.y;
                const float slo = jj ? sv.z : sv.x, shi = jj ? sv.w : sv.y;
                const uint32_t a0 = (w0 << 4) & 0xF0F0F0F0u, a1 = w0 & 0xF0F0F0F0u;
                const uint32_t a2 = (w1 << 4) & 0xF0F0F0F0u, a3 = w1 & 0xF0F0F0F0u;
                const int j = 2 * jp + jj;
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const uint2 b = *reinterpret_cast<const uint2*>(bbase + (size_t)c * 8 * cs + j * 32);
                    int32_t dd[4];
                    mma_bias(dd, a0, a1, a2, a3, b.x, b.y);
                    if (DUMP) {
#pragma unroll
                        for (int q2 = 0; q2 < 2; ++q2) {
                            const int i = c * 8 + 2 * t4 + q2;
                            const int64_t r = rrow0 + i;
                            if (i < prows && r >= drow0 && r < drow0 + dnrows) {
                                if (GU) {
                                    int32_t* base = dump + (r - drow0) * 2 * p.hmax * ng;
                                    const int n = rb * 8 + gid;
                                    base[(int64_t)n * ng + j] = partial_of(dd[q2]);
                                    base[(int64_t)(p.hmax + n) * ng + j] = partial_of(dd[2 + q2]);
                                } else {
                                    const int m = rb * 16 + gid;
                                    dump[((r - drow0) * p.d + m) * ngh + j] = partial_of(dd[q2]);
                                    dump[((r - drow0) * p.d + m + 8) * ngh + j] = partial_of(dd[2 + q2]);
                                }
                            }
                        }
                    }
                    promote2(alo[c][0], alo[c][1], dd[0], dd[1], slo);
                    promote2(ahi[c][0], ahi[c][1], dd[2], dd[3], shi);
                }
            }
        };
        // full stages unrolled without a bound check per K-group pair; the last, partial stage looped
        if (njs == kStageJP) {
#pragma unroll
            for (int q = 0; q < kStageJP; ++q) stage_q(q);
        } else {
#pragma unroll 1
            for (int q = 0; q < njs; ++q) stage_q(q);
        }
        __syncwarp();
        if (lane == 0 && sc + S.nring() < S.ntot) S.issue(sc + S.nring());
    }
    return true;
}

// SwiGLU of row i's gate and up accumulators (the row's activation scale sxr applied to both)
__device__ __forceinline__ float swiglu_row(float g, float u, float sxr) {
    const float gv = __fmul_rn(g, sxr), uv = __fmul_rn(u, sxr);
    const float silu = __fdiv_rn(gv, __fadd_rn(1.0f, expf(-gv)));
    return __fmul_rn(silu, uv);
}

// The GEMV of one warp over one pass of up to 8 * NCH rows, then its
// epilogue.  Returns false if a bounded wait gave up (nothing is written).
template <bool GU, bool DUMP, int NCH, int NR>
__device__ __forceinline__ bool warp_pass(const Plan& p, const WarpStream<NR>& S, const uint8_t* codes, int cs,
                                          const float* shs, int lane, int rb, int64_t rrow0, int prows,
                                          int32_t* dump, int64_t drow0, int64_t dnrows)
{
    const int gid = lane >> 2, t4 = lane & 3;
    float alo[NCH][2], ahi[NCH][2];
    if (!warp_gemv<GU, DUMP, NCH>(p, S, codes, cs, lane, rb, rrow0, prows, dump, drow0, dnrows, alo, ahi))
        return false;
    if (DUMP) return true;

    if (GU) {
        // the (gate, up) pairs times the rows' activation scales (shs, staged by the caller); the
        // requantisation launch applies the SwiGLU
        const int n = rb * 8 + gid;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int i = c * 8 + 2 * t4 + q;
                if (i >= prows) continue;
                const int64_t r = rrow0 + i;
                const float sxr = shs[i];
                reinterpret_cast<float2*>(p.act)[r * p.hmax + n] =
                    make_float2(__fmul_rn(alo[c][q], sxr), __fmul_rn(ahi[c][q], sxr));
            }
        }
    } else {
        const int m0 = rb * 16 + gid;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int i = c * 8 + 2 * t4 + q;
                if (i >= prows) continue;
                const int64_t r = rrow0 + i;
                const float s = shs[i];
                const float olo = __fmul_rn(alo[c][q], s), ohi = __fmul_rn(ahi[c][q], s);
                if (p.deterministic) {
                    p.obuf[r * p.d + m0] = olo;
                    p.obuf[r * p.d + m0 + 8] = ohi;
                } else {
                    const float gt = __ldcg(p.row_gate + r);
                    float* yr = p.y + (int64_t)__ldcg(p.row_src + r) * p.d;
                    atomicAdd(yr + m0, __fmul_rn(gt, olo));
                    atomicAdd(yr + m0 + 8, __fmul_rn(gt, ohi));
                }
            }
        }
    }
    return true;
}

// grid: (groups that can have rows) x nbpg blocks; block: W warps, warp w
// handles weight-row block blk * W + w of group dec_groups[blockIdx.x / nbpg].
// The group's rows go in passes of up to kPassRows; each pass stages their
// codes (B-fragment order inside each 32-group) and streams the weights again
// (from L2 after the first pass).  Shared memory: mbarriers | row scales |
// W rings of nring stages | codes [kPassRows][K + 32].
template <bool GU, bool DUMP>
__global__ void __launch_bounds__(kMaxWarps * 32)
expert_decode_kernel(Plan p, int nbpg, int nring, int32_t* dump, int64_t drow0, int64_t dnrows)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int W = blockDim.x >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    float* shs = reinterpret_cast<float*>(smem + 256);
    uint8_t* ring = smem + kHeadBytes;
    uint8_t* codes = ring + W * nring * kStageBytes;

    pdl_trigger();
    if (GU && !DUMP && !p.deterministic && p.y) {
        // y is accumulated by the down launch: clear it here, spread over every CTA (the
        // router launch before this one does not touch y, so no wait is needed)
        const int64_t n4 = p.T * p.d / 4;
        const int64_t per = (n4 + gridDim.x - 1) / gridDim.x;
        const int64_t a = (int64_t)blockIdx.x * per, b = a + per < n4 ? a + per : n4;
        float4* y4 = reinterpret_cast<float4*>(p.y);
        for (int64_t i = a + tid; i < b; i += blockDim.x) y4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }

    // group slot 0 is always the shared expert (rows Tk .. Tk + T - 1), known before the
    // previous launch has finished; every other slot waits for the routing
    const int gi = blockIdx.x / nbpg, blk = blockIdx.x % nbpg;
    const bool shared = gi == 0;
    if (!shared) {
        pdl_wait();
        if (gi >= *p.dec_ngroups) return;
    }
    const int g = shared ? p.E : p.dec_groups[gi];
    const int hid = g == p.E ? p.hs : p.h;
    const int K = GU ? p.d : hid;
    const int nrb = GU ? hid / 8 : p.d / 16;
    const int rb0 = blk * W;
    if (rb0 >= nrb) return;
    const int nrows = shared ? (int)p.T : p.counts[g];
    const int64_t row0 = shared ? p.Tk : p.offsets[g];
    if (GU && !DUMP && !shared && tid == 0 &&  // routed CTAs have waited for the routing here
        (int64_t)(*p.dec_ngroups) * ((int64_t)p.d * p.h * 5 / 8) <= kDownPrefetchLimit) {
        // this CTA's share of the group's down weights toward L2, for the next launch (only when all
        // selected down weights fit easily in L2 next to the gate/up weights streaming through it)
        const int nblk = (nrb + W - 1) / W;
        const int64_t dbytes = (int64_t)p.d * hid * 5 / 8;
        const int64_t per = ((dbytes / nblk) + 15) / 16 * 16;
        const int64_t o0 = (int64_t)blk * per;
        if (o0 < dbytes)
            prefetch_range(p.w_down_d + (int64_t)g * ((int64_t)p.d * p.h * 5 / 8) + o0,
                           o0 + per <= dbytes ? per : dbytes - o0);
    }
    const int NJ = K / 64;
    const int cs = K + 32;
    const int ngr = K / 32;
    const int rb = rb0 + warp;
    const bool wact = rb < nrb;
    WarpStream<0> S;
    S.src = (GU ? p.w_gate_up_d + (int64_t)g * ((int64_t)p.h * p.d * 5 / 4)
                : p.w_down_d + (int64_t)g * ((int64_t)p.d * p.h * 5 / 8)) +
            (int64_t)rb * NJ * kJP;
    S.ring = ring + warp * nring * kStageBytes;
    S.bars = bars + warp * kRingMax;
    S.NJ = NJ;
    S.nst = (NJ + kStageJP - 1) / kStageJP;
    S.sc0 = 0;
    S.nring_rt = nring;
    S.pstride = 0;  // every pass of rows streams the same block again (from L2 after the first)
    S.base = 0;
    const int npass = (nrows + kPassRows - 1) / kPassRows;
    S.ntot = npass * S.nst;  // the ring runs on into the next pass
    if (lane == 0) {
        for (int s = 0; s < nring; ++s) mbar_init(&S.bars[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    bool alive = wact;                    // false once this warp's bounded wait gave up
    for (int pass = 0; pass < npass; ++pass, S.sc0 += S.nst) {
        const int prow0 = pass * kPassRows;
        const int prows = nrows - prow0 < kPassRows ? nrows - prow0 : kPassRows;
        const int nch = (prows + 7) >> 3;
        const int64_t rrow0 = row0 + prow0;
        if (pass > 0) __syncthreads();  // every warp is done with the previous pass's codes
        if (pass == 0 && alive && lane == 0)
            for (int s = 0; s < nring && s < S.ntot; ++s) S.issue(s);
        if (pass == 0 && shared) pdl_wait();  // weights are in flight; now the previous launch's outputs

        // codes of this pass's rows, zero rows up to a multiple of 8
        if (GU) {
            for (int i = tid; i < nch * 8; i += blockDim.x) shs[i] = i < prows ? p.sx[p.row_src[rrow0 + i]] : 0.0f;
            for (int it = tid; it < nch * 8 * ngr; it += blockDim.x) {
                const int i = it / ngr, j = it % ngr;
                uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
                if (i < prows) {
                    const int64_t t = p.row_src[rrow0 + i];
                    const uint4* s4 = reinterpret_cast<const uint4*>(p.xq + (p.Tk + t) * p.d + j * 32);
                    u0 = s4[0];
                    u1 = s4[1];
                }
                uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)i * cs + j * 32);
                dst[0] = make_uint4(u0.x, u1.x, u0.y, u1.y);
                dst[1] = make_uint4(u0.z, u1.z, u0.w, u1.w);
            }
        } else {
            // the group's requantised SwiGLU rows (h_q and s_h from the requantisation launch between the
            // two GEMV launches), zero rows up to a multiple of 8
            for (int i = tid; i < nch * 8; i += blockDim.x) shs[i] = i < prows ? p.sh[rrow0 + i] : 0.0f;
            for (int it = tid; it < nch * 8 * ngr; it += blockDim.x) {
                const int i = it / ngr, j = it % ngr;
                uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
                if (i < prows) {
                    const uint4* q4 = reinterpret_cast<const uint4*>(p.hq + (rrow0 + i) * p.hmax + j * 32);
                    u0 = q4[0];
                    u1 = q4[1];
                }
                uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)i * cs + j * 32);
                dst[0] = make_uint4(u0.x, u1.x, u0.y, u1.y);
                dst[1] = make_uint4(u0.z, u1.z, u0.w, u1.w);
            }
        }
        __syncthreads();
        if (alive)  // a warp that gave up keeps taking the CTA barriers but issues and computes nothing
            alive = nch == 1 ? warp_pass<GU, DUMP, 1>(p, S, codes, cs, shs, lane, rb, rrow0, prows, dump, drow0,
                                                      dnrows)
                             : warp_pass<GU, DUMP, 2>(p, S, codes, cs, shs, lane, rb, rrow0, prows, dump, drow0,
                                                      dnrows);
    }
}

// ------------------------------------------------------------------ one-launch decode (T <= kCMaxT)
// The whole layer (or a stack of layers) for a handful of tokens in one launch of clusters of CS CTAs:
//   - every CTA computes the activation scales of all tokens and the FP32 router products of its
//     K slice (d / CS rows of W_r) for every token; the slices' partial logits go to every CTA of the
//     cluster through distributed shared memory and, after a cluster barrier, each CTA adds them in
//     rank order (the same sums in every CTA of every cluster), then runs gating, top-k and the
//     permutation of the routing slots itself;
//   - the groups with rows (the shared expert first, then the selected experts in ascending order)
//     go to the clusters in turn; CTA r of a cluster takes the weight-row blocks r W + w, r W + w + CS W,
//     ... of the group's gate/up and then of its down weights, streamed as in the four-launch path
//     (a ring of bulk copies per warp, mma.sync m16n8k32 with the weights as A).  A cluster's first
//     stream starts before the permutation (the shared expert's before the layer's x is there), each
//     warp's down stream as soon as its gate/up blocks are done;
//   - each CTA writes the SwiGLU values of its hidden features into every CTA's copy of the group's
//     rows (distributed shared memory); after one cluster barrier every CTA requantises the whole rows
//     itself (absmax / 127 and the INT8 codes, as K4's requantisation) for its down blocks;
//   - by default the down outputs, times their gates, are added into y with atomics (cluster 0 clears
//     every layer's y first and counts that in a flag).  In deterministic mode they go to a row buffer
//     instead; per token and CTA rank a counter in global memory counts the k + 1 contributions, and
//     the CTA that brings the last one adds them in the fixed order of Eq. (*) (shared expert, then
//     the selected experts in top-k order) over its rank's output columns and resets the counter.
// Waits: for this CTA's own bulk copies, the cluster barriers (every CTA of a cluster reaches them
// equally often), once for the cleared-y flag, and in a stack for the previous layer's y (a counter);
// all bounded.  The grid is the number of clusters that can be resident at once, so the waits between
// clusters end.
constexpr int kCMaxT = 8;
constexpr int kCWarps = 8;
constexpr int kCThreads = kCWarps * 32;
constexpr int kCMaxCS = 16;
constexpr int kCMaxSlots = kCMaxT * kMaxTopK;
constexpr int kMaxChain = kDecChainMax;

// One layer's weights and outputs (the layers of one launch share every shape).
struct LayerW {
    const float* w_router;
    const float* router_bias;
    const uint8_t* w_gate_up_d;
    const uint8_t* w_down_d;
    float* y;             // [T, d]
    int32_t* out_idx;     // optional copies of the routing for the caller: [T, k]
    float* out_gate;      // [T, k]
    int32_t* out_counts;  // [E + 1]
};

struct CArgs {
    uint32_t* cnt;        // [kCMaxT][CS] contribution counters, zero at launch (the last user resets one)
    float* obuf;          // [kCMaxT * (kMaxTopK + 1)][d] expert outputs, rows as in the permutation
    uint32_t* chain;      // [3]: y columns combined (fixed order) or groups finished by CTAs (atomics) over
                          // the launch, CTAs that left, CTAs of cluster 0 that cleared y (zero at launch;
                          // reset by the last CTA to leave)
    int nl;               // layers in this launch; layer l + 1 reads layer l's y rounded to BF16
    int off_x, off_codes, off_act, off_wr, off_u;  // dynamic shared memory offsets
    int wr_in_ring;       // 1: the W_r slice shares the rings' space (fetched at the start of each layer)
    LayerW layers[kMaxChain];
};

struct CShared {
    uint64_t bars[kCWarps * kRingMax];
    uint64_t wbar, xbar;
    float sxs[kCMaxT];             // activation scales of the tokens
    float shs[8];                  // per row of the current group: activation scale, then SwiGLU scale
    int idx[kCMaxSlots];
    float gate[kCMaxSlots];
    int slot_row[kCMaxSlots];
    int row_tok[kCMaxSlots];       // routed row -> token
    float row_gate[kCMaxSlots];    //              -> gate
    int cnt[kMaxExperts];
    int offs[kMaxExperts + 2];
    int groups[kMaxExperts + 1];
    int nslots;
    int last[8];
    int flag;
};

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t peer_addr(const void* p, int rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(su32(p)), "r"(rank));
    return a;
}
__device__ __forceinline__ void st_peer(const void* p, int rank, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_addr(p, rank)), "r"(v) : "memory");
}
__device__ __forceinline__ void st_peer(const void* p, int rank, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(peer_addr(p, rank)), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

// position of word v (features 4v .. 4v + 3) of a 32-element group in the B-fragment order of an operand
// row: words 0, 4, 1, 5, 2, 6, 3, 7
__device__ __forceinline__ int bfrag_pos(int v) { return v < 4 ? 2 * v : 2 * (v - 4) + 1; }

// number of passes pi >= 0 with first + pi * step < n
// The router's FP32 partial logits of one expert over kq K rows of a slice (four per step), for NT token
// rows of x (NT >= T: rows past T are summed too and never read); out[t * 64] = row t's sum.
template <int NT>
__device__ __forceinline__ void router_partials(const uint16_t* xk, const float* wk, int d, int E, int kq, float* out,
                                                bool on) {
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
    if (on) {
#pragma unroll 2
        for (int kk = 0; kk < kq; kk += 4) {
            const float w0 = wk[kk * E], w1 = wk[(kk + 1) * E], w2 = wk[(kk + 2) * E], w3 = wk[(kk + 3) * E];
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint2 xv = *reinterpret_cast<const uint2*>(xk + t * d + kk);
                acc[t] = fmaf(bf16_to_f32(xv.x & 0xffffu), w0, acc[t]);
                acc[t] = fmaf(bf16_to_f32(xv.x >> 16), w1, acc[t]);
                acc[t] = fmaf(bf16_to_f32(xv.y & 0xffffu), w2, acc[t]);
                acc[t] = fmaf(bf16_to_f32(xv.y >> 16), w3, acc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) out[t * 64] = acc[t];
}

// Position of the set bit of m with n set bits below it (m has more than n set bits).
__device__ __forceinline__ int nth_set_bit(uint32_t m, int n) {
    int pos = 0;
#pragma unroll
    for (int w = 16; w > 0; w >>= 1) {
        const int c = __popc(m & ((1u << w) - 1u));
        if (n >= c) {
            n -= c;
            m >>= w;
            pos += w;
        }
    }
    return pos;
}

__device__ __forceinline__ int npasses(int first, int step, int n) { return first < n ? (n - first + step - 1) / step : 0; }

// two floats rounded to BF16 (round to nearest even; finite inputs), packed low | high << 16
__device__ __forceinline__ uint32_t bf16_pair_rn(float a, float b) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a)) |
           ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b)) << 16);
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* a) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

// Adds v at GPU scope with acquire-release semantics and returns the old value.  Called after a CTA
// barrier, it publishes every write of the CTA made before the barrier to whoever acquires the count,
// and the caller sees what the earlier adders published.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* a, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(a), "r"(v) : "memory");
    return old;
}

// The same without the old value and the acquire half.
__device__ __forceinline__ void red_add_release(uint32_t* a, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}

// One thread's L2 prefetch of this CTA's gate/up and down row blocks of a layer's shared expert (expert
// E of the decode-layout arrays gu, dn).  Not inlined: one copy of code that one thread runs.
__device__ __noinline__ void prefetch_shared_expert(const uint8_t* gu, const uint8_t* dn, int rank, int cs, int d,
                                                    int h, int hs, int E) {
    const int W = kCWarps, NJ = d / 64, NJd = hs / 64, nrb = hs / 8, nrbd = d / 16, rstep = cs * W;
    const int64_t gu_stride = (int64_t)h * d * 5 / 4, dn_stride = (int64_t)d * h * 5 / 8;
    for (int b = rank * W; b < nrb; b += rstep)
        prefetch_range(gu + E * gu_stride + (int64_t)b * NJ * kJP, (int64_t)min(W, nrb - b) * NJ * kJP);
    for (int b = rank * W; b < nrbd; b += rstep)
        prefetch_range(dn + E * dn_stride + (int64_t)b * NJd * kJP, (int64_t)min(W, nrbd - b) * NJd * kJP);
}

// The gate/up weight stream of one warp over group g of a layer: row blocks rb0, rb0 + CS W, ...
template <int CS>
__device__ __forceinline__ void gu_stream(WarpStream<kRingMax>& S, const Plan& p, const LayerW& Lw, int g, int rb0, int base) {
    const int hid = g == p.E ? p.hs : p.h, nrb = hid / 8, NJ = p.d / 64;
    const int np = npasses(rb0, CS * kCWarps, nrb);
    S.src = Lw.w_gate_up_d + (int64_t)g * ((int64_t)p.h * p.d * 5 / 4) + (int64_t)rb0 * NJ * kJP;
    S.pstride = (int64_t)CS * kCWarps * NJ * kJP;
    S.NJ = NJ;
    S.nst = (NJ + kStageJP - 1) / kStageJP;
    S.ntot = np * S.nst;
    S.base = base;
}

template <int CS>
__global__ void __launch_bounds__(kCThreads, 1) decode_cluster_kernel(Plan p, CArgs ca)
{
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ CShared st;
    constexpr int W = kCWarps;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gid = lane >> 2, t4 = lane & 3;
    const int T = (int)p.T, d = p.d, E = p.E, k = p.k, Tk = (int)p.Tk;
    const int rank = (int)cluster_rank();
    const int cid = (int)blockIdx.x / CS, ncl = (int)gridDim.x / CS;
    const int ks = d / CS;
    const bool keeper = cid == 0 && rank == 0;  // writes the routing and permutation for inspection
    float* part_recv0 = reinterpret_cast<float*>(smem);                      // [2][CS][kCMaxT][64]
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + ca.off_x);             // [T][d]
    uint8_t* codes = smem + ca.off_codes;                                    // [8][max(d, hmax) + 32]
    float* act_all = reinterpret_cast<float*>(smem + ca.off_act);            // [8 rows][hmax] SwiGLU values
    float* wr = reinterpret_cast<float*>(smem + (ca.wr_in_ring ? ca.off_u : ca.off_wr));  // this CTA's W_r slice
    uint8_t* ring = smem + ca.off_u;                                         // the warps' rings
    const uint32_t wbytes = (uint32_t)(ks * E * 4);

    // first half of a cluster barrier: this CTA has started (its shared memory may be written by peers
    // once the second half has been waited for)
    cluster_arrive_relaxed();
    pdl_trigger();
    if (tid == 0) {
        for (int i = 0; i < W * kRingMax; ++i) mbar_init(&st.bars[i], 1);
        mbar_init(&st.wbar, 1);
        mbar_init(&st.xbar, 1);
        fence_barrier_init();
        // layer 0's K slice of W_r, rows [rank ks, (rank + 1) ks): weights, not outputs of the previous launch
        mbar_expect_tx(&st.wbar, wbytes);
        bulk_load(wr, ca.layers[0].w_router + (int64_t)rank * ks * E, wbytes, &st.wbar);
    }
    __syncthreads();  // the mbarriers are initialised
    pdl_wait();       // x, and the buffers the previous launch used
    // y is added with atomics unless the combine must be in a fixed order: cluster 0 clears every layer's y
    // first, and counts that in chain[2] for the CTAs that add
    const bool fixed = p.deterministic != 0;
    if (!fixed && cid == 0) {
        const int n4 = T * d / 4, per = (n4 + CS - 1) / CS, i0 = rank * per, i1 = min(n4, i0 + per);
        for (int l = 0; l < ca.nl; ++l) {
            float4* y4 = reinterpret_cast<float4*>(ca.layers[l].y);
            for (int i = i0 + tid; i < i1; i += kCThreads) y4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
        __syncthreads();
        if (tid == 0) red_add_release(ca.chain + 2, 1u);
    }
    bool y_clear = fixed;  // this CTA has seen every layer's y cleared
    uint32_t ctarget = 0;  // y columns combined (fixed order), or groups done by CTAs (atomics), before layer l
    bool ok = true;
    int wsc = 0;      // this warp's running stage count (ring slot and phase), over all layers
    bool alive = true;  // false once one of this warp's bounded waits gave up
    WarpStream<kRingMax> S;
    S.ring = ring + warp * kRingMax * kStageBytes;
    S.bars = st.bars + warp * kRingMax;
    S.nring_rt = kRingMax;
    const int rb0 = rank * W + warp;  // this warp's first row block of every stream

    for (int l = 0; l < ca.nl; ++l) {
        const LayerW Lw = ca.layers[l];  // (a copy: its fields stay in registers for the whole layer)
        // partial logits from every CTA of the cluster, one copy per layer parity: a peer that has moved on
        // to the next layer (possible when this cluster has no group in this layer) writes the other copy
        float* part_recv = part_recv0 + (l & 1) * (CS * kCMaxT * 64);
        // the shared expert is cluster 0's first group whatever the routing: its gate/up stream starts before
        // this layer's x is there, and the rest of this CTA's share of it goes toward L2 (unless the W_r slice
        // is about to use the rings' space)
        const bool early0 = cid == 0 && !ca.wr_in_ring;
        if (early0) {
            gu_stream<CS>(S, p, Lw, E, rb0, wsc);
            if (alive && lane < kRingMax && lane < S.ntot) S.issue(lane);
            if (tid == 32)
                prefetch_shared_expert(Lw.w_gate_up_d, Lw.w_down_d, rank, CS, d, p.h, p.hs, E);
        }
        // ------------------------------------------------------------ this layer's x
        if (l == 0) {
            if (tid == 0) {
                const uint32_t xbytes = (uint32_t)(T * d * 2);
                mbar_expect_tx(&st.xbar, xbytes);
                bulk_load(xs, p.x, xbytes, &st.xbar);
            }
            ok = wait_bounded(&st.xbar, 0) && ok;
        } else {
            // every combine of layer l - 1 is done, so its y is complete; x = its BF16 rounding
            if (tid == 0) {
                int good = 1;
                const uint32_t target = ctarget;
                if (ld_acquire(ca.chain) < target) {
                    const long long t0 = clk();
                    while (ld_acquire(ca.chain) < target) {
                        if (clk() - t0 > p.wait_limit) {
                            good = 0;
                            set_error(p, 42);
                            break;
                        }
                    }
                }
                st.flag = good;
            }
            __syncthreads();
            ok = ok && st.flag;
            if (ca.wr_in_ring && tid == 0) {
                mbar_expect_tx(&st.wbar, wbytes);
                bulk_load(wr, Lw.w_router + (int64_t)rank * ks * E, wbytes, &st.wbar);
            }
            const float4* y4 = reinterpret_cast<const float4*>(ca.layers[l - 1].y);
            uint2* x2 = reinterpret_cast<uint2*>(xs);
#pragma unroll 1
            for (int i = tid; i < T * d / 4; i += kCThreads) {
                const float4 v = __ldcg(y4 + i);
                x2[i] = make_uint2(bf16_pair_rn(v.x, v.y), bf16_pair_rn(v.z, v.w));
            }
            __syncthreads();
        }
        // activation scales: warp t, the absmax of token t over d (the magnitude bits of a BF16 value order
        // like its magnitude, so an integer maximum over eight values per 16-byte word finds it exactly)
        for (int t = warp; t < T; t += W) {
            const uint4* xr = reinterpret_cast<const uint4*>(xs + t * d);
            uint32_t m2 = 0u;
            for (int i = lane; i < d / 8; i += 32) {
                const uint4 v = xr[i];
                m2 = __vmaxu2(m2, __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                                           __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu)));
            }
            const uint32_t mb = __reduce_max_sync(0xffffffffu, max(m2 & 0xffffu, m2 >> 16));
            if (lane == 0) st.sxs[t] = __fdiv_rn(bf16_to_f32(mb), 127.0f);
        }
        ok = wait_bounded(&st.wbar, (uint32_t)(l & 1)) && ok;
        if (!ok && tid == 0) set_error(p, 40);

        // ------------------------------------------------------------ router
        {
            const int e = tid & 63, q = tid >> 6, kq = ks / 4;
            const uint16_t* xk = xs + rank * ks + q * kq;
            const float* wk = wr + (q * kq) * E + e;
            float* rq = act_all;  // scratch until the first group's SwiGLU: [4][kCMaxT][64]
            const bool on = e < E && ok;
            if (T == 1)
                router_partials<1>(xk, wk, d, E, kq, rq + q * kCMaxT * 64 + e, on);
            else if (T == 2)
                router_partials<2>(xk, wk, d, E, kq, rq + q * kCMaxT * 64 + e, on);
            else if (T <= 4)
                router_partials<4>(xk, wk, d, E, kq, rq + q * kCMaxT * 64 + e, on);
            else
                router_partials<kCMaxT>(xk, wk, d, E, kq, rq + q * kCMaxT * 64 + e, on);
        }
        __syncthreads();
        if (l + 1 < ca.nl && !ca.wr_in_ring && tid == 0) {
            // every thread is done with this layer's W_r slice: the next layer's goes in now
            mbar_expect_tx(&st.wbar, wbytes);
            bulk_load(wr, ca.layers[l + 1].w_router + (int64_t)rank * ks * E, wbytes, &st.wbar);
        }
        if (l == 0) cluster_wait();  // every CTA of the cluster has started
#pragma unroll 1
        for (int i = tid; i < T * 16; i += kCThreads) {
            const int t = i >> 4, e4 = (i & 15) * 4;
            const float* rq = act_all;
            float v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int o = t * 64 + e4 + c;
                v[c] = __fadd_rn(__fadd_rn(__fadd_rn(rq[o], rq[kCMaxT * 64 + o]), rq[2 * kCMaxT * 64 + o]),
                                 rq[3 * kCMaxT * 64 + o]);
            }
            const float4 v4 = make_float4(v[0], v[1], v[2], v[3]);
#pragma unroll 4
            for (int c = 0; c < CS; ++c) st_peer(part_recv + (rank * kCMaxT + t) * 64 + e4, c, v4);
        }
        cluster_sync();  // every slice's partial logits are here
        // gating and top-k: warp t adds token t's slices in rank order, then selects and normalises
        for (int t = warp; t < T; t += W) {
            float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
            for (int c = 0; c < CS; ++c) {
                s0 = __fadd_rn(s0, part_recv[(c * kCMaxT + t) * 64 + lane]);
                s1 = __fadd_rn(s1, part_recv[(c * kCMaxT + t) * 64 + lane + 32]);
            }
            const float l0 = lane < E ? biased_logit(p, Lw.router_bias, s0, lane) : -INFINITY;
            const float l1 = lane + 32 < E ? biased_logit(p, Lw.router_bias, s1, lane + 32) : -INFINITY;
            gate_topk_warp(p, Lw.router_bias, t, l0, l1, lane, st.idx, st.gate, keeper ? p.logits : nullptr);
        }
        __syncthreads();
        if (!early0) {
            // this cluster's first group from the set of selected experts (groups are the shared expert, then
            // the selected experts in ascending order): its gate/up stream starts now, before the permutation
            const int e0 = lane < Tk ? st.idx[lane] : -1, e1 = lane + 32 < Tk ? st.idx[lane + 32] : -1;
            const uint32_t lo = __reduce_or_sync(0xffffffffu, (e0 >= 0 && e0 < 32 ? 1u << e0 : 0u) |
                                                                  (e1 >= 0 && e1 < 32 ? 1u << e1 : 0u));
            const uint32_t hi = __reduce_or_sync(0xffffffffu, (e0 >= 32 ? 1u << (e0 - 32) : 0u) |
                                                                  (e1 >= 32 ? 1u << (e1 - 32) : 0u));
            const int nlo = __popc(lo);
            if (cid <= nlo + __popc(hi)) {
                const int g = cid == 0 ? E : cid - 1 < nlo ? nth_set_bit(lo, cid - 1) : 32 + nth_set_bit(hi, cid - 1 - nlo);
                gu_stream<CS>(S, p, Lw, g, rb0, wsc);
                if (alive && lane < kRingMax && lane < S.ntot) S.issue(lane);
            }
        }
        // ------------------------------------------------------------ permutation (warp 0)
        if (warp == 0) {
            // per-expert counts (experts lane, lane + 32) and each slot's rank among the earlier slots of its
            // expert (slots lane, lane + 32), by one pass over the slots
            const int s0 = lane, s1 = lane + 32;
            const int e0 = s0 < Tk ? st.idx[s0] : -1, e1 = s1 < Tk ? st.idx[s1] : -1;
            int c0 = 0, c1 = 0, r0 = 0, r1 = 0;
#pragma unroll 4
            for (int sl = 0; sl < Tk; ++sl) {
                const int e = st.idx[sl];
                c0 += e == lane;
                c1 += e == lane + 32;
                r0 += sl < s0 && e == e0;
                r1 += sl < s1 && e == e1;
            }
            if (lane >= E) c0 = 0;
            if (lane + 32 >= E) c1 = 0;
            st.cnt[lane] = c0;
            st.cnt[lane + 32] = c1;
            int i0 = c0, i1 = c1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u0 = __shfl_up_sync(0xffffffffu, i0, o), u1 = __shfl_up_sync(0xffffffffu, i1, o);
                if (lane >= o) { i0 += u0; i1 += u1; }
            }
            i1 += __shfl_sync(0xffffffffu, i0, 31);
            const unsigned lt = (1u << lane) - 1u;
            const unsigned b0 = __ballot_sync(0xffffffffu, c0 > 0), b1 = __ballot_sync(0xffffffffu, c1 > 0);
            st.offs[lane] = i0 - c0;
            st.offs[lane + 32] = i1 - c1;
            if (c0) st.groups[1 + __popc(b0 & lt)] = lane;
            if (c1) st.groups[1 + __popc(b0) + __popc(b1 & lt)] = lane + 32;
            __syncwarp();
            if (lane == 0) {
                st.groups[0] = E;
                st.nslots = 1 + __popc(b0) + __popc(b1);
                st.offs[E] = Tk;
                st.offs[E + 1] = Tk + T;
            }
            __syncwarp();
            if (e0 >= 0) {
                const int r = st.offs[e0] + r0;
                st.slot_row[s0] = r;
                st.row_tok[r] = s0 / k;
                st.row_gate[r] = st.gate[s0];
            }
            if (e1 >= 0) {
                const int r = st.offs[e1] + r1;
                st.slot_row[s1] = r;
                st.row_tok[r] = s1 / k;
                st.row_gate[r] = st.gate[s1];
            }
        }
        __syncthreads();
        const int nslots = st.nslots;
        ctarget += fixed ? (uint32_t)(T * CS) : (uint32_t)(nslots * CS);
        int nmine = 0;  // groups of this layer done by this CTA
        // ------------------------------------------------------------ the groups of this cluster
        for (int s = cid; s < nslots; s += ncl) {
            const int g = st.groups[s];
            const bool shared = g == E;
            const int hid = shared ? p.hs : p.h;
            const int nrows = shared ? T : st.cnt[g];
            const int row0 = shared ? Tk : st.offs[g];
            // -------------------------------------------------- gate/up: blocks of 8 gate + 8 up rows
            const int nrb = hid / 8, csz = d + 32, ngr = d / 32;
            const int np = npasses(rb0, CS * W, nrb);
            if (s != cid) {  // (the first group's stream was started before the permutation)
                gu_stream<CS>(S, p, Lw, g, rb0, wsc);
                if (alive && lane < kRingMax && lane < S.ntot) S.issue(lane);
            }
            // the rows' activation codes (one word of four per item, at its place in the B-fragment order of
            // its 32-group); the operand rows past nrows keep stale codes, whose products land only in
            // accumulator columns that are never read
            for (int it = tid; it < nrows * ngr * 8; it += kCThreads) {
                const int i = it / (ngr * 8), j = (it >> 3) % ngr, v = it & 7;
                const int t = shared ? i : st.row_tok[row0 + i];
                const uint2 u = *reinterpret_cast<const uint2*>(xs + t * d + j * 32 + v * 4);
                *reinterpret_cast<uint32_t*>(codes + (size_t)i * csz + j * 32 + 4 * bfrag_pos(v)) =
                    pack_codes(bf16_to_f32(u.x & 0xffffu), bf16_to_f32(u.x >> 16), bf16_to_f32(u.y & 0xffffu),
                               bf16_to_f32(u.y >> 16), st.sxs[t]);
            }
            if (tid < 8) st.shs[tid] = tid < nrows ? st.sxs[shared ? tid : st.row_tok[row0 + tid]] : 0.0f;
            __syncthreads();
            for (int pi = 0; pi < np; ++pi) {
                const int rb = rb0 + pi * CS * W;
                float alo[1][2], ahi[1][2];
                S.sc0 = pi * S.nst;
                if (alive)
                    alive = warp_gemv<true, false, 1>(p, S, codes, csz, lane, rb, row0, nrows, nullptr, 0, 0, alo, ahi);
                // SwiGLU of rows 2 t4, 2 t4 + 1 at feature n, into every CTA's copy of the rows (and into act)
                const int n = rb * 8 + gid;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int i = 2 * t4 + q;
                    if (i >= nrows) continue;
                    const float a = alive ? swiglu_row(alo[0][q], ahi[0][q], st.shs[i]) : 0.0f;
#pragma unroll 4
                    for (int c = 0; c < CS; ++c) st_peer(act_all + i * p.hmax + n, c, __float_as_uint(a));
                }
            }
            wsc += S.ntot;
            if (!y_clear) {
                // before the first atomics into y: cluster 0 has cleared every layer's y (long since)
                if (tid == 0) {
                    const long long t0 = clk();
                    while (ld_acquire(ca.chain + 2) < (uint32_t)CS) {
                        if (clk() - t0 > p.wait_limit) {
                            set_error(p, 43);
                            break;
                        }
                    }
                }
                y_clear = true;  // (the barriers below order the other threads' atomics after the wait)
            }
            // this warp's down blocks start streaming now
            const int nrbd = d / 16, NJd = hid / 64, cszd = hid + 32, ngh = hid / 32;
            const int npd = npasses(rb0, CS * W, nrbd);
            WarpStream<kRingMax> D = S;
            D.src = Lw.w_down_d + (int64_t)g * ((int64_t)d * p.h * 5 / 8) + (int64_t)rb0 * NJd * kJP;
            D.pstride = (int64_t)CS * W * NJd * kJP;
            D.NJ = NJd;
            D.nst = (NJd + kStageJP - 1) / kStageJP;
            D.ntot = npd * D.nst;
            D.base = wsc;
            __syncwarp();
            if (alive && lane < kRingMax && lane < D.ntot) D.issue(lane);
            // -------------------------------------------------- requantisation of the whole rows, in every CTA
            cluster_sync();  // every CTA's SwiGLU features are in every CTA's copy
            if (warp < nrows) {
                float m = 0.0f;
                for (int n = lane; n < hid; n += 32) m = fmaxf(m, fabsf(act_all[warp * p.hmax + n]));
                m = warp_max(m);
                if (lane == 0) {
                    const float sv = __fdiv_rn(m, 127.0f);
                    st.shs[warp] = sv;
                    if (rank == 0) p.sh[row0 + warp] = sv;
                }
            } else if (warp < 8 && lane == 0) {
                st.shs[warp] = 0.0f;
            }
            __syncthreads();
            for (int it = tid; it < nrows * ngh * 8; it += kCThreads) {
                const int i = it / (ngh * 8), j = (it >> 3) % ngh, v = it & 7;
                const float4 a = *reinterpret_cast<const float4*>(act_all + i * p.hmax + j * 32 + v * 4);
                const uint32_t word = pack_codes(a.x, a.y, a.z, a.w, st.shs[i]);
                if (rank == 0) *reinterpret_cast<uint32_t*>(p.hq + (int64_t)(row0 + i) * p.hmax + j * 32 + v * 4) = word;
                *reinterpret_cast<uint32_t*>(codes + (size_t)i * cszd + j * 32 + 4 * bfrag_pos(v)) = word;
            }
            // before this cluster's next group, no CTA may write its SwiGLU values into a copy whose codes
            // are still being taken
            if (s + ncl < nslots)
                cluster_sync();
            else
                __syncthreads();
            // -------------------------------------------------- down: blocks of 16 output rows
            for (int pi = 0; pi < npd; ++pi) {
                const int rb = rb0 + pi * CS * W;
                float alo[1][2], ahi[1][2];
                D.sc0 = pi * D.nst;
                if (alive)
                    alive =
                        warp_gemv<false, false, 1>(p, D, codes, cszd, lane, rb, row0, nrows, nullptr, 0, 0, alo, ahi);
                const int m0 = rb * 16 + gid;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int i = 2 * t4 + q;
                    if (i >= nrows) continue;
                    const float sv = st.shs[i];
                    if (fixed) {
                        ca.obuf[(int64_t)(row0 + i) * d + m0] = __fmul_rn(alo[0][q], sv);
                        ca.obuf[(int64_t)(row0 + i) * d + m0 + 8] = __fmul_rn(ahi[0][q], sv);
                    } else {
                        // gate x row output straight into y (the shared expert's gate is 1)
                        const int t = shared ? i : st.row_tok[row0 + i];
                        const float g = shared ? 1.0f : st.row_gate[row0 + i];
                        float* yr = Lw.y + (int64_t)t * d + m0;
                        atomicAdd(yr, __fmul_rn(g, __fmul_rn(alo[0][q], sv)));
                        atomicAdd(yr + 8, __fmul_rn(g, __fmul_rn(ahi[0][q], sv)));
                    }
                }
            }
            wsc += D.ntot;
            if (!fixed) {
                ++nmine;
                if (s + ncl < nslots) __syncthreads();  // the next group's codes go where this one's were read
                continue;
            }
            // -------------------------------------------------- combine of the tokens whose last contribution this is
            __syncthreads();  // the CTA's row outputs are written; the counts below publish them
            if (tid < 8) {
                int t = -1;
                if (tid < nrows) {
                    const int tt = shared ? tid : st.row_tok[row0 + tid];
                    if (atom_add_acq_rel(ca.cnt + tt * CS + rank, 1u) == (uint32_t)k) t = tt;
                }
                st.last[tid] = t;
            }
            __syncthreads();
            const int npdmax = npasses(rank * W, CS * W, nrbd);
            int ncomb = 0;
#pragma unroll 1
            for (int i = 0; i < 8; ++i) {
                const int t = st.last[i];
                if (t < 0) continue;
                ++ncomb;
#pragma unroll 1
                for (int it = tid; it < npdmax * W * 4; it += kCThreads) {
                    const int pi = it / (W * 4), w = (it >> 2) % W, c4 = it & 3;
                    const int rb = rank * W + w + pi * CS * W;
                    if (rb >= nrbd) continue;
                    const int m = rb * 16 + c4 * 4;
                    float4 yv = __ldcg(reinterpret_cast<const float4*>(ca.obuf + (int64_t)(Tk + t) * d + m));
                    for (int j = 0; j < k; ++j) {
                        const float gj = st.gate[t * k + j];
                        const float4 o = __ldcg(
                            reinterpret_cast<const float4*>(ca.obuf + (int64_t)st.slot_row[t * k + j] * d + m));
                        yv.x = __fadd_rn(yv.x, __fmul_rn(gj, o.x));
                        yv.y = __fadd_rn(yv.y, __fmul_rn(gj, o.y));
                        yv.z = __fadd_rn(yv.z, __fmul_rn(gj, o.z));
                        yv.w = __fadd_rn(yv.w, __fmul_rn(gj, o.w));
                    }
                    *reinterpret_cast<float4*>(Lw.y + (int64_t)t * d + m) = yv;
                }
                if (tid == 0) ca.cnt[t * CS + rank] = 0u;
            }
            if (ca.nl > 1 && ncomb > 0) {
                // these tokens' columns of y are complete: count them for the next layer's wait
                __syncthreads();
                if (tid == 0) red_add_release(ca.chain, (uint32_t)ncomb);
            }
        }
        if (!fixed && ca.nl > 1 && nmine > 0) {
            // this CTA's rows of its groups are in y: count the groups for the next layer's wait
            __syncthreads();
            if (tid == 0) red_add_release(ca.chain, (uint32_t)nmine);
        }
        if (keeper) {
            // the routing and the permutation, as the four-launch path leaves them (of the last layer); here,
            // where the CTA would otherwise wait for the next layer's x
#pragma unroll 1
            for (int i = tid; i < Tk; i += kCThreads) {
                p.idx[i] = st.idx[i];
                p.gate[i] = st.gate[i];
                p.slot_row[i] = st.slot_row[i];
                p.row_src[st.slot_row[i]] = i / k;
                p.row_gate[st.slot_row[i]] = st.gate[i];
                if (Lw.out_idx) Lw.out_idx[i] = st.idx[i];
                if (Lw.out_gate) Lw.out_gate[i] = st.gate[i];
            }
#pragma unroll 1
            for (int t = tid; t < T; t += kCThreads) {
                p.sx[t] = st.sxs[t];
                p.row_src[Tk + t] = t;
                p.row_gate[Tk + t] = 1.0f;
            }
#pragma unroll 1
            for (int e = tid; e <= E + 1; e += kCThreads) {
                p.offsets[e] = st.offs[e];
                if (e <= E) {
                    const int c = e < E ? st.cnt[e] : T;
                    p.counts[e] = c;
                    if (Lw.out_counts) Lw.out_counts[e] = c;
                }
            }
#pragma unroll 1
            for (int i = tid; i < st.nslots; i += kCThreads) p.dec_groups[i] = st.groups[i];
            if (tid == 0) *p.dec_ngroups = st.nslots;
        }
        if (cid == 0) {
            // the shared rows' activation codes (this CTA's K slice), kept for inspection
#pragma unroll 1
            for (int i = tid; i < T * (ks / 4); i += kCThreads) {
                const int t = i / (ks / 4), v = i % (ks / 4);
                const uint16_t* xr = xs + t * d + rank * ks + v * 4;
                *reinterpret_cast<uint32_t*>(p.xq + (int64_t)(Tk + t) * d + rank * ks + v * 4) = pack_codes(
                    bf16_to_f32(xr[0]), bf16_to_f32(xr[1]), bf16_to_f32(xr[2]), bf16_to_f32(xr[3]), st.sxs[t]);
            }
        }
    }
    if (!alive && lane == 0) set_error(p, 41);
    if (ca.nl > 1 || !fixed) {
        // the last CTA to leave resets the chain counters for the next launch (after every CTA's counts:
        // each released them before leaving)
        __syncthreads();
        if (tid == 0 && atom_add_acq_rel(ca.chain + 1, 1u) == gridDim.x - 1) {
            ca.chain[0] = 0u;
            ca.chain[1] = 0u;
            ca.chain[2] = 0u;
        }
    }
}

// INT4 interchange layout -> decode layout (see the top of this file).  For
// gate/up, row block rb holds gate rows 8 rb .. 8 rb + 7 (the A rows 0-7) and
// the matching up rows (A rows 8-15); for down, output rows 16 rb .. 16 rb + 15.
// Lane (gid, t4) of K-group pair jp gets, for each of the two groups, the
// words of A-fragment columns 4 t4 .. 4 t4 + 3 and 16 + 4 t4 .. 16 + 4 t4 + 3:
// byte b = (code of row gid + 8) << 4 | (code of row gid).
__global__ void retile_decode_kernel(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn,
                                     uint8_t* gu_d, uint8_t* dn_d, int d, int h, int hs, int E)
{
    const int g = blockIdx.y;
    const bool down = blockIdx.z == 1;
    const int hid = g == E ? hs : h;
    const int K = down ? hid : d;
    const int nrb = down ? d / 16 : hid / 8;
    const int NJ = K / 64;
    const uint8_t* w = down ? dn + (int64_t)g * d * (h / 2) : gu + (int64_t)g * 2 * h * (d / 2);
    const float* s = down ? sdn + (int64_t)g * d * (h / kGroup) : sgu + (int64_t)g * 2 * h * (d / kGroup);
    uint8_t* dst = down ? dn_d + (int64_t)g * ((int64_t)d * h * 5 / 8) : gu_d + (int64_t)g * ((int64_t)h * d * 5 / 4);
    const int rowb = K / 2, rows_s = K / kGroup;
    const int64_t units = (int64_t)nrb * NJ * 32;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units; u += (int64_t)gridDim.x * blockDim.x) {
        const int lane = (int)(u & 31);
        const int64_t q = u >> 5;
        const int jp = (int)(q % NJ), rb = (int)(q / NJ);
        const int gid = lane >> 2, t4 = lane & 3;
        const int rlo = down ? rb * 16 + gid : rb * 8 + gid;
        const int rhi = down ? rlo + 8 : hid + rb * 8 + gid;
        uint32_t wv[4];
        for (int jj = 0; jj < 2; ++jj)
            for (int wd = 0; wd < 2; ++wd) {
                uint32_t word = 0;
                for (int b = 0; b < 4; ++b) {
                    const int kk = (2 * jp + jj) * 32 + wd * 16 + 4 * t4 + b;
                    const uint32_t nlo = (w[(int64_t)rlo * rowb + kk / 2] >> (4 * (kk & 1))) & 0xFu;
                    const uint32_t nhi = (w[(int64_t)rhi * rowb + kk / 2] >> (4 * (kk & 1))) & 0xFu;
                    word |= ((nhi << 4) | nlo) << (8 * b);
                }
                wv[jj * 2 + wd] = word;
            }
        uint8_t* o = dst + ((int64_t)rb * NJ + jp) * kJP;
        *reinterpret_cast<uint4*>(o + lane * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        if (t4 == 0) {
            const int j0 = 2 * jp, j1 = j0 + 1;
            *reinterpret_cast<float4*>(o + 512 + gid * 16) =
                make_float4(s[(int64_t)rlo * rows_s + j0], s[(int64_t)rhi * rows_s + j0],
                            s[(int64_t)rlo * rows_s + j1], s[(int64_t)rhi * rows_s + j1]);
        }
    }
}

// Raises a kernel's dynamic shared-memory opt-in to at least `bytes`, never
// lowering it (handles of different sizes share the kernels) and calling the
// runtime only when it grows (keeps the call out of stream captures).
// `granted` holds the current opt-in per device.
int g_router_smem[64] = {};

cudaError_t raise_smem(const void* kern, int (&granted)[64], size_t bytes) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (granted[dev] >= (int)bytes) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) granted[dev] = (int)bytes;
    return e;
}

int sm_count() {
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!n[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

size_t expert_smem(int W, int64_t T, int K, int nring) {
    const int64_t rows = T < kPassRows ? T : kPassRows;
    return (size_t)kHeadBytes + (size_t)W * nring * kStageBytes + (size_t)((rows + 7) / 8) * 8 * (K + 32);
}

// Stages in flight per warp: all of a row block's stages when they are at most kRingMax,
// else 3 (keeps two 8-warp CTAs per SM).
int pick_ring(int K) {
    const int nst = (K / 64 + kStageJP - 1) / kStageJP;
    return nst <= kRingMax ? nst : 3;
}

// warps per CTA: as many as keep at least two CTAs per SM busy
int pick_warps(int64_t items) {
    int W = kMaxWarps;
    while (W > 1 && (items + W - 1) / W < 2 * sm_count()) W >>= 1;
    return W;
}

template <bool GU>
cudaError_t launch_expert(const Plan& p, cudaStream_t s, int32_t* dump, int64_t r0, int64_t nr) {
    if (p.T == 0) return cudaSuccess;
    const int gmax = (int)(p.Tk < p.E ? p.Tk : p.E) + 1;
    const int max_nrb = GU ? p.hmax / 8 : p.d / 16;
    const int W = pick_warps((int64_t)gmax * max_nrb);
    const int nbpg = (max_nrb + W - 1) / W;
    const int nring = pick_ring(GU ? p.d : p.hmax);
    const size_t smem = expert_smem(W, p.T, GU ? p.d : p.hmax, nring);
    auto kern = dump ? expert_decode_kernel<GU, true> : expert_decode_kernel<GU, false>;
    static int granted[2][64] = {};
    cudaError_t e = raise_smem((const void*)kern, granted[dump ? 1 : 0], smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(gmax * nbpg), 1, 1);
    cfg.blockDim = dim3((unsigned)(W * 32), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p, nbpg, nring, dump, r0, nr);
}

size_t align128(size_t v) { return (v + 127) / 128 * 128; }

// Dynamic shared memory of the one-launch decode and its offsets: partial logits from every CTA of
// the cluster (two copies) | x (BF16, up to kCMaxT tokens) | operand buffer of 8 rows | SwiGLU values of
// the group's rows (also the router's scratch) | the W_r slice | the rings.  Where that exceeds the SM's
// shared memory the W_r slice lives in the rings' space instead (a layer's slice is then fetched when
// the layer starts, not during the previous layer).
size_t cluster_layout(int d, int h, int hs, int E, int CS, CArgs* ca) {
    const int hmax = h > hs ? h : hs;
    size_t o = align128((size_t)2 * CS * kCMaxT * 64 * 4);
    const size_t off_x = o;
    o = align128(o + (size_t)kCMaxT * d * 2);
    const size_t off_codes = o;
    o = align128(o + (size_t)8 * ((d > hmax ? d : hmax) + 32));
    const size_t off_act = o;
    o = align128(o + std::max((size_t)8 * hmax * 4, (size_t)4 * kCMaxT * 64 * 4));
    const size_t wr_bytes = align128((size_t)(d / CS) * E * 4), ring_bytes = (size_t)kCWarps * kRingMax * kStageBytes;
    const bool apart = o + wr_bytes + ring_bytes + sizeof(CShared) <= (size_t)kSmemLimit;
    const size_t off_wr = o;
    if (apart) o += wr_bytes;
    const size_t off_u = o;
    o += std::max(ring_bytes, apart ? (size_t)0 : wr_bytes);
    if (ca) {
        ca->off_x = (int)off_x;
        ca->off_codes = (int)off_codes;
        ca->off_act = (int)off_act;
        ca->off_wr = (int)off_wr;
        ca->off_u = (int)off_u;
        ca->wr_in_ring = apart ? 0 : 1;
    }
    return o;
}

template <int CS>
cudaLaunchConfig_t cluster_config(size_t smem, int nclusters, cudaStream_t s, cudaLaunchAttribute (&at)[2]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nclusters * CS), 1, 1);
    cfg.blockDim = dim3(kCThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = CS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cfg;
}

// Clusters of CS CTAs of the one-launch decode the device holds at once for this shape (0: none).
template <int CS>
int cluster_capacity(int d, int h, int hs, int E) {
    if (d % (CS * 16)) return 0;  // each CTA's K slice of the router: a multiple of 16 rows
    const size_t smem = cluster_layout(d, h, hs, E, CS, nullptr);
    if (smem + sizeof(CShared) > (size_t)kSmemLimit) return 0;
    static int granted[64] = {};
    if (raise_smem((const void*)decode_cluster_kernel<CS>, granted, smem) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (CS > 8 && cudaFuncSetAttribute(decode_cluster_kernel<CS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                      cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchAttribute at[2];
    cudaLaunchConfig_t cfg = cluster_config<CS>(smem, 1, nullptr, at);
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_cluster_kernel<CS>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

}  // namespace
}  // namespace dec

int dec_fused_max_tokens() { return dec::kCMaxT; }

DecFusedShape dec_fused_shape(int d, int h, int hs, int E) {
    DecFusedShape r{};
    if (E > kMaxExperts || d % 64 || h % 64 || hs % 64) return r;
    r.clusters8 = dec::cluster_capacity<8>(d, h, hs, E);
    r.clusters16 = dec::cluster_capacity<16>(d, h, hs, E);
    return r;
}

size_t dec_fused_counter_words() { return (size_t)dec::kCMaxT * dec::kCMaxCS; }
size_t dec_fused_obuf_floats(int d) { return (size_t)dec::kCMaxT * (kMaxTopK + 1) * d; }

size_t dec_chain_counter_words() { return 3; }

cudaError_t launch_decode_chain(const Plan& p, const DecFusedShape& shape, uint32_t* cnt, float* obuf,
                                uint32_t* chain, const DecChainLayer* layers, int nl, cudaStream_t s) {
    if (p.T == 0) return cudaSuccess;
    if (p.T > dec::kCMaxT || nl < 1 || nl > dec::kMaxChain || !cnt || !obuf || !chain) return cudaErrorInvalidValue;
    for (int l = 0; l < nl; ++l)
        if (!layers[l].y) return cudaErrorInvalidValue;
    dec::CArgs ca{};
    ca.cnt = cnt;
    ca.obuf = obuf;
    ca.chain = chain;
    ca.nl = nl;
    for (int l = 0; l < nl; ++l) {
        ca.layers[l].w_router = layers[l].w_router;
        ca.layers[l].router_bias = layers[l].router_bias;
        ca.layers[l].w_gate_up_d = layers[l].w_gate_up_d;
        ca.layers[l].w_down_d = layers[l].w_down_d;
        ca.layers[l].y = layers[l].y;
        ca.layers[l].out_idx = layers[l].out_idx;
        ca.layers[l].out_gate = layers[l].out_gate;
        ca.layers[l].out_counts = layers[l].out_counts;
    }
    // 16-CTA clusters when one or two tokens leave few groups and every warp of such a cluster has a
    // row block of a routed expert; else 8
    const bool big = shape.clusters16 > 0 && p.T <= 2 && std::min(p.h / 8, p.d / 16) >= 16 * dec::kCWarps;
    cudaLaunchAttribute at[2];
    if (big) {
        const size_t smem = dec::cluster_layout(p.d, p.h, p.hs, p.E, 16, &ca);
        cudaLaunchConfig_t cfg = dec::cluster_config<16>(smem, shape.clusters16, s, at);
        return cudaLaunchKernelEx(&cfg, dec::decode_cluster_kernel<16>, p, ca);
    }
    if (shape.clusters8 <= 0) return cudaErrorInvalidConfiguration;
    const size_t smem = dec::cluster_layout(p.d, p.h, p.hs, p.E, 8, &ca);
    cudaLaunchConfig_t cfg = dec::cluster_config<8>(smem, shape.clusters8, s, at);
    return cudaLaunchKernelEx(&cfg, dec::decode_cluster_kernel<8>, p, ca);
}

cudaError_t launch_decode_fused(const Plan& p, const DecFusedShape& shape, uint32_t* cnt, float* obuf,
                                uint32_t* chain, int32_t* out_idx, float* out_gate, int32_t* out_counts,
                                cudaStream_t s) {
    DecChainLayer one{p.w_router, p.router_bias, p.w_gate_up_d, p.w_down_d, p.y, out_idx, out_gate, out_counts};
    return launch_decode_chain(p, shape, cnt, obuf, chain, &one, 1, s);
}

bool dec_supported(int d, int h, int hs) { return d % 64 == 0 && h % 64 == 0 && hs % 64 == 0; }

int dec_max_tokens(int d, int hmax) {
    const int K = d > hmax ? d : hmax;
    int T = dec::kMaxT;
    while (T > 0 && dec::expert_smem(dec::kMaxWarps, T, K, dec::kRingMax) > (size_t)dec::kSmemLimit) T -= 8;
    return T;
}

// CTAs per router cluster: 16 (non-portable size) where the device runs it,
// else 8, 4, 2, 1; each CTA's K slice must be a multiple of 64 (whole chunks of
// the W_r pieces) and its x and W_r slices must fit in shared memory.  0: no
// size works (the decode path is then off).
int dec_router_cluster(int d, int E) {
    for (int cs = 16; cs >= 1; cs >>= 1) {
        const size_t smem = dec::router_smem(d, cs);
        if (d % (cs * kRouterKChunk) || smem > (size_t)dec::kSmemLimit) continue;
        if (dec::raise_smem((const void*)dec::router_decode_kernel, dec::g_router_smem, smem) != cudaSuccess) {
            cudaGetLastError();
            continue;
        }
        if (cs > 8 &&
            cudaFuncSetAttribute(dec::router_decode_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess) {
            cudaGetLastError();
            continue;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cs, 1, 1);
        cfg.blockDim = dim3(dec::kRThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = cs;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, dec::router_decode_kernel, &cfg) == cudaSuccess && n > 0) return cs;
        cudaGetLastError();
    }
    return 0;
}

cudaError_t launch_router_dec(const Plan& p, int cluster, cudaStream_t s) {
    if (p.T == 0) return cudaSuccess;
    const size_t smem = dec::router_smem(p.d, cluster);
    cudaError_t e = dec::raise_smem((const void*)dec::router_decode_kernel, dec::g_router_smem, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cluster, 1, 1);
    cfg.blockDim = dim3(dec::kRThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, dec::router_decode_kernel, p, cluster);
}

cudaError_t launch_gate_up_dec(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    return dec::launch_expert<true>(p, s, dump, row0, nrows);
}

cudaError_t launch_down_dec(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    return dec::launch_expert<false>(p, s, dump, row0, nrows);
}

cudaError_t launch_retile_dec(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn,
                              uint8_t* gu_d, uint8_t* dn_d, int d, int h, int hs, int E, cudaStream_t s) {
    dim3 grid(64, (unsigned)(E + 1), 2);
    dec::retile_decode_kernel<<<grid, 256, 0, s>>>(gu, sgu, dn, sdn, gu_d, dn_d, d, h, hs, E);
    return cudaGetLastError();
}

}  // namespace mmoe
