// Grouped expert GEMMs on the 5th-generation tensor cores with exact integer
// group partials computed by kind::f16 MMAs.
//
// MobileMoE pages (paper-archivist reading): every expert runs its contiguous
// token slice as one batched matmul, gate and up projections in one GEMM per
// expert, then SwiGLU, the down projection and the weighted scatter back to
// token order (section "custom MoE kernel"); weights are symmetric group-32
// INT4 with FP32 scales (Eq. (6)), activations INT8 (section "QAT").
//
// Why f16 operands for an INT8 x INT4 product.  Every 32-element K group has its
// own FP32 weight scale, so each group's partial sum P_j must leave the tensor
// cores on its own and be promoted, acc = fma(P_j, s_j, acc), by the CUDA
// cores.  The activation codes (|x| <= 127) and the weight codes (-8 .. 7) are
// exact in f16, every product is exact, and a 32-term sum stays below 2^15, so
// an f16 MMA with an FP32 accumulator returns P_j exactly, already as a float.
// Against kind::i8 (S32 partials) that halves the MMA rate but removes the
// integer-to-float conversion, and it doubles the MMA time per TMEM column,
// which is what bounds this kernel: each group's 128 x 128 partials must be
// read out of TMEM (the only way out of the tensor cores) before the buffer can
// take the next group.  Measured on B200 in an isolated loop of the exact
// promotion: i8 8.0 % and f16 14.8 % of the nominal INT8 MMA rate.
//
// A persistent kernel (one CTA per SM) walks over tiles of 256 weight rows
// (two halves of 128) x 128 token rows, each over the whole K range:
//   gate/up: half 0 = the gate rows of 128 hidden features, half 1 = the up
//            rows of the same features, so one thread holds a feature's gate and
//            up sums and applies SwiGLU in registers; K = d_model.
//   down:    the two halves are output rows mb*256 .. +127 and +128 .. +255;
//            K = hidden size of the group's expert.
// Roles (12 warps, three warpgroups):
//   warp 0      producer: per 64-element K stage, two 1-D bulk copies of the
//               halves' weight stage images (f16 codes, already in the
//               canonical K-major 128-byte-swizzle layout, written at load
//               time) and a 2-D TMA load (128-byte swizzle) of the 128 x 64
//               f16 activation-code tile, running ahead across tiles;
//   warp 1      allocates TMEM (512 columns: two buffers of 2 x 128); one lane
//               issues the MMAs (M = 128, N = 128, K = 16): per 32-element
//               group 2 per half into one buffer, then a commit;
//   warps 2-3   idle (they complete warpgroup 0, whose registers go to the
//               promotion warpgroups);
//   warps 4-11  promotion: warp w owns TMEM lane quarter w % 4 (32 weight rows
//               of each half) and token columns 64 * ((w - 4) / 4) .. + 63; per
//               group it reads its 4 x 32 partials per row (each load overlapped
//               with the promotion of the previous one), hands the buffer back
//               and accumulates acc = fma(P_j, s_j, acc) in packed FP32 pairs;
//               after the K range it runs the tile's epilogue from registers
//               (SwiGLU and the FP32 store, or the down projection's output),
//               while the MMA already fills both buffers with the next tile.
// The promotion order (j ascending, fused multiply-add) is the oracle's, so
// the FP32 sums equal it exactly.  Every mbarrier wait is bounded; a wait that
// gives up raises the handle's error flag and the CTA drains and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstddef>

#include "mmoe_internal.cuh"
#include "sm100_tc.cuh"

namespace mmoe {
namespace tf {

constexpr int BMH = 128;                   // weight rows of one half of a tile
constexpr int BN = kTcTileRows;            // token rows per tile (128)
constexpr int BK = 64;                     // K elements per stage (128 bytes of f16 per row)
constexpr int kGroupsPerStage = BK / kGroup;
constexpr int kStages = 4;
constexpr int kBufs = 2;                   // TMEM buffers of 2 x BN columns
constexpr int kBufCols = 2 * BN;
constexpr int kTmemCols = kBufs * kBufCols;
#ifndef MMOE_F16_PROMO_WARPS
#define MMOE_F16_PROMO_WARPS 8
#endif
// 8 or 16: two or four per SM sub-partition.  Measured on c4 (gate/up, down): 2.90 / 1.54 ms with 8,
// 2.80 / 1.95 ms with 16 (32 token columns per thread); the build uses 8.
constexpr int kPromoWarps = MMOE_F16_PROMO_WARPS;
constexpr int kPromoWarp0 = 4;             // promotion warps are the warpgroups after the first
constexpr int kThreads = 128 + kPromoWarps * 32;
// Register split (setmaxnreg): the launch gives every thread kRegsLaunch registers (what fits the SM's
// 65536 when the sub-partition with the most warps holds ceil(warps / 4) of them); warpgroup 0
// (producer, MMA issuer, two idle warps) drops to 32 and the promotion warpgroups rise to kRegsHigh.
constexpr int kRegsLaunch = kPromoWarps == 8 ? 168 : 96;
constexpr int kRegsLow = 32;
constexpr int kRegsHigh = kPromoWarps == 8 ? 232 : 112;
static_assert(kPromoWarps == 8 || kPromoWarps == 16, "8 or 16 promotion warps");
static_assert(128 * kRegsLow + kPromoWarps * 32 * kRegsHigh <= kThreads * kRegsLaunch, "register split");
constexpr int kColGroups = kPromoWarps / 4;  // token-column groups (one warp per lane quarter each)
constexpr int kCols = BN / kColGroups;     // token columns per promotion thread (per half)
constexpr int kChunks = 2 * kCols / 16;    // 16-column TMEM loads per thread and group (both halves)

constexpr int kImgBytes = BMH * BK * 2;    // one half's weight stage image: 16 KB
constexpr int kBBytes = BN * BK * 2;       // activation-code tile: 16 KB
constexpr int kStageBytes = 2 * kImgBytes + kBBytes;
constexpr long long kDrainClk = 4000000000ll;  // about 2 s of SM clock: the limit of the waits while draining

constexpr uint32_t kIdesc = tc5::idesc_f16(BN);

enum Epi { kEpiSwiGLU = 0, kEpiDown = 1 };

constexpr int kMaxCluster = 8;             // CTAs sharing a token tile when the requantisation is fused

constexpr int kTInfo = 4;                  // tile-info ring entries
constexpr int kTInfoConsumers = 1 + kPromoWarps;  // MMA lane, promotion warps

// What every role needs to know about one tile, gathered by the producer warp.
struct TileInfo {
    int row0, nr, mb, nks, tile0, end;
    int skip;            // fused requantisation: this CTA has no feature block of the tile's group
    float colf[BN];      // per token column: activation scale (gate/up) or SwiGLU scale (down)
    float colg[BN];      // per token column: gate of the row (down)
    int colrow[BN];      // per token column: token id (down)
};

struct Smem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t accf[kBufs];    // a buffer holds a finished group
    uint64_t acce[kBufs];    // a buffer has been read (free for the next group)
    uint64_t tfull[kTInfo];
    uint64_t tempty[kTInfo];
    uint64_t never;          // signalled by nothing: the injected stall of the failure-detection tests
    uint64_t xbar[2];        // fused requantisation: the cluster's per-token maxima of a tile have arrived
    uint64_t pbar;           // fused requantisation: the promotion warps' two meeting points of a tile
    uint32_t tmem_base;
    int abort;
    TileInfo ti[kTInfo];
    // fused requantisation: per-token |SwiGLU| maxima of this CTA's 128 features, per TMEM lane quarter,
    // and the maxima received from every CTA of the cluster (two tiles in flight)
    uint32_t amax_part[4][BN];
    alignas(16) float recv[2][kMaxCluster][BN];  // written with 16-byte st.async: 16-byte aligned
};
static_assert(offsetof(Smem, recv) % 16 == 0, "st.async needs 16-byte aligned destinations");

using async::bulk_load;
using async::clk;
using async::fence_barrier_init;
using async::mbar_arrive;
using async::mbar_expect_tx;
using async::mbar_init;
using async::mbar_try_wait;

struct ErrFlags {
    int* dev;
    int* host;
    long long limit;
};

// Waits for the phase of the given parity; gives up after `limit` SM clocks or
// once another thread of the CTA has given up, recording `where` in both error
// flags.  Returns false on giving up.
__device__ __forceinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, Smem* sm, ErrFlags err, int where) {
    const long long t0 = clk();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&sm->abort)) return false;
        if (clk() - t0 > err.limit) {
            atomicExch(&sm->abort, 1);
            if (err.dev) *reinterpret_cast<volatile int*>(err.dev) = where;
            if (err.host) *reinterpret_cast<volatile int*>(err.host) = where;
            __threadfence_system();
            return false;
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Smem* sm, ErrFlags err, int where) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, sm, err, where);
}

// Bounded wait used while draining after an abort: ignores the abort flag and
// the per-call limit, gives up only after kDrainClk.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const long long t0 = clk();
    while (!mbar_try_wait(bar, parity))
        if (clk() - t0 > kDrainClk) return;
}

// One lane waits, the warp follows.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Smem* sm, ErrFlags ef, int where) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, sm, ef, where);
    return __shfl_sync(0xffffffffu, ok, 0);
}

struct Args {
    const uint16_t* wimg;   // weight stage images (f16 codes) of the expert kind
    const float* simg;      // their group scales: per image, 2 groups x 128 rows
    int64_t expert_stride;  // stage images per routed expert
    int mblocks_routed;     // tiles of 256 weight rows per routed expert (gate/up: h/128, down: d/256)
    int mblocks_shared;
    int ks_routed;          // K stages of a routed expert (gate/up: d/64, down: h/64)
    int ks_shared;
    int fblocks;            // weight-row tiles per token tile in the launch (the larger of the two)
    int cluster;            // fused requantisation: CTAs per cluster (= fblocks), else 1
    int32_t* dump;          // optional INT32 partial dump
    int64_t drow0, dnrows;
};

struct Tile {
    int g, mb, nks, nr, row0, tile0;
    bool valid;
};

// Tile L of the launch: weight-row tile L % fblocks of token tile L / fblocks.
__device__ __forceinline__ Tile decode_tile(const Plan& p, const Args& a, int L) {
    Tile t;
    const int fb = L % a.fblocks;
    const int ti = L / a.fblocks;
    const int code = p.tiles[ti];
    t.g = code >> 24;
    const int tin = code & 0xffffff;
    const bool shared_grp = t.g == p.E;
    t.valid = fb < (shared_grp ? a.mblocks_shared : a.mblocks_routed);
    t.mb = fb;
    t.nks = shared_grp ? a.ks_shared : a.ks_routed;
    const int cnt = p.offsets[t.g + 1] - p.offsets[t.g];
    t.row0 = p.offsets[t.g] + tin * BN;
    t.nr = min(BN, cnt - tin * BN);
    // half 0 is image block 2 mb, half 1 block 2 mb + 1; each block has nks stage images
    t.tile0 = (int)(t.g * a.expert_stride) + 2 * fb * t.nks;
    return t;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(async::su32(p)), "r"(rank));
    return a;
}

// 16 bytes into a peer's shared memory, counted on the peer's mbarrier as bytes of its transaction.
__device__ __forceinline__ void st_async_peer(uint32_t dst, uint32_t bar, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(dst),
                 "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar)
                 : "memory");
}

// acc[c] = fma((P[2c], P[2c+1]), (s, s), acc[c]) for 8 pairs of columns: the
// partials arrive from TMEM as the bits of exact FP32 integers.
__device__ __forceinline__ void promote8(float2* acc, const uint32_t (&v)[16], float s) {
    const float2 s2 = make_float2(s, s);
#pragma unroll
    for (int c = 0; c < 8; ++c)
        acc[c] = __ffma2_rn(make_float2(__uint_as_float(v[2 * c]), __uint_as_float(v[2 * c + 1])), s2, acc[c]);
}

// SwiGLU of one feature from its gate and up sums and the token's activation scale:
// silu(g sx) * (u sx), silu(v) = v / (1 + exp(-v)), each step an IEEE FP32 operation
__device__ __forceinline__ float swiglu(float g, float u, float sx) {
    const float gv = __fmul_rn(g, sx);
    const float uv = __fmul_rn(u, sx);
    const float silu = __fdiv_rn(gv, __fadd_rn(1.0f, expf(-gv)));
    return __fmul_rn(silu, uv);
}

// INT32 partials of 16 columns (one TMEM load) for the inspection entry point.
template <int kEpi>
__device__ __forceinline__ void dump16(const Plan& p, const Args& a, const TileInfo& ti, int half, int row, int c0,
                                       const uint32_t (&v)[16], int j) {
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
        const int cc = c0 + c;
        const int64_t grow = (int64_t)ti.row0 + cc;
        if (cc >= ti.nr || grow < a.drow0 || grow >= a.drow0 + a.dnrows) continue;
        const int32_t pv = (int32_t)__uint_as_float(v[c]);
        if (kEpi == kEpiSwiGLU) {
            const int f = ti.mb * BMH + row;
            const int n = half == 0 ? f : p.hmax + f;
            a.dump[((grow - a.drow0) * 2 * p.hmax + n) * (p.d / kGroup) + j] = pv;
        } else {
            const int m = ti.mb * 2 * BMH + half * BMH + row;
            a.dump[((grow - a.drow0) * p.d + m) * (p.hmax / kGroup) + j] = pv;
        }
    }
}

template <int kEpi, bool kDump, bool kFuse>
__global__ void __launch_bounds__(kThreads, 1)
expert_gemm_f16_kernel(const __grid_constant__ CUtensorMap bmap, Plan p, Args a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = base;
    Smem* sm = reinterpret_cast<Smem*>(base + kStages * kStageBytes);

    // Fused requantisation: the CTAs of a cluster share each token tile, rank r taking feature block r;
    // they all walk the same tiles and leave together (no early exit: peers write into each other's
    // shared memory until the final cluster barrier).
    const int C = kFuse ? a.cluster : 1;
    const int crank = kFuse ? (int)cluster_ctarank() : 0;
    const int cid = (int)blockIdx.x / C, ncl = (int)gridDim.x / C;
    if (!kFuse) {
        // nothing to do after an earlier wait gave up
        if (p.err && *reinterpret_cast<volatile int*>(p.err)) return;
    }
    const int total = kFuse ? *p.tile_count : (*p.tile_count) * a.fblocks;
    if (!kFuse && (int)blockIdx.x >= total) return;
    const ErrFlags ef{p.err, p.err_host, p.wait_limit};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < kBufs; ++b) {
            mbar_init(&sm->accf[b], 1);
            mbar_init(&sm->acce[b], kPromoWarps);
        }
        for (int b = 0; b < kTInfo; ++b) {
            mbar_init(&sm->tfull[b], 32);
            mbar_init(&sm->tempty[b], kTInfoConsumers);
        }
        mbar_init(&sm->never, 1);
        mbar_init(&sm->xbar[0], 1);
        mbar_init(&sm->xbar[1], 1);
        mbar_init(&sm->pbar, kPromoWarps);
        sm->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tc5::tmem_alloc(&sm->tmem_base, kTmemCols);
        tc5::before_sync();
    }
    __syncthreads();
    tc5::after_sync();
    // the peers' barriers exist before anyone signals them
    if (kFuse) cluster_sync_all();
    const uint32_t tmem = sm->tmem_base;
    if (warp < kPromoWarp0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
        if (warp == 0) {
            // ------------------------------------------------------------ producer (whole warp)
            int sc = 0, tcount = 0;
            bool ok = true;
            for (int L = kFuse ? cid : (int)blockIdx.x; ok; L += kFuse ? ncl : (int)gridDim.x) {
                Tile t{};
                const bool last = L >= total;  // past the last tile: publish the end marker and stop
                if (!last) {
                    // fused: token tile L, feature block = cluster rank
                    if (lane == 0) t = decode_tile(p, a, kFuse ? L * a.fblocks + crank : L);
                    t.valid = __shfl_sync(0xffffffffu, t.valid, 0);
                    if (!t.valid && !kFuse) continue;
                    if (!t.valid) t.nks = 0;  // published with no K stages: the CTA joins the exchange only
                    t.mb = __shfl_sync(0xffffffffu, t.mb, 0);
                    t.nks = __shfl_sync(0xffffffffu, t.nks, 0);
                    t.nr = __shfl_sync(0xffffffffu, t.nr, 0);
                    t.row0 = __shfl_sync(0xffffffffu, t.row0, 0);
                    t.tile0 = __shfl_sync(0xffffffffu, t.tile0, 0);
                }
                const int b = tcount % kTInfo;
                if (tcount >= kTInfo && !warp_wait(&sm->tempty[b], ((tcount / kTInfo) - 1) & 1, sm, ef, 16)) {
                    ok = false;
                    break;
                }
                TileInfo& ti = sm->ti[b];
                if (lane == 0) {
                    ti.end = last ? 1 : 0;
                    ti.skip = (!last && !t.valid) ? 1 : 0;
                    ti.row0 = t.row0; ti.nr = t.nr; ti.mb = t.mb; ti.nks = t.nks; ti.tile0 = t.tile0;
                }
                if (!last) {
                    for (int c = lane; c < BN; c += 32) {
                        const int r = t.row0 + (c < t.nr ? c : 0);
                        if (kEpi == kEpiSwiGLU) {
                            ti.colf[c] = p.sx[p.row_src[r]];
                        } else {
                            ti.colf[c] = p.sh[r];
                            ti.colg[c] = p.row_gate[r];
                            ti.colrow[c] = p.row_src[r];
                        }
                    }
                }
                mbar_arrive(&sm->tfull[b]);
                ++tcount;
                if (last) break;
                if (lane == 0) {
                    for (int ks = 0; ks < t.nks; ++ks, ++sc) {
                        const int s = sc % kStages;
                        if (sc >= kStages && !mbar_wait(&sm->empty[s], ((sc / kStages) - 1) & 1, sm, ef, 11)) {
                            ok = false;
                            break;
                        }
                        uint8_t* st = stages + s * kStageBytes;
                        mbar_expect_tx(&sm->full[s], kStageBytes);
                        bulk_load(st, a.wimg + ((int64_t)t.tile0 + ks) * (kImgBytes / 2), kImgBytes, &sm->full[s]);
                        bulk_load(st + kImgBytes, a.wimg + ((int64_t)t.tile0 + t.nks + ks) * (kImgBytes / 2), kImgBytes,
                                  &sm->full[s]);
                        tc5::tma_load_2d(st + 2 * kImgBytes, &bmap, ks * BK, t.row0, &sm->full[s]);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
            }
            // every issued copy has landed before the CTA may exit
            if (lane == 0)
                for (int i = sc > kStages ? sc - kStages : 0; i < sc; ++i)
                    mbar_wait_drain(&sm->full[i % kStages], (i / kStages) & 1);
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                int sc = 0, pc = 0, tcount = 0;
                bool ok = true;
                // injected stall (tests only): a wait that can never complete runs out after the
                // handle's limit, exactly like a real stall, and the CTA drains and exits
                if (p.debug_stall && blockIdx.x == 0) ok = mbar_wait(&sm->never, 0, sm, ef, 20);
                while (ok) {
                    const int tb = tcount % kTInfo;
                    if (!mbar_wait(&sm->tfull[tb], (tcount / kTInfo) & 1, sm, ef, 17)) break;
                    const int nks = sm->ti[tb].nks, end = sm->ti[tb].end;
                    mbar_arrive(&sm->tempty[tb]);
                    ++tcount;
                    if (end) break;
                    for (int ks = 0; ks < nks && ok; ++ks, ++sc) {
                        const int s = sc % kStages;
                        if (!mbar_wait(&sm->full[s], (sc / kStages) & 1, sm, ef, 12)) { ok = false; break; }
                        tc5::after_sync();
                        uint8_t* st = stages + s * kStageBytes;
                        const uint64_t a0 = tc5::smem_desc_sw128(st);
                        const uint64_t a1 = tc5::smem_desc_sw128(st + kImgBytes);
                        const uint64_t bd = tc5::smem_desc_sw128(st + 2 * kImgBytes);
    #pragma unroll
                        for (int jj = 0; jj < kGroupsPerStage; ++jj, ++pc) {
                            const int b = pc & 1;
                            if (!mbar_wait(&sm->acce[b], (pc >> 1) & 1, sm, ef, 13)) { ok = false; break; }
                            tc5::after_sync();
                            const uint32_t d0 = tmem + b * kBufCols;
                            // a 32-element group = two K = 16 steps, 32 bytes each (2 descriptor units)
                            const uint64_t k0 = (uint64_t)(4 * jj), k1 = k0 + 2;
                            tc5::mma_f16<kIdesc>(d0, a0 + k0, bd + k0, 0u);
                            tc5::mma_f16<kIdesc>(d0, a0 + k1, bd + k1, 1u);
                            tc5::mma_f16<kIdesc>(d0 + BN, a1 + k0, bd + k0, 0u);
                            tc5::mma_f16<kIdesc>(d0 + BN, a1 + k1, bd + k1, 1u);
                            tc5::commit(&sm->accf[b]);
                        }
                        tc5::commit(&sm->empty[s]);
                    }
                }
                // every MMA issued has completed before TMEM is released
                if (pc > 0) mbar_wait_drain(&sm->accf[(pc - 1) & 1], ((pc - 1) >> 1) & 1);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        // ------------------------------------------------------------ promotion + epilogue
        const int pw = warp - kPromoWarp0;    // 0..7
        const int hc = pw >> 2;               // token-column group
        const int quarter = warp & 3;         // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;  // weight row of this thread within each half
        const int col0 = hc * kCols;
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)col0;
        // every buffer starts free: completion 0 of both acce barriers
        if (lane == 0)
            for (int b = 0; b < kBufs; ++b) mbar_arrive(&sm->acce[b]);
        int pc = 0, tcount = 0;
        bool ok = true;
        while (ok) {
            const int tb = tcount % kTInfo;
            if (!warp_wait(&sm->tfull[tb], (tcount / kTInfo) & 1, sm, ef, 19)) break;
            const TileInfo& ti = sm->ti[tb];
            if (ti.end) break;
            const int nks = ti.nks, nr = ti.nr, mb = ti.mb, skip = ti.skip;
            const int64_t row0 = ti.row0;
            // group scales: half 0 at sp[j * 128], half 1 at sp[half1 + j * 128]
            const float* sp = a.simg + (size_t)ti.tile0 * (kGroupsPerStage * BMH) + row;
            const size_t half1 = (size_t)nks * (kGroupsPerStage * BMH);
            float2 acc0[kCols / 2], acc1[kCols / 2];
#pragma unroll
            for (int c = 0; c < kCols / 2; ++c) acc0[c] = acc1[c] = make_float2(0.0f, 0.0f);
            const int ng = nks * kGroupsPerStage;
            float s0 = 0.0f, s1 = 0.0f;
            if (ng > 0) {
                s0 = __ldg(sp);
                s1 = __ldg(sp + half1);
            }
            for (int j = 0; j < ng; ++j, ++pc) {
                const int b = pc & 1;
                float n0 = 0.0f, n1 = 0.0f;
                if (j + 1 < ng) {
                    n0 = __ldg(sp + (size_t)(j + 1) * BMH);
                    n1 = __ldg(sp + half1 + (size_t)(j + 1) * BMH);
                }
                if (!warp_wait(&sm->accf[b], (pc >> 1) & 1, sm, ef, 15)) { ok = false; break; }
                tc5::after_sync();
                const uint32_t ta = tl + b * kBufCols;
                // loads of 16 columns (half 0, then half 1), each overlapped with the promotion of the
                // one before; the buffer goes back to the MMA as soon as the last has landed
                constexpr int kPerHalf = kChunks / 2;
                uint32_t va[16], vb[16];
                tc5::tmem_ld16(ta, va);
#pragma unroll
                for (int ch = 0; ch < kChunks; ++ch) {
                    uint32_t (&cur)[16] = (ch & 1) ? vb : va;
                    uint32_t (&nxt)[16] = (ch & 1) ? va : vb;
                    tc5::tmem_wait_ld(cur);
                    if (ch < kChunks - 1) {
                        const int nc = ch + 1;
                        tc5::tmem_ld16(ta + (nc / kPerHalf) * BN + (nc % kPerHalf) * 16, nxt);
                    } else {
                        tc5::before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm->acce[b]);
                    }
                    const int half = ch / kPerHalf;
                    float2* acc = half ? acc1 : acc0;
                    promote8(acc + (ch % kPerHalf) * 8, cur, half ? s1 : s0);
                    if (kDump) dump16<kEpi>(p, a, ti, half, row, col0 + (ch % kPerHalf) * 16, cur, j);
                }
                s0 = n0;
                s1 = n1;
            }
            if (!ok || *reinterpret_cast<volatile int*>(&sm->abort)) break;
            // the tile's epilogue, from registers; for a fixed column a warp writes 32 consecutive floats.
            // The inspection launch (kDump) runs the same K loop with the partials' stores added and no
            // epilogue: its plan has no output buffers.
            if (kDump) {
            } else if (kEpi == kEpiSwiGLU && kFuse) {
                // SwiGLU in registers (kept in acc0), then the per-token requantisation over all
                // hidden features: this CTA's maxima over its 128 features (a warp reduction per
                // column, then the four lane quarters through shared memory), sent to every CTA of
                // the cluster, the cluster's maximum, the codes of this CTA's features
                const int slot = tcount & 1;
#pragma unroll
                for (int c = 0; c < kCols; ++c) {
                    const int cc = col0 + c;
                    const float g = (c & 1) ? acc0[c >> 1].y : acc0[c >> 1].x;
                    const float u = (c & 1) ? acc1[c >> 1].y : acc1[c >> 1].x;
                    const float av = (!skip && cc < nr) ? swiglu(g, u, ti.colf[cc]) : 0.0f;
                    if (c & 1) acc0[c >> 1].y = av;
                    else acc0[c >> 1].x = av;
                }
                uint32_t mine[kCols / 32];
#pragma unroll
                for (int c = 0; c < kCols; ++c) {
                    const float av = (c & 1) ? acc0[c >> 1].y : acc0[c >> 1].x;
                    const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(av)));
                    if ((c & 31) == lane) mine[c >> 5] = m;
                }
#pragma unroll
                for (int i = 0; i < kCols / 32; ++i) sm->amax_part[quarter][col0 + 32 * i + lane] = mine[i];
                // every promotion warp has written its maxima: the first of the tile's two phases of pbar
                // (a bounded wait, unlike a named barrier, so that a warp that gave up cannot hang the rest)
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->pbar);
                if (!warp_wait(&sm->pbar, 0, sm, ef, 22)) { ok = false; break; }
                mbar_try_wait(&sm->pbar, 0);  // this lane's own acquire of the phase
                const int pt = pw * 32 + lane;  // 0 .. promotion threads - 1
                if (pt == 0) mbar_expect_tx(&sm->xbar[slot], (uint32_t)(C * BN * 4));
                if (pt < C * 32) {
                    // thread pt sends columns 4 (pt % 32) .. + 3 to cluster rank pt / 32
                    const int c4 = 4 * (pt & 31);
                    uint32_t v[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        v[i] = max(max(sm->amax_part[0][c4 + i], sm->amax_part[1][c4 + i]),
                                   max(sm->amax_part[2][c4 + i], sm->amax_part[3][c4 + i]));
                    const uint32_t dst = (uint32_t)(pt >> 5);
                    st_async_peer(peer_addr(&sm->recv[slot][crank][c4], dst), peer_addr(&sm->xbar[slot], dst), v[0],
                                  v[1], v[2], v[3]);
                }
                // every sender has read the maxima before the next tile overwrites them: the second phase
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->pbar);
                if (!warp_wait(&sm->pbar, 1, sm, ef, 23)) { ok = false; break; }
                if (!warp_wait(&sm->xbar[slot], (tcount >> 1) & 1, sm, ef, 21)) { ok = false; break; }
                mbar_try_wait(&sm->xbar[slot], (tcount >> 1) & 1);  // this lane's own acquire of the phase
                if (!skip) {
                    uint16_t* out = p.hq16 + row0 * p.hmax + mb * BMH + row;
#pragma unroll
                    for (int c = 0; c < kCols; ++c) {
                        const int cc = col0 + c;
                        float m = 0.0f;
                        for (int r = 0; r < C; ++r) m = fmaxf(m, sm->recv[slot][r][cc]);
                        const float sh = __fdiv_rn(m, 127.0f);
                        const float av = (c & 1) ? acc0[c >> 1].y : acc0[c >> 1].x;
                        if (cc < nr) {
                            out[(int64_t)cc * p.hmax] = (uint16_t)code_f16(quant_i8(av, sh));
                            if (crank == 0 && quarter == 0 && lane == (c & 31)) p.sh[row0 + cc] = sh;
                        }
                    }
                }
            } else if (kEpi == kEpiSwiGLU) {
                // the (gate, up) pair of each feature times the row's activation scale; the SwiGLU itself
                // is applied by the requantisation pass, off this loop's critical path
                float2* out = reinterpret_cast<float2*>(p.act) + row0 * p.hmax + mb * BMH + row;
#pragma unroll
                for (int c = 0; c < kCols; ++c) {
                    const int cc = col0 + c;
                    if (cc < nr) {
                        const float g = (c & 1) ? acc0[c >> 1].y : acc0[c >> 1].x;
                        const float u = (c & 1) ? acc1[c >> 1].y : acc1[c >> 1].x;
                        const float f = ti.colf[cc];
                        out[(int64_t)cc * p.hmax] = make_float2(__fmul_rn(g, f), __fmul_rn(u, f));
                    }
                }
            } else {
                const int m = mb * 2 * BMH + row;
#pragma unroll
                for (int c = 0; c < kCols; ++c) {
                    const int cc = col0 + c;
                    if (cc < nr) {
                        const float f = ti.colf[cc];
                        const float o0 = __fmul_rn((c & 1) ? acc0[c >> 1].y : acc0[c >> 1].x, f);
                        const float o1 = __fmul_rn((c & 1) ? acc1[c >> 1].y : acc1[c >> 1].x, f);
                        if (p.deterministic) {
                            float* o = p.obuf + (row0 + cc) * p.d + m;
                            o[0] = o0;
                            o[BMH] = o1;
                        } else {
                            const float gt = ti.colg[cc];
                            float* yr = p.y + (int64_t)ti.colrow[cc] * p.d + m;
                            atomicAdd(yr, __fmul_rn(gt, o0));
                            atomicAdd(yr + BMH, __fmul_rn(gt, o1));
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->tempty[tb]);
            ++tcount;
        }
    }

    __syncthreads();
    // no CTA of a cluster leaves while a peer may still write into its shared memory
    if (kFuse) cluster_sync_all();
    if (warp == 1) {
        tc5::after_sync();
        tc5::tmem_dealloc(tmem, kTmemCols);
    }
}

// --------------------------------------------------------------- weight stage images (load time)
// Image (g, blk, ks) of an expert: 128 weight rows x 64 K values as f16 codes, row r at byte 128 r, its
// 16-byte chunk c (K values ks*64 + 8c .. + 7) stored at chunk c ^ (r & 7) (the 128-byte swizzle the
// MMA's shared-memory descriptor expects at a 1024-byte aligned stage).  Blocks: gate/up block 2i holds
// the gate rows of features 128 i .. + 127, block 2i + 1 the up rows of the same features; down block i
// holds output rows 128 i .. + 127.  Scales: per image, group ks*2 + jj at [(image * 2 + jj) * 128 + r].

// one thread per 16-byte chunk of an image row (8 K values)
__global__ void retile_f16_kernel(const uint8_t* __restrict__ src, const float* __restrict__ ssrc,
                                  uint16_t* __restrict__ dst, float* __restrict__ sdst, int E, int K_routed,
                                  int K_shared, int blk_routed, int blk_shared, int gate_up, int h, int hs,
                                  int64_t total_chunks)
{
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= total_chunks) return;
    const int64_t per_routed = (int64_t)blk_routed * (K_routed / BK) * BMH * 8;  // chunks of a routed expert
    int g;
    int64_t r;
    if (q < per_routed * E) { g = (int)(q / per_routed); r = q % per_routed; }
    else { g = E; r = q - per_routed * E; }
    const int K = g < E ? K_routed : K_shared;
    const int nks = K / BK;
    const int chunk = (int)(r % 8);
    const int trow = (int)((r / 8) % BMH);
    const int64_t img = r / (8 * BMH);  // blk * nks + ks
    const int ks = (int)(img % nks);
    const int blk = (int)(img / nks);
    const int hid = g < E ? h : hs;
    int64_t srow;  // row inside the expert's interchange block
    if (gate_up) srow = (blk & 1) ? (int64_t)hid + (blk >> 1) * BMH + trow : (int64_t)(blk >> 1) * BMH + trow;
    else srow = (int64_t)blk * BMH + trow;
    // interchange block of expert g starts at g * (routed block size)
    const int64_t src_rows_routed = gate_up ? 2 * (int64_t)h : (int64_t)blk_routed * BMH;
    const int64_t src_expert_bytes = src_rows_routed * ((int64_t)K_routed / 2);
    const uint8_t* s = src + (int64_t)g * src_expert_bytes + srow * (K / 2) + (int64_t)ks * (BK / 2) + chunk * 4;
    const uint32_t w = *reinterpret_cast<const uint32_t*>(s);  // 8 codes, low nibble first
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int c0 = ((int)(w >> (8 * i)) << 28) >> 28;        // sign-extended nibbles
        const int c1 = ((int)(w >> (8 * i + 4)) << 28) >> 28;
        o[i] = (uint32_t)__half_as_ushort(__int2half_rn(c0)) | ((uint32_t)__half_as_ushort(__int2half_rn(c1)) << 16);
    }
    const int64_t dst_imgs_routed = (int64_t)blk_routed * (K_routed / BK);
    const int64_t dimg = (int64_t)g * dst_imgs_routed + img;
    uint4* rowp = reinterpret_cast<uint4*>(dst + dimg * (kImgBytes / 2) + trow * BK);
    rowp[chunk ^ (trow & 7)] = make_uint4(o[0], o[1], o[2], o[3]);
    if ((chunk & 3) == 0) {
        const int jj = chunk >> 2;
        const int64_t src_expert_scales = src_rows_routed * ((int64_t)K_routed / kGroup);
        sdst[(dimg * 2 + jj) * BMH + trow] =
            ssrc[(int64_t)g * src_expert_scales + srow * (K / kGroup) + ks * kGroupsPerStage + jj];
    }
}

}  // namespace tf

// ------------------------------------------------------------------ host side
bool f16tc_supported(int d, int h, int hs) { return d % 256 == 0 && h % 128 == 0 && hs % 128 == 0; }

size_t f16tc_smem_bytes() { return 1024 + tf::kStages * tf::kStageBytes + sizeof(tf::Smem); }
static_assert(1024 + tf::kStages * tf::kStageBytes + sizeof(tf::Smem) <= 232448, "shared memory");

size_t f16tc_image_elems(int d, int h, int hs, int E, bool gate_up) {
    // f16 codes: one per weight
    return gate_up ? (size_t)(E * 2 * (size_t)h + 2 * (size_t)hs) * d : (size_t)(E * (size_t)h + hs) * d;
}

cudaError_t launch_retile_f16(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn,
                              uint16_t* gu_t, float* sgu_t, uint16_t* dn_t, float* sdn_t, int d, int h, int hs, int E,
                              cudaStream_t s) {
    // gate/up: blocks of 128 rows over 2*hid rows, K = d
    const int64_t gu_chunks = ((int64_t)E * (2 * h / tf::BMH) + (2 * hs / tf::BMH)) * (d / tf::BK) * tf::BMH * 8;
    tf::retile_f16_kernel<<<(unsigned)((gu_chunks + 255) / 256), 256, 0, s>>>(gu, sgu, gu_t, sgu_t, E, d, d,
                                                                               2 * h / tf::BMH, 2 * hs / tf::BMH, 1, h,
                                                                               hs, gu_chunks);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // down: blocks of 128 output rows, K = hid
    const int64_t dn_chunks = ((int64_t)E * (h / tf::BK) + (hs / tf::BK)) * (d / tf::BMH) * tf::BMH * 8;
    tf::retile_f16_kernel<<<(unsigned)((dn_chunks + 255) / 256), 256, 0, s>>>(dn, sdn, dn_t, sdn_t, E, h, hs,
                                                                               d / tf::BMH, d / tf::BMH, 0, h, hs,
                                                                               dn_chunks);
    return cudaGetLastError();
}

static int sm_count_f16() {
    static int n[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!n[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

int f16tc_fused_clusters(int c);

template <int kEpi, bool kDump, bool kFuse>
static cudaError_t launch_f16(const Plan& p, cudaStream_t s, const CUtensorMap* map, tf::Args a) {
    auto kern = tf::expert_gemm_f16_kernel<kEpi, kDump, kFuse>;
    const size_t smem = f16tc_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (!kFuse) {
        // persistent: one CTA per SM (never more CTAs than the largest possible tile count)
        a.cluster = 1;
        const int64_t upper = p.max_tiles * (int64_t)a.fblocks;
        const unsigned grid = (unsigned)(upper < sm_count_f16() ? upper : sm_count_f16());
        kern<<<grid, tf::kThreads, smem, s>>>(*map, p, a);
        return cudaGetLastError();
    }
    // fused requantisation: clusters of fblocks CTAs, as many as the device holds at once (each CTA
    // takes a whole SM), never more than the largest possible token-tile count
    a.cluster = a.fblocks;
    const int ncl_max = f16tc_fused_clusters(a.fblocks);
    if (ncl_max <= 0) return cudaErrorNotSupported;
    const int64_t ncl = p.max_tiles < ncl_max ? p.max_tiles : ncl_max;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(ncl * a.cluster), 1, 1);
    cfg.blockDim = dim3(tf::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)a.cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, *map, p, a);
}

// Clusters of `c` CTAs of the fused gate/up GEMM that fit on the device at once (0: none); queried
// once per device and cluster size.
int f16tc_fused_clusters(int c) {
    static int cache[64][tf::kMaxCluster + 1] = {};
    static bool done[64][tf::kMaxCluster + 1] = {};
    if (c < 1 || c > tf::kMaxCluster) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (done[dev][c]) return cache[dev][c];
    auto kern = tf::expert_gemm_f16_kernel<tf::kEpiSwiGLU, false, true>;
    const size_t smem = f16tc_smem_bytes();
    int n = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)c, 1, 1);
        cfg.blockDim = dim3(tf::kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = (unsigned)c;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cache[dev][c] = n;
    done[dev][c] = true;
    return n;
}

cudaError_t launch_gate_up_f16(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    if (p.T == 0) return cudaSuccess;
    tf::Args a{};
    a.wimg = p.w_gate_up_f16;
    a.simg = p.s_gate_up_t;
    a.mblocks_routed = p.h / tf::BMH;
    a.mblocks_shared = p.hs / tf::BMH;
    a.ks_routed = a.ks_shared = p.d / tf::BK;
    a.expert_stride = (int64_t)(2 * a.mblocks_routed) * a.ks_routed;
    a.fblocks = p.hmax / tf::BMH;
    a.dump = dump;
    a.drow0 = row0;
    a.dnrows = nrows;
    const CUtensorMap* map = static_cast<const CUtensorMap*>(p.tmap_xq);
    if (dump) return launch_f16<tf::kEpiSwiGLU, true, false>(p, s, map, a);
    return p.fuse_requant ? launch_f16<tf::kEpiSwiGLU, false, true>(p, s, map, a)
                          : launch_f16<tf::kEpiSwiGLU, false, false>(p, s, map, a);
}

cudaError_t launch_down_f16(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    if (p.T == 0) return cudaSuccess;
    tf::Args a{};
    a.wimg = p.w_down_f16;
    a.simg = p.s_down_t;
    a.mblocks_routed = a.mblocks_shared = p.d / (2 * tf::BMH);
    a.ks_routed = p.h / tf::BK;
    a.ks_shared = p.hs / tf::BK;
    a.expert_stride = (int64_t)(p.d / tf::BMH) * a.ks_routed;
    a.fblocks = p.d / (2 * tf::BMH);
    a.dump = dump;
    a.drow0 = row0;
    a.dnrows = nrows;
    const CUtensorMap* map = static_cast<const CUtensorMap*>(p.tmap_hq);
    return dump ? launch_f16<tf::kEpiDown, true, false>(p, s, map, a) : launch_f16<tf::kEpiDown, false, false>(p, s, map, a);
}

}  // namespace mmoe
