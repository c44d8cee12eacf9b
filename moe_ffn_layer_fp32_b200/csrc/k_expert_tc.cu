// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, kind::i8).
//
// MobileMoE pages (paper-archivist reading): every expert runs its contiguous
// token slice as one batched matmul, gate and up projections in one GEMM per
// expert, then SwiGLU, the down projection and the weighted scatter back to
// token order (section "custom MoE kernel"); weights are symmetric group-32
// INT4 with FP32 scales (Eq. (6)), activations INT8 (section "QAT").
//
// A persistent kernel (one CTA per SM) walks over 128 x 128 output tiles:
// 128 weight rows (M) x 128 token rows (N), each over the whole K range.
//   gate/up: the 128 weight rows are 64 gate rows and the 64 up rows of the
//            same 64 hidden features, so one MMA per K group yields both
//            halves of SwiGLU; K = d_model.
//   down:    128 output features; K = hidden size of the group's expert.
// Roles (18 warps):
//   warp 0      producer: one 1-D bulk copy of the weight stage (128 rows x
//               128 K as INT8 holding 16 x the INT4 code, already in the
//               canonical K-major SW128 layout: expanded once at load time,
//               twice the INT4 bytes, so no warp unpacks in the hot loop) and
//               a 2-D TMA load (128B swizzle) of the 128 x 128 INT8 activation
//               tile, running ahead across tile boundaries;
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M=128, N=128,
//               K=32, INT8 x INT8 -> INT32), one instruction per 32-element
//               K group into one of 4 TMEM buffers of 128 columns, handed
//               over to the promotion warps two groups (a pair of buffers) at
//               a time;
//   warps 2-17  promotion: read each group's INT32 partials from TMEM and
//               accumulate acc = fma(float(P_j), s_j, acc) in registers
//               (4 warpgroups x 32 token columns, one weight row per thread),
//               then park the finished tile in shared memory; its epilogue
//               runs one step after each buffer pair of the next tile, while
//               the warps would otherwise wait for the MMA.  Each group is
//               one MMA that overwrites its buffer, so a pair of buffers goes
//               back to the MMA as soon as it has been read.  The weights
//               enter as 16 x their code, so a partial
//               arrives as 16 P; added as an integer to the bit pattern of
//               1.5 * 2^19 it is the float 1.5 * 2^19 + P (exact for
//               |16 P| < 2^22), and one exact subtraction converts it.
// The exact INT32 group partial is needed because every 32-element group of K
// has its own FP32 weight scale; the promotion order (j ascending, fused
// multiply-add) is the oracle's, so the FP32 result is identical to it.
// Every mbarrier wait is bounded; a wait that gives up raises the handle's
// error flag and the CTA drains and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mmoe_internal.cuh"
#include "sm100_async.cuh"

namespace mmoe {
namespace tc {

constexpr int BM = 128;                    // weight rows per tile
constexpr int BN = kTcTileRows;            // token rows per tile (128)
constexpr int BK = 128;                    // K elements (bytes of INT8) per stage
constexpr int kStages = 4;
constexpr int kBufs = 4;                   // TMEM accumulator buffers, 128 columns each
constexpr int kPairs = kBufs / 2;          // buffers are handed over two at a time
constexpr int kPromoWarpgroups = 4;        // each covers 32 token columns of all 128 weight rows
constexpr int kPromoThreads = kPromoWarpgroups * 128;
constexpr int kThreads = 64 + kPromoThreads;    // producer, MMA, promotion warps
constexpr int kCols = BN / kPromoWarpgroups;    // token columns per promotion thread

constexpr int kAI8Bytes = BM * BK;         // 16 KB: the weight stage image (INT8, SW128)
constexpr int kBBytes = BN * BK;           // 16 KB
constexpr int kStageBytes = kAI8Bytes + kBBytes;
constexpr int kXchBytes = BM * BN * 4;     // finished FP32 tile handed to the epilogue, [column][row]
constexpr long long kTimeoutClk = 4000000000ll;  // about 2 s of SM clock

enum Epi { kEpiSwiGLU = 0, kEpiCombine = 1 };

constexpr int kTInfo = 4;                  // tile-info ring entries
constexpr int kTInfoConsumers = 1 + kPromoWarpgroups * 4;  // MMA lane, promotion warps

// What every role needs to know about one tile, gathered by the producer warp
// ahead of time (tile decode, per-column data, the first two group scales).
struct TileInfo {
    int row0, nr, mb, nks, tile0, end;
    float colf[BN];      // per token column: activation scale (gate/up) or SwiGLU scale (down)
    float colg[BN];      // per token column: gate of the row (down)
    int colrow[BN];      // per token column: token id (down)
    float s01[2][BM];    // scales of groups 0 and 1, per weight row
};

struct Smem {
    // stage buffers are carved from the 1024-aligned base: [A_i8 | B] x kStages
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t accf[kPairs];   // a pair of buffers holds two finished groups
    uint64_t acce[kPairs];   // a pair of buffers has been read (free for the next MMAs)
    uint64_t tfull[kTInfo];  // tile info written
    uint64_t tempty[kTInfo]; // tile info no longer needed
    uint32_t tmem_base;
    int abort;
    TileInfo ti[kTInfo];
};

// ---------------------------------------------------------------- PTX helpers
using async::su32;
using async::mbar_init;
using async::mbar_expect_tx;
using async::mbar_arrive;
using async::mbar_try_wait;
using async::clk;
using async::bulk_load;
using async::fence_barrier_init;

// Waits for the phase of the given parity; gives up after kTimeoutClk SM
// clocks or once another thread of the CTA has given up.  On giving up it
// records `where` in the device flag (read by every later CTA, which then
// exits at once) and in the host-visible flag.  Returns false on giving up.
struct ErrFlags {
    int* dev;
    int* host;
};

__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, Smem* sm, ErrFlags err, int where) {
    const long long t0 = clk();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&sm->abort)) return false;
        if (clk() - t0 > kTimeoutClk) {
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

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(su32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(su32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major operand in the 128-byte swizzle layout: 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
    const uint64_t a = (su32(p) >> 4) & 0x3fff;
    return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// kind::i8: signed A and B, S32 accumulator, both K-major, M = 128, N = BN.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// D = A * B: a 32-element K group is exactly one instruction, so the buffer
// receives that group's partial alone and needs no clearing in between.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(0)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, int32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }


// The weights enter the MMA as 16 x their INT4 code (the code in the high nibble
// of a byte), so a group's result is v = 16 P.  Added as an integer to the bit
// pattern of 1.5 * 2^19, whose float ulp is 1/16, it gives the bits of the float
// 1.5 * 2^19 + P exactly (|16 P| < 2^22 since |P| <= 32 * 8 * 127), and one exact
// subtraction leaves P.
constexpr uint32_t kMagicBits = 0x49400000u;  // 1.5 * 2^19
constexpr float kMagic = 786432.0f;

// Two columns at once, the FP32 steps as paired instructions (each half is an
// ordinary IEEE operation, so the results equal the scalar ones):
// (a0, a1) = fma((P0, P1), s, (a0, a1)) with P = float(bits(1.5 * 2^19) + v) - 1.5 * 2^19
__device__ __forceinline__ void promote2(float& a0, float& a1, int32_t v0, int32_t v1, float s) {
    const uint32_t b0 = (uint32_t)v0 + kMagicBits, b1 = (uint32_t)v1 + kMagicBits;
    asm("{\n\t.reg .b64 t, acc, sc, mg;\n\t"
        "mov.b64 t, {%2, %3};\n\t"
        "mov.b64 acc, {%0, %1};\n\t"
        "mov.b64 mg, {%5, %5};\n\t"
        "mov.b64 sc, {%4, %4};\n\t"
        "sub.rn.f32x2 t, t, mg;\n\t"
        "fma.rn.f32x2 acc, t, sc, acc;\n\t"
        "mov.b64 {%0, %1}, acc;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "r"(b0), "r"(b1), "f"(s), "f"(kMagic));
}

// SwiGLU of one feature from its gate and up sums and the token's activation scale:
// silu(g sx) * (u sx), silu(v) = v / (1 + exp(-v)), each step an IEEE FP32 operation
__device__ __forceinline__ float swiglu(float g, float u, float sx) {
    const float gv = __fmul_rn(g, sx);
    const float uv = __fmul_rn(u, sx);
    const float silu = __fdiv_rn(gv, __fadd_rn(1.0f, expf(-gv)));
    return __fmul_rn(silu, uv);
}

struct TcArgs {
    const uint8_t* wtiles;  // weight stage images (INT8, SW128) of the expert kind (gate/up or down)
    const float* stiles;    // pre-tiled group scales
    int64_t w_expert_stride_tiles;  // stage images (of kAI8Bytes) per routed expert
    int mblocks_routed;     // weight-row blocks of a routed expert (gate/up: h/64, down: d/128)
    int mblocks_shared;
    int ks_routed;          // K stages of a routed expert (gate/up: d/128, down: h/128)
    int ks_shared;
    int fblocks;            // weight-row blocks per token tile in the launch (the larger of the two)
    int32_t* dump;          // optional INT32 partial dump
    int64_t drow0, dnrows;
};

// Bounded wait used while draining after an abort: ignores the abort flag,
// gives up only on time.
__device__ __noinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const long long t0 = clk();
    while (!mbar_try_wait(bar, parity))
        if (clk() - t0 > kTimeoutClk) return;
}

// --------------------------------------------------------------- the kernel
struct Tile {
    int g, mb, nks, nr;
    int row0;           // first row of the token tile
    bool valid;
    int tile0;          // first weight tile (index into the pre-tiled arrays)
};

// Tile L of the launch: weight-row block L % fblocks of token tile L / fblocks.
__device__ __forceinline__ Tile decode_tile(const Plan& p, const TcArgs& a, int L) {
    Tile t;
    const int fb = L % a.fblocks;
    const int ti = L / a.fblocks;
    const int code = p.tiles[ti];
    t.g = code >> 24;
    const int tin = code & 0xffffff;
    const bool shared_grp = t.g == p.E;
    const int mblocks = shared_grp ? a.mblocks_shared : a.mblocks_routed;
    t.valid = fb < mblocks;
    t.mb = fb;
    t.nks = shared_grp ? a.ks_shared : a.ks_routed;
    const int cnt = p.offsets[t.g + 1] - p.offsets[t.g];
    t.row0 = p.offsets[t.g] + tin * BN;
    t.nr = min(BN, cnt - tin * BN);
    t.tile0 = t.g * (int)a.w_expert_stride_tiles + fb * t.nks;
    return t;
}

// One lane waits, the warp follows.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Smem* sm, ErrFlags ef, int where) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, sm, ef, where);
    return __shfl_sync(0xffffffffu, ok, 0);
}

// One step of a parked tile's epilogue for one promotion warp: the warp of
// lane quarter `quarter` in the warpgroup whose token columns start at col0
// finishes columns cq .. cq + 7 (cq = col0 + 8 quarter) in kEpiSteps steps,
// reading whole columns of the exchange buffer ([column][row]) and storing
// 16 bytes per lane.
template <int kEpi>
constexpr int kEpiSteps = kEpi == kEpiSwiGLU ? kCols / 8 : kCols / 4;

template <int kEpi>
__device__ __forceinline__ void epilogue_step(const Plan& p, const TileInfo& ti, const float* xch, int col0,
                                              int quarter, int lane, int step) {
    const int cq = col0 + quarter * (kCols / 4);
    const int nr = ti.nr, mb = ti.mb;
    const int64_t row0 = ti.row0;
    if (kEpi == kEpiSwiGLU) {
        // rows 0..63 hold the gate of feature mb*64 + row, rows 64..127 the up of the same feature;
        // lanes 0-15 take column cq + 2 step, lanes 16-31 the next, each lane features 4 (lane & 15) .. + 3
        const int fl4 = 4 * (lane & 15);
        const int cc = cq + 2 * step + (lane >> 4);
        if (cc >= nr) return;
        const float sx = ti.colf[cc];
        const float4 g4 = *reinterpret_cast<const float4*>(&xch[cc * BM + fl4]);
        const float4 u4 = *reinterpret_cast<const float4*>(&xch[cc * BM + 64 + fl4]);
        // (gate, up) pairs times the activation scale; the requantisation pass applies the SwiGLU
        float4* out = reinterpret_cast<float4*>(p.act + ((row0 + cc) * p.hmax + mb * 64 + fl4) * 2);
        out[0] = make_float4(__fmul_rn(g4.x, sx), __fmul_rn(u4.x, sx), __fmul_rn(g4.y, sx), __fmul_rn(u4.y, sx));
        out[1] = make_float4(__fmul_rn(g4.z, sx), __fmul_rn(u4.z, sx), __fmul_rn(g4.w, sx), __fmul_rn(u4.w, sx));
    } else {
        // column cq + step; lane l covers outputs mb*128 + 4 l .. + 3
        const int cc = cq + step;
        if (cc >= nr) return;
        const int m4 = mb * BM + 4 * lane;
        const float f = ti.colf[cc];
        const float4 v = *reinterpret_cast<const float4*>(&xch[cc * BM + 4 * lane]);
        const float4 o = make_float4(__fmul_rn(v.x, f), __fmul_rn(v.y, f), __fmul_rn(v.z, f), __fmul_rn(v.w, f));
        if (p.deterministic) {
            *reinterpret_cast<float4*>(p.obuf + (row0 + cc) * p.d + m4) = o;
        } else {
            const float g = ti.colg[cc];
            float* yr = p.y + (int64_t)ti.colrow[cc] * p.d + m4;
            atomicAdd(yr, __fmul_rn(g, o.x));
            atomicAdd(yr + 1, __fmul_rn(g, o.y));
            atomicAdd(yr + 2, __fmul_rn(g, o.z));
            atomicAdd(yr + 3, __fmul_rn(g, o.w));
        }
    }
}

template <int kEpi, bool kDump>
// 18 warps: the SM sub-partitions holding 5 of them bound a thread to 96 registers
__global__ void __launch_bounds__(kThreads, 1)
expert_gemm_tc_kernel(const __grid_constant__ CUtensorMap bmap, Plan p, TcArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = base;
    float* xch = reinterpret_cast<float*>(base + kStages * kStageBytes);
    Smem* sm = reinterpret_cast<Smem*>(base + kStages * kStageBytes + kXchBytes);

    // nothing to do after an earlier wait gave up
    if (p.err && *reinterpret_cast<volatile int*>(p.err)) return;
    const int total = (*p.tile_count) * a.fblocks;
    if ((int)blockIdx.x >= total) return;
    const ErrFlags ef{p.err, p.err_host};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < kPairs; ++b) {
            mbar_init(&sm->accf[b], 1);
            mbar_init(&sm->acce[b], kPromoThreads / 32);
        }
        for (int b = 0; b < kTInfo; ++b) {
            mbar_init(&sm->tfull[b], 32);
            mbar_init(&sm->tempty[b], kTInfoConsumers);
        }
        sm->abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&sm->tmem_base)),
                     "r"(kBufs * 128)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_before_sync();
    }
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = sm->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (whole warp)
        int sc = 0, tcount = 0;
        bool ok = true;
        for (int L = blockIdx.x; ok; L += gridDim.x) {
            Tile t{};
            const bool last = L >= total;  // past the last tile: publish the end marker and stop
            if (!last) {
                if (lane == 0) t = decode_tile(p, a, L);
                t.valid = __shfl_sync(0xffffffffu, t.valid, 0);
                if (!t.valid) continue;
                t.mb = __shfl_sync(0xffffffffu, t.mb, 0);
                t.nks = __shfl_sync(0xffffffffu, t.nks, 0);
                t.nr = __shfl_sync(0xffffffffu, t.nr, 0);
                t.row0 = __shfl_sync(0xffffffffu, t.row0, 0);
                t.tile0 = __shfl_sync(0xffffffffu, t.tile0, 0);
            }
            // publish the tile's information (or the end marker)
            const int b = tcount % kTInfo;
            if (tcount >= kTInfo && !warp_wait(&sm->tempty[b], ((tcount / kTInfo) - 1) & 1, sm, ef, 6)) { ok = false; break; }
            TileInfo& ti = sm->ti[b];
            if (lane == 0) {
                ti.end = last ? 1 : 0;
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
                const float* sp = a.stiles + (size_t)t.tile0 * (BK / kGroup) * BM;
                for (int r = lane; r < 2 * BM; r += 32) ti.s01[r / BM][r % BM] = __ldg(sp + r);
            }
            mbar_arrive(&sm->tfull[b]);
            ++tcount;
            if (last) break;
            // the tile's stages
            if (lane == 0) {
                for (int ks = 0; ks < t.nks; ++ks, ++sc) {
                    const int s = sc % kStages;
                    if (sc >= kStages && !mbar_wait(&sm->empty[s], ((sc / kStages) - 1) & 1, sm, ef, 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = stages + s * kStageBytes;
                    mbar_expect_tx(&sm->full[s], kAI8Bytes + kBBytes);
                    bulk_load(st, a.wtiles + ((int64_t)t.tile0 + ks) * kAI8Bytes, kAI8Bytes, &sm->full[s]);
                    tma_load_2d(st + kAI8Bytes, &bmap, ks * BK, t.row0, &sm->full[s]);
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
            while (ok) {
                const int tb = tcount % kTInfo;
                if (!mbar_wait(&sm->tfull[tb], (tcount / kTInfo) & 1, sm, ef, 7)) break;
                const int nks = sm->ti[tb].nks, end = sm->ti[tb].end;
                mbar_arrive(&sm->tempty[tb]);
                ++tcount;
                if (end) break;
                for (int ks = 0; ks < nks && ok; ++ks, ++sc) {
                    const int s = sc % kStages;
                    if (!mbar_wait(&sm->full[s], (sc / kStages) & 1, sm, ef, 2)) { ok = false; break; }
                    tc_after_sync();
                    uint8_t* st = stages + s * kStageBytes;
                    const uint64_t ad = smem_desc_sw128(st);
                    const uint64_t bd = smem_desc_sw128(st + kAI8Bytes);
#pragma unroll
                    for (int pp = 0; pp < (BK / kGroup) / 2; ++pp, ++pc) {
                        const int b = pc & 1;
                        if (!mbar_wait(&sm->acce[b], (pc >> 1) & 1, sm, ef, 3)) { ok = false; break; }
                        tc_after_sync();
#pragma unroll
                        for (int gg = 0; gg < 2; ++gg) {
                            const int jj = pp * 2 + gg;
                            mma_i8(tmem + (2 * b + gg) * 128, ad + (uint64_t)(jj * 2), bd + (uint64_t)(jj * 2));
                        }
                        mma_commit(&sm->accf[b]);
                    }
                    mma_commit(&sm->empty[s]);
                }
            }
            // every MMA issued has completed before TMEM is released
            if (pc > 0) mbar_wait_drain(&sm->accf[(pc - 1) & 1], ((pc - 1) >> 1) & 1);
        }
    } else {
        // ------------------------------------------------------------ promotion + epilogue
        const int pw = warp - 2;            // 0..15
        const int wg = pw >> 2;             // token-column quarter
        const int quarter = warp & 3;       // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;  // weight row of this thread (0..127)
        const int col0 = wg * kCols;
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)col0;
        // every buffer starts free: completion 0 of both acce barriers
        if (lane == 0)
            for (int b = 0; b < kPairs; ++b) mbar_arrive(&sm->acce[b]);
        int pc = 0, tcount = 0;
        int ptb = -1, pstep = 0;  // tile-info slot of the parked tile whose epilogue is pending, next step
        bool ok = true;
        while (ok) {
            const int tb = tcount % kTInfo;
            if (!warp_wait(&sm->tfull[tb], (tcount / kTInfo) & 1, sm, ef, 9)) break;
            const TileInfo& ti = sm->ti[tb];
            if (ti.end) break;
            const int nks = ti.nks, nr = ti.nr, mb = ti.mb, row0 = ti.row0;
            const float* sp = a.stiles + (size_t)ti.tile0 * (BK / kGroup) * BM + row;
            float acc[kCols];
#pragma unroll
            for (int c = 0; c < kCols; ++c) acc[c] = 0.0f;
            const int ng = nks * (BK / kGroup);
            float s0 = ti.s01[0][row], s1 = ti.s01[1][row];
            for (int j = 0; j < ng; j += 2, ++pc) {
                const int b = pc & 1;
                const float sa = s0, sb = s1;
                if (j + 2 < ng) {
                    s0 = __ldg(sp + (j + 2) * BM);
                    s1 = __ldg(sp + (j + 3) * BM);
                }
                if (!warp_wait(&sm->accf[b], (pc >> 1) & 1, sm, ef, 5)) { ok = false; break; }
                tc_after_sync();
                // both halves of a group leave TMEM behind one wait; the pair goes back to the MMA
                // as soon as its second group has been read, before that group's arithmetic
#pragma unroll 1
                for (int gg = 0; gg < 2; ++gg) {
                    const float sc = gg ? sb : sa;
                    const uint32_t ta = tl + (2 * b + gg) * 128;
                    int32_t v[16], w[16];
                    tmem_ld16(ta, v);
                    tmem_ld16(ta + 16, w);
                    tmem_wait_ld();
                    if (gg == 1) {
                        tc_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm->acce[b]);
                    }
#pragma unroll
                    for (int c = 0; c < 16; c += 2) promote2(acc[c], acc[c + 1], v[c], v[c + 1], sc);
#pragma unroll
                    for (int c = 0; c < 16; c += 2) promote2(acc[16 + c], acc[17 + c], w[c], w[c + 1], sc);
                    if (kDump) {
                        // INT32 partials of rows [drow0, drow0 + dnrows) for the inspection entry point
                        const int jg = j + gg;
#pragma unroll
                        for (int c = 0; c < kCols; ++c) {
                            const int cc = col0 + c;
                            const int64_t grow = (int64_t)row0 + cc;
                            if (cc >= nr || grow < a.drow0 || grow >= a.drow0 + a.dnrows) continue;
                            const int32_t pv = (c < 16 ? v[c & 15] : w[c & 15]) >> 4;
                            if (kEpi == kEpiSwiGLU) {
                                const int f = mb * 64 + (row & 63);
                                const int n = row < 64 ? f : p.hmax + f;
                                a.dump[((grow - a.drow0) * 2 * p.hmax + n) * (p.d / kGroup) + jg] = pv;
                            } else {
                                const int m = mb * BM + row;
                                a.dump[((grow - a.drow0) * p.d + m) * (p.hmax / kGroup) + jg] = pv;
                            }
                        }
                    }
                }
                // one step of the previous tile's epilogue while the MMAs of the next pair run
                if (!kDump && ptb >= 0) {
                    epilogue_step<kEpi>(p, sm->ti[ptb], xch, col0, quarter, lane, pstep);
                    if (++pstep == kEpiSteps<kEpi>) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm->tempty[ptb]);
                        ptb = -1;
                    }
                }
            }
            if (!ok || *reinterpret_cast<volatile int*>(&sm->abort)) break;
            // the rest of the previous tile's epilogue (a K loop shorter than its steps)
            if (ptb >= 0) {
                for (; pstep < kEpiSteps<kEpi>; ++pstep) epilogue_step<kEpi>(p, sm->ti[ptb], xch, col0, quarter, lane, pstep);
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->tempty[ptb]);
                ptb = -1;
            }
            // park the tile in shared memory ([column][row]); its epilogue runs during the next tile's pairs
            const int named = 1 + wg;
            asm volatile("bar.sync %0, %1;" ::"r"(named), "r"(128) : "memory");  // previous tile's readers are done
#pragma unroll
            for (int c = 0; c < kCols; ++c) xch[(col0 + c) * BM + row] = acc[c];
            asm volatile("bar.sync %0, %1;" ::"r"(named), "r"(128) : "memory");
            if (kDump) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->tempty[tb]);
            } else {
                ptb = tb;
                pstep = 0;
            }
            ++tcount;
        }
        // the last parked tile's epilogue
        if (ok && ptb >= 0 && !*reinterpret_cast<volatile int*>(&sm->abort))
            for (; pstep < kEpiSteps<kEpi>; ++pstep) epilogue_step<kEpi>(p, sm->ti[ptb], xch, col0, quarter, lane, pstep);
    }

    __syncthreads();
    if (warp == 1) {
        tc_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kBufs * 128) : "memory");
    }
}

// --------------------------------------------------------------- weight re-tiling (load time)
// gate/up stage (g, fb, ks): 128 rows x 128 K; rows 0..63 are gate rows fb*64 .. fb*64+63, rows 64..127 the up
// rows of the same features; down stage (g, mb, ks): output rows mb*128 ..  Each row holds K values
// ks*128 .. ks*128+127 as bytes 16 x code, its 16-byte chunk c stored at chunk c ^ (row & 7) (the 128-byte
// swizzle the MMA's shared-memory descriptor expects at a 1024-byte aligned stage).  Scales (g, fb, j): 128
// floats, one per stage row.

// 8 nibbles (K order, low nibble first) -> 8 bytes 16 x code: (K 0..3), (K 4..7)
__device__ __forceinline__ void expand_nibbles(uint32_t v, uint32_t& a, uint32_t& b) {
    a = b = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        a |= ((v >> (4 * i)) & 15u) << (8 * i + 4);
        b |= ((v >> (4 * (i + 4))) & 15u) << (8 * i + 4);
    }
}

// one thread per 16-byte chunk of packed codes (32 K values) of a stage row
__global__ void retile_weights_kernel(const uint8_t* __restrict__ src, const float* __restrict__ ssrc,
                                      uint8_t* __restrict__ dst, float* __restrict__ sdst, int E, int K_routed,
                                      int K_shared, int rows_routed, int rows_shared, int gate_up, int h, int hs,
                                      int64_t total_chunks)
{
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= total_chunks) return;
    // q -> (expert, stage, row, chunk)
    const int64_t per_routed = (int64_t)rows_routed / BM * (K_routed / BK) * BM * 4;  // chunks of a routed expert
    int g;
    int64_t r;
    if (q < per_routed * E) { g = (int)(q / per_routed); r = q % per_routed; }
    else { g = E; r = q - per_routed * E; }
    const int K = g < E ? K_routed : K_shared;
    const int nks = K / BK;
    const int chunk = (int)(r % 4);
    const int trow = (int)((r / 4) % BM);
    const int64_t tile = r / (4 * BM);  // mb * nks + ks
    const int ks = (int)(tile % nks);
    const int mb = (int)(tile / nks);
    const int hid = g < E ? h : hs;
    int64_t srow;  // row inside the expert's interchange block
    if (gate_up) srow = trow < 64 ? (int64_t)mb * 64 + trow : (int64_t)hid + mb * 64 + (trow - 64);
    else srow = (int64_t)mb * BM + trow;
    // interchange block of expert g starts at g * (routed block size)
    const int64_t src_rows_routed = gate_up ? 2 * (int64_t)h : (int64_t)rows_routed;
    const int64_t src_row_bytes = K / 2;
    const int64_t src_expert_bytes = src_rows_routed * ((int64_t)K_routed / 2);
    const uint8_t* s = src + (int64_t)g * src_expert_bytes + srow * src_row_bytes + (int64_t)ks * 64 + chunk * 16;
    const uint4 w = *reinterpret_cast<const uint4*>(s);
    uint4 o0, o1;  // K 32 chunk + 0..15 and 16..31
    expand_nibbles(w.x, o0.x, o0.y);
    expand_nibbles(w.y, o0.z, o0.w);
    expand_nibbles(w.z, o1.x, o1.y);
    expand_nibbles(w.w, o1.z, o1.w);
    const int64_t dst_tiles_routed = (int64_t)rows_routed / BM * (K_routed / BK);
    const int64_t dtile = (int64_t)g * dst_tiles_routed + tile;
    uint4* row = reinterpret_cast<uint4*>(dst + dtile * kAI8Bytes + trow * 128);
    row[(2 * chunk) ^ (trow & 7)] = o0;
    row[(2 * chunk + 1) ^ (trow & 7)] = o1;
    // scale of group (ks*4 + chunk) of this row
    const int64_t src_expert_scales = src_rows_routed * ((int64_t)K_routed / kGroup);
    const float sc = ssrc[(int64_t)g * src_expert_scales + srow * (K / kGroup) + ks * 4 + chunk];
    sdst[(dtile * 4 + chunk) * BM + trow] = sc;
}

}  // namespace tc

// ------------------------------------------------------------------ host side
bool tc_supported(int d, int h, int hs) { return d % 128 == 0 && h % 128 == 0 && hs % 128 == 0; }

size_t tc_smem_bytes() { return 1024 + tc::kStages * tc::kStageBytes + tc::kXchBytes + sizeof(tc::Smem); }
static_assert(1024 + tc::kStages * tc::kStageBytes + tc::kXchBytes + sizeof(tc::Smem) <= 232448, "shared memory");

cudaError_t launch_retile(const uint8_t* gu, const float* sgu, const uint8_t* dn, const float* sdn, uint8_t* gu_t,
                          float* sgu_t, uint8_t* dn_t, float* sdn_t, int d, int h, int hs, int E, cudaStream_t s) {
    // gate/up: rows of a tile are 128 (64 features x 2); "rows" counted as 2*hid
    const int64_t gu_chunks = ((int64_t)E * (2 * h / tc::BM) + (2 * hs / tc::BM)) * (d / tc::BK) * tc::BM * 4;
    tc::retile_weights_kernel<<<(unsigned)((gu_chunks + 255) / 256), 256, 0, s>>>(gu, sgu, gu_t, sgu_t, E, d, d, 2 * h,
                                                                                   2 * hs, 1, h, hs, gu_chunks);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t dn_chunks = ((int64_t)E * (h / tc::BK) + (hs / tc::BK)) * (d / tc::BM) * tc::BM * 4;
    tc::retile_weights_kernel<<<(unsigned)((dn_chunks + 255) / 256), 256, 0, s>>>(dn, sdn, dn_t, sdn_t, E, h, hs, d, d,
                                                                                   0, h, hs, dn_chunks);
    return cudaGetLastError();
}

size_t tensor_map_bytes() { return sizeof(CUtensorMap); }

cudaError_t make_tensor_map(void* map_, void* base, uint64_t inner_elems, uint64_t rows, uint64_t row_stride_bytes,
                            int elem_bytes) {
    CUtensorMap* map = static_cast<CUtensorMap*>(map_);
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (elem_bytes != 1 && elem_bytes != 2) return cudaErrorInvalidValue;
    // boxes of 128 bytes (one swizzle row) x 128 rows
    const cuuint64_t dims[2] = {inner_elems, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), 128u};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base,
                        dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

static int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            n = 148;
    }
    return n;
}

template <int kEpi, bool kDump>
static cudaError_t launch_tc(const Plan& p, cudaStream_t s, const CUtensorMap* map, tc::TcArgs a, int fblocks) {
    auto kern = tc::expert_gemm_tc_kernel<kEpi, kDump>;
    const size_t smem = tc_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    a.fblocks = fblocks;
    // persistent: one CTA per SM (never more CTAs than the largest possible tile count)
    const int64_t upper = p.max_tiles * (int64_t)fblocks;
    const unsigned grid = (unsigned)(upper < sm_count() ? upper : sm_count());
    kern<<<grid, tc::kThreads, smem, s>>>(*map, p, a);
    return cudaGetLastError();
}

cudaError_t launch_gate_up_tc(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    if (p.T == 0) return cudaSuccess;
    tc::TcArgs a{};
    a.wtiles = p.w_gate_up_t;
    a.stiles = p.s_gate_up_t;
    a.mblocks_routed = p.h / 64;
    a.mblocks_shared = p.hs / 64;
    a.ks_routed = a.ks_shared = p.d / tc::BK;
    a.w_expert_stride_tiles = (int64_t)a.mblocks_routed * a.ks_routed;
    a.dump = dump;
    a.drow0 = row0;
    a.dnrows = nrows;
    const int gx = p.hmax / 64;
    const CUtensorMap* map = static_cast<const CUtensorMap*>(p.tmap_xq);
    return dump ? launch_tc<tc::kEpiSwiGLU, true>(p, s, map, a, gx)
                : launch_tc<tc::kEpiSwiGLU, false>(p, s, map, a, gx);
}

cudaError_t launch_down_tc(const Plan& p, cudaStream_t s, int32_t* dump, int64_t row0, int64_t nrows) {
    if (p.T == 0) return cudaSuccess;
    tc::TcArgs a{};
    a.wtiles = p.w_down_t;
    a.stiles = p.s_down_t;
    a.mblocks_routed = a.mblocks_shared = p.d / tc::BM;
    a.ks_routed = p.h / tc::BK;
    a.ks_shared = p.hs / tc::BK;
    a.w_expert_stride_tiles = (int64_t)a.mblocks_routed * a.ks_routed;
    a.dump = dump;
    a.drow0 = row0;
    a.dnrows = nrows;
    const int gx = p.d / tc::BM;
    const CUtensorMap* map = static_cast<const CUtensorMap*>(p.tmap_hq);
    return dump ? launch_tc<tc::kEpiCombine, true>(p, s, map, a, gx)
                : launch_tc<tc::kEpiCombine, false>(p, s, map, a, gx);
}

}  // namespace mmoe
