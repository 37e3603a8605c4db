// Compress step on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…", section "TurboQuant" steps 1-4
// (normalize, rotate by R^T, Gaussian Lloyd-Max, pack nibbles + fp32 norm) and
// section "注意力计算的特殊挑战与QJL校正" (keys: sign(S r), gamma = ||r||);
// [TQ-RS] "TurboQuant : compresser le KV-cache…", "Couche 1" (randomized
// Walsh-Hadamard rotation).
//
// 2-CTA clusters (one CTA per SM) walk 256-vector tiles of the flattened
// [T*Hkv, 128] input, 128 rows per CTA; every MMA is a cta_group::2 pair issued
// by the even CTA (M = 256, each CTA holding its own x rows and half of the
// operand image rows, each CTA's tensor memory receiving its own 128 rows):
//   warps 0..4n-1  epilogue, n teams of four warps (one per TMEM lane quarter,
//                  one thread per row); team t takes the cluster's tiles k with
//                  k % n == t in TMEM buffer t, so one team's waits overlap the
//                  other teams' arithmetic (values n = 4, keys n = 3)
//   warp 4n        TMA producer: this CTA's 128 x 128 fp16 rows of the tile
//   warp 4n+1      TMEM owner; even CTA: rotation issuer; odd CTA: forwards its
//                  stage-full and operands-ready events to the even CTA
//   warp 4n+2      keys, even CTA: sketch issuer (a second issuing thread)
// Rotation: D[v][n] = sum_k x[v][k] B[n][k] with B the rotation split into
// fp16 parts held in shared memory for the whole kernel:
//   Haar      B = 16 R^T = hi + lo (two passes, x is exact in fp16, products are
//             exact, fp32 accumulation, the small lo pass first)  -> acc = 16 y
//   Hadamard  B = H D (entries +-1, exact, one pass)  -> acc = sqrt(d) y
// Values: ||x|| comes from the fp16 tile in shared memory (exact squares, fp32
// sums), read while the rotation runs; the codes only need acc within the 1e-6
// window.  Keys: ||x|| = ||acc|| / (acc / y) from the accumulator itself.
// In both cases v = sqrt(d) y / ||x||; the epilogue works in cell units u = v * scale of a shared-memory
// table of uniform cells (each holds at most one boundary): round(u) addresses
// the cell, one fp32 compare with its boundary gives the code (values: of
// u - round(u) with the boundary's offset in the cell, from one 4-byte read;
// keys: of u with the boundary, from one 16-byte read that also holds the levels).
// Keys (prod mode): the residual d = u - c[code] (cell units) gives
// gamma = ||x - x_hat|| and rho = 32 (v - c[code]), and the sign sketch
//   S (x - x_hat) = (S R) (y - y_hat)
// is a second contraction whose A operand rho (split into fp16 hi + lo) the
// epilogue writes back into tensor memory over the accumulator columns it has
// just read; the sketches, in tile order, share one accumulator:
//   Haar      acc2 = rho_lo M_hi + rho_hi M_lo + rho_hi M_hi   (M = S R)
//   Hadamard  acc2 = (rho_lo + rho_hi) M',   M' = S D H integer, exact in fp16
// sign bit j = [acc2_j >= 0].  Every wait is bounded (TQ_DEVERR_TIMEOUT).
#include <atomic>
#include <cmath>

#include <cuda.h>

#include "device_util.cuh"
#include "sm100.cuh"
#include "tc_params.h"

namespace tq {
namespace {

using namespace sm100;

constexpr int kTeamWarps = 4;  // one per TMEM lane quarter, one thread per row
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 fp16 operand
constexpr uint32_t kHalf = kTile / 2;      // one 128-byte-swizzled K-half
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kSmemMax = 232448;

// TMEM (512 columns): buffer t (columns [128 t, 128 t + 128)) holds team t's tile.
// Values: four teams, each buffer a rotation accumulator.  Keys: three teams; the
// buffer holds the rotation accumulator, then rho: the 16 coordinates of K-step st
// (columns [16 st, 16 st + 16)) become 8 columns of rho_hi pairs followed by 8 of
// rho_lo pairs, written by the thread that has just read those columns.  The
// sketches, issued in tile order, share the accumulator at column kColSketch.
constexpr uint32_t kColSketch = 384;

template <int ROT, bool PROD, bool PAIR>
struct Cfg {
    static constexpr int kRotImages = ROT == 0 ? 2 : 1;
    static constexpr int kQjlImages = PROD ? (ROT == 0 ? 2 : 1) : 0;
    static constexpr int kImages = kRotImages + kQjlImages;
    // this CTA's part of an operand image: all 128 rows, or (pair) 64 of them
    static constexpr uint32_t kImgBytes = PAIR ? kTile / 2 : kTile;
    static constexpr uint32_t kImgHalf = kImgBytes / 2;  // K-half stride inside an image
    static constexpr int kLutBytes = PROD ? kLutBytesProd : kLutBytesMse;
    static constexpr uint32_t kPartBytes = 0;
    static constexpr uint32_t kBarBytes = 512;
    static constexpr uint32_t kFixed = kImages * kImgBytes + kLutBytes + kPartBytes + kBarBytes;
    static constexpr int kStagesFit = (int)((kSmemMax - kFixed) / kTile);
    static constexpr int kStages = kStagesFit > 4 ? 4 : kStagesFit;
    static constexpr uint32_t kOffImg = 0;
    static constexpr uint32_t kOffX = kOffImg + kImages * kImgBytes;
    static constexpr uint32_t kOffLut = kOffX + kStages * kTile;
    static constexpr uint32_t kOffPart = kOffLut + kLutBytes;
    static constexpr uint32_t kOffBar = kOffPart + kPartBytes;
    static constexpr uint32_t kSmem = kOffBar + kBarBytes;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kTeams = PROD ? 3 : 4;
    static constexpr int kEpiWarps = 4 * kTeams;
    static constexpr int kWarpProducer = kEpiWarps;
    static constexpr int kWarpMma = kEpiWarps + 1;     // rotations
    static constexpr int kWarpSketch = kEpiWarps + 2;  // keys: the sketches, from a second thread
    static constexpr int kThreads = kEpiWarps * 32 + (PROD ? 96 : 64);
    // registers: warps get them in fours (one per SM sub-partition), so keys (15 warps)
    // run at up to 128 and values (18 warps) at up to 112
    static constexpr int kBound = kThreads;
    static constexpr uint32_t kBufCols = 128;
    static_assert(kStages >= 1, "shared memory budget");
    static_assert(kSmem <= kSmemMax, "shared memory budget");
};

// barrier indices
enum : int {
    kBarConst = 0,
    kBarXFull = 1,     // +stage (4)
    kBarXEmpty = 5,    // +stage (4)
    kBarRotFull = 9,    // +team (4): rotation accumulator ready
    kBarRotEmpty = 13,  // +team (4): the team is done with its buffer
    kBarRhoFull = 17,   // +team (3): rho written (keys)
    kBarQjlFull = 20,   // +team (3): sketch ready (keys)
    kBarSketchEmpty = 23,  // the sketch accumulator has been read (keys)
    kBarDrain = 24,      // +issuer (2): the issuer's MMAs are complete
    kBarPeerConst = 26,  // pair: the odd CTA's operand images are in (arrived from it)
    kNumBars = 27
};

struct TcArgs {
    const int32_t* slots;
    uint8_t* cache;
    int N;  // rows = T * H
    int H;
    int num_blocks;
    const uint8_t* images;  // kImages pre-swizzled 32 KB operands
    const uint8_t* lut;     // bucketize table
    ChunkLayout lay;
    float lut_kscale;  // keys: sqrt(d) * table scale, u = acc * lut_kscale / ||acc|| is v in cell units
    float lut_xscale;  // values: sqrt(d) * table scale / (acc / y), u = acc * lut_xscale / ||x||
    float lut_magic;   // 1.5 * 2^23 + cells / 2
    float rho_scale;   // 32 / table scale: rho = 32 (v - c) from the cell-unit residual
    float n_scale;     // ||x|| = n_scale * ||acc||
    float gamma_scale; // n_scale / (sqrt(d) * table scale): gamma = ||d|| ||acc|| gamma_scale
    uint32_t* err;
    int stall;         // test hook: load no x tile (every wait for one runs out)
};

__device__ __forceinline__ void set_abort(volatile int* abort, uint32_t* err) {
    *abort = 1;
    atomicOr(err, TQ_DEVERR_TIMEOUT);
}

// 1/sqrt(x) for finite x > 0: the hardware estimate and one Newton step
// r' = r + r (1 - x r^2) / 2, within about an ulp.
__device__ __forceinline__ float rsqrt_refined(float x) {
    const float r = rsqrtf(x);
    const float e = fmaf(-x * r, r, 1.0f);
    return fmaf(0.5f * r, e, r);
}

// A read-only global load that stays where it is written (not sunk to its use).
__device__ __forceinline__ int ldg_early(const int32_t* p) {
    int v;
    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Table reads at a 32-bit shared-memory address.
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t x;
    asm("ld.shared.u32 %0, [%1];" : "=r"(x) : "r"(addr));
    return x;
}
__device__ __forceinline__ void lds_v4(uint32_t addr, uint32_t& x, uint32_t& y, uint32_t& z, uint32_t& w) {
    asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(x), "=r"(y), "=r"(z), "=r"(w) : "r"(addr));
}
// in program order with the other volatile accesses (bounds how far loads are hoisted)
__device__ __forceinline__ void lds_v4_ordered(uint32_t addr, uint32_t& x, uint32_t& y, uint32_t& z, uint32_t& w) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(x), "=r"(y), "=r"(z), "=r"(w) : "r"(addr));
}

// s0 += lo^2, s1 += hi^2 for the two fp16 halves of w (exact squares, fp32 sums).
__device__ __forceinline__ void sq_acc2(uint32_t w, float& s0, float& s1) {
    asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "fma.rn.f32.f16 %0, a, a, %0;\n\tfma.rn.f32.f16 %1, b, b, %1;\n\t}"
        : "+f"(s0), "+f"(s1)
        : "r"(w));
}

template <int ROT, bool PROD, int W, bool PAIR>
__global__ void __launch_bounds__(Cfg<ROT, PROD, PAIR>::kBound, 1) compress_tc_kernel(const __grid_constant__ CUtensorMap tmap, TcArgs a) {
    using C = Cfg<ROT, PROD, PAIR>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (sbase & 1023u) {  // the swizzled operands need 1024-byte alignment
        if (threadIdx.x == 0) atomicOr(a.err, TQ_DEVERR_INTERNAL);
        return;
    }
    const uint32_t bars = sbase + C::kOffBar;
    auto bar = [&](int i) -> uint32_t { return bars + 8u * (uint32_t)i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffBar + 8 * kNumBars);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffBar + 8 * kNumBars + 4);
    // Tiles: 128 rows per CTA, or (pair) 256 rows per 2-CTA cluster, the even CTA taking
    // the first 128; worker u (CTA or cluster) takes tiles u, u + workers, ...
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool lead = rank == 0;
    const int workers = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
    const int uid = PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x;
    constexpr int kTileRows = PAIR ? 256 : 128;
    const int ntiles = (a.N + kTileRows - 1) / kTileRows;
    const int my_tiles = uid < ntiles ? (ntiles - 1 - uid) / workers + 1 : 0;
    auto row0_of = [&](int k) -> int { return (uid + k * workers) * kTileRows + (int)rank * 128; };
    // barriers that the odd CTA of a pair also arrives on count both CTAs' arrivals
    constexpr int kBoth = PAIR ? 2 : 1;

    if (threadIdx.x == 0) {
        mbar_init(bar(kBarConst), 1);
        for (int s = 0; s < C::kStages; ++s) {
            // pair: the even CTA's stage is full once its own copy landed and the odd CTA
            // has reported its copy (an arrival forwarded by its MMA warp)
            mbar_init(bar(kBarXFull + s), PAIR && lead ? 2 : 1);
            // released by the rotation MMAs and, for values, by the team that reads ||x||
            mbar_init(bar(kBarXEmpty + s), PROD ? 1 : 1 + kTeamWarps);
        }
        for (int t = 0; t < C::kTeams; ++t) {
            mbar_init(bar(kBarRotFull + t), 1);
            mbar_init(bar(kBarRotEmpty + t), kBoth * kTeamWarps);
            if (PROD) {
                mbar_init(bar(kBarRhoFull + t), kBoth * kTeamWarps);
                mbar_init(bar(kBarQjlFull + t), 1);
            }
        }
        mbar_init(bar(kBarSketchEmpty), kBoth * kTeamWarps);
        mbar_init(bar(kBarDrain), 1);
        mbar_init(bar(kBarDrain + 1), 1);
        mbar_init(bar(kBarPeerConst), 1);
        *abort = 0;
        fence_mbar_init();
        // the operand images (pair: this CTA's 64 rows of each K-half) and the table (set
        // up by tq_init, not by the kernel before)
        mbar_arrive_expect_tx(bar(kBarConst), C::kImages * C::kImgBytes + C::kLutBytes);
        for (int i = 0; i < C::kImages; ++i)
            for (int h = 0; h < 2; ++h)
                bulk_g2s(sbase + C::kOffImg + i * C::kImgBytes + h * C::kImgHalf,
                         a.images + (size_t)i * kTile + h * kHalf + rank * C::kImgHalf, C::kImgHalf, bar(kBarConst));
        bulk_g2s(sbase + C::kOffLut, a.lut, C::kLutBytes, bar(kBarConst));
    }
    if (warp == C::kWarpMma) {
        if (PAIR) {
            tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();  // both CTAs' barriers are initialised before either signals the other
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();  // the inputs, the slot mapping and the cache may come from the kernel before
    griddep_launch_dependents();

    if (warp == C::kWarpProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            const int to_load = a.stall ? 0 : my_tiles;
            for (int k = 0; k < to_load; ++k) {
                const int s = k % C::kStages;
                const uint32_t ph = (uint32_t)(k / C::kStages) & 1u;
                if (!mbar_wait(bar(kBarXEmpty + s), ph ^ 1u, abort, kWaitNs)) {
                    set_abort(abort, a.err);
                    break;
                }
                const int row0 = row0_of(k);
                mbar_arrive_expect_tx(bar(kBarXFull + s), kTile);
                tma_load_2d(sbase + C::kOffX + s * kTile, &tmap, 0, row0, bar(kBarXFull + s));
                tma_load_2d(sbase + C::kOffX + s * kTile + kHalf, &tmap, 64, row0, bar(kBarXFull + s));
                ++issued;
            }
            // every copy this CTA started lands before the CTA can exit
            const volatile int never = 0;
            mbar_wait(bar(kBarConst), 0, &never, kWaitNs);
            for (int k = issued - C::kStages < 0 ? 0 : issued - C::kStages; k < issued; ++k)
                mbar_wait(bar(kBarXFull + k % C::kStages), (uint32_t)(k / C::kStages) & 1u, &never, kWaitNs);
        }
        __syncwarp();
    } else if (warp == C::kWarpMma && PAIR && !lead) {
        // ------------------------------------------------------------ odd CTA of a pair
        // Forwards to the even CTA that this CTA's operand images are in and, stage by
        // stage, that the x tile it loaded is full.
        if (lane == 0) {
            bool ok = mbar_wait(bar(kBarConst), 0, abort, kWaitNs);
            if (ok) mbar_arrive_remote(bar(kBarPeerConst), 0);
            for (int k = 0; ok && k < my_tiles; ++k) {
                const int s = k % C::kStages;
                ok = mbar_wait(bar(kBarXFull + s), (uint32_t)(k / C::kStages) & 1u, abort, kWaitNs);
                if (ok) mbar_arrive_remote(bar(kBarXFull + s), 0);
            }
            if (!ok) set_abort(abort, a.err);
        }
        __syncwarp();
    } else if ((warp == C::kWarpMma || (PROD && warp == C::kWarpSketch)) && (!PAIR || lead)) {
        // ------------------------------------------------------------ MMA issuers
        // Rotations from one thread, the keys' sketches from another (on another SM
        // sub-partition), so that neither waits for the other's MMA issue.
        const bool rot_issuer = warp == C::kWarpMma;
        if (lane == 0) {
            // pair: M = 256 (each CTA's 128 rows of x), each CTA holding 64 of the image rows
            const uint32_t idesc = idesc_f16(PAIR ? 256 : 128, 128);
            // barriers that the odd CTA also arrives on are tested at cluster scope
            auto test = [](uint32_t b, uint32_t parity) -> bool {
                return PAIR ? mbar_test_wait_cluster(b, parity) : mbar_test_wait(b, parity);
            };
            bool ok = mbar_wait(bar(kBarConst), 0, abort, kWaitNs);
            if (PAIR && ok) {  // the odd CTA's images
                const uint64_t t0 = globaltimer_ns();
                for (uint32_t it = 0; !test(bar(kBarPeerConst), 0); ++it)
                    if ((it & 31u) == 31u && (*abort || globaltimer_ns() - t0 > kWaitNs)) {
                        ok = false;
                        break;
                    }
            }
            auto mma_ss = [](uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
                if (PAIR) umma_ss_pair(d, ad, bd, id, acc);
                else umma_ss(d, ad, bd, id, acc);
            };
            auto mma_ts = [](uint32_t d, uint32_t at, uint64_t bd, uint32_t id, uint32_t acc) {
                if (PAIR) umma_ts_pair(d, at, bd, id, acc);
                else umma_ts(d, at, bd, id, acc);
            };
            auto commit_both = [](uint32_t b) {  // on this CTA's barrier and (pair) the odd CTA's
                if (PAIR) umma_commit_pair_both(b);
                else umma_commit(b);
            };
            // descriptors as low halves: operand i of the images, stage s of x, and
            // the offset of K-step st (16 elements) inside an operand (x: 128 rows, K-halves
            // 16 KB apart; images: this CTA's rows, K-halves kImgHalf apart)
            constexpr uint32_t kTileU = kTile >> 4;
            constexpr uint32_t kImgU = C::kImgBytes >> 4;
            const uint32_t img = sw128_desc_lo(sbase + C::kOffImg);
            const uint32_t x0 = sw128_desc_lo(sbase + C::kOffX);
            auto kdesc = [](uint32_t lo, int step) {
                return sw128_desc(lo + (((uint32_t)(step >> 2) * kHalf + (uint32_t)(step & 3) * 32u) >> 4));
            };
            auto bdesc = [](uint32_t lo, int step) {
                return sw128_desc(lo + (((uint32_t)(step >> 2) * C::kImgHalf + (uint32_t)(step & 3) * 32u) >> 4));
            };
            // rotation of local tile k into its team's buffer; false when not ready yet
            auto try_rot = [&](int k) -> bool {
                const int s = k % C::kStages;
                const int t = k % C::kTeams;
                const uint32_t use = (uint32_t)(k / C::kTeams);
                if (!test(bar(kBarXFull + s), (uint32_t)(k / C::kStages) & 1u)) return false;
                if (!test(bar(kBarRotEmpty + t), (use & 1u) ^ 1u)) return false;
                tc_fence_after();
                const uint32_t dA = tmem + C::kBufCols * (uint32_t)t;
                const uint32_t xs = x0 + (uint32_t)s * kTileU;
                uint32_t accA = 0u;
                if (ROT == 0) {  // the small lo pass first, then the hi pass
#pragma unroll
                    for (int st = 0; st < 8; ++st) {
                        mma_ss(dA, kdesc(xs, st), bdesc(img + kImgU, st), idesc, accA);
                        accA = 1u;
                    }
                }
#pragma unroll
                for (int st = 0; st < 8; ++st) {
                    mma_ss(dA, kdesc(xs, st), bdesc(img, st), idesc, accA);
                    accA = 1u;
                }
                commit_both(bar(kBarXEmpty + s));
                commit_both(bar(kBarRotFull + t));
                return true;
            };
            // sketch of local tile k (keys); false when its rho is not written yet or
            // the sketch of tile k - 1 has not been read
            auto try_qjl = [&](int k) -> bool {
                const int t = k % C::kTeams;
                if (!test(bar(kBarRhoFull + t), (uint32_t)(k / C::kTeams) & 1u)) return false;
                if (!test(bar(kBarSketchEmpty), ((uint32_t)k & 1u) ^ 1u)) return false;
                tc_fence_after();
                const uint32_t buf = tmem + C::kBufCols * (uint32_t)t;
                const uint32_t d = tmem + kColSketch;
                const uint32_t m0 = img + C::kRotImages * kImgU;
                // rho of K-step st: columns 16 st (hi pairs) and 16 st + 8 (lo pairs)
                auto rho_col = [&](int st) { return buf + 16u * (uint32_t)st; };
                uint32_t acc2 = 0u;
                // the small terms first: rho_lo M_hi (+ rho_hi M_lo for Haar), then rho_hi M_hi
#pragma unroll
                for (int st = 0; st < 8; ++st) {
                    mma_ts(d, rho_col(st) + 8u, bdesc(m0, st), idesc, acc2);
                    acc2 = 1u;
                }
                if (ROT == 0) {
#pragma unroll
                    for (int st = 0; st < 8; ++st) mma_ts(d, rho_col(st), bdesc(m0 + kImgU, st), idesc, 1u);
                }
#pragma unroll
                for (int st = 0; st < 8; ++st) mma_ts(d, rho_col(st), bdesc(m0, st), idesc, 1u);
                commit_both(bar(kBarQjlFull + t));
                return true;
            };
            // Each issuer goes in tile order.  Polls with a bound on time without progress.
            int next = 0;
            uint64_t t_last = globaltimer_ns();
            uint32_t spins = 0;
            while (ok && next < my_tiles) {
                if (rot_issuer ? try_rot(next) : try_qjl(next)) {
                    ++next;
                    spins = 0;
                    t_last = globaltimer_ns();
                } else if ((++spins & 31u) == 0) {
                    if (*abort || globaltimer_ns() - t_last > kWaitNs) ok = false;
                }
            }
            if (!ok) set_abort(abort, a.err);
            // this thread's MMAs (pair: of both CTAs) complete before the tensor memory is released
            const int drain = kBarDrain + (rot_issuer ? 0 : 1);
            if (PAIR) umma_commit_pair_local(bar(drain));
            else umma_commit(bar(drain));
            const volatile int never = 0;
            mbar_wait(bar(drain), 0, &never, kWaitNs);
        }
        __syncwarp();
    } else if (warp < C::kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int team = warp >> 2;    // tiles k with k % kTeams == team, buffer team
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const uint32_t buf = tmem + lane_addr + C::kBufCols * (uint32_t)team;
        const uint32_t sketch = tmem + lane_addr + kColSketch;  // keys
        // table entry of u: bits(u + magic) * 128 + lut_off, in this lane's copy
        // (bits(u + magic) = bits(1.5 * 2^23) + cells / 2 + round(u), see tc_params.h)
        const uint32_t lut_off = sbase + C::kOffLut +
                                 (PROD ? 16u * (uint32_t)(lane & (kLutReplProd - 1)) : 4u * (uint32_t)lane) -
                                 __float_as_uint(12582912.0f) * 128u;
        const float2 magic2 = make_float2(a.lut_magic, a.lut_magic);
        const float2 mone2 = make_float2(-1.f, -1.f);
        // code of u from its cell's entry e and fr = u - round(u) (exact)
        auto code_of = [](uint32_t e, float fr) -> uint32_t { return (e & 15u) + (__uint_as_float(e) < fr ? 1u : 0u); };
        const float2 rho_k = make_float2(a.rho_scale, a.rho_scale);
        constexpr int kPer = 32 / W;       // codes per 32-bit word
        constexpr int kQW = 32 / kPer;     // words of 32 columns' codes
        const bool ok = mbar_wait_warp(bar(kBarConst), 0, abort, kWaitNs);
        if (!ok) set_abort(abort, a.err);

        // slot of this thread's row of a tile, and the row's destination: the chunk
        // pointer with the row inside the page in its low 4 bits (chunks are
        // 16-byte aligned), or null
        // row vi = row0 + row of this CTA's 128 rows from row0 (a multiple of 128) is
        // (token vi / H, head vi % H); when H divides 128 a block of 128 rows holds
        // 128 / H whole tokens and this thread's token offset and head are the same in
        // every block
        const bool hdiv = (128 % a.H) == 0;
        const int tok_per_block = hdiv ? 128 / a.H : 0;
        const int row_tok = hdiv ? row / a.H : 0, row_head = hdiv ? row % a.H : 0;
        auto token_of = [&](int row0, int vi) -> int { return hdiv ? (row0 >> 7) * tok_per_block + row_tok : vi / a.H; };
        // (a volatile load: issued where it is written, a tile before its use)
        auto slot_of = [&](int row0) -> int {
            const int vi = row0 + row;
            return vi < a.N ? ldg_early(a.slots + token_of(row0, vi)) : -1;
        };
        auto dest = [&](int row0, int slot) -> uint8_t* {
            const int vi = row0 + row;
            if (vi >= a.N || slot < 0) return nullptr;
            if (slot >= a.num_blocks * kPage) {
                atomicOr(a.err, TQ_DEVERR_SLOT);
                return nullptr;
            }
            const int head = hdiv ? row_head : vi % a.H;
            return a.cache + ((size_t)(slot >> 4) * a.H + head) * (size_t)a.lay.bytes + (size_t)(slot & (kPage - 1));
        };
        // codes of columns [32 q, 32 q + 32) of the row
        auto store_codes = [&](uint8_t* d, int q, const uint32_t (&w)[kQW]) {
            if (!d) return;
            const int pr = (int)((uintptr_t)d & 15u);
            uint8_t* cp = d - pr + pr * a.lay.code_row + q * (4 * kQW);
            // streaming stores: the cache lines leave L2 first (nothing here reads them again)
            if (kQW == 4) __stcs(reinterpret_cast<uint4*>(cp), make_uint4(w[0], w[1 % kQW], w[2 % kQW], w[3 % kQW]));
            else if (kQW == 2) __stcs(reinterpret_cast<uint2*>(cp), make_uint2(w[0], w[1 % kQW]));
            else __stcs(reinterpret_cast<unsigned int*>(cp), w[0]);
        };
        auto store_tail = [&](uint8_t* d, float norm, float gamma, const uint32_t (&sg)[4]) {
            if (!d) return;
            const int pr = (int)((uintptr_t)d & 15u);
            uint8_t* chunk = d - pr;
            if (PROD) __stcs(reinterpret_cast<uint4*>(chunk + a.lay.signs_off + pr * (kDim / 8)), make_uint4(sg[0], sg[1], sg[2], sg[3]));
            __stcs(reinterpret_cast<float*>(chunk + a.lay.norm_off) + pr, norm);
            if (PROD) __stcs(reinterpret_cast<float*>(chunk + a.lay.gamma_off) + pr, gamma);
        };

        // the buffer-release arrivals of both CTAs of a pair go to the even CTA's issuer
        auto release = [&](int b) {
            if (PAIR) mbar_arrive_remote_warp(bar(b), 0);
            else mbar_arrive_warp(bar(b));
        };
        // the destination of the team's current tile and the slot of its next one; the
        // next tile's destination and the slot of the one after it are worked out while
        // the team waits for the rotation (values) or after the tile's stores (keys)
        int slot_next = team + C::kTeams < my_tiles ? slot_of(row0_of(team + C::kTeams)) : -1;
        uint8_t* dst = team < my_tiles ? dest(row0_of(team), slot_of(row0_of(team))) : nullptr;
        uint8_t* dst_next = nullptr;
        auto advance = [&](int k) {
            dst_next = k + C::kTeams < my_tiles ? dest(row0_of(k + C::kTeams), slot_next) : nullptr;
            if (k + 2 * C::kTeams < my_tiles) slot_next = slot_of(row0_of(k + 2 * C::kTeams));
        };
        for (int k = team; k < my_tiles; k += C::kTeams) {
            const uint32_t use = (uint32_t)(k / C::kTeams);
            float nsq;
            if (!PROD) {
                // ---- ||x||^2 of the row from the swizzled fp16 tile (logical 16-byte
                // chunk c of a 128-byte row sits at chunk c ^ (row % 8))
                const int stg = k % C::kStages;
                bool good = mbar_wait_warp(bar(kBarXFull + stg), (uint32_t)(k / C::kStages) & 1u, abort, kWaitNs);
                good = __all_sync(0xffffffffu, good && !*abort);
                if (!good) {
                    set_abort(abort, a.err);
                    break;
                }
                float sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    const uint32_t xr = sbase + C::kOffX + stg * kTile + kb * kHalf + row * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint32_t w0, w1, w2, w3;
                        lds_v4_ordered(xr + (uint32_t)((c ^ (row & 7)) << 4), w0, w1, w2, w3);
                        sq_acc2(w0, sq[0], sq[1]);
                        sq_acc2(w1, sq[2], sq[3]);
                        sq_acc2(w2, sq[0], sq[1]);
                        sq_acc2(w3, sq[2], sq[3]);
                    }
                }
                fence_proxy_async_shared();  // these reads before the next TMA write of the stage
                mbar_arrive_warp(bar(kBarXEmpty + stg));
                nsq = (sq[0] + sq[1]) + (sq[2] + sq[3]);
                advance(k);
                good = mbar_wait_warp(bar(kBarRotFull + team), use & 1u, abort, kWaitNs);
                if (!good) {
                    set_abort(abort, a.err);
                    break;
                }
                tc_fence_after();
            } else {
                bool good = mbar_wait_warp(bar(kBarRotFull + team), use & 1u, abort, kWaitNs);
                good = __all_sync(0xffffffffu, good && !*abort);
                if (!good) {
                    set_abort(abort, a.err);
                    break;
                }
                tc_fence_after();
                // ---- ||acc||^2 of the row
                float2 q2[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) q2[i] = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t r0[32];
                    tmem_ld32(buf + 32 * c, r0);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 v = make_float2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
                        q2[i & 3] = __ffma2_rn(v, v, q2[i & 3]);
                    }
                }
                nsq = ((q2[0].x + q2[0].y) + (q2[1].x + q2[1].y)) + ((q2[2].x + q2[2].y) + (q2[3].x + q2[3].y));
            }
            // rows with inf / nan inputs are quantized as zero vectors (their norm stays non-finite)
            const bool finite = nsq <= 3.4e38f;
            const bool live = finite && nsq > 0.f;
            const float rn = live ? rsqrt_refined(nsq) : 0.f;  // 1 / ||acc|| (keys), 1 / ||x|| (values)
            const float nacc = nsq * rn;
            const float sc = (PROD ? a.lut_kscale : a.lut_xscale) * rn;
            const float2 s2 = make_float2(sc, sc);
            const bool any_bad = __any_sync(0xffffffffu, !finite);
            const float norm = live ? (PROD ? nacc * a.n_scale : nacc) : (finite ? 0.f : sqrtf(nsq));

            // ---- bucketize + pack (+ residual, rho for keys): 32 columns (two K-steps)
            // per iteration, their codes stored at once
            float2 gs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
              uint32_t words[kQW];
#pragma unroll
              for (int i = 0; i < kQW; ++i) words[i] = 0u;
              if (PROD) {
                // both K-steps of the 32 columns at once: 16 independent column pairs
                const uint32_t col = buf + 32 * q;
                float2 av[16];
                {
                    uint32_t r0[32];
                    tmem_ld32(col, r0);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) av[i] = make_float2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
                }
                if (any_bad && !finite) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) av[i] = make_float2(0.f, 0.f);
                }
                // K-step 2 q + h: its rho goes over its A columns (already read), hi pairs
                // at the first 8 and lo pairs at the next 8, as soon as they are known
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t rho_hi[8], rho_lo[8];
#pragma unroll
                    for (int ii = 0; ii < 8; ++ii) {
                        const int i = 8 * h + ii;
                        const float2 u = __fmul2_rn(av[i], s2);
                        const float2 gg = __fadd2_rn(u, magic2);
                        uint32_t b0, base0, lo0, hi0, b1, base1, lo1, hi1;
                        lds_v4(__float_as_uint(gg.x) * 128u + lut_off, b0, base0, lo0, hi0);
                        lds_v4(__float_as_uint(gg.y) * 128u + lut_off, b1, base1, lo1, hi1);
                        const bool p0 = __uint_as_float(b0) < u.x;
                        const bool p1 = __uint_as_float(b1) < u.y;
                        const uint32_t code0 = base0 + (p0 ? 1u : 0u);
                        const uint32_t code1 = base1 + (p1 ? 1u : 0u);
                        const float c0 = __uint_as_float(p0 ? hi0 : lo0);
                        const float c1 = __uint_as_float(p1 ? hi1 : lo1);
                        const float2 d = __ffma2_rn(av[i], s2, make_float2(-c0, -c1));  // residual, cell units
                        gs[i & 1] = __ffma2_rn(d, d, gs[i & 1]);
                        // rho = 32 (v - c) = hi + lo in fp16: hi keeps the top 11 significant bits
                        // (exact in fp16 for |rho| < 65504), lo = rho - hi exactly
                        const float2 rho = __fmul2_rn(d, rho_k);
                        const float2 hf = make_float2(__uint_as_float(__float_as_uint(rho.x) & 0xffffe000u),
                                                      __uint_as_float(__float_as_uint(rho.y) & 0xffffe000u));
                        const float2 rem = __fadd2_rn(rho, make_float2(-hf.x, -hf.y));
                        const __half2 hi = __floats2half2_rn(hf.x, hf.y);
                        const __half2 lo = __floats2half2_rn(rem.x, rem.y);
                        rho_hi[ii] = *reinterpret_cast<const uint32_t*>(&hi);
                        rho_lo[ii] = *reinterpret_cast<const uint32_t*>(&lo);
                        const int j = 2 * i;  // column within the 32
                        words[j / kPer] += code0 << (W * (j % kPer));
                        words[(j + 1) / kPer] += code1 << (W * ((j + 1) % kPer));
                    }
                    tmem_st8(col + 16 * h, rho_hi);
                    tmem_st8(col + 16 * h + 8, rho_lo);
                }
              } else {
#pragma unroll
              for (int sub = 0; sub < 2; ++sub) {
                const uint32_t col = buf + 32 * q + 16 * sub;
                float2 av[8];
                {  // one accumulator
                    uint32_t r0[16];
                    tmem_ld16(col, r0);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 8; ++i) av[i] = make_float2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
                }
                if (any_bad && !finite) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) av[i] = make_float2(0.f, 0.f);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 u = __fmul2_rn(av[i], s2);
                    const float2 gg = __fadd2_rn(u, magic2);
                    const float2 fr = __fadd2_rn(u, __ffma2_rn(gg, mone2, magic2));  // u - round(u)
                    const uint32_t code0 = code_of(lds_u32(__float_as_uint(gg.x) * 128u + lut_off), fr.x);
                    const uint32_t code1 = code_of(lds_u32(__float_as_uint(gg.y) * 128u + lut_off), fr.y);
                    const int j = 16 * sub + 2 * i;  // column within the 32
                    words[j / kPer] += code0 << (W * (j % kPer));
                    words[(j + 1) / kPer] += code1 << (W * ((j + 1) % kPer));
                }
              }
              }
              store_codes(dst, q, words);
            }
            if (!PROD) {
                tc_fence_before();
                release(kBarRotEmpty + team);
                const uint32_t none[4] = {0u, 0u, 0u, 0u};
                store_tail(dst, norm, 0.f, none);
                dst = dst_next;
                continue;
            }
            // ---- keys: release rho; gamma; then the sketch as sign bits
            tmem_st_wait();
            tc_fence_before();
            release(kBarRhoFull + team);
            const float gsq = (gs[0].x + gs[0].y) + (gs[1].x + gs[1].y);
            const float gamma = (live && gsq > 0.f) ? gsq * rsqrt_refined(gsq) * nacc * a.gamma_scale : 0.f;
            const bool sk = mbar_wait_warp(bar(kBarQjlFull + team), use & 1u, abort, kWaitNs);
            if (!sk) {
                set_abort(abort, a.err);
                break;
            }
            // the sketch is done with rho: the buffer is free for the team's next rotation
            tc_fence_after();
            release(kBarRotEmpty + team);
            uint32_t sg[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t q[32];
                tmem_ld32(sketch + 32 * c, q);
                tmem_ld_wait();
                uint32_t neg = 0u;  // bit j = sign bit of column 32 c + j
#pragma unroll
                for (int j = 31; j >= 0; --j) neg = __funnelshift_l(q[j], neg, 1);
                sg[c] = live ? ~neg : 0xffffffffu;
            }
            tc_fence_before();
            release(kBarSketchEmpty);
            store_tail(dst, norm, gamma, sg);
            advance(k);
            dst = dst_next;
        }
    }
    __syncthreads();
    // pair: neither CTA leaves, or frees tensor memory the even CTA's MMAs write, while
    // the other may still signal it
    if (PAIR) cluster_sync();
    if (warp == C::kWarpMma) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem, C::kTmemCols);
        else tmem_dealloc(tmem, C::kTmemCols);
    }
}

// One launch over N rows: 2-CTA clusters (pair) or single CTAs, as many as are
// resident at once and no more than there are tiles; programmatic stream
// serialization lets the setup above griddep_wait overlap the end of the kernel before.
template <int ROT, bool PROD, int W, bool PAIR>
cudaError_t launch_tc(const CUtensorMap& tmap, const TcArgs& a, int sm_count, cudaStream_t stream) {
    using C = Cfg<ROT, PROD, PAIR>;
    auto k = compress_tc_kernel<ROT, PROD, W, PAIR>;
    // CTAs (pair: clusters) of this kernel resident at once, per device; computed once
    // and published atomically (two threads computing it at once store the same value)
    static std::atomic<int> resident_of[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int resident = resident_of[dev].load(std::memory_order_relaxed);
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = PAIR ? 2 : 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (resident == 0) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
        if (e != cudaSuccess) return e;
        int n = PAIR ? sm_count / 2 : sm_count;
        if (PAIR) {
            cfg.gridDim = dim3(2 * (unsigned)n);
            int clusters = 0;
            e = cudaOccupancyMaxActiveClusters(&clusters, k, &cfg);
            if (e != cudaSuccess) return e;
            if (clusters > 0 && clusters < n) n = clusters;
        }
        resident = n > 0 ? n : 1;
        resident_of[dev].store(resident, std::memory_order_relaxed);
    }
    const int rows = PAIR ? 256 : 128;
    const int ntiles = (a.N + rows - 1) / rows;
    const int workers = ntiles < resident ? (ntiles > 0 ? ntiles : 1) : resident;
    cfg.gridDim = dim3((unsigned)(PAIR ? 2 * workers : workers));
    return cudaLaunchKernelEx(&cfg, k, tmap, a);
}

}  // namespace

cudaError_t launch_compress_tc(const tq_ctx* ctx, int kind, const uint16_t* x, int T, int H, const int32_t* slots,
                               uint8_t* cache, int num_blocks, cudaStream_t stream) {
    const bool value = (kind == TQ_KIND_VALUE);
    const ChunkLayout& lay = value ? ctx->lay_value : ctx->lay_key;
    const TcTables& tabs = ctx->tc;
    const int rot = ctx->host.rotation;
    const int N = T * H;
    CUtensorMap tmap;
    if (!encode_rows_tmap(&tmap, x, N)) return cudaErrorInvalidValue;
    const bool prod = lay.prod;
    TcArgs a{};
    a.slots = slots;
    a.cache = cache;
    a.N = N;
    a.H = H;
    a.num_blocks = num_blocks;
    a.images = tabs.images;
    a.lut = value ? tabs.lut_value : tabs.lut_key;
    const LutParams& lp = value ? tabs.lp_value : tabs.lp_key;
    a.lut_kscale = (float)(std::sqrt((double)kDim) * (double)lp.scale);
    // values: acc = 16 y (Haar) or sqrt(d) y (Hadamard)
    a.lut_xscale = (float)(std::sqrt((double)kDim) * (double)lp.scale / (rot == TQ_ROT_HAAR ? 16.0 : std::sqrt((double)kDim)));
    a.lut_magic = lp.magic;
    a.rho_scale = (float)(32.0 / (double)lp.scale);
    const double n_scale = rot == TQ_ROT_HAAR ? 1.0 / 16.0 : 1.0 / std::sqrt(128.0);
    a.n_scale = (float)n_scale;
    a.gamma_scale = (float)(n_scale / (std::sqrt((double)kDim) * (double)lp.scale));
    a.lay = lay;
    a.err = ctx->dev_error;
    a.stall = take_stall(ctx) ? 1 : 0;
    const int W = container_width(value ? ctx->host.vbits : ctx->host.kbits);
    cudaError_t e = cudaErrorInvalidValue;
    // every kind runs as MMA pairs on the two SMs of 2-CTA clusters, 256 rows a tile
#define TQ_TC_CASE(R, P, WW) \
    if (rot == R && prod == P && W == WW) e = launch_tc<R, P, WW, true>(tmap, a, ctx->sm_count, stream);
    TQ_TC_CASE(0, false, 4)
    TQ_TC_CASE(0, false, 2)
    TQ_TC_CASE(1, false, 4)
    TQ_TC_CASE(1, false, 2)
    TQ_TC_CASE(0, true, 4)
    TQ_TC_CASE(0, true, 2)
    TQ_TC_CASE(0, true, 1)
    TQ_TC_CASE(1, true, 4)
    TQ_TC_CASE(1, true, 2)
    TQ_TC_CASE(1, true, 1)
#undef TQ_TC_CASE
    if (e == cudaSuccess) count_launches(1);
    return e;
}

cudaError_t launch_compress(const tq_ctx* ctx, int kind, const uint16_t* x, int T, int H, const int32_t* slots,
                            uint8_t* cache, int num_blocks, cudaStream_t stream) {
    return launch_compress_tc(ctx, kind, x, T, H, slots, cache, num_blocks, stream);
}

}  // namespace tq
