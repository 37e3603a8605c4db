// Compress step on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…", section "TurboQuant" steps 1-4
// (normalize, rotate by R^T, Gaussian Lloyd-Max, pack nibbles + fp32 norm) and
// section "注意力计算的特殊挑战与QJL校正" (keys: sign(S r), gamma = ||r||);
// [TQ-RS] "TurboQuant : compresser le KV-cache…", "Couche 1" (randomized
// Walsh-Hadamard rotation).
//
// One CTA per SM walks 128-vector tiles of the flattened [T*Hkv, 128] input:
//   warp 0       TMA producer: 128x128 fp16 tiles (two 128-byte-swizzled boxes)
//   warp 1       TMEM owner and single-thread MMA issuer
//   warps 2..17  epilogue, four warps per TMEM lane quarter (32 columns each)
// Rotation: D[v][n] = sum_k x[v][k] B[n][k] with B the rotation split into
// fp16 parts held in shared memory for the whole kernel:
//   Haar      B = 16 R^T = hi + lo (two passes, x is exact in fp16, products are
//             exact, fp32 accumulation)  -> acc = 16 y
//   Hadamard  B = H D (entries +-1, exact, one pass)  -> acc = sqrt(d) y
// The tensor core rounds each accumulation step; to keep ||x|| and gamma within
// 1e-6 the rotation goes to two accumulators, A = (lo pass) + K-steps 0-3 of the
// hi pass and B = K-steps 4-7, summed in registers (acc = A + B).
// In both cases v = sqrt(d) y / ||x|| = sqrt(d) acc / ||acc||, so the epilogue
// only needs ||acc||.  Codes come from a 2 KB shared-memory table of uniform
// cells over v (each cell holds at most one boundary), one exact fp32 compare.
// Keys (prod mode): r = acc - c[code] ||acc|| / sqrt(d) (the residual in the
// rotated domain, scaled), gamma = ||r|| / scale, and the sign sketch
//   S (x - x_hat) = (S R) (y - y_hat)
// is a second contraction whose A operand rho ~ r (split into fp16 hi + lo) is
// written by the epilogue straight into tensor memory (over the tile's own,
// already read, accumulator A; the sketch accumulates over B):
//   Haar      acc2 = rho_hi M_hi + rho_lo M_hi + rho_hi M_lo   (M = S R)
//   Hadamard  acc2 = (rho_hi + rho_lo) M',   M' = S D H integer, exact in fp16
// sign bit j = [acc2_j >= 0].  Every wait is bounded (TQ_DEVERR_TIMEOUT).
#include <cuda.h>

#include "device_util.cuh"
#include "sm100.cuh"
#include "tc_params.h"

namespace tq {
namespace {

using namespace sm100;

constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kSpan = 4 * 128 / kEpiWarps;  // columns per epilogue thread
constexpr int kQ = 128 / kSpan;             // epilogue threads per row
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 fp16 operand
constexpr uint32_t kHalf = kTile / 2;      // one 128-byte-swizzled K-half
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint32_t kSmemMax = 232448;

// TMEM (512 columns).  Values: two tile buffers [A 128 | B 128] at 0 and 256.
// Keys: one rotation buffer [A | B] at 0 (released as soon as it has been read, so
// the next tile's rotation overlaps this tile's epilogue) and a sketch region at
// 256: rho_hi [256,320), rho_lo [320,384) (the A operand, fp16 pairs) and the
// sketch accumulator [384,512).  The epilogue reads tile k-1's sketch before it
// writes tile k's rho, so the sketch contraction overlaps the epilogue too.
constexpr uint32_t kBufCols = 256;
constexpr uint32_t kColB = 128;
constexpr uint32_t kColRhoHi = 256;
constexpr uint32_t kColRhoLo = 320;
constexpr uint32_t kColQjl = 384;

template <int ROT, bool PROD>
struct Cfg {
    static constexpr int kRotImages = ROT == 0 ? 2 : 1;
    static constexpr int kQjlImages = PROD ? (ROT == 0 ? 2 : 1) : 0;
    static constexpr int kImages = kRotImages + kQjlImages;
    static constexpr int kCells = PROD ? kLutCellsProd : kLutCellsMse;
    static constexpr int kLutBytes = PROD ? kLutBytesProd : kLutBytesMse;
    static constexpr uint32_t kPartBytes = 2 * 2 * kQ * 128 * 4;  // [tile parity][norm, gamma][span][row]
    static constexpr uint32_t kBarBytes = 512;
    static constexpr uint32_t kFixed = kImages * kTile + kLutBytes + kPartBytes + kBarBytes;
    static constexpr int kStagesFit = (int)((kSmemMax - kFixed) / kTile);
    static constexpr int kStages = kStagesFit > 4 ? 4 : kStagesFit;
    static constexpr uint32_t kOffImg = 0;
    static constexpr uint32_t kOffX = kOffImg + kImages * kTile;
    static constexpr uint32_t kOffLut = kOffX + kStages * kTile;
    static constexpr uint32_t kOffPart = kOffLut + kLutBytes;
    static constexpr uint32_t kOffBar = kOffPart + kPartBytes;
    static constexpr uint32_t kSmem = kOffBar + kBarBytes;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kStages >= 1, "shared memory budget");
    static_assert(kSmem <= kSmemMax, "shared memory budget");
};

// barrier indices
enum : int {
    kBarConst = 0,
    kBarXFull = 1,    // +stage (4)
    kBarXEmpty = 5,   // +stage (4)
    kBarRotFull = 9,  // +buffer (2)
    kBarRotEmpty = 11,
    kBarRhoFull = 13,
    kBarQjlFull = 14,
    kBarDrain = 15,
    kNumBars = 16
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
    float lut_scale, lut_magic;
    float n2_scale;  // ||x||^2 = n2_scale * ||acc||^2
    uint32_t* err;
};

struct LutMse {
    float bnd;
    int base;
};
struct LutProd {
    float bnd;
    int base;
    float c_lo, c_hi;
};

__device__ __forceinline__ void set_abort(volatile int* abort, uint32_t* err) {
    *abort = 1;
    atomicOr(err, TQ_DEVERR_TIMEOUT);
}

template <int ROT, bool PROD, int W>
__global__ void __launch_bounds__(kThreads, 1) compress_tc_kernel(const __grid_constant__ CUtensorMap tmap, TcArgs a) {
    using C = Cfg<ROT, PROD>;
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
    const int ntiles = (a.N + 127) / 128;
    const int my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        mbar_init(bar(kBarConst), 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(bar(kBarXFull + s), 1);
            mbar_init(bar(kBarXEmpty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar(kBarRotFull + b), 1);
            mbar_init(bar(kBarRotEmpty + b), kEpiThreads);
        }
        mbar_init(bar(kBarRhoFull), kEpiThreads);
        mbar_init(bar(kBarQjlFull), 1);
        mbar_init(bar(kBarDrain), 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(kBarConst), C::kImages * kTile + C::kLutBytes);
            for (int i = 0; i < C::kImages; ++i)
                bulk_g2s(sbase + C::kOffImg + i * kTile, a.images + (size_t)i * kTile, kTile, bar(kBarConst));
            bulk_g2s(sbase + C::kOffLut, a.lut, C::kLutBytes, bar(kBarConst));
            int issued = 0;
            for (int k = 0; k < my_tiles; ++k) {
                const int s = k % C::kStages;
                const uint32_t ph = (uint32_t)(k / C::kStages) & 1u;
                if (!mbar_wait(bar(kBarXEmpty + s), ph ^ 1u, abort, kWaitNs)) {
                    set_abort(abort, a.err);
                    break;
                }
                const int row0 = ((int)blockIdx.x + k * (int)gridDim.x) * 128;
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
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_f16(128, 128);
            const uint32_t img = sbase + C::kOffImg;
            bool ok = mbar_wait(bar(kBarConst), 0, abort, kWaitNs);
            auto kdesc = [](uint32_t base, int step) {  // K-step of 16 elements inside a 128x128 operand
                return smem_desc_sw128(base + (uint32_t)(step >> 2) * kHalf + (uint32_t)(step & 3) * 32u);
            };
            auto issue_rot = [&](int k) -> bool {
                const int s = k % C::kStages;
                const int b = PROD ? 0 : (k & 1);
                const uint32_t use = PROD ? (uint32_t)k : (uint32_t)(k >> 1);  // use count of buffer b
                if (!mbar_wait(bar(kBarXFull + s), (uint32_t)(k / C::kStages) & 1u, abort, kWaitNs)) return false;
                if (!mbar_wait(bar(kBarRotEmpty + b), (use & 1u) ^ 1u, abort, kWaitNs)) return false;
                tc_fence_after();
                const uint32_t dA = tmem + kBufCols * b, dB = dA + kColB;
                const uint32_t xs = sbase + C::kOffX + s * kTile;
                uint32_t accA = 0u;
                if (ROT == 0) {  // the small lo pass first, then K-steps 0-3 of the hi pass
#pragma unroll
                    for (int st = 0; st < 8; ++st) {
                        umma_ss(dA, kdesc(xs, st), kdesc(img + kTile, st), idesc, accA);
                        accA = 1u;
                    }
                }
#pragma unroll
                for (int st = 0; st < 4; ++st) {
                    umma_ss(dA, kdesc(xs, st), kdesc(img, st), idesc, accA);
                    accA = 1u;
                }
#pragma unroll
                for (int st = 4; st < 8; ++st) umma_ss(dB, kdesc(xs, st), kdesc(img, st), idesc, st > 4 ? 1u : 0u);
                umma_commit(bar(kBarXEmpty + s));
                umma_commit(bar(kBarRotFull + b));
                return true;
            };
            auto issue_qjl = [&](int k) -> bool {
                if (!mbar_wait(bar(kBarRhoFull), (uint32_t)k & 1u, abort, kWaitNs)) return false;
                tc_fence_after();
                const uint32_t d = tmem + kColQjl;
                const uint32_t m0 = img + C::kRotImages * kTile;
                uint32_t acc2 = 0u;
                // the small terms first: rho_lo M_hi (+ rho_hi M_lo for Haar), then rho_hi M_hi
#pragma unroll
                for (int st = 0; st < 8; ++st) {
                    umma_ts(d, tmem + kColRhoLo + 8u * st, kdesc(m0, st), idesc, acc2);
                    acc2 = 1u;
                }
                if (ROT == 0) {
#pragma unroll
                    for (int st = 0; st < 8; ++st) umma_ts(d, tmem + kColRhoHi + 8u * st, kdesc(m0 + kTile, st), idesc, 1u);
                }
#pragma unroll
                for (int st = 0; st < 8; ++st) umma_ts(d, tmem + kColRhoHi + 8u * st, kdesc(m0, st), idesc, 1u);
                umma_commit(bar(kBarQjlFull));
                return true;
            };
            if (ok && my_tiles > 0) ok = issue_rot(0);
            for (int k = 0; ok && k < my_tiles; ++k) {
                if (k + 1 < my_tiles) ok = issue_rot(k + 1);
                if (ok && PROD) ok = issue_qjl(k);
            }
            if (!ok) set_abort(abort, a.err);
            // all MMAs of this CTA complete before its tensor memory is released
            umma_commit(bar(kBarDrain));
            const volatile int never = 0;
            mbar_wait(bar(kBarDrain), 0, &never, kWaitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int h = ew >> 2;         // column span [kSpan h, kSpan (h+1))
        const int row = quarter * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        float* part = reinterpret_cast<float*>(smem + C::kOffPart);
        // this lane's replica of the bucketize table (see tc_params.h)
        const uint8_t* lut = smem + C::kOffLut + (PROD ? 16 * (lane & (kLutReplProd - 1)) : 8 * (lane & (kLutReplMse - 1)));
        const float sqrt_d = 11.313708498984761f;
        constexpr int kPer = 32 / W;          // codes per 32-bit word
        constexpr int kWords = kSpan / kPer;  // words of this thread's span
        bool ok = mbar_wait(bar(kBarConst), 0, abort, kWaitNs);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) set_abort(abort, a.err);

        // destination of this thread's row of a tile: the chunk pointer with the row
        // inside the page in its low 4 bits (chunks are 16-byte aligned), or null
        auto dest = [&](int tile) -> uint8_t* {
            const int vi = tile * 128 + row;
            if (vi >= a.N) return nullptr;
            const int t = vi / a.H, head = vi - t * a.H;
            const long s = a.slots[t];
            if (s >= (long)a.num_blocks * kPage) {
                if (h == 0) atomicOr(a.err, TQ_DEVERR_SLOT);
                return nullptr;
            }
            if (s < 0) return nullptr;
            return a.cache + ((size_t)(s / kPage) * a.H + head) * (size_t)a.lay.bytes + (size_t)(s % kPage);
        };
        auto store = [&](uint8_t* d, const uint32_t (&words)[kWords], float norm, float gamma, uint32_t sg) {
            if (!d) return;
            const int pr = (int)((uintptr_t)d & 15u);
            uint8_t* chunk = d - pr;
            uint8_t* cp = chunk + pr * a.lay.code_row + h * (a.lay.code_row / kQ);
            if (kWords == 4) {
                *reinterpret_cast<uint4*>(cp) = make_uint4(words[0], words[1], words[2], words[kWords - 1]);
            } else if (kWords == 2) {
                *reinterpret_cast<uint2*>(cp) = make_uint2(words[0], words[kWords - 1]);
            } else {
                *reinterpret_cast<uint32_t*>(cp) = words[0];
            }
            if (PROD) *reinterpret_cast<uint32_t*>(chunk + a.lay.signs_off + pr * (kDim / 8) + h * 4) = sg;
            if (h == 0) {
                reinterpret_cast<float*>(chunk + a.lay.norm_off)[pr] = norm;
                if (PROD) reinterpret_cast<float*>(chunk + a.lay.gamma_off)[pr] = gamma;
            }
        };
        // read tile k's sketch accumulator and turn it into sign bits (bit set when >= 0)
        auto read_signs = [&](int k, bool nonzero, uint32_t& sg) -> bool {
            bool ok3 = mbar_wait(bar(kBarQjlFull), (uint32_t)k & 1u, abort, kWaitNs);
            ok3 = __all_sync(0xffffffffu, ok3);
            if (!ok3) return false;
            tc_fence_after();
            uint32_t q[32];
            tmem_ld32(tmem + lane_addr + kColQjl + kSpan * h, q);
            tmem_ld_wait();
            uint32_t n0 = 0u;
#pragma unroll
            for (int j = 0; j < 32; ++j) n0 |= (q[j] >> 31) << j;
            sg = nonzero ? ~n0 : 0xffffffffu;
            return true;
        };
        auto sum4 = [&](const float* pp) {
            return (pp[row] + pp[128 + row]) + (pp[256 + row] + pp[384 + row]);
        };

        // the previous tile's outputs wait here until its sketch is ready (keys)
        uint32_t pw[kWords];
        float pnorm = 0.f, pgamma = 0.f;
        bool pnz = false;
        uint8_t* pdst = nullptr;
        for (int k = 0; k < my_tiles; ++k) {
            const int tile = (int)blockIdx.x + k * (int)gridDim.x;
            const int b = PROD ? 0 : (k & 1);
            const uint32_t use = PROD ? (uint32_t)k : (uint32_t)(k >> 1);
            float* pn = part + ((k & 1) * 2 + 0) * (kQ * 128);
            float* pg = part + ((k & 1) * 2 + 1) * (kQ * 128);
            uint8_t* dst = dest(tile);  // issued early: the slot load overlaps the wait below
            // ---- rotation accumulators A + B -> registers
            float acc[kSpan];
            const uint32_t buf = tmem + lane_addr + kBufCols * (uint32_t)b + kSpan * h;
            ok = !*abort && mbar_wait(bar(kBarRotFull + b), use & 1u, abort, kWaitNs);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                uint32_t r0[32], r1[32];
                tmem_ld32(buf, r0);
                tmem_ld32(buf + kColB, r1);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(bar(kBarRotEmpty + b));
#pragma unroll
                for (int j = 0; j < kSpan; ++j) acc[j] = __uint_as_float(r0[j]) + __uint_as_float(r1[j]);
            } else {
                set_abort(abort, a.err);
#pragma unroll
                for (int j = 0; j < kSpan; ++j) acc[j] = 0.f;
            }
            // ---- ||acc||^2: 8 interleaved partial sums, then the spans of the row
            float ps[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) ps[i] = 0.f;
#pragma unroll
            for (int j = 0; j < kSpan; ++j) ps[j & 7] = fmaf(acc[j], acc[j], ps[j & 7]);
            pn[h * 128 + row] = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            named_barrier(1, kEpiThreads);
            if (*abort) break;
            const float nsq = sum4(pn);
            const float nacc = sqrtf(nsq);
            const float inv = nacc > 0.f ? sqrt_d / nacc : 0.f;
            const float norm = sqrtf(nsq * a.n2_scale);

            // ---- bucketize + pack (+ residual for keys)
            uint32_t words[kWords];
#pragma unroll
            for (int i = 0; i < kWords; ++i) words[i] = 0u;
            uint32_t rho_hi[kSpan / 2], rho_lo[kSpan / 2];
            float gs[4] = {0.f, 0.f, 0.f, 0.f};
            const float chat_scale = nacc / sqrt_d;
            const float kappa = nacc > 0.f ? 32.f * sqrt_d / nacc : 0.f;
#pragma unroll
            for (int j = 0; j < kSpan; j += 2) {
                float rho2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const float v = acc[j + u] * inv;
                    const float gg = fmaf(v, a.lut_scale, a.lut_magic);
                    const int cell = __float_as_int(gg) & (C::kCells - 1);
                    int code;
                    if (PROD) {
                        const LutProd e = *reinterpret_cast<const LutProd*>(lut + cell * 128);
                        const bool upc = e.bnd < v;
                        code = e.base + (upc ? 1 : 0);
                        const float r = fmaf(upc ? -e.c_hi : -e.c_lo, chat_scale, acc[j + u]);
                        gs[(j + u) & 3] = fmaf(r, r, gs[(j + u) & 3]);
                        rho2[u] = r * kappa;
                    } else {
                        const LutMse e = *reinterpret_cast<const LutMse*>(lut + cell * 128);
                        code = e.base + (e.bnd < v ? 1 : 0);
                    }
                    words[(j + u) / kPer] |= (uint32_t)code << (W * ((j + u) % kPer));
                }
                if (PROD) {  // rho = hi + lo in fp16
                    const __half2 hi = __floats2half2_rn(rho2[0], rho2[1]);
                    const float2 hf = __half22float2(hi);
                    const __half2 lo = __floats2half2_rn(rho2[0] - hf.x, rho2[1] - hf.y);
                    rho_hi[j >> 1] = *reinterpret_cast<const uint32_t*>(&hi);
                    rho_lo[j >> 1] = *reinterpret_cast<const uint32_t*>(&lo);
                }
            }
            if (!PROD) {
                store(dst, words, norm, 0.f, 0u);
                continue;
            }
            pg[h * 128 + row] = (gs[0] + gs[1]) + (gs[2] + gs[3]);
            // tile k-1's sketch leaves the sketch region before tile k's rho enters it
            uint32_t sg = 0xffffffffu;
            bool have_prev = (k > 0) && !*abort;
            if (have_prev && !read_signs(k - 1, pnz, sg)) {
                set_abort(abort, a.err);
                have_prev = false;
            }
            if (!*abort) {
                tmem_st16(tmem + lane_addr + kColRhoHi + (kSpan / 2) * h, rho_hi);
                tmem_st16(tmem + lane_addr + kColRhoLo + (kSpan / 2) * h, rho_lo);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(kBarRhoFull));
            }
            named_barrier(1, kEpiThreads);
            if (*abort) break;
            if (have_prev) store(pdst, pw, pnorm, pgamma, sg);
            // this tile's outputs wait for its sketch
#pragma unroll
            for (int i = 0; i < kWords; ++i) pw[i] = words[i];
            pnorm = norm;
            pgamma = sqrtf(sum4(pg) * a.n2_scale);
            pnz = nsq > 0.f;
            pdst = dst;
        }
        if (PROD && my_tiles > 0 && !*abort) {
            uint32_t sg;
            if (read_signs(my_tiles - 1, pnz, sg))
                store(pdst, pw, pnorm, pgamma, sg);
            else
                set_abort(abort, a.err);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int ROT, bool PROD, int W>
cudaError_t launch_tc(const CUtensorMap& tmap, const TcArgs& a, int grid, cudaStream_t stream) {
    using C = Cfg<ROT, PROD>;
    auto k = compress_tc_kernel<ROT, PROD, W>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, C::kSmem, stream>>>(tmap, a);
    return cudaGetLastError();
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
    a.lut_scale = lp.scale;
    a.lut_magic = lp.magic;
    a.n2_scale = rot == TQ_ROT_HAAR ? 1.0f / 256.0f : 1.0f / 128.0f;
    a.lay = lay;
    a.err = ctx->dev_error;
    const int ntiles = (N + 127) / 128;
    const int grid = ntiles < ctx->sm_count ? ntiles : ctx->sm_count;
    const int W = container_width(value ? ctx->host.vbits : ctx->host.kbits);
    cudaError_t e = cudaErrorInvalidValue;
#define TQ_TC_CASE(R, P, WW) \
    if (rot == R && prod == P && W == WW) e = launch_tc<R, P, WW>(tmap, a, grid, stream);
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
