// Causal prefill attention of one sequence over its compressed, paged cache, on
// tensor cores, with the keys and values decompressed on the fly.
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…":
//   - section "架构设计": the fused prefill attention kernel (queries of many positions
//     against the compressed keys, dequantized inline);
//   - section "注意力计算的特殊挑战与QJL校正": the score estimator
//       <q,k> ~ <q,k_hat> + gamma sqrt(pi/2)/d <S q, sign(S r)>.
// Query i of the chunk (position q_start + i) attends to the tokens 0 .. q_start + i
// of the sequence, whose keys and values are already in the cache.  As in the
// decode, everything happens in the rotated domain: scores <R^T q, c[idx]> n/sqrt(d)
// (+ the sign term against S q), values accumulated as sum_t p_t n_t c[idx_t]/sqrt(d)
// and un-rotated once per query row (o = R acc / l).
//
// One CTA of 8 warps per (block of 128 queries, query head); warp w takes 16 queries.
//   prologue  R^T (fp16 hi, lo) and S staged in shared memory (16-byte async copies,
//             rows swizzled); each warp computes q' and s of its 16 queries on
//             mma.sync and keeps them as fp16 A fragments in registers.
//   pages     per step of two 16-token pages up to the block's last query: the CTA's
//             threads decode the key codes, sign bits and value codes (fetched a step
//             ahead) into fp16 [token][coordinate] tiles in shared memory; each warp
//             takes scores S[16 queries x 32 tokens] (four n-tiles, key term and sign
//             term; B fragments by ldmatrix), the causal mask, an online-softmax step
//             (base 2), and O += P' V (B fragments by transposing ldmatrix).
//   epilogue  R (fp16 hi, lo) staged over R^T; o = R (O / l) / sqrt(d) on mma.sync
//             (three passes), stored fp16 or fp32.
#include <cmath>

#include "device_util.cuh"
#include "mma_sync.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

constexpr int kPW = 8;                 // warps per CTA
constexpr int kPThreads = kPW * 32;
constexpr int kPQ = 16 * kPW;          // queries per CTA
constexpr int kPT = 2 * kPage;         // tokens per step: two pages
constexpr int kKS = kDim + 8;          // tile row stride (halves): rows 16 bytes apart in banks
// Shared memory: [0, 96 KiB) staged matrices (R^T hi | R^T lo | S, then R hi | R lo),
// then the page tiles and the per-token scalars.
constexpr uint32_t kPOffMat = 0;
constexpr uint32_t kPMatBytes = 3 * kDim * kDim * 2;
constexpr uint32_t kPOffK = kPOffMat + kPMatBytes;                  // half [32][kKS]: c[key code]
constexpr uint32_t kPOffS = kPOffK + kPT * kKS * 2;                 // half [32][kKS]: +-1 signs
constexpr uint32_t kPOffV = kPOffS + kPT * kKS * 2;                 // half [32][kKS]: c[value code]
constexpr uint32_t kPOffT = kPOffV + kPT * kKS * 2;                 // float [3][32]: key norm, gamma, value norm
constexpr uint32_t kPOffCB = kPOffT + 3 * kPT * 4;                  // half [2][16]: key, value levels
constexpr uint32_t kPSmem = kPOffCB + 2 * 16 * 2;

struct PrefillArgs {
    const uint16_t* q;  // [Tq][Hq][128] fp16
    const uint8_t* kc;
    const uint8_t* vc;
    int num_blocks;
    const int32_t* block_table;  // [max_blocks]
    int max_blocks;
    int q_start, Tq, Hq, Hkv, G;
    const uint16_t* RTh;  // fp16 R^T hi / lo, S (row-major)
    const uint16_t* RTl;
    const uint16_t* Sh;
    const uint16_t* Rh;   // fp16 R hi / lo (row-major)
    const uint16_t* Rl;
    Codebook cbk, cbv;
    ChunkLayout lk, lv;
    float qscale, sscale;  // scale*log2(e)/sqrt(d), scale*log2(e)*sqrt(pi/2)/d
    void* out;             // [Tq][Hq][128]
    int out_fp32;
    uint32_t* err;
};

// 16-byte async copies of n matrices of 128 x 128 fp16 from src[] into shared memory
// at dst, row r's 16-byte pieces in the order k ^ (r % 8).
__device__ __forceinline__ void stage_matrices(uint32_t dst, const uint16_t* const* src, int n) {
    constexpr int kPieces = kDim * kDim * 2 / 16;
    for (int i = threadIdx.x; i < n * kPieces; i += kPThreads) {
        const int mtx = i / kPieces, o = (i - mtx * kPieces) * 16;
        const int r = o >> 8, k16 = (o >> 4) & 15;
        sm100::cp_async16(dst + mtx * (kPieces * 16) + r * 256 + ((k16 ^ (r & 7)) << 4),
                          reinterpret_cast<const uint8_t*>(src[mtx]) + o);
    }
    sm100::cp_async_commit();
}

// Four 8x8 fp16 matrices from shared memory (lane l gives the address of row l % 8 of
// matrix l / 8); register j holds matrix j in the mma fragment layout.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// The same, each matrix transposed: register j holds column (not row) pairs of matrix j.
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// Word w (two halves: columns 2w, 2w + 1) of row r of a staged matrix.
__device__ __forceinline__ uint32_t staged_word(const uint8_t* m, int r, int w) {
    return *reinterpret_cast<const uint32_t*>(m + r * 256 + ((((w >> 2) ^ (r & 7)) << 4) | ((w & 3) << 2)));
}

// The 16 packed codes of width W from bit 16 W t8 of a row (t8 = 0..7): 2 W bytes at a
// 2 W-aligned offset.
template <int W>
__device__ __forceinline__ uint64_t load_codes16(const uint8_t* row, int t8) {
    if (W == 4) return *reinterpret_cast<const uint64_t*>(row + 8 * t8);
    if (W == 2) return *reinterpret_cast<const uint32_t*>(row + 4 * t8);
    return *reinterpret_cast<const uint16_t*>(row + 2 * t8);
}

// One step's bytes for thread i (page i / 128 of the step's two, token i % 16,
// coordinates 16 (i / 16 % 8) .. + 15): its packed key codes, sign bits and value
// codes, and (threads i % 128 < 16) the token's scalars.  Loaded a step ahead of use.
static_assert(kPThreads == 256, "one thread per (page, token, 16 coordinates) of a step");
struct PageBytes {
    uint64_t kw, vw;
    uint32_t sw;
    float kn, kg, vn;
};
template <int WK, int WV>
__device__ __forceinline__ PageBytes fetch_page(const PrefillArgs& a, int blk, int hk) {
    PageBytes r{};
    if (blk < 0 || blk >= a.num_blocks) return r;
    const uint8_t* kch = a.kc + ((size_t)blk * a.Hkv + hk) * a.lk.bytes;
    const uint8_t* vch = a.vc + ((size_t)blk * a.Hkv + hk) * a.lv.bytes;
    const int t = threadIdx.x & 15, t8 = (threadIdx.x >> 4) & 7;
    r.kw = load_codes16<WK>(kch + t * a.lk.code_row, t8);
    r.vw = load_codes16<WV>(vch + t * a.lv.code_row, t8);
    if (a.lk.prod) r.sw = *reinterpret_cast<const uint16_t*>(kch + a.lk.signs_off + t * (kDim / 8) + 2 * t8);
    if ((threadIdx.x & 127) < kPage) {
        r.kn = reinterpret_cast<const float*>(kch + a.lk.norm_off)[t] * a.qscale;
        r.kg = a.lk.prod ? reinterpret_cast<const float*>(kch + a.lk.gamma_off)[t] * a.sscale : 0.f;
        r.vn = reinterpret_cast<const float*>(vch + a.lv.norm_off)[t];
    }
    return r;
}

// A step's fp16 tiles from its bytes (levels from the shared-memory codebooks ck, cv;
// code widths WK, WV):
// each thread writes its token's 16 coordinates of the three [token][coordinate] tiles
// as two 16-byte stores each (eight consecutive tokens of a quarter-warp cover the 32
// banks once: rows are 16 bytes apart modulo 128).
template <int WK, int WV>
__device__ __forceinline__ void store_page_tiles(const PrefillArgs& a, const PageBytes& r, uint8_t* smem,
                                                 const __half* ck, const __half* cv) {
    float* ts = reinterpret_cast<float*>(smem + kPOffT);
    const int t = (threadIdx.x >> 7) * kPage + (threadIdx.x & 15), j0 = 16 * ((threadIdx.x >> 4) & 7);
    constexpr uint32_t mk = (1u << WK) - 1u, mv = (1u << WV) - 1u;
    const uint32_t row = (uint32_t)(t * kKS + j0) * 2;
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {  // coordinates j0 + 8 hb .. + 7: one 16-byte store per tile
        uint32_t kw[4], sw[4], vw[4];
#pragma unroll
        for (int jj = 0; jj < 8; jj += 2) {
            const int j = 8 * hb + jj;
            const __half k0 = ck[(uint32_t)(r.kw >> (j * WK)) & mk], k1 = ck[(uint32_t)(r.kw >> ((j + 1) * WK)) & mk];
            const __half v0 = cv[(uint32_t)(r.vw >> (j * WV)) & mv], v1 = cv[(uint32_t)(r.vw >> ((j + 1) * WV)) & mv];
            kw[jj / 2] = h2bits(k0, k1);
            vw[jj / 2] = h2bits(v0, v1);
            // +-1 in fp16: 0xBC00 (-1) with bit 15 cleared where the sign bit is set
            sw[jj / 2] = 0xBC00BC00u ^ (((r.sw >> j) & 1u) << 15) ^ (((r.sw >> (j + 1)) & 1u) << 31);
        }
        *reinterpret_cast<uint4*>(smem + kPOffK + row + 16 * hb) = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        *reinterpret_cast<uint4*>(smem + kPOffV + row + 16 * hb) = make_uint4(vw[0], vw[1], vw[2], vw[3]);
        if (a.lk.prod)
            *reinterpret_cast<uint4*>(smem + kPOffS + row + 16 * hb) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
    }
    if ((threadIdx.x & 127) < kPage) {
        ts[t] = r.kn;
        ts[kPT + t] = r.kg;
        ts[2 * kPT + t] = r.vn;
    }
}

template <int WK, int WV>
__global__ void __launch_bounds__(kPThreads) prefill_attn_kernel(PrefillArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int h = blockIdx.y, hk = h / a.G;
    const int i0 = blockIdx.x * kPQ + 16 * warp;  // this warp's first query (chunk index)
    const uint32_t mat = sm100::smem_u32(smem) + kPOffMat;
    const uint8_t* mp = smem + kPOffMat;
    {
        const uint16_t* src[3] = {a.RTh, a.RTl, a.Sh};
        stage_matrices(mat, src, 3);
    }
    __half* ck = reinterpret_cast<__half*>(smem + kPOffCB);
    __half* cv = ck + 16;
    if (threadIdx.x < 16) {
        ck[threadIdx.x] = __float2half_rn(threadIdx.x < a.cbk.levels ? a.cbk.c[threadIdx.x] : 0.f);
        cv[threadIdx.x] = __float2half_rn(threadIdx.x < a.cbv.levels ? a.cbv.c[threadIdx.x] : 0.f);
    }
    // q rows i0 + g, i0 + g + 8 as A fragments (zero past the chunk)
    const bool r0 = i0 + g < a.Tq, r1 = i0 + g + 8 < a.Tq;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + ((size_t)(r0 ? i0 + g : 0) * a.Hq + h) * kDim);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + ((size_t)(r1 ? i0 + g + 8 : 0) * a.Hq + h) * kDim);
    uint32_t qa[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        qa[ks][0] = r0 ? q0[8 * ks + c] : 0u;
        qa[ks][1] = r1 ? q1[8 * ks + c] : 0u;
        qa[ks][2] = r0 ? q0[8 * ks + c + 4] : 0u;
        qa[ks][3] = r1 ? q1[8 * ks + c + 4] : 0u;
    }
    sm100::cp_async_wait<0>();
    __syncthreads();
    // ---- q' = R^T q and s = S q (fp32 accumulation), kept as fp16 A fragments: output
    // tiles 2ks, 2ks + 1 of the rotation form K-step ks of the score contraction (their
    // rows g, g + 8 are the fragment's registers 0, 1 and 2, 3)
    uint32_t ra[8][4], sa[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int n = (2 * ks + half) * 8 + g;  // output row of R^T / S for this lane's B column
            float dq[4], ds[4];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t h0 = staged_word(mp, n, 8 * k + c), h1 = staged_word(mp, n, 8 * k + c + 4);
                const uint32_t l0 = staged_word(mp + kDim * kDim * 2, n, 8 * k + c);
                const uint32_t l1 = staged_word(mp + kDim * kDim * 2, n, 8 * k + c + 4);
                const uint32_t s0 = staged_word(mp + 2 * kDim * kDim * 2, n, 8 * k + c);
                const uint32_t s1 = staged_word(mp + 2 * kDim * kDim * 2, n, 8 * k + c + 4);
                if (k == 0) {
                    mma16816_z(dq, qa[0][0], qa[0][1], qa[0][2], qa[0][3], l0, l1);
                    mma16816_z(ds, qa[0][0], qa[0][1], qa[0][2], qa[0][3], s0, s1);
                } else {
                    mma16816(dq, qa[k][0], qa[k][1], qa[k][2], qa[k][3], l0, l1);
                    mma16816(ds, qa[k][0], qa[k][1], qa[k][2], qa[k][3], s0, s1);
                }
                mma16816(dq, qa[k][0], qa[k][1], qa[k][2], qa[k][3], h0, h1);
            }
            ra[ks][2 * half] = f2h2(dq[0], dq[1]);
            ra[ks][2 * half + 1] = f2h2(dq[2], dq[3]);
            sa[ks][2 * half] = f2h2(ds[0], ds[1]);
            sa[ks][2 * half + 1] = f2h2(ds[2], ds[3]);
        }
    }

    // ---- pages up to the block's last query
    const int last_q = min(a.Tq, (int)blockIdx.x * kPQ + kPQ) - 1;  // chunk index
    const int n_tok = a.q_start + last_q + 1;
    const int n_pages = (n_tok + kPage - 1) / kPage;
    const int qp0 = a.q_start + i0 + g, qp1 = qp0 + 8;  // positions of this lane's rows
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float acc[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const uint32_t kt_addr = sm100::smem_u32(smem) + kPOffK, st_addr = sm100::smem_u32(smem) + kPOffS;
    const uint32_t vt_addr = sm100::smem_u32(smem) + kPOffV;
    const float* ts = reinterpret_cast<const float*>(smem + kPOffT);
    static_assert(kPOffK % 16 == 0 && kPOffS % 16 == 0 && kPOffV % 16 == 0 && (kKS * 2) % 16 == 0,
                  "ldmatrix rows and tile stores 16-byte aligned");
    // steps of two pages: this thread's page id two steps ahead, its bytes one step ahead
    const int sub = threadIdx.x >> 7;  // the page of the step this thread fetches
    const int n_steps = (n_pages + 1) / 2;
    auto block_of = [&](int pg) {
        return pg < n_pages && TQ_DCHECK(pg < a.max_blocks, a.err) ? a.block_table[pg] : -1;
    };
    int blk_next = block_of(sub);
    PageBytes nxt = fetch_page<WK, WV>(a, blk_next, hk);
    int blk_after = block_of(2 + sub);
    for (int step = 0; step < n_steps; ++step) {
        // pages of the step with a valid block (a page past the last is masked by the
        // causal limit: its positions exceed every query's)
        const int b0 = block_of(2 * step), b1 = block_of(2 * step + 1);
        const bool ok0 = b0 >= 0 && b0 < a.num_blocks;
        const bool ok1 = (2 * step + 1 >= n_pages) || (b1 >= 0 && b1 < a.num_blocks);
        __syncthreads();  // the previous step's tiles are read
        if (blk_next >= 0 && blk_next < a.num_blocks) store_page_tiles<WK, WV>(a, nxt, smem, ck, cv);
        // the next step's bytes, in flight during this step's contractions
        if (step + 1 < n_steps) {
            blk_next = blk_after;
            nxt = fetch_page<WK, WV>(a, blk_next, hk);
            blk_after = block_of(2 * (step + 2) + sub);
        }
        if (threadIdx.x == 0 && !(ok0 && ok1)) atomicOr(a.err, TQ_DEVERR_BLOCK);
        __syncthreads();
        // scores of tokens nt*8 + 2c + e (nt = 0..3) for rows g (i = 0), g + 8 (i = 1)
        float sc[4][2][2];  // [nt][i][e]
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            // B fragments of two K-steps per ldmatrix.x4: lane l addresses token nt*8 + l % 8,
            // coordinates 16 (ks + l / 16) + 8 (l / 8 % 2)
            const uint32_t krow = (uint32_t)((nt * 8 + (lane & 7)) * kKS + 8 * ((lane >> 3) & 1) + 16 * (lane >> 4)) * 2;
            float d1[4], d2[4];
#pragma unroll
            for (int ks = 0; ks < 8; ks += 2) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(kt_addr + krow + 32 * ks, b0, b1, b2, b3);
                if (ks == 0) mma16816_z(d1, ra[0][0], ra[0][1], ra[0][2], ra[0][3], b0, b1);
                else mma16816(d1, ra[ks][0], ra[ks][1], ra[ks][2], ra[ks][3], b0, b1);
                mma16816(d1, ra[ks + 1][0], ra[ks + 1][1], ra[ks + 1][2], ra[ks + 1][3], b2, b3);
            }
            if (a.lk.prod) {
#pragma unroll
                for (int ks = 0; ks < 8; ks += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(st_addr + krow + 32 * ks, b0, b1, b2, b3);
                    if (ks == 0) mma16816_z(d2, sa[0][0], sa[0][1], sa[0][2], sa[0][3], b0, b1);
                    else mma16816(d2, sa[ks][0], sa[ks][1], sa[ks][2], sa[ks][3], b0, b1);
                    mma16816(d2, sa[ks + 1][0], sa[ks + 1][1], sa[ks + 1][2], sa[ks + 1][3], b2, b3);
                }
            } else {
                d2[0] = d2[1] = d2[2] = d2[3] = 0.f;
            }
            const bool okp = nt < 2 ? ok0 : ok1;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int tt = nt * 8 + 2 * c + e, pos = step * kPT + tt;
                const float kn = ts[tt], kg = ts[kPT + tt];
                const float s0 = fmaf(kg, d2[e], kn * d1[e]), s1 = fmaf(kg, d2[2 + e], kn * d1[2 + e]);
                sc[nt][0][e] = okp && pos <= qp0 ? s0 : -INFINITY;
                sc[nt][1][e] = okp && pos <= qp1 ? s1 : -INFINITY;
            }
        }
        // online softmax per row (the row's 32 scores sit in the quad's 4 lanes)
        uint32_t pa[2][4];  // [K-step: tokens 0-15 / 16-31][A register]
        float mnew[2], corr[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(sc[nt][i][0], sc[nt][i][1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mnew[i] = fmaxf(m[i], mx);
            corr[i] = (m[i] == -INFINITY) ? 0.f : exp2f(m[i] - mnew[i]);
        }
        // rescale O only when a row of the warp has a new maximum (after the first steps
        // of a long sequence, seldom)
        if (__any_sync(0xffffffffu, corr[0] != 1.f || corr[1] != 1.f)) {
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                acc[nt][0] *= corr[0];
                acc[nt][1] *= corr[0];
                acc[nt][2] *= corr[1];
                acc[nt][3] *= corr[1];
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float pw[4][2];
            float sum = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float pr = (sc[nt][i][e] == -INFINITY) ? 0.f : exp2f(sc[nt][i][e] - mnew[i]);
                    sum += pr;
                    // (a masked token's value norm is not read: it may be anything)
                    pw[nt][e] = pr > 0.f ? pr * ts[2 * kPT + nt * 8 + 2 * c + e] : 0.f;
                }
            l[i] = l[i] * corr[i] + sum;
            m[i] = mnew[i];
            // P' as A fragments of the value contraction (K-steps: tokens 0-15, 16-31)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                pa[k][i] = f2h2(pw[2 * k][0], pw[2 * k][1]);          // tokens 16k + 2c, + 1
                pa[k][2 + i] = f2h2(pw[2 * k + 1][0], pw[2 * k + 1][1]);  // tokens 16k + 2c + 8, + 9
            }
        }
        // O[16 x 128] += P' V: n-tile nt = coordinates 8 nt .. 8 nt + 7; one transposing
        // ldmatrix.x4 gives both K-steps' B fragments (lane l addresses token l,
        // coordinates 8 nt .. 8 nt + 7)
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(vt_addr + (uint32_t)(lane * kKS + 8 * nt) * 2, b0, b1, b2, b3);
            mma16816(acc[nt], pa[0][0], pa[0][1], pa[0][2], pa[0][3], b0, b1);
            mma16816(acc[nt], pa[1][0], pa[1][1], pa[1][2], pa[1][3], b2, b3);
        }
    }

    // ---- epilogue: o = R acc / (l sqrt(d)) for each row
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
    }
    __syncthreads();  // every warp is done with the staged R^T, S
    {
        const uint16_t* src[2] = {a.Rh, a.Rl};
        stage_matrices(mat, src, 2);
    }
    const float inv0 = l[0] > 0.f ? 0.08838834764831845f / l[0] : 0.f;
    const float inv1 = l[1] > 0.f ? 0.08838834764831845f / l[1] : 0.f;
    uint32_t ah[8][4], al[8][4];  // a = acc / (l sqrt(d)) as fp16 hi + lo A fragments
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const float* d = acc[2 * ks + half];
            const float x0 = d[0] * inv0, x1 = d[1] * inv0, x2 = d[2] * inv1, x3 = d[3] * inv1;
            const __half2 h01 = __floats2half2_rn(x0, x1), h23 = __floats2half2_rn(x2, x3);
            const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
            const __half2 l01 = __floats2half2_rn(x0 - f01.x, x1 - f01.y), l23 = __floats2half2_rn(x2 - f23.x, x3 - f23.y);
            ah[ks][2 * half] = *reinterpret_cast<const uint32_t*>(&h01);
            ah[ks][2 * half + 1] = *reinterpret_cast<const uint32_t*>(&h23);
            al[ks][2 * half] = *reinterpret_cast<const uint32_t*>(&l01);
            al[ks][2 * half + 1] = *reinterpret_cast<const uint32_t*>(&l23);
        }
    sm100::cp_async_wait<0>();
    __syncthreads();  // R landed
#pragma unroll 1
    for (int nt = 0; nt < 16; ++nt) {  // outputs 8 nt .. 8 nt + 7
        const int n = nt * 8 + g;
        float d[4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t h0 = staged_word(mp, n, 8 * ks + c), h1 = staged_word(mp, n, 8 * ks + c + 4);
            const uint32_t l0 = staged_word(mp + kDim * kDim * 2, n, 8 * ks + c);
            const uint32_t l1 = staged_word(mp + kDim * kDim * 2, n, 8 * ks + c + 4);
            if (ks == 0) mma16816_z(d, al[0][0], al[0][1], al[0][2], al[0][3], h0, h1);
            else mma16816(d, al[ks][0], al[ks][1], al[ks][2], al[ks][3], h0, h1);
            mma16816(d, ah[ks][0], ah[ks][1], ah[ks][2], ah[ks][3], l0, l1);
            mma16816(d, ah[ks][0], ah[ks][1], ah[ks][2], ah[ks][3], h0, h1);
        }
        const int col = nt * 8 + 2 * c;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int qi = i0 + g + 8 * i;
            if (qi >= a.Tq) continue;
            const size_t oi = ((size_t)qi * a.Hq + h) * kDim + col;
            if (a.out_fp32) {
                *reinterpret_cast<float2*>(static_cast<float*>(a.out) + oi) = make_float2(d[2 * i], d[2 * i + 1]);
            } else {
                *reinterpret_cast<__half2*>(static_cast<__half*>(a.out) + oi) = __floats2half2_rn(d[2 * i], d[2 * i + 1]);
            }
        }
    }
}

}  // namespace

cudaError_t launch_prefill(const tq_ctx* ctx, const uint16_t* q, const uint8_t* kc, const uint8_t* vc, int num_blocks,
                           const int32_t* block_table, int max_blocks, int q_start, int Tq, int Hq, int Hkv, float scale,
                           void* out, int out_fp32, cudaStream_t stream) {
    PrefillArgs a{};
    a.q = q;
    a.kc = kc;
    a.vc = vc;
    a.num_blocks = num_blocks;
    a.block_table = block_table;
    a.max_blocks = max_blocks;
    a.q_start = q_start;
    a.Tq = Tq;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = Hq / Hkv;
    a.RTh = ctx->dev.RTh;
    a.RTl = ctx->dev.RTl;
    a.Sh = ctx->dev.Sh;
    a.Rh = ctx->dev.Rh;
    a.Rl = ctx->dev.Rl;
    a.cbk = ctx->cb_key;
    a.cbv = ctx->cb_value;
    a.lk = ctx->lay_key;
    a.lv = ctx->lay_value;
    const float scale_log2 = scale * 1.4426950408889634f;
    a.qscale = scale_log2 / sqrtf((float)kDim);
    a.sscale = scale_log2 * 1.2533141373155003f / (float)kDim;
    a.out = out;
    a.out_fp32 = out_fp32;
    a.err = ctx->dev_error;
    // code container widths (key, value): TQ4 and 3/4-bit MSE keys (4, 4), bits 3 prod
    // keys (2, 4), TQ2 (1, 2), 2-bit MSE keys (2, 2)
    void (*kern)(PrefillArgs) = nullptr;
    const int wk = a.cbk.width, wv = a.cbv.width;
    if (wk == 4 && wv == 4) kern = prefill_attn_kernel<4, 4>;
    else if (wk == 2 && wv == 4) kern = prefill_attn_kernel<2, 4>;
    else if (wk == 1 && wv == 2) kern = prefill_attn_kernel<1, 2>;
    else if (wk == 2 && wv == 2) kern = prefill_attn_kernel<2, 2>;
    else return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPSmem);
    if (e != cudaSuccess) return e;
    const dim3 grid((Tq + kPQ - 1) / kPQ, Hq);
    kern<<<grid, kPThreads, kPSmem, stream>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace tq
