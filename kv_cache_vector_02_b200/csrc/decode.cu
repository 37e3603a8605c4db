// Split-K decode attention over the paged compressed cache, on tensor cores, in one
// kernel launch.
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…":
//   - section "注意力计算的特殊挑战与QJL校正": score estimator
//       <q,k> ~ <q,k_hat> + gamma sqrt(pi/2)/d <S q, sign(S r)>
//   - section "架构设计" / "关键工程改进": Paged Decode as split-K FlashDecoding.
// Everything happens in the rotated domain: <q, k_hat> = n/sqrt(d) <R^T q, c[idx]>,
// the value sum is accumulated as sum_t p_t n_t c[idx_t]/sqrt(d) and un-rotated
// once per query head (o = R acc / l).
//
// One kernel (decode_attn_kernel), cooperative: one persistent CTA per SM over an
// equal range of the pages of all (sequence, kv head) units, all CTAs resident.
//   prologue  R^T (fp16 hi, lo) staged in shared memory; the CTA's own page prefix
//             sums of the sequences; the lookup tables; q' = R^T q and s = S q of the
//             units of the range (mma.sync) into the CTA's workspace slots.
//   pages     pages p, p + 1 (p = 2 (w + kNW j)) of a unit's piece (the range's part
//             of one unit) go to warp w.  Each warp streams its own pairs of pages
//             (16-byte async copies by every lane of the key and the value chunks,
//             one commit group per pair) into its ring of shared-memory stages, its
//             issue cursor running ahead across pieces, and per pair of 16-token pages:
//               scores  D[16 tok x 8 heads] = sum_k Khat[tok][k] q'[k][h]  (mma m16n8k16)
//                       plus the sign term with +-1 fragments against s, per page
//               softmax online, base 2, per head column, one update for both pages
//               values  D[16 coords x 8 heads] += Vhat^T[coord][tok] P'[tok][h], per page
//             The warps of the CTA merge their states per piece into the slot (unit
//             + CTA); a piece that does not start its unit publishes the slot with
//             the launch's tag.
//   epilogue  the CTA that holds a unit's first page waits (bounded) for the later
//             slots of the unit, combines them by log-sum-exp, adds the residual
//             window, un-rotates (o = R a on mma.sync, R staged in shared memory) and
//             stores, 16 query heads at a time.
//
// Packed codes become fp16 MMA fragments in registers:
//   - 3-bit key codes (nibbles): byte permutes of an 8-entry register table;
//   - value codes: two tokens' codes of one coordinate are merged into one "pair
//     byte" (two ALU ops per 4 or 8 pair bytes), and one PRMT builds the full
//     shared-memory address of the pair byte's entry in a lane-replicated table
//     (tables sit at shared address 64 KiB, 256 bytes per entry, so the address is
//     0x10000 | byte << 8 | lane offset); one LDS then gives the fragment register;
//   - sign bits (and 1- or 2-bit key codes, taken as +-1 bit planes): one LDS.128
//     per sign byte from an 8-fold replicated table gives four +-1 fragment
//     registers.
// Inside a page the token order is permuted (row r holds token r ^ ((r >> 1) & 1))
// so that a warp's loads of four tokens' value bytes meet at most two to a bank.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <mutex>

#include "device_util.cuh"
#include "mma_sync.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

constexpr int kNW = 8;                        // warps per CTA (one CTA per SM, two per scheduler)
constexpr int kThreads = kNW * 32;
constexpr int kPartStride = kDim + 2;         // m, l, acc[128]
constexpr int kStages = 6;                    // page stages per warp: 3 pairs
constexpr uint32_t kStageBytes = 2496;        // >= key chunk + value chunk at every bit width (16-byte multiple)
constexpr uint32_t kTabAddr = 65536;          // shared-window address of the lookup tables
constexpr uint32_t kTabBytes = 65536;         // 256 entries x 256 bytes
// Stages: the first kLowStages below the tables (after the fields below), the rest
// from kRingAddr on (see stage_addr).
constexpr int kLowStages = 12;
constexpr uint32_t kRingAddr = kTabAddr + kTabBytes;
constexpr uint32_t kSmemBytes = kRingAddr + (kNW * kStages - kLowStages) * kStageBytes;  // any window base >= 0
// Below the tables, from the window base: the warps' (m, l), the CTA merge area (4
// heads at a time), the low stages.
constexpr uint32_t kOffML = 0;                                  // [kNW][2][4] float: m, l
constexpr uint32_t kOffMerge = kOffML + kNW * 2 * 4 * 4;        // [kNW][4][128] float
constexpr uint32_t kOffLowStages = (kOffMerge + kNW * 4 * kDim * 4 + 127) & ~127u;
constexpr uint32_t kLowBytes = kOffLowStages + kLowStages * kStageBytes;
// The page prefix sums of up to kPreCap - 1 sequences sit in the rest of the window
// below the tables (more sequences: the CTA's copy in the workspace).
constexpr uint32_t kEpiBytes = 45056;  // the epilogue's scratch (EpiSmem) from kOffMerge on
constexpr uint32_t kOffPre = (kLowBytes > kOffMerge + kEpiBytes ? kLowBytes : kOffMerge + kEpiBytes);
constexpr int kPreCap = 3840;
static_assert(kOffPre + kPreCap * 4 + 1024 <= kTabAddr, "prefix sums below the tables");
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint64_t kWaitNs = 2000000000ull;  // bounded waits for another CTA's slot

enum KMode { kKPrmt = 0, kKByte4 = 1, kKByte2 = 2, kKBit1 = 3 };
enum VMode { kVByte4 = 0, kVByte2 = 1 };

struct DecodeArgs {
    const uint16_t* q;
    float* qf;  // [slots][G][2][128] fp32: q' then s of unit u in slot u + CTA
    const uint8_t* kc;
    const uint8_t* vc;
    int num_blocks;
    const int32_t* block_table;
    int max_blocks;
    const int32_t* seq_lens;
    int B, Hq, Hkv, G, max_seq_len;
    float* partial;    // [slots][G][130]: m, l, acc (rotated domain) of unit u's piece in CTA c: slot u + c
    unsigned long long* flags;  // [slots]: = epoch once the slot's partial is complete
    unsigned long long epoch;   // this launch's tag (never repeats within the process)
    int* prefix;       // [grid][B + 1]: each CTA's own page prefix sums (pages of sequences < b)
    const uint16_t* RTh;   // fp16 R^T hi / lo, S (row-major)
    const uint16_t* RTl;
    const uint16_t* Sh;
    const uint16_t* Rh;    // fp16 R hi / lo (row-major)
    const uint16_t* Rl;
    float qscale, sscale;  // scale*log2(e)/sqrt(d), scale*log2(e)*sqrt(pi/2)/d
    float kscale;          // 1-bit keys: the level c[1] (key term = c1 <q', 2b - 1>)
    float kalpha, kbeta;   // 2-bit keys: c[code] = alpha (2 b1 - 1) + beta (2 b0 - 1)
    Codebook cbk, cbv;
    ChunkLayout lk, lv;
    void* out;
    int out_fp32;
    int stall;             // test hook: no piece publishes its partial (the merges wait out their limit)
    // residual window: fp16 keys / values [B][tail_cap][Hkv][128] of the last tail_lens[b]
    // tokens of each sequence, uncompressed (tail_k == NULL: none)
    const uint16_t* tail_k;
    const uint16_t* tail_v;
    const int32_t* tail_lens;
    int tail_cap;
    float scale_log2;      // softmax scale * log2(e)
    uint32_t* err;
};

__device__ __forceinline__ bool seq_len_ok(const DecodeArgs& a, int L) {
    return L >= 0 && L <= a.max_blocks * kPage && L <= a.max_seq_len;
}

// ------------------------------------------------------------------ helpers

// Transpose of an 8x8 fp16 matrix held as m8n8 fragments (thread 4 g + c holds row g,
// columns 2c, 2c + 1): afterwards it holds row g of the transpose.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ __half cb_half(const Codebook& cb, int code) {
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxLevels; ++k) v = (k == code) ? cb.c[k] : v;
    return __float2half_rn(v);
}

// Table reads at 32-bit shared-window addresses (the table is written once, before
// a CTA barrier, and never again).
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t x;
    asm("ld.shared.u32 %0, [%1];" : "=r"(x) : "r"(addr));
    return x;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 x;
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(x.x), "=r"(x.y) : "r"(addr));
    return x;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 x;
    asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w) : "r"(addr));
    return x;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

// Shared-window address of the table entry of byte K of p: 0x10000 | p.byte[K] << 8 |
// L.byte[X], where L holds this lane's offsets inside an entry in bytes 0 and 1 and
// 0x01, 0x00 in bytes 2 and 3 (one PRMT).
template <int K, int X>
__device__ __forceinline__ uint32_t taddr(uint32_t p, uint32_t L) {
    return __byte_perm(p, L, 0x7600u | (K << 4) | (4 + X));
}

// 2^x by the hardware approximation (flushes denormal results to 0; relative error
// about 2^-22), for the softmax weights.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Lazy softmax rescaling: the running maximum only moves when a page exceeds it by
// more than 2^kSlack (log2 units), so exponentials stay <= 2^kSlack in fp32 / fp16.
constexpr float kSlack = 8.f;

// Token of page row r (see the file comment).
__host__ __device__ constexpr int row_token(int r) { return r ^ ((r >> 1) & 1); }

// ------------------------------------------------------------------ page loop: tables
// Entry e (a byte) of the 64 KiB table at kTabAddr is 256 bytes:
//   bytes   0..127  region A, values:
//                     nibble pair bytes (low nibble: token t, high: token t + 1):
//                       half2(c[e & 15], c[e >> 4]), 32 copies (lane * 4);
//                     crumb pair bytes (crumbs: tokens t, t + 1 of a coordinate j,
//                     then of coordinate j + 2): {half2 of j, half2 of j + 2}, 16
//                     copies ((lane % 16) * 8)
//   bytes 128..255  region B, keys:
//                     sign bytes (bit = 1 -> +1): four half2 {bits 0,1 | 2,3 | 4,5 |
//                     6,7}, 8 copies (128 + (lane % 8) * 16) -- the QJL signs and the
//                     bit planes of 1- and 2-bit key codes;
//                     or (4-bit MSE keys) nibble pair bytes of one token:
//                     half2(c[e & 15], c[e >> 4]), 32 copies (128 + lane * 4)
template <int KM, int VM, bool PROD>
__device__ void build_tables(const DecodeArgs& a, int e) {
    const uint32_t row = kTabAddr + 256u * (uint32_t)e;
    if (VM == kVByte4) {
        const uint32_t w = h2bits(cb_half(a.cbv, e & 15), cb_half(a.cbv, e >> 4));
#pragma unroll
        for (int i = 0; i < 8; ++i) sts128(row + 16 * i, w, w, w, w);
    } else {
        const uint32_t x = h2bits(cb_half(a.cbv, e & 3), cb_half(a.cbv, (e >> 2) & 3));
        const uint32_t y = h2bits(cb_half(a.cbv, (e >> 4) & 3), cb_half(a.cbv, e >> 6));
#pragma unroll
        for (int i = 0; i < 8; ++i) sts128(row + 16 * i, x, y, x, y);
    }
    constexpr bool kSignTab = PROD || KM == kKByte2 || KM == kKBit1;
    if (kSignTab) {
        const __half one = __float2half_rn(1.f), mone = __float2half_rn(-1.f);
        auto pm = [&](int bit) { return ((e >> bit) & 1) ? one : mone; };
        const uint32_t x = h2bits(pm(0), pm(1)), y = h2bits(pm(2), pm(3));
        const uint32_t z = h2bits(pm(4), pm(5)), w = h2bits(pm(6), pm(7));
#pragma unroll
        for (int i = 0; i < 8; ++i) sts128(row + 128 + 16 * i, x, y, z, w);
    } else if (KM == kKByte4) {
        const uint32_t w = h2bits(cb_half(a.cbk, e & 15), cb_half(a.cbk, e >> 4));
#pragma unroll
        for (int i = 0; i < 8; ++i) sts128(row + 128 + 16 * i, w, w, w, w);
    }
}

// ------------------------------------------------------------------ page loop: pieces
// The CTA's range [pos, end) of the pages of all units in order (unit u = b Hkv + h
// holds the pages of sequence b), cut into pieces by unit.
struct Pieces {
    const int* pre;  // the CTA's page prefix sums
    long pos, end;
    int b;
    __device__ void init(const DecodeArgs& a, const int* prefix, long p, long e) {
        pre = prefix;
        pos = p;
        end = e;
        b = 0;
        if (pos < end) {  // the last sequence b with Hkv * pre[b] <= pos
            int lo = 0, hi = a.B - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if ((long)a.Hkv * pre[mid] <= pos) lo = mid;
                else hi = mid - 1;
            }
            b = lo;
        }
    }
    // next piece: sequence bb, kv head hk, pages [p0, p1) of the sequence
    __device__ bool next(const DecodeArgs& a, int& bb, int& hk, int& p0, int& p1) {
        while (pos < end && b < a.B) {
            const int np = pre[b + 1] - pre[b];
            const long off = pos - (long)a.Hkv * pre[b];
            if (np == 0 || off >= (long)a.Hkv * np) {
                ++b;
                continue;
            }
            hk = (int)(off / np);
            p0 = (int)(off - (long)hk * np);
            p1 = (int)min((long)np, p0 + (end - pos));
            pos += p1 - p0;
            bb = b;
            return true;
        }
        return false;
    }
};

// The page pairs of one warp (p0 + 2 warp + {0, 1}, + 2 kNW, ...) of every piece of the
// CTA, in order, with their block ids: lane l holds the block id of page l % 2 of
// the warp's pair wbase + l / 2 of the piece (-2: past the piece's end), and the next
// 16 pairs are loaded 8 pairs ahead of their use.
constexpr int kNoPage = -2;
struct PageCursor {
    Pieces it;
    int b, hk, p0, p1, ji, nj;
    bool live;
    int win, win_next, wbase;
    uint32_t kb, vb;                    // chunk bytes
    const uint8_t *kbase, *vbase;       // this lane's 16 bytes of kv head hk's chunks in physical block 0
    __device__ int load_win(const DecodeArgs& a, int warp, int lane, int base) const {
        const int jj = base + (lane >> 1), p = p0 + 2 * warp + (lane & 1) + jj * (2 * kNW);
        return jj < nj && p < p1 ? a.block_table[(size_t)b * a.max_blocks + p] : kNoPage;
    }
    __device__ void enter(const DecodeArgs& a, int warp, int lane) {  // the next piece with pages for this warp
        live = false;
        while (it.next(a, b, hk, p0, p1)) {
            nj = p0 + 2 * warp < p1 ? (p1 - p0 - 2 * warp + 2 * kNW - 1) / (2 * kNW) : 0;
            if (nj == 0) continue;
            ji = 0;
            wbase = 0;
            win = load_win(a, warp, lane, 0);
            win_next = kNoPage;
            kbase = a.kc + (size_t)hk * kb + 16 * lane;
            vbase = a.vc + (size_t)hk * vb + 16 * lane;
            live = true;
            return;
        }
    }
    __device__ void init(const DecodeArgs& a, const int* pre, long pos, long end, int warp, int lane, uint32_t kbytes,
                         uint32_t vbytes) {
        kb = kbytes;
        vb = vbytes;
        it.init(a, pre, pos, end);
        enter(a, warp, lane);
    }
    // block id of page h (0, 1) of the current pair (warp-uniform; every lane calls it)
    __device__ int block(int h) const { return __shfl_sync(0xffffffffu, win, 2 * (ji - wbase) + h); }
    __device__ void advance(const DecodeArgs& a, int warp, int lane) {
        ++ji;
        if (ji >= nj) {
            enter(a, warp, lane);
            return;
        }
        if (ji - wbase == 8 && wbase + 16 < nj) win_next = load_win(a, warp, lane, wbase + 16);
        if (ji - wbase == 16) {
            wbase = ji;
            win = win_next;
        }
    }
};

// ------------------------------------------------------------------ page loop: one page
template <int KM, int VM, bool PROD>
struct PageRegs {
    uint32_t k[2][4];    // key code bytes of token rows g, g+8 (coords 32c .. 32c+31)
    uint32_t s[2];       // sign word c of rows g, g+8
    float kn[2], kg[2];  // key norm * qscale, gamma * sscale of rows g, g+8
    uint32_t v[4][2];    // value code bytes of rows 2c, 2c+1, 2c+8, 2c+9 (coords 16g .. 16g+15)
    float vn[2];         // value norm of rows g, g+8
};

// Byte geometry of a page's key and value chunks (the same as the library's chunk
// layouts, fixed by the code widths; checked against the context at launch).
template <int KM, int VM, bool PROD>
struct PageGeom {
    static constexpr int kRow = KM == kKBit1 ? 16 : (KM == kKByte2 ? 32 : 64);  // key code bytes per token
    static constexpr int kSigns = 16 * kRow;
    static constexpr int kNorm = PROD ? kSigns + 16 * 16 : 16 * kRow;
    static constexpr int kGamma = kNorm + 64;
    static constexpr int kBytes = PROD ? kGamma + 64 : kNorm + 64;               // key chunk
    static constexpr int vRow = VM == kVByte4 ? 64 : 32;
    static constexpr int vNorm = 16 * vRow;
    static constexpr int vBytes = vNorm + 64;                                   // value chunk
    static constexpr int kPer = KM == kKBit1 ? 4 : (KM == kKByte2 ? 8 : 16);    // key bytes per thread per row
    static constexpr int vPer = VM == kVByte4 ? 8 : 4;                          // value bytes per thread per token
};

// Per-thread byte offsets inside a stage (key chunk at 0, value chunk at kBytes):
// rows g, g+8 of the scores are tokens tk0, tk0 + 8; the value rows are tokens tv0,
// tv1 and tv0 + 8, tv1 + 8 (see row_token).
struct PageOffs {
    uint32_t key, sign, norm, val0, val1;
};
template <int KM, int VM, bool PROD>
__device__ __forceinline__ PageOffs page_offsets(int tk0, int tv0, int tv1, int g, int c) {
    using P = PageGeom<KM, VM, PROD>;
    PageOffs o;
    o.key = tk0 * P::kRow + P::kPer * c;
    o.sign = P::kSigns + tk0 * 16 + 4 * c;
    o.norm = 4 * tk0;
    o.val0 = P::kBytes + tv0 * P::vRow + P::vPer * g;
    o.val1 = P::kBytes + tv1 * P::vRow + P::vPer * g;
    return o;
}

// Fragment bytes of one page from its stage st (a generic pointer to shared memory).
template <int KM, int VM, bool PROD>
__device__ __forceinline__ void load_page(PageRegs<KM, VM, PROD>& r, const uint8_t* st, const PageOffs& o,
                                          float qscale, float sscale) {
    using P = PageGeom<KM, VM, PROD>;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint8_t* row = st + o.key + i * 8 * P::kRow;
        if (P::kPer == 16) {
            const uint4 w = *reinterpret_cast<const uint4*>(row);
            r.k[i][0] = w.x, r.k[i][1] = w.y, r.k[i][2] = w.z, r.k[i][3] = w.w;
        } else if (P::kPer == 8) {
            const uint2 w = *reinterpret_cast<const uint2*>(row);
            r.k[i][0] = w.x, r.k[i][1] = w.y;
        } else {
            r.k[i][0] = *reinterpret_cast<const uint32_t*>(row);
        }
        const uint8_t* nb = st + o.norm + i * 32;
        if (PROD) {
            r.s[i] = *reinterpret_cast<const uint32_t*>(st + o.sign + i * 128);
            r.kg[i] = *reinterpret_cast<const float*>(nb + P::kGamma) * sscale;
        }
        r.kn[i] = *reinterpret_cast<const float*>(nb + P::kNorm) * qscale;
        r.vn[i] = *reinterpret_cast<const float*>(nb + P::kBytes + P::vNorm);  // (1/sqrt(d) in the epilogue)
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint8_t* row = st + ((i & 1) ? o.val1 : o.val0) + (i >> 1) * 8 * P::vRow;
        if (P::vPer == 8) {
            const uint2 w = *reinterpret_cast<const uint2*>(row);
            r.v[i][0] = w.x, r.v[i][1] = w.y;
        } else {
            r.v[i][0] = *reinterpret_cast<const uint32_t*>(row);
        }
    }
}

template <int KM>
struct KeyTerm {
    static constexpr int kSteps = KM == kKByte2 ? 16 : 8;  // 2-bit codes: 128 coordinates x 2 bit planes
};

// Base-2 logits of one page (ntok valid rows; 0: none): sc[nt][i][e] for rows g, g + 8
// (i) and heads nt*8 + 2c + e.  The key term (even and odd K-steps in separate
// accumulators) and the sign term on mma.sync.
template <int KM, int VM, bool PROD, int NT>
__device__ __forceinline__ void page_logits(const PageRegs<KM, VM, PROD>& cur, int ntok, const int (&tk)[2],
                                            uint32_t klo0, uint32_t klo1, uint32_t khi0, uint32_t khi1,
                                            uint32_t LA, uint32_t LB,
                                            const uint32_t (&bq)[NT][KeyTerm<KM>::kSteps][2],
                                            const uint32_t (&bs)[NT][8][2], float (&sc)[NT][2][2]) {
    float d1[NT][2][4], d2[NT][2][4];  // the first MMA of each accumulator starts it
    if (KM == kKPrmt || KM == kKByte4) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t ak[2][2];  // [row g / g+8][coords 32c+4ks+{0,1} / +{2,3}]
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint32_t w = cur.k[i][ks >> 1];
                if (KM == kKPrmt) {
                    const uint32_t sel = (ks & 1) ? (w >> 16) : w;
                    const uint32_t lo = __byte_perm(klo0, klo1, sel);
                    const uint32_t hi = __byte_perm(khi0, khi1, sel);
                    ak[i][0] = __byte_perm(lo, hi, 0x5140);
                    ak[i][1] = __byte_perm(lo, hi, 0x7362);
                } else if (ks & 1) {
                    ak[i][0] = lds32(taddr<2, 1>(w, LA));
                    ak[i][1] = lds32(taddr<3, 1>(w, LA));
                } else {
                    ak[i][0] = lds32(taddr<0, 1>(w, LA));
                    ak[i][1] = lds32(taddr<1, 1>(w, LA));
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                if (ks < 2) mma16816_z(d1[nt][ks & 1], ak[0][0], ak[1][0], ak[0][1], ak[1][1], bq[nt][ks][0], bq[nt][ks][1]);
                else mma16816(d1[nt][ks & 1], ak[0][0], ak[1][0], ak[0][1], ak[1][1], bq[nt][ks][0], bq[nt][ks][1]);
        }
    } else {
        // +-1 bit planes: byte b of the thread's key bytes -> K-steps 2b, 2b+1
        constexpr int kB = KM == kKByte2 ? 8 : 4;
#pragma unroll
        for (int b = 0; b < kB; ++b) {
            uint4 t[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint32_t w = cur.k[i][b >> 2];
                switch (b & 3) {
                    case 0: t[i] = lds128(taddr<0, 0>(w, LB)); break;
                    case 1: t[i] = lds128(taddr<1, 0>(w, LB)); break;
                    case 2: t[i] = lds128(taddr<2, 0>(w, LB)); break;
                    default: t[i] = lds128(taddr<3, 0>(w, LB)); break;
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (b == 0) {
                    mma16816_z(d1[nt][0], t[0].x, t[1].x, t[0].y, t[1].y, bq[nt][0][0], bq[nt][0][1]);
                    mma16816_z(d1[nt][1], t[0].z, t[1].z, t[0].w, t[1].w, bq[nt][1][0], bq[nt][1][1]);
                } else {
                    mma16816(d1[nt][0], t[0].x, t[1].x, t[0].y, t[1].y, bq[nt][2 * b][0], bq[nt][2 * b][1]);
                    mma16816(d1[nt][1], t[0].z, t[1].z, t[0].w, t[1].w, bq[nt][2 * b + 1][0], bq[nt][2 * b + 1][1]);
                }
            }
        }
    }
    if (PROD) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            uint4 t[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint32_t w = cur.s[i];
                switch (b) {
                    case 0: t[i] = lds128(taddr<0, 0>(w, LB)); break;
                    case 1: t[i] = lds128(taddr<1, 0>(w, LB)); break;
                    case 2: t[i] = lds128(taddr<2, 0>(w, LB)); break;
                    default: t[i] = lds128(taddr<3, 0>(w, LB)); break;
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (b == 0) {
                    mma16816_z(d2[nt][0], t[0].x, t[1].x, t[0].y, t[1].y, bs[nt][0][0], bs[nt][0][1]);
                    mma16816_z(d2[nt][1], t[0].z, t[1].z, t[0].w, t[1].w, bs[nt][1][0], bs[nt][1][1]);
                } else {
                    mma16816(d2[nt][0], t[0].x, t[1].x, t[0].y, t[1].y, bs[nt][2 * b][0], bs[nt][2 * b][1]);
                    mma16816(d2[nt][1], t[0].z, t[1].z, t[0].w, t[1].w, bs[nt][2 * b + 1][0], bs[nt][2 * b + 1][1]);
                }
            }
        }
    }
    const bool full = ntok >= kPage;
    const bool valid0 = full || tk[0] < ntok, valid1 = full || tk[1] < ntok;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float x = cur.kn[i] * (d1[nt][0][2 * i + e] + d1[nt][1][2 * i + e]);
                if (PROD) x = fmaf(cur.kg[i], d2[nt][0][2 * i + e] + d2[nt][1][2 * i + e], x);
                sc[nt][i][e] = x;
            }
            if (!full) {
                sc[nt][0][e] = valid0 ? sc[nt][0][e] : -INFINITY;
                sc[nt][1][e] = valid1 ? sc[nt][1][e] : -INFINITY;
            }
        }
}

// Value accumulation of one page: acc += Vhat^T P' (v: the page's value code bytes,
// pb: its P').
template <int VM, int NT>
__device__ __forceinline__ void page_values(const uint32_t (&v)[4][2], const uint32_t (&pb)[NT][2], uint32_t LA,
                                            uint32_t LB, float (&acc)[NT][8][4]) {
    // ---- values: m-tile mt, row g -> coordinate c0(mt) of the thread's 16, row g+8 -> c0 + 1
    if (VM == kVByte4) {
        // pair bytes of rows (2c, 2c+1) and (2c+8, 2c+9): lo -> even coordinates, hi -> odd
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            constexpr uint32_t M4 = 0x0F0F0F0Fu;
            const uint32_t A = v[0][hf], B = v[1][hf], C = v[2][hf], D = v[3][hf];
            const uint32_t pl0 = (A & M4) | ((B << 4) & ~M4), ph0 = ((A >> 4) & M4) | (B & ~M4);
            const uint32_t pl1 = (C & M4) | ((D << 4) & ~M4), ph1 = ((C >> 4) & M4) | (D & ~M4);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t a0, a1, a2, a3;
                switch (k) {
                    case 0: a0 = lds32(taddr<0, 0>(pl0, LA)), a1 = lds32(taddr<0, 0>(ph0, LA)),
                            a2 = lds32(taddr<0, 0>(pl1, LA)), a3 = lds32(taddr<0, 0>(ph1, LA)); break;
                    case 1: a0 = lds32(taddr<1, 0>(pl0, LA)), a1 = lds32(taddr<1, 0>(ph0, LA)),
                            a2 = lds32(taddr<1, 0>(pl1, LA)), a3 = lds32(taddr<1, 0>(ph1, LA)); break;
                    case 2: a0 = lds32(taddr<2, 0>(pl0, LA)), a1 = lds32(taddr<2, 0>(ph0, LA)),
                            a2 = lds32(taddr<2, 0>(pl1, LA)), a3 = lds32(taddr<2, 0>(ph1, LA)); break;
                    default: a0 = lds32(taddr<3, 0>(pl0, LA)), a1 = lds32(taddr<3, 0>(ph0, LA)),
                             a2 = lds32(taddr<3, 0>(pl1, LA)), a3 = lds32(taddr<3, 0>(ph1, LA)); break;
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma16816(acc[nt][4 * hf + k], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
        }
    } else {
        // crumb pair bytes: X -> coordinates 4m, 4m+2 of the 16, Y -> 4m+1, 4m+3
        constexpr uint32_t M2 = 0x33333333u;
        const uint32_t A = v[0][0], B = v[1][0], C = v[2][0], D = v[3][0];
        const uint32_t x0 = (A & M2) | ((B << 2) & ~M2), y0 = ((A >> 2) & M2) | (B & ~M2);
        const uint32_t x1 = (C & M2) | ((D << 2) & ~M2), y1 = ((C >> 2) & M2) | (D & ~M2);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint2 tx0, ty0, tx1, ty1;
            switch (k) {
                case 0: tx0 = lds64(taddr<0, 1>(x0, LB)), ty0 = lds64(taddr<0, 1>(y0, LB)),
                        tx1 = lds64(taddr<0, 1>(x1, LB)), ty1 = lds64(taddr<0, 1>(y1, LB)); break;
                case 1: tx0 = lds64(taddr<1, 1>(x0, LB)), ty0 = lds64(taddr<1, 1>(y0, LB)),
                        tx1 = lds64(taddr<1, 1>(x1, LB)), ty1 = lds64(taddr<1, 1>(y1, LB)); break;
                case 2: tx0 = lds64(taddr<2, 1>(x0, LB)), ty0 = lds64(taddr<2, 1>(y0, LB)),
                        tx1 = lds64(taddr<2, 1>(x1, LB)), ty1 = lds64(taddr<2, 1>(y1, LB)); break;
                default: tx0 = lds64(taddr<3, 1>(x0, LB)), ty0 = lds64(taddr<3, 1>(y0, LB)),
                         tx1 = lds64(taddr<3, 1>(x1, LB)), ty1 = lds64(taddr<3, 1>(y1, LB)); break;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma16816(acc[nt][2 * k], tx0.x, ty0.x, tx1.x, ty1.x, pb[nt][0], pb[nt][1]);
                mma16816(acc[nt][2 * k + 1], tx0.y, ty0.y, tx1.y, ty1.y, pb[nt][0], pb[nt][1]);
            }
        }
    }
}

// Two pages (A, B) of one piece: logits of both, one online-softmax update over
// their 32 rows, then both value contractions.  Lazy maximum: each lane checks its
// own four logits per column against m + kSlack; only when one exceeds it is the
// maximum reduced over the column's lanes and the state rescaled.  l holds this
// lane's partial sum (its rows), reduced over the column's lanes once per piece.
template <int KM, int VM, bool PROD, int NT>
__device__ __forceinline__ void process_pair(const PageRegs<KM, VM, PROD>& ra, const PageRegs<KM, VM, PROD>& rb,
                                             int ntok_a, int ntok_b, const int (&tk)[2], uint32_t klo0,
                                             uint32_t klo1, uint32_t khi0, uint32_t khi1, uint32_t LA, uint32_t LB,
                                             const uint32_t (&bq)[NT][KeyTerm<KM>::kSteps][2],
                                             const uint32_t (&bs)[NT][8][2], float (&m)[NT][2], float (&l)[NT][2],
                                             float (&acc)[NT][8][4]) {
    float sa[NT][2][2], sb[NT][2][2];
    page_logits<KM, VM, PROD, NT>(ra, ntok_a, tk, klo0, klo1, khi0, khi1, LA, LB, bq, bs, sa);
    page_logits<KM, VM, PROD, NT>(rb, ntok_b, tk, klo0, klo1, khi0, khi1, LA, LB, bq, bs, sb);
    // value norms of the rows past a page's valid tokens are not used (a partial page's
    // unused rows may hold anything)
    float van[2], vbn[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        van[i] = (ntok_a >= kPage || tk[i] < ntok_a) ? ra.vn[i] : 0.f;
        vbn[i] = (ntok_b >= kPage || tk[i] < ntok_b) ? rb.vn[i] : 0.f;
    }
    uint32_t pa[NT][2], pbb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        bool over = false;
#pragma unroll
        for (int e = 0; e < 2; ++e)
            over |= fmaxf(fmaxf(sa[nt][0][e], sa[nt][1][e]), fmaxf(sb[nt][0][e], sb[nt][1][e])) > m[nt][e] + kSlack;
        if (__any_sync(0xffffffffu, over)) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float mx = fmaxf(fmaxf(sa[nt][0][e], sa[nt][1][e]), fmaxf(sb[nt][0][e], sb[nt][1][e]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float mnew = mx > m[nt][e] + kSlack ? mx : m[nt][e];
                const float corr = ex2(m[nt][e] - mnew);  // 1 when unchanged, 0 from -inf
                l[nt][e] *= corr;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    acc[nt][mt][e] *= corr;
                    acc[nt][mt][2 + e] *= corr;
                }
                m[nt][e] = mnew;
            }
        }
        float wa[2][2], wb[2][2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float a0 = ex2(sa[nt][0][e] - m[nt][e]), a1 = ex2(sa[nt][1][e] - m[nt][e]);
            const float b0 = ex2(sb[nt][0][e] - m[nt][e]), b1 = ex2(sb[nt][1][e] - m[nt][e]);
            l[nt][e] += (a0 + a1) + (b0 + b1);
            wa[0][e] = a0 * van[0];
            wa[1][e] = a1 * van[1];
            wb[0][e] = b0 * vbn[0];
            wb[1][e] = b1 * vbn[1];
        }
        // P' to the B-operand layout: each 8-row half of the C fragment (row g, heads
        // 2c, 2c + 1) transposed in registers to (rows 2c, 2c + 1, head g)
        pa[nt][0] = movmatrix_trans(f2h2(wa[0][0], wa[0][1]));
        pa[nt][1] = movmatrix_trans(f2h2(wa[1][0], wa[1][1]));
        pbb[nt][0] = movmatrix_trans(f2h2(wb[0][0], wb[0][1]));
        pbb[nt][1] = movmatrix_trans(f2h2(wb[1][0], wb[1][1]));
    }
    page_values<VM, NT>(ra.v, pa, LA, LB, acc);
    page_values<VM, NT>(rb.v, pbb, LA, LB, acc);
}

// Coordinate of row g of m-tile mt among the thread's 16 (16 g + c0; row g+8 -> c0 + 1).
template <int VM>
__device__ __forceinline__ int coord_of(int mt) {
    return VM == kVByte4 ? 2 * mt : 4 * (mt >> 1) + 2 * (mt & 1);
}

// ------------------------------------------------------------------ prologue helpers
// Unit (b Hkv + hk) of page position p of the CTA's page order (0 <= p < total).
__device__ __forceinline__ int unit_at(const DecodeArgs& a, const int* pre, long p) {
    int lo = 0, hi = a.B - 1;  // the last sequence with Hkv pre[b] <= p (it has pages)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((long)a.Hkv * pre[mid] <= p) lo = mid;
        else hi = mid - 1;
    }
    const int np = pre[lo + 1] - pre[lo];
    return lo * a.Hkv + (int)((p - (long)a.Hkv * pre[lo]) / np);
}

// [q' | s] = q [R | S^T] of the query heads of units u_lo .. u_hi (rows u G + h of q,
// contiguous) into the CTA's slots (row u G + h + CTA G of qf), on mma.sync: fp16
// inputs, fp32 accumulation; R^T enters as fp16 hi + lo, S (+-1) is exact and read from
// global memory.  rt: the shared-memory copies [R^T hi | R^T lo], row-major fp16 with the 16-byte pieces of
// row n in the order k ^ (n % 8) (the eight rows of a fragment load meet no bank
// twice).  Per 16-row tile of q (A fragments loaded once) warp w takes the 8-column
// output tiles w, w + kNW, ... of the 32 (q' then s), two at a time.
static_assert(kNW == 8, "rotate_queries: warp w takes the output tiles w, w + 8 (q') and w + 16, w + 24 (s)");
__device__ void rotate_queries(const DecodeArgs& a, const uint8_t* rt, int u_lo, int u_hi, int warp, int lane) {
    const int g = lane >> 2, c = lane & 3;
    const int r_lo = u_lo * a.G, r_end = (u_hi + 1) * a.G;
    const size_t slot_rows = (size_t)blockIdx.x * a.G;
    auto word = [&](const uint8_t* row, int w) {  // word w of a row: piece (w / 4) ^ g, word w % 4
        return *reinterpret_cast<const uint32_t*>(row + ((((w >> 2) ^ g) << 4) | ((w & 3) << 2)));
    };
    // S fragments of the tiles w + 16, w + 24 (rows 8 (w + 8 t) + g of S), loaded with
    // the first tile's q rows
    uint32_t sb[2][8][2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const uint32_t* ps = reinterpret_cast<const uint32_t*>(a.Sh + (size_t)((warp + 8 * t) * 8 + g) * kDim);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) sb[t][ks][0] = ps[8 * ks + c], sb[t][ks][1] = ps[8 * ks + c + 4];
    }
    for (int r0 = r_lo; r0 < r_end; r0 += 16) {
        const bool v0 = r0 + g < r_end, v1 = r0 + g + 8 < r_end;
        const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + (size_t)(v0 ? r0 + g : r_lo) * kDim);
        const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + (size_t)(v1 ? r0 + g + 8 : r_lo) * kDim);
        uint32_t A[8][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            A[ks][0] = v0 ? q0[8 * ks + c] : 0u;
            A[ks][1] = v1 ? q1[8 * ks + c] : 0u;
            A[ks][2] = v0 ? q0[8 * ks + c + 4] : 0u;
            A[ks][3] = v1 ? q1[8 * ks + c + 4] : 0u;
        }
        float d[4][4];  // tiles w, w + 8 (q'), w + 16, w + 24 (s): four independent chains
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int n = (warp + 8 * t) * 8 + g;
                const uint8_t* ph = rt + n * kDim * 2;
                const uint8_t* pl = rt + kDim * kDim * 2 + n * kDim * 2;
                if (ks == 0) mma16816_z(d[t], A[0][0], A[0][1], A[0][2], A[0][3], word(ph, c), word(ph, c + 4));
                else mma16816(d[t], A[ks][0], A[ks][1], A[ks][2], A[ks][3], word(ph, 8 * ks + c), word(ph, 8 * ks + c + 4));
                mma16816(d[t], A[ks][0], A[ks][1], A[ks][2], A[ks][3], word(pl, 8 * ks + c), word(pl, 8 * ks + c + 4));
                if (ks == 0) mma16816_z(d[2 + t], A[0][0], A[0][1], A[0][2], A[0][3], sb[t][0][0], sb[t][0][1]);
                else mma16816(d[2 + t], A[ks][0], A[ks][1], A[ks][2], A[ks][3], sb[t][ks][0], sb[t][ks][1]);
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int col = (warp + 8 * (t & 1)) * 8 + 2 * c, which = t >> 1;
            if (v0)
                *reinterpret_cast<float2*>(a.qf + ((slot_rows + r0 + g) * 2 + which) * kDim + col) =
                    make_float2(d[t][0], d[t][1]);
            if (v1)
                *reinterpret_cast<float2*>(a.qf + ((slot_rows + r0 + g + 8) * 2 + which) * kDim + col) =
                    make_float2(d[t][2], d[t][3]);
        }
    }
}

// ------------------------------------------------------------------ epilogue helpers
// Slot flags: a piece that does not start its unit publishes its partial with the
// launch's epoch; the CTA holding the unit's first page waits for them (bounded).
__device__ __forceinline__ void flag_publish(unsigned long long* f, unsigned long long epoch) {
    __threadfence();
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(f), "l"(epoch) : "memory");
}
__device__ __forceinline__ unsigned long long flag_load(const unsigned long long* f) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
    return v;
}
// Warp-collective bounded wait: each active lane waits for its own flag to reach
// `epoch`; false for a lane whose flag did not within the limit (or once another warp
// of the CTA gave up).
__device__ bool flag_wait_lanes(const unsigned long long* f, bool active, unsigned long long epoch,
                                volatile int* gave_up) {
    bool ok = !active || flag_load(f) == epoch;
    if (__all_sync(0xffffffffu, ok)) return true;
    const uint64_t t0 = sm100::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (!ok) ok = flag_load(f) == epoch;
        if (__all_sync(0xffffffffu, ok) || *gave_up) break;
        if ((it & 63u) == 0 && sm100::globaltimer_ns() - t0 > kWaitNs) {
            *gave_up = 1;
            break;
        }
        __nanosleep(64);
    }
    return ok;
}

// Epilogue scratch in the merge area and the low stages (free once the pages are done).
struct EpiSmem {
    float arow[16][kDim + 4];  // a = acc / l of the compressed part (rotated), then o = R a (rows padded)
    float ml[16][2];       // its M, L
    float trow[16][kDim + 4];  // window: acc (original domain)
    float tml[16][2];      // window: M, L
    float sq[16][kDim];    // window: q of the unit's heads
    float ts[kDecodeTailMax][16];  // window: scores, then probabilities
    float red[2][kNW][16];
    int gave_up;
};
static_assert(sizeof(EpiSmem) <= kEpiBytes, "epilogue scratch fits below the prefix sums");
static_assert(2 * kDim * kDim * 2 <= (kNW * kStages - kLowStages) * kStageBytes, "R hi, lo fit the ring");

// The residual window of unit u (sequence b, kv head hk) for its G heads: rows r0 + h.
__device__ void window_unit(const DecodeArgs& a, EpiSmem& e, int b, int hk, int r0) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = a.G;
    int tl = a.tail_lens[b];
    if (tl < 0 || tl > a.tail_cap) {
        if (tid == 0 && hk == 0) atomicOr(a.err, TQ_DEVERR_SEQLEN);
        tl = 0;
    }
    for (int k = tid; k < G * kDim; k += kThreads) {
        const int h = k / kDim, i = k - h * kDim;
        e.sq[h][i] = __half2float(__ushort_as_half(a.q[((size_t)b * a.Hq + hk * G + h) * kDim + i]));
    }
    __syncthreads();
    float mx[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
    for (int t = tid; t < tl; t += kThreads) {  // scores: a thread per token
        const uint4* kr = reinterpret_cast<const uint4*>(a.tail_k + (((size_t)b * a.tail_cap + t) * a.Hkv + hk) * kDim);
        float sc[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) sc[h] = 0.f;
#pragma unroll 1
        for (int c8 = 0; c8 < kDim / 8; ++c8) {
            const uint4 w = kr[c8];
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const float2 kk = __half22float2(*reinterpret_cast<const __half2*>(&ww[jj]));
#pragma unroll
                for (int h = 0; h < 16; ++h)
                    if (h < G) sc[h] = fmaf(e.sq[h][8 * c8 + 2 * jj + 1], kk.y, fmaf(e.sq[h][8 * c8 + 2 * jj], kk.x, sc[h]));
            }
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            sc[h] *= a.scale_log2;
            e.ts[t][h] = sc[h];
            mx[h] = fmaxf(mx[h], sc[h]);
        }
    }
#pragma unroll
    for (int h = 0; h < 16; ++h) {
        for (int off = 16; off > 0; off >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], off));
        if (lane == 0) e.red[0][warp][h] = mx[h];
    }
    __syncthreads();
    float gm[16], sm[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) {
        gm[h] = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNW; ++w) gm[h] = fmaxf(gm[h], e.red[0][w][h]);
        sm[h] = 0.f;
    }
    for (int t = tid; t < tl; t += kThreads)
#pragma unroll
        for (int h = 0; h < 16; ++h) {
            const float pr = h < G ? exp2f(e.ts[t][h] - gm[h]) : 0.f;
            e.ts[t][h] = pr;
            sm[h] += pr;
        }
#pragma unroll
    for (int h = 0; h < 16; ++h) {
        for (int off = 16; off > 0; off >>= 1) sm[h] += __shfl_xor_sync(0xffffffffu, sm[h], off);
        if (lane == 0) e.red[1][warp][h] = sm[h];
    }
    __syncthreads();
    for (int h = warp; h < G; h += kNW) {  // values: (head h, coordinates 4 lane ..)
        float tL = 0.f;
#pragma unroll
        for (int w = 0; w < kNW; ++w) tL += e.red[1][w][h];
        float4 tA = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int t = 0; t < tl; ++t) {
            const uint2 w = reinterpret_cast<const uint2*>(a.tail_v + (((size_t)b * a.tail_cap + t) * a.Hkv + hk) * kDim)[lane];
            const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
            const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
            const float pr = e.ts[t][h];
            tA.x = fmaf(pr, v0.x, tA.x);
            tA.y = fmaf(pr, v0.y, tA.y);
            tA.z = fmaf(pr, v1.x, tA.z);
            tA.w = fmaf(pr, v1.y, tA.w);
        }
        reinterpret_cast<float4*>(e.trow[r0 + h])[lane] = tA;
        if (lane == 0) e.tml[r0 + h][0] = tl > 0 ? gm[h] : -INFINITY, e.tml[r0 + h][1] = tL;
    }
    __syncthreads();
}

// ------------------------------------------------------------------ the decode kernel
// One persistent CTA per SM (cooperative launch: all CTAs resident) over an equal
// range of the pages of all (sequence, kv head) units:
//   prologue  the CTA's own page prefix sums (last warp) while the other warps build
//             the lookup tables; the page stream starts; q' and s of the units of the
//             range into the CTA's slots;
//   pages     per piece (the range's part of one unit) the warps' online softmax
//             states, merged per piece into the slot (unit + CTA); a piece that does
//             not hold its unit's first page publishes the slot (epoch flag);
//   epilogue  the CTA that holds a unit's first page (or, for units without pages, the
//             CTA of that position) combines the unit's slots by log-sum-exp, adds the
//             residual window, un-rotates (o = R a on mma.sync, R as fp16 hi + lo) and
//             stores, 16 query heads at a time.
template <int KM, int VM, bool PROD, int NT>
__global__ void __launch_bounds__(kThreads, 1) decode_attn_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t base = sm100::smem_u32(smem);
    if (base + kOffPre > kTabAddr) {  // the window leaves no room below the tables
        if (tid == 0) atomicOr(a.err, TQ_DEVERR_INTERNAL);
        return;
    }
    // shared-window address of stage st
    auto stage_addr = [&](uint32_t st) -> uint32_t {
        return st < (uint32_t)kLowStages ? base + kOffLowStages + st * kStageBytes
                                         : kRingAddr + (st - kLowStages) * kStageBytes;
    };
    // ---- prologue: R^T hi and R^T lo into the ring by 16-byte copies (parameters,
    // nothing to wait for; row n's pieces swizzled, see rotate_queries), meanwhile the
    // page prefix sums of the sequences (exclusive; invalid lengths count as empty and
    // raise the error word), this CTA's own copy, and the lookup tables
    {
        constexpr int kPieces = kDim * kDim * 2 / 16;  // per matrix
        for (int i = tid; i < 2 * kPieces; i += kThreads) {
            const int mtx = i / kPieces, o = (i - mtx * kPieces) * 16;
            const int n = o >> 8, k16 = (o >> 4) & 15;
            const uint16_t* src = mtx == 0 ? a.RTh : a.RTl;
            sm100::cp_async16(kRingAddr + mtx * (kPieces * 16) + n * 256 + ((k16 ^ (n & 7)) << 4),
                              reinterpret_cast<const uint8_t*>(src) + o);
        }
        sm100::cp_async_commit();
    }
    int* pre = a.B + 1 <= kPreCap && base + kOffPre + (a.B + 1) * 4 <= kTabAddr
                   ? reinterpret_cast<int*>(smem + kOffPre)
                   : a.prefix + (size_t)blockIdx.x * (a.B + 1);
    if (warp == kNW - 1) {
        int carry = 0;
        for (int b0 = 0; b0 < a.B; b0 += 32) {
            const int b = b0 + lane;
            int n = 0;
            if (b < a.B) {
                const int L = a.seq_lens[b];
                if (seq_len_ok(a, L)) n = (L + kPage - 1) / kPage;
                else if (blockIdx.x == 0) atomicOr(a.err, TQ_DEVERR_SEQLEN);
            }
            int x = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (b < a.B) pre[b] = carry + x - n;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) pre[a.B] = carry;
    }
    if (tid < 256) build_tables<KM, VM, PROD>(a, tid);
    sm100::cp_async_wait<0>();
    __syncthreads();
    const long total = (long)a.Hkv * pre[a.B];
    const long pos0 = total * (long)blockIdx.x / gridDim.x;
    const long end = total * (long)(blockIdx.x + 1) / gridDim.x;
    // q' and s of the units the range touches
    if (pos0 < end)
        rotate_queries(a, smem + (kRingAddr - base), unit_at(a, pre, pos0), unit_at(a, pre, end - 1), warp, lane);
    __syncthreads();  // the slots are written, the ring is free
    using P = PageGeom<KM, VM, PROD>;
    constexpr uint32_t kb = P::kBytes, vb = P::vBytes;
    static_assert(kb % 16 == 0 && vb % 16 == 0 && kb + vb <= kStageBytes, "page chunks in 16-byte pieces");
    static_assert(2 * kDim * kDim * 2 <= (kNW * kStages - kLowStages) * kStageBytes, "R^T hi, lo fit the ring");
    const size_t kstride = (size_t)a.Hkv * kb, vstride = (size_t)a.Hkv * vb;  // bytes per physical block

    // ---- this warp's page stream, by pairs of pages: the issue cursor runs kPairs pairs
    // ahead; pair k of the warp goes to stages 2 (k % kPairs) and + 1 as 16-byte copies
    // by every lane, one commit group per pair (empty past the end), so waiting for all
    // but the newest kPairs - 1 groups means pair k has landed.  vmask bit s: stage s
    // holds a page with a valid block id.
    constexpr int kPairs = kStages / 2;
    PageCursor icur;
    icur.init(a, pre, pos0, end, warp, lane, kb, vb);
    uint32_t issued = 0, vmask = 0;
    // the warp's stages are consecutive (kLowStages is a multiple of kStages)
    static_assert(kLowStages % kStages == 0 && kStages % 2 == 0, "a warp's stages in one region, in pairs");
    const uint32_t wstage_addr = stage_addr(warp * kStages) + 16 * lane;
    const uint8_t* wstage = smem + (stage_addr(warp * kStages) - base);
    auto issue_next = [&]() {
        if (icur.live) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int blk = icur.block(h);
                const uint32_t s = 2 * (issued % kPairs) + h;
                const bool v = blk >= 0 && blk < a.num_blocks;
                vmask = (vmask & ~(1u << s)) | ((uint32_t)v << s);
                if (v) {
                    const uint32_t dst = wstage_addr + s * kStageBytes;
                    const uint8_t* ks = icur.kbase + (size_t)blk * kstride;
                    const uint8_t* vs = icur.vbase + (size_t)blk * vstride;
#pragma unroll
                    for (int i = 0; i < (int)(kb / 512 + 1); ++i)
                        if (i * 32 + lane < (int)(kb / 16)) sm100::cp_async16(dst + 512 * i, ks + 512 * i);
#pragma unroll
                    for (int i = 0; i < (int)(vb / 512 + 1); ++i)
                        if (i * 32 + lane < (int)(vb / 16)) sm100::cp_async16(dst + kb + 512 * i, vs + 512 * i);
                } else if (blk != kNoPage && lane == 0) {
                    atomicOr(a.err, TQ_DEVERR_BLOCK);
                }
            }
            icur.advance(a, warp, lane);
        }
        sm100::cp_async_commit();
        ++issued;
    };
#pragma unroll 1
    for (int i = 0; i < kPairs; ++i) issue_next();

    // ---------------------------------------------------------------- pages
    const int g = lane >> 2, c = lane & 3;
    // rows of this thread in the page: score rows g, g+8; value rows 2c, 2c+1, 2c+8, 2c+9
    const int tk[2] = {row_token(g), row_token(g + 8)};
    const PageOffs po = page_offsets<KM, VM, PROD>(row_token(g), row_token(2 * c), row_token(2 * c + 1), g, c);
    // lane offsets inside a table entry: LA = {lane*4 (A), 128 + lane*4 (B)}, LB = {128 +
    // (lane%8)*16 (B, 16-byte entries), (lane%16)*8 (A, 8-byte entries)}; bytes 2, 3 = 0x01, 0x00
    const uint32_t LA = (uint32_t)(lane * 4) | ((uint32_t)(128 + lane * 4) << 8) | 0x10000u;
    const uint32_t LB = (uint32_t)(128 + (lane & 7) * 16) | ((uint32_t)((lane & 15) * 8) << 8) | 0x10000u;
    // 3-bit key codes: low / high bytes of the 8 fp16 levels
    uint32_t klo0 = 0, klo1 = 0, khi0 = 0, khi1 = 0;
    if (KM == kKPrmt) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t hb = __half_as_ushort(cb_half(a.cbk, k));
            if (k < 4) {
                klo0 |= (hb & 0xffu) << (8 * k);
                khi0 |= (hb >> 8) << (8 * k);
            } else {
                klo1 |= (hb & 0xffu) << (8 * (k - 4));
                khi1 |= (hb >> 8) << (8 * (k - 4));
            }
        }
    }
    float* wml = reinterpret_cast<float*>(smem + kOffML);      // [warp][2][4]: m then l
    float* wacc = reinterpret_cast<float*>(smem + kOffMerge);  // [warp][4 heads][128]
    uint32_t cnt = 0;  // pages this warp has consumed (all pieces)
    Pieces it;
    it.init(a, pre, pos0, end);
    int b, hk, p0, p1;
    constexpr int KS = KeyTerm<KM>::kSteps;
    const long n_slots = (long)a.B * a.Hkv + gridDim.x;
    while (it.next(a, b, hk, p0, p1)) {
        const int unit = b * a.Hkv + hk;
        if (!TQ_DCHECK(unit >= 0 && unit + (long)blockIdx.x < n_slots && p0 >= 0 && p1 <= a.max_blocks, a.err)) break;
        const int Ls = a.seq_lens[b];  // valid: the sequence has pages
        // query fragments (B operand) of heads nt*8 + g: key term and sign term
        uint32_t bq[NT][KS][2], bs[NT][8][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = nt * 8 + g;
            if (h < a.G) {
                const float4* src =
                    reinterpret_cast<const float4*>(a.qf + (((size_t)(unit + blockIdx.x) * a.G + h) * 2) * kDim + 32 * c);
                float4 x[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = src[i];
                if (KM == kKByte2) {
#pragma unroll
                    for (int ks = 0; ks < 16; ++ks) {
                        const float4 v = x[ks >> 1];
                        const float q0 = (ks & 1) ? v.z : v.x, q1 = (ks & 1) ? v.w : v.y;
                        bq[nt][ks][0] = f2h2(a.kbeta * q0, a.kalpha * q0);
                        bq[nt][ks][1] = f2h2(a.kbeta * q1, a.kalpha * q1);
                    }
                } else {
                    const float ksc = a.kscale;
#pragma unroll
                    for (int ks = 0; ks < KS && ks < 8; ++ks) {
                        bq[nt][ks][0] = f2h2(ksc * x[ks].x, ksc * x[ks].y);
                        bq[nt][ks][1] = f2h2(ksc * x[ks].z, ksc * x[ks].w);
                    }
                }
                if (PROD) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float4 v = src[i + kDim / 4];
                        bs[nt][i][0] = f2h2(v.x, v.y);
                        bs[nt][i][1] = f2h2(v.z, v.w);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < KS; ++i) bq[nt][i][0] = bq[nt][i][1] = 0u;
#pragma unroll
                for (int i = 0; i < 8; ++i) bs[nt][i][0] = bs[nt][i][1] = 0u;
            }
        }
        float m[NT][2], l[NT][2], acc[NT][8][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) acc[nt][mt][0] = acc[nt][mt][1] = acc[nt][mt][2] = acc[nt][mt][3] = 0.f;
        }

        // ---- the warp's page pairs of the piece: p0 + 2 warp + {0, 1}, + 2 kNW, ...
        const int nj = p0 + 2 * warp < p1 ? (p1 - p0 - 2 * warp + 2 * kNW - 1) / (2 * kNW) : 0;
        for (int j = 0; j < nj; ++j) {
            const uint32_t s = 2 * (cnt % kPairs);
            sm100::cp_async_wait<kPairs - 1>();  // this lane's copies of the pair
            __syncwarp();                          // ... and every other lane's
            const int page = p0 + 2 * warp + j * (2 * kNW);
            // the pages' bytes into registers, then the stages go back to the stream
            // before the pages are worked, so every stage is in flight meanwhile
            const bool va = (vmask >> s) & 1u, vbb = (vmask >> (s + 1)) & 1u;
            PageRegs<KM, VM, PROD> ra, rb;
            if (va) load_page<KM, VM, PROD>(ra, wstage + s * kStageBytes, po, a.qscale, a.sscale);
            else ra = PageRegs<KM, VM, PROD>{};
            if (vbb) load_page<KM, VM, PROD>(rb, wstage + (s + 1) * kStageBytes, po, a.qscale, a.sscale);
            else rb = PageRegs<KM, VM, PROD>{};
            __syncwarp();  // every lane is done with the stages before they are refilled
            ++cnt;
            issue_next();
            const int ntok_a = va ? min(kPage, Ls - page * kPage) : 0;
            const int ntok_b = vbb && page + 1 < p1 ? min(kPage, Ls - (page + 1) * kPage) : 0;
            process_pair<KM, VM, PROD, NT>(ra, rb, ntok_a, ntok_b, tk, klo0, klo1, khi0, khi1, LA, LB, bq, bs, m, l,
                                           acc);
        }

        // ---- merge the CTA's warps (one tile of 8 heads at a time; coordinates back in order)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {  // l over the column's lanes
                l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], 4);
                l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], 8);
                l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], 16);
            }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {  // heads nt*8 + 4 qq + (0..3)
                if (nt * 8 + 4 * qq >= a.G) break;
                __syncthreads();  // the previous merge is done with the area
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int hh = 2 * c + e;
                    if ((hh >> 2) != qq) continue;
                    const int hl = hh & 3;
                    if (g == 0) {
                        wml[(warp * 2 + 0) * 4 + hl] = m[nt][e];
                        wml[(warp * 2 + 1) * 4 + hl] = l[nt][e];
                    }
#pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        const int c0 = 16 * g + coord_of<VM>(mt);
                        wacc[(warp * 4 + hl) * kDim + c0] = acc[nt][mt][e];
                        wacc[(warp * 4 + hl) * kDim + c0 + 1] = acc[nt][mt][2 + e];
                    }
                }
                __syncthreads();
                // thread = (head hl = warp, coordinates 4 lane .. 4 lane + 3) for the first 4 warps
                const int hl = warp, h = nt * 8 + 4 * qq + hl;
                if (hl < 4 && h < a.G) {
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kNW; ++w) M = fmaxf(M, wml[(w * 2) * 4 + hl]);
                    float Lsum = 0.f;
                    float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int w = 0; w < kNW; ++w) {
                        const float mw = wml[(w * 2) * 4 + hl];
                        const float wt = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
                        Lsum = fmaf(wt, wml[(w * 2 + 1) * 4 + hl], Lsum);
                        const float4 v = reinterpret_cast<const float4*>(wacc + (w * 4 + hl) * kDim)[lane];
                        A.x = fmaf(wt, v.x, A.x);
                        A.y = fmaf(wt, v.y, A.y);
                        A.z = fmaf(wt, v.z, A.z);
                        A.w = fmaf(wt, v.w, A.w);
                    }
                    float* part = a.partial + (((size_t)unit + blockIdx.x) * a.G + h) * kPartStride;
                    if (lane == 0) *reinterpret_cast<float2*>(part) = make_float2(M, Lsum);
                    reinterpret_cast<float2*>(part + 2)[2 * lane] = make_float2(A.x, A.y);
                    reinterpret_cast<float2*>(part + 2)[2 * lane + 1] = make_float2(A.z, A.w);
                }
            }
        // a piece that does not start its unit publishes the slot for the unit's merge
        if (p0 > 0) {
            __syncthreads();  // every head of the slot is written
            if (tid == 0 && !a.stall) flag_publish(a.flags + unit + blockIdx.x, a.epoch);
        }
    }
    sm100::cp_async_wait<0>();  // only empty groups remain; nothing is in flight
    __syncthreads();            // the stage ring is free for the epilogue

    // ---------------------------------------------------------------- epilogue
    EpiSmem& ep = *reinterpret_cast<EpiSmem*>(smem + kOffMerge);
    if (tid == 0) ep.gave_up = 0;
    // R hi and lo into the ring, row i's 16-byte pieces in the order k ^ (i % 8) (the
    // fragment loads below meet no bank twice); they land while the slots are read
    {
        constexpr int kPieces = kDim * kDim * 2 / 16;  // per matrix
        for (int i = tid; i < 2 * kPieces; i += kThreads) {
            const int mtx = i / kPieces, o = (i - mtx * kPieces) * 16;
            const int n = o >> 8, k16 = (o >> 4) & 15;
            sm100::cp_async16(kRingAddr + mtx * (kPieces * 16) + n * 256 + ((k16 ^ (n & 7)) << 4),
                              reinterpret_cast<const uint8_t*>(mtx == 0 ? a.Rh : a.Rl) + o);
        }
        sm100::cp_async_commit();
    }
    const uint8_t* rsm = smem + (kRingAddr - base);
    __syncthreads();
    const int grid = gridDim.x, cta = blockIdx.x;
    // The units this CTA finishes: first page position in [pos0, end), or (last CTA) at
    // total -- units without pages sit at their sequence's position.  Sequences from the
    // first one that reaches pos0, in batches of 16 / G units (16 rows).
    int b_lo;
    {
        int lo = 0, hi = a.B;  // first b with Hkv pre[b] >= pos0 or Hkv pre[b + 1] > pos0
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if ((long)a.Hkv * pre[mid] >= pos0 || (long)a.Hkv * pre[mid + 1] > pos0) hi = mid;
            else lo = mid + 1;
        }
        b_lo = lo;
    }
    const bool last_cta = cta == grid - 1;
    const int per_batch = 16 / a.G;
    int ulist[16];
    int nu = 0;
    auto finish_batch = [&]() {
        const int rows = nu * a.G;
        // 1. log-sum-exp of each row's slots, thread = (row r, coordinates 4 lane ..);
        // the slots' flags and (m, l) a lane per slot, 32 slots at a time
        for (int r = warp; r < 16; r += kNW) {
            float M = -INFINITY, L = 0.f;
            float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < rows) {
                const int j = r / a.G, h = r - j * a.G;
                const int u = ulist[j], b = u / a.Hkv, hk = u - b * a.Hkv;
                const int np = pre[b + 1] - pre[b];
                if (np > 0) {
                    const long first = (long)a.Hkv * pre[b] + (long)hk * np, last = first + np - 1;
                    const int ncon = (int)(((last + 1) * grid - 1) / total) - cta + 1;  // slots u + cta ..
                    for (int i0 = 0; i0 < ncon; i0 += 32) {
                        const int i = i0 + lane;
                        const bool later = i > 0 && i < ncon;
                        const bool ok = flag_wait_lanes(a.flags + u + cta + (later ? i : 0), later, a.epoch, &ep.gave_up);
                        if (!__all_sync(0xffffffffu, ok) && lane == 0)
                            atomicOr(a.err, TQ_DEVERR_TIMEOUT);  // (the slot is read all the same)
                        const size_t row0 = ((size_t)u + cta + i0) * a.G + h;  // slot u + cta + i0, head h
                        const int n = min(32, ncon - i0);
                        // the first (up to) 8 slots' coordinates are loaded with the (m, l)
                        float4 pa[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            pa[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (k < n) {
                                const float* pp = a.partial + (row0 + (size_t)k * a.G) * kPartStride + 2;
                                const float2 x = __ldcg(reinterpret_cast<const float2*>(pp) + 2 * lane);
                                const float2 y = __ldcg(reinterpret_cast<const float2*>(pp) + 2 * lane + 1);
                                pa[k] = make_float4(x.x, x.y, y.x, y.y);
                            }
                        }
                        float2 mli = make_float2(-INFINITY, 0.f);
                        if (i < ncon) mli = __ldcg(reinterpret_cast<const float2*>(a.partial + (row0 + (size_t)lane * a.G) * kPartStride));
                        float mx = mli.x;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                        const float mn = fmaxf(M, mx);
                        if (mn == -INFINITY) continue;  // nothing in these slots yet
                        const float sa = M == -INFINITY ? 0.f : exp2f(M - mn);
                        const float wi = mli.x == -INFINITY ? 0.f : exp2f(mli.x - mn);
                        float li = wi * mli.y;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) li += __shfl_xor_sync(0xffffffffu, li, o);
                        L = fmaf(L, sa, li);
                        A.x *= sa, A.y *= sa, A.z *= sa, A.w *= sa;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float w = __shfl_sync(0xffffffffu, wi, k);  // 0 past n
                            A.x = fmaf(w, pa[k].x, A.x);
                            A.y = fmaf(w, pa[k].y, A.y);
                            A.z = fmaf(w, pa[k].z, A.z);
                            A.w = fmaf(w, pa[k].w, A.w);
                        }
#pragma unroll 4
                        for (int k = 8; k < n; ++k) {
                            const float w = __shfl_sync(0xffffffffu, wi, k);
                            const float* pp = a.partial + (row0 + (size_t)k * a.G) * kPartStride + 2;
                            const float2 x = __ldcg(reinterpret_cast<const float2*>(pp) + 2 * lane);
                            const float2 y = __ldcg(reinterpret_cast<const float2*>(pp) + 2 * lane + 1);
                            A.x = fmaf(w, x.x, A.x);
                            A.y = fmaf(w, x.y, A.y);
                            A.z = fmaf(w, y.x, A.z);
                            A.w = fmaf(w, y.y, A.w);
                        }
                        M = mn;
                    }
                }
            }
            // a = acc / (l sqrt(d)): the value norms entered without their 1/sqrt(d)
            const float inv = L > 0.f ? 0.08838834764831845f / L : 0.f;
            reinterpret_cast<float4*>(ep.arow[r])[lane] = make_float4(A.x * inv, A.y * inv, A.z * inv, A.w * inv);
            if (lane == 0) ep.ml[r][0] = M, ep.ml[r][1] = L;
        }
        // 2. the residual windows of the batch's units
        if (a.tail_k)
            for (int j = 0; j < nu; ++j) window_unit(a, ep, ulist[j] / a.Hkv, ulist[j] % a.Hkv, j * a.G);
        __syncthreads();  // a, ml complete
        // 3. o = R a: rows = the batch's heads, columns = outputs; warp w < 8 takes the
        // output tiles w and w + 8 (B fragments: column n = output i, K-pair =
        // consecutive j of row i of R)
        sm100::cp_async_wait<0>();
        __syncthreads();  // R landed (every thread's copies)
        float d[2][4];
        if (warp < 8) {
            uint32_t ah[8][4], al[8][4];
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {  // rows g / g + 8, k-columns 2c.. / 2c + 8..
                    const float2 x = *reinterpret_cast<const float2*>(&ep.arow[g + 8 * (q4 & 1)][16 * ks + 8 * (q4 >> 1) + 2 * c]);
                    const __half2 hi = __floats2half2_rn(x.x, x.y);
                    const float2 hif = __half22float2(hi);
                    const __half2 lo = __floats2half2_rn(x.x - hif.x, x.y - hif.y);
                    ah[ks][q4] = *reinterpret_cast<const uint32_t*>(&hi);
                    al[ks][q4] = *reinterpret_cast<const uint32_t*>(&lo);
                }
#pragma unroll
            for (int t = 0; t < 2; ++t) {
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) d[t][e4] = 0.f;
                const int i = (warp + 8 * t) * 8 + g;
                const uint8_t* rh = rsm + i * 256;
                const uint8_t* rl = rsm + kDim * kDim * 2 + i * 256;
                auto word = [&](const uint8_t* row, int w) {  // word w: piece (w / 4) ^ g
                    return *reinterpret_cast<const uint32_t*>(row + ((((w >> 2) ^ g) << 4) | ((w & 3) << 2)));
                };
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t h0 = word(rh, 8 * ks + c), h1 = word(rh, 8 * ks + c + 4);
                    const uint32_t l0 = word(rl, 8 * ks + c), l1 = word(rl, 8 * ks + c + 4);
                    mma16816(d[t], al[ks][0], al[ks][1], al[ks][2], al[ks][3], h0, h1);
                    mma16816(d[t], ah[ks][0], ah[ks][1], ah[ks][2], ah[ks][3], l0, l1);
                    mma16816(d[t], ah[ks][0], ah[ks][1], ah[ks][2], ah[ks][3], h0, h1);
                }
            }
        }
        __syncthreads();  // every warp has read a
        if (warp < 8) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int col = (warp + 8 * t) * 8 + 2 * c;
                *reinterpret_cast<float2*>(&ep.arow[g][col]) = make_float2(d[t][0], d[t][1]);
                *reinterpret_cast<float2*>(&ep.arow[g + 8][col]) = make_float2(d[t][2], d[t][3]);
            }
        }
        __syncthreads();
        // 4. combine with the window and store: thread = (row r, coordinates 4 lane ..)
        for (int r = warp; r < rows; r += kNW) {
            const int j = r / a.G, h = r - j * a.G;
            float4 o = reinterpret_cast<const float4*>(ep.arow[r])[lane];
            if (a.tail_k) {
                const float Mc = ep.ml[r][0], Lc = ep.ml[r][1], tM = ep.tml[r][0], tL = ep.tml[r][1];
                const float4 tA = reinterpret_cast<const float4*>(ep.trow[r])[lane];
                const float Mx = fmaxf(Mc, tM);
                const float wc = Lc > 0.f ? exp2f(Mc - Mx) * Lc : 0.f;
                const float et = tL > 0.f ? exp2f(tM - Mx) : 0.f;
                const float den = wc + et * tL;
                const float inv = den > 0.f ? 1.f / den : 0.f;
                o = make_float4((wc * o.x + et * tA.x) * inv, (wc * o.y + et * tA.y) * inv,
                                (wc * o.z + et * tA.z) * inv, (wc * o.w + et * tA.w) * inv);
            }
            const size_t oi = ((size_t)ulist[j] * a.G + h) * kDim + 4 * lane;
            if (a.out_fp32) {
                *reinterpret_cast<float4*>(static_cast<float*>(a.out) + oi) = o;
            } else {
                const __half2 lo = __floats2half2_rn(o.x, o.y), hi = __floats2half2_rn(o.z, o.w);
                *reinterpret_cast<uint2*>(static_cast<__half*>(a.out) + oi) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
            }
        }
        __syncthreads();  // the scratch is free for the next batch
        nu = 0;
    };
    for (int b = b_lo; b < a.B; ++b) {
        const long s0 = (long)a.Hkv * pre[b];
        if (s0 >= end && !(last_cta && s0 == total)) break;
        const int np = pre[b + 1] - pre[b];
        for (int hk = 0; hk < a.Hkv; ++hk) {
            const long first = s0 + (long)hk * np;
            if (!((first >= pos0 && first < end) || (last_cta && first == total))) continue;
            if (!TQ_DCHECK(nu < per_batch && b * a.Hkv + hk + (long)cta < n_slots, a.err)) continue;
            ulist[nu++] = b * a.Hkv + hk;
            if (nu == per_batch) finish_batch();
        }
    }
    if (nu > 0) finish_batch();
}

int kmode_of(const tq_ctx* ctx) {
    const int w = ctx->cb_key.width;
    if (w == 4) return ctx->cb_key.levels <= 8 ? kKPrmt : kKByte4;
    if (w == 2) return kKByte2;
    return kKBit1;
}

template <int KM, int VM, bool PROD, int NT>
cudaError_t launch_attn(const DecodeArgs& a, int grid, cudaStream_t stream) {
    using P = PageGeom<KM, VM, PROD>;
    if (a.lk.bytes != P::kBytes || a.lv.bytes != P::vBytes || a.lk.code_row != P::kRow ||
        a.lv.code_row != P::vRow || a.lk.norm_off != P::kNorm || a.lv.norm_off != P::vNorm ||
        (PROD && (a.lk.signs_off != P::kSigns || a.lk.gamma_off != P::kGamma)))
        return cudaErrorInvalidValue;  // the kernel's fixed geometry must be the context's
    auto k = decode_attn_kernel<KM, VM, PROD, NT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    // cooperative: every CTA resident at once (a unit's merge waits for later CTAs' slots)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, a);
}

// Launch tags: a process-wide counter from a time-derived start, so that no two
// launches share one and stale or foreign workspace contents never match.
std::atomic<unsigned long long> g_epoch{0};
unsigned long long next_epoch() {
    unsigned long long e = g_epoch.fetch_add(1, std::memory_order_relaxed);
    if (e == 0) {  // first use: start from the clock, away from 0 and all-ones patterns
        const unsigned long long t =
            (unsigned long long)std::chrono::high_resolution_clock::now().time_since_epoch().count();
        unsigned long long expect = 1;
        const unsigned long long start = (t * 0x9E3779B97F4A7C15ull) | (1ull << 40);
        g_epoch.compare_exchange_strong(expect, start + 1, std::memory_order_relaxed);
        return start;
    }
    return e;
}

}  // namespace

DecodePlan plan_decode(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_seq_len) {
    DecodePlan p{};
    p.max_pages = (max_seq_len + kPage - 1) / kPage;
    const long resident = (long)ctx->sm_count;  // one CTA per SM
    const long units = (long)B * Hkv;
    // every SM, but at least 2 pages (one pair) per warp for small batches (llama8b,
    // 2048 pages: 128 CTAs took 25 us against 27.5 with 64 and 29 with 148)
    long grid = (units * p.max_pages + 2 * kNW - 1) / (2 * kNW);
    if (grid > resident) grid = resident;
    if (grid < 1) grid = 1;
    p.grid = (int)grid;
    p.slots = (int)(units + grid);
    const int G = Hkv > 0 ? Hq / Hkv : 0;
    auto take = [](size_t& off, size_t n) {
        const size_t at = off;
        off = (off + n + 255) & ~size_t(255);
        return at;
    };
    size_t off = 0;
    p.qprep_off = take(off, (size_t)p.slots * G * 2 * kDim * sizeof(float));
    p.partial_off = take(off, (size_t)p.slots * G * kPartStride * sizeof(float));
    p.flags_off = take(off, (size_t)p.slots * sizeof(unsigned long long));
    p.prefix_off = take(off, (size_t)grid * (B + 1) * sizeof(int));
    p.bytes = off;
    return p;
}

cudaError_t launch_decode(const tq_ctx* ctx, const DecodePlan& plan, const uint16_t* q, const uint8_t* kc,
                          const uint8_t* vc, int num_blocks, const int32_t* block_table, int max_blocks,
                          const int32_t* seq_lens, int B, int Hq, int Hkv, int max_seq_len, const DecodeTail& tail,
                          float scale, void* out, int out_fp32, void* workspace, cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecodeArgs a{};
    a.q = q;
    a.qf = reinterpret_cast<float*>(ws + plan.qprep_off);
    a.kc = kc;
    a.vc = vc;
    a.num_blocks = num_blocks;
    a.block_table = block_table;
    a.max_blocks = max_blocks;
    a.seq_lens = seq_lens;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = Hq / Hkv;
    a.max_seq_len = max_seq_len;
    const float scale_log2 = scale * 1.4426950408889634f;
    a.scale_log2 = scale_log2;
    a.tail_k = tail.k;
    a.tail_v = tail.v;
    a.tail_lens = tail.lens;
    a.tail_cap = tail.cap;
    a.qscale = scale_log2 / sqrtf((float)kDim);
    a.sscale = scale_log2 * 1.2533141373155003f / (float)kDim;
    a.partial = reinterpret_cast<float*>(ws + plan.partial_off);
    a.flags = reinterpret_cast<unsigned long long*>(ws + plan.flags_off);
    a.epoch = next_epoch();
    a.prefix = reinterpret_cast<int*>(ws + plan.prefix_off);
    a.RTh = ctx->dev.RTh;
    a.RTl = ctx->dev.RTl;
    a.Sh = ctx->dev.Sh;
    a.Rh = ctx->dev.Rh;
    a.Rl = ctx->dev.Rl;
    a.cbk = ctx->cb_key;
    a.cbv = ctx->cb_value;
    a.lk = ctx->lay_key;
    a.lv = ctx->lay_value;
    a.out = out;
    a.out_fp32 = out_fp32;
    a.err = ctx->dev_error;
    const int KM = kmode_of(ctx);
    // +-1 bit planes of low-bit key codes (symmetric codebooks, exact up to rounding):
    // 1 bit: c[b] = c1 (2b - 1); 2 bits: c[2 b1 + b0] = alpha (2 b1 - 1) + beta (2 b0 - 1)
    const float* ck = ctx->cb_key.c;
    a.kscale = KM == kKBit1 ? 0.5f * (ck[1] - ck[0]) : 1.f;
    a.kalpha = KM == kKByte2 ? 0.25f * (ck[3] + ck[2] - ck[1] - ck[0]) : 0.f;
    a.kbeta = KM == kKByte2 ? 0.25f * (ck[3] - ck[2] + ck[1] - ck[0]) : 0.f;
    a.stall = take_stall(ctx) ? 1 : 0;

    const int VM = ctx->cb_value.width == 4 ? kVByte4 : kVByte2;
    const bool prod = ctx->lay_key.prod;
    const int NT = a.G <= 8 ? 1 : 2;
    const int grid = plan.grid;
    cudaError_t e = cudaErrorInvalidValue;
#define TQ_DEC_CASE(K_, V_, P_, N_) \
    if (KM == K_ && VM == V_ && prod == P_ && NT == N_) e = launch_attn<K_, V_, P_, N_>(a, grid, stream);
#define TQ_DEC_NT(K_, V_, P_) TQ_DEC_CASE(K_, V_, P_, 1) TQ_DEC_CASE(K_, V_, P_, 2)
    TQ_DEC_NT(kKPrmt, kVByte4, true)    // bits 4, prod keys (3-bit codes)
    TQ_DEC_NT(kKByte2, kVByte4, true)   // bits 3, prod keys (2-bit codes)
    TQ_DEC_NT(kKBit1, kVByte2, true)    // bits 2, prod keys (1-bit codes)
    TQ_DEC_NT(kKByte4, kVByte4, false)  // bits 4, MSE keys
    TQ_DEC_NT(kKPrmt, kVByte4, false)   // bits 3, MSE keys
    TQ_DEC_NT(kKByte2, kVByte2, false)  // bits 2, MSE keys
#undef TQ_DEC_NT
#undef TQ_DEC_CASE
    if (e != cudaSuccess) return e;
    count_launches(1);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ allocation-free variant
// The scratch of tq_decode_attention_noalloc: one array per device, reserved when
// the module loads and kept until the process exits.  Host code cannot use the
// symbol itself (that is a host-side stand-in); its device address is looked up
// once per device with cudaGetSymbolAddress and cached.
namespace {
__device__ __align__(256) uint8_t g_noalloc_scratch[TQ_NOALLOC_SCRATCH_BYTES];
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

cudaError_t noalloc_scratch(int device, void** out) {
    if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[device]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // with `device` current
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[device] = p;
    }
    *out = g_noalloc_ptr[device];
    return cudaSuccess;
}

}  // namespace tq

extern "C" tq_status tq_decode_attention_noalloc(const tq_ctx* ctx, const uint16_t* q, const uint8_t* k_cache,
                                                 const uint8_t* v_cache, int num_blocks, const int32_t* block_table,
                                                 int max_blocks, const int32_t* seq_lens, int B, int Hq, int Hkv,
                                                 int max_seq_len, float scale, void* out, int out_fp32,
                                                 void* stream) {
    if (!ctx || ctx->host_only) return TQ_ERR_INVALID_ARG;
    if (B > 0) {
        const size_t need = tq_decode_workspace_bytes(ctx, B, Hq, Hkv, max_seq_len);
        if (need > TQ_NOALLOC_SCRATCH_BYTES) return TQ_ERR_INVALID_ARG;
    }
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) {
        cudaGetLastError();
        return TQ_ERR_CUDA;
    }
    if (cur != ctx->device) return TQ_ERR_INVALID_ARG;
    void* scratch = nullptr;
    if (tq::noalloc_scratch(cur, &scratch) != cudaSuccess) {
        cudaGetLastError();
        return TQ_ERR_CUDA;
    }
    return tq_decode_attention(ctx, q, k_cache, v_cache, num_blocks, block_table, max_blocks, seq_lens, B, Hq, Hkv,
                               max_seq_len, scale, out, out_fp32, scratch, TQ_NOALLOC_SCRATCH_BYTES, stream);
}
