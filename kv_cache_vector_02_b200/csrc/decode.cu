// Split-K decode attention over the paged compressed cache, on tensor cores.
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…":
//   - section "注意力计算的特殊挑战与QJL校正": score estimator
//       <q,k> ~ <q,k_hat> + gamma sqrt(pi/2)/d <S q, sign(S r)>
//   - section "架构设计" / "关键工程改进": Paged Decode as split-K FlashDecoding.
// Everything happens in the rotated domain: <q, k_hat> = n/sqrt(d) <R^T q, c[idx]>,
// the value sum is accumulated as sum_t p_t n_t c[idx_t]/sqrt(d) and un-rotated
// once per query head (o = R acc / l).
//
// Kernels:
//   prep   one CTA per (sequence, kv head): q' = R^T q and s = S q for its G query
//          heads, stored fp16.
//   split  persistent CTAs over items (sequence, kv head, page range); each warp
//          takes one 16-token page at a time:
//            scores  D[16 tok x 8 heads] = sum_k Khat[tok][k] q'[k][h]   (mma m16n8k16)
//                    plus the sign term with +-1 fragments against s
//            softmax online, base 2, per head column
//            values  D[16 coords x 8 heads] += Vhat^T[coord][tok] P'[tok][h]
//          Packed codes become fp16 fragments in registers: key codes (<= 8 levels)
//          through byte permutes of an 8-entry table, sign nibbles and value bytes
//          through small shared-memory tables (the value table is replicated per
//          lane so a warp's 32 lookups never share a bank).  Coordinates are
//          permuted inside each contraction so that a thread's fragment elements
//          are contiguous packed bytes.  The warps of a CTA merge their states;
//          each item's partial (m, l, acc) goes to the workspace.
//   merge  log-sum-exp combination of the splits, division by l, un-rotation.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "device_util.cuh"
#include "sm100.cuh"

namespace tq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxG = 16;
constexpr int kPartStride = kDim + 2;  // m, l, acc[128]

enum KMode { kKPrmt = 0, kKByte4 = 1, kKByte2 = 2, kKBit1 = 3 };
enum VMode { kVByte4 = 0, kVByte2 = 1 };

struct DecodeArgs {
    const uint16_t* q;
    __half* qf;  // [B][Hq][2][128] fp16: q' then s
    const uint8_t* kc;
    const uint8_t* vc;
    int num_blocks;
    const int32_t* block_table;
    int max_blocks;
    const int32_t* seq_lens;
    int B, Hq, Hkv, G, max_seq_len;
    float scale_log2;  // softmax scale * log2(e)
    float* partial;    // [slots][G][130]: m, l, acc (rotated domain)
    int* prefix;       // [B + 1] pages of the sequences before b (prep writes it)
    int split_grid;    // CTAs of the split kernel
    int merge_sg;      // merge: groups of 128 threads per item, each on every merge_sg-th slot
    const float* RT;       // row-major R^T (fp32)
    const uint16_t* RTh;   // fp16 R^T hi / lo, S (row-major)
    const uint16_t* RTl;
    const uint16_t* Sh;
    float qscale, sscale;  // scale*log2(e)/sqrt(d), scale*log2(e)*sqrt(pi/2)/d
    Codebook cbk, cbv;
    ChunkLayout lk, lv;
    void* out;
    int out_fp32;
    uint32_t* err;
};

__device__ __forceinline__ bool seq_len_ok(const DecodeArgs& a, int L) {
    return L >= 0 && L <= a.max_blocks * kPage && L <= a.max_seq_len;
}

// ------------------------------------------------------------------ helpers
using sm100::griddep_wait;
using sm100::griddep_launch_dependents;

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ prep
// [q' | s] = q [R | S^T] for 16 query heads per CTA, on mma.sync (fp16 inputs, fp32
// accumulation; R^T enters as fp16 hi + lo, S is exact).  CTA (x, y), warp w
// computes output columns 8 (8 y + w) .. +7 of the 256 (q' then s).
constexpr int kPrepThreads = 256;
__global__ void __launch_bounds__(kPrepThreads) decode_prep_kernel(DecodeArgs a) {
    griddep_wait();  // q and seq_lens may come from the kernel before
    const int NQ = a.B * a.Hq;
    const int h0 = blockIdx.x * 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const bool r0 = h0 + g < NQ, r1 = h0 + g + 8 < NQ;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + (size_t)(r0 ? h0 + g : 0) * kDim);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + (size_t)(r1 ? h0 + g + 8 : 0) * kDim);
    if (blockIdx.x == 0 && blockIdx.y == 0) {
        // pages per sequence (invalid lengths count as empty and raise the error
        // word) and their exclusive prefix sum, in chunks of 256 sequences
        __shared__ int sc[kPrepThreads];
        int carry = 0;
        for (int b0 = 0; b0 < a.B; b0 += kPrepThreads) {
            const int b = b0 + (int)threadIdx.x;
            int n = 0;
            if (b < a.B) {
                const int L = a.seq_lens[b];
                if (seq_len_ok(a, L)) n = (L + kPage - 1) / kPage;
                else atomicOr(a.err, TQ_DEVERR_SEQLEN);
            }
            sc[threadIdx.x] = n;
            __syncthreads();
            for (int off = 1; off < kPrepThreads; off <<= 1) {  // inclusive scan
                const int v = threadIdx.x >= off ? sc[threadIdx.x - off] : 0;
                __syncthreads();
                sc[threadIdx.x] += v;
                __syncthreads();
            }
            if (b < a.B) a.prefix[b] = carry + sc[threadIdx.x] - n;
            carry += sc[kPrepThreads - 1];
            __syncthreads();
        }
        if (threadIdx.x == 0) a.prefix[a.B] = carry;
    }
    griddep_launch_dependents();  // the split kernel may start its prologue
    uint32_t A[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        A[ks][0] = r0 ? q0[8 * ks + c] : 0u;
        A[ks][1] = r1 ? q1[8 * ks + c] : 0u;
        A[ks][2] = r0 ? q0[8 * ks + c + 4] : 0u;
        A[ks][3] = r1 ? q1[8 * ks + c + 4] : 0u;
    }
    {
        const int nt = blockIdx.y * 8 + warp;  // 0..15 -> q', 16..31 -> s
        const bool isq = nt < 16;
        const int n = (nt & 15) * 8 + g;
        const uint32_t* bh = reinterpret_cast<const uint32_t*>((isq ? a.RTh : a.Sh) + (size_t)n * kDim);
        const uint32_t* bl = reinterpret_cast<const uint32_t*>(a.RTl + (size_t)n * kDim);
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            mma16816(d, A[ks][0], A[ks][1], A[ks][2], A[ks][3], bh[8 * ks + c], bh[8 * ks + c + 4]);
            if (isq) mma16816(d, A[ks][0], A[ks][1], A[ks][2], A[ks][3], bl[8 * ks + c], bl[8 * ks + c + 4]);
        }
        const int col = (nt & 15) * 8 + 2 * c, which = isq ? 0 : 1;
        if (r0)
            *reinterpret_cast<__half2*>(a.qf + ((size_t)(h0 + g) * 2 + which) * kDim + col) = __floats2half2_rn(d[0], d[1]);
        if (r1)
            *reinterpret_cast<__half2*>(a.qf + ((size_t)(h0 + g + 8) * 2 + which) * kDim + col) =
                __floats2half2_rn(d[2], d[3]);
    }
}

// Transpose of an 8x8 fp16 matrix held as m8n8 fragments (thread 4 g + c holds row g,
// columns 2c, 2c + 1): afterwards it holds row g of the transpose.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ uint32_t h2bits(__half lo, __half hi) {
    return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

__device__ __forceinline__ __half cb_half(const Codebook& cb, int code) {
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxLevels; ++k) v = (k == code) ? cb.c[k] : v;
    return __float2half_rn(v);
}

// Raw bytes of one page that one thread needs (lane = 4 g + c), with the per-token
// scalars already multiplied by the constants of the score and of P'.
template <int KM, int VM, bool PROD>
struct PageRegs {
    uint32_t k[2][4];    // key code bytes of token rows g, g+8 (coords 32c .. 32c+31)
    uint32_t s[2];       // sign word c of rows g, g+8
    float kn[2], kg[2];  // key norm * qscale, gamma * sscale of tokens g, g+8
    uint32_t v[4][2];    // value code bytes of token rows 2c, 2c+1, 2c+8, 2c+9 (coords 16g .. 16g+15)
    float vn[2];         // value norm / sqrt(d) of tokens g, g+8
};

// Fragment bytes of one page from its shared-memory stage (key chunk at kst, value
// chunk at vst).
template <int KM, int VM, bool PROD>
__device__ __forceinline__ void load_page(PageRegs<KM, VM, PROD>& r, const uint8_t* kst, const uint8_t* vst,
                                          const DecodeArgs& a, int g, int c) {
    constexpr int kBytes = KM == kKBit1 ? 4 : (KM == kKByte2 ? 8 : 16);  // per key row per thread
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint8_t* row = kst + (g + 8 * i) * a.lk.code_row + kBytes * c;
        if (kBytes == 16) {
            const uint4 w = *reinterpret_cast<const uint4*>(row);
            r.k[i][0] = w.x, r.k[i][1] = w.y, r.k[i][2] = w.z, r.k[i][3] = w.w;
        } else if (kBytes == 8) {
            const uint2 w = *reinterpret_cast<const uint2*>(row);
            r.k[i][0] = w.x, r.k[i][1] = w.y;
        } else {
            r.k[i][0] = *reinterpret_cast<const uint32_t*>(row);
        }
        if (PROD) {
            r.s[i] = reinterpret_cast<const uint32_t*>(kst + a.lk.signs_off + (g + 8 * i) * 16)[c];
            r.kg[i] = reinterpret_cast<const float*>(kst + a.lk.gamma_off)[g + 8 * i] * a.sscale;
        }
        r.kn[i] = reinterpret_cast<const float*>(kst + a.lk.norm_off)[g + 8 * i] * a.qscale;
        r.vn[i] = reinterpret_cast<const float*>(vst + a.lv.norm_off)[g + 8 * i] * 0.08838834764831845f;
    }
    constexpr int vBytes = VM == kVByte4 ? 8 : 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int tok = 2 * c + (i & 1) + 8 * (i >> 1);
        const uint8_t* row = vst + tok * a.lv.code_row + vBytes * g;
        if (vBytes == 8) {
            const uint2 w = *reinterpret_cast<const uint2*>(row);
            r.v[i][0] = w.x, r.v[i][1] = w.y;
        } else {
            r.v[i][0] = *reinterpret_cast<const uint32_t*>(row);
        }
    }
}

// Shared memory of the split kernel (byte offsets; V at offset 0).
//   V    value byte table, lane-replicated: [256][32] half2 (nibbles) or [256][16] 2 x half2 (crumbs)
//   K    key byte table (same layouts) when keys are not byte-permuted
//   S    sign nibble table [16] 2 x half2 of +-1 (bit set -> +1)
//   K1   1-bit key nibble table [16] 2 x half2 of c[bit]
//   M    per warp m[16], l[16]
//   Bar  per warp kStagesD mbarriers of the page ring
//   Ring per warp kStagesD stages of one page (key chunk, then value chunk), filled
//        by bulk copies; after the page loop the same bytes hold the warps'
//        accumulators for the CTA merge (Acc: per warp acc[16 heads][128])
constexpr int kTabBytes = 32768;
constexpr int kStagesD = 4;
constexpr int kStageBytes = 2496;  // >= key chunk + value chunk for every bit width (16-byte multiple)

template <int KM, int VM, bool PROD>
struct SmemLayout {
    static constexpr bool kKTab = (KM == kKByte4 || KM == kKByte2);
    static constexpr uint32_t kOffV = 0;
    static constexpr uint32_t kOffK = kOffV + kTabBytes;
    static constexpr uint32_t kOffS = kOffK + (kKTab ? kTabBytes : 0);
    static constexpr uint32_t kOffK1 = kOffS + 128;
    static constexpr uint32_t kOffM = kOffK1 + 128;
    static constexpr uint32_t kOffBar = kOffM + kWarps * 2 * kMaxG * 4;
    static constexpr uint32_t kOffRing = (kOffBar + kWarps * kStagesD * 8 + 127) & ~127u;
    static constexpr uint32_t kRingBytes = kWarps * kStagesD * kStageBytes;
    static constexpr uint32_t kAccBytes = kWarps * kMaxG * kDim * 4;
    static constexpr uint32_t kOffAcc = kOffRing;
    static constexpr uint32_t kBytes = kOffRing + (kRingBytes > kAccBytes ? kRingBytes : kAccBytes);
};

template <int KM, int VM, bool PROD>
__device__ void build_tables(uint8_t* smem, const DecodeArgs& a) {
    using L = SmemLayout<KM, VM, PROD>;
    const int tid = threadIdx.x;
    for (int e = tid; e < 256; e += kThreads) {
        if (VM == kVByte4) {
            const uint32_t w = h2bits(cb_half(a.cbv, e & 15), cb_half(a.cbv, e >> 4));
            uint32_t* t = reinterpret_cast<uint32_t*>(smem + L::kOffV) + e * 32;
#pragma unroll
            for (int l = 0; l < 32; ++l) t[l] = w;
        } else {
            const uint2 w = make_uint2(h2bits(cb_half(a.cbv, e & 3), cb_half(a.cbv, (e >> 2) & 3)),
                                       h2bits(cb_half(a.cbv, (e >> 4) & 3), cb_half(a.cbv, e >> 6)));
            uint2* t = reinterpret_cast<uint2*>(smem + L::kOffV) + e * 16;
#pragma unroll
            for (int l = 0; l < 16; ++l) t[l] = w;
        }
        if (KM == kKByte4) {
            const uint32_t w = h2bits(cb_half(a.cbk, e & 15), cb_half(a.cbk, e >> 4));
            uint32_t* t = reinterpret_cast<uint32_t*>(smem + L::kOffK) + e * 32;
#pragma unroll
            for (int l = 0; l < 32; ++l) t[l] = w;
        } else if (KM == kKByte2) {
            const uint2 w = make_uint2(h2bits(cb_half(a.cbk, e & 3), cb_half(a.cbk, (e >> 2) & 3)),
                                       h2bits(cb_half(a.cbk, (e >> 4) & 3), cb_half(a.cbk, e >> 6)));
            uint2* t = reinterpret_cast<uint2*>(smem + L::kOffK) + e * 16;
#pragma unroll
            for (int l = 0; l < 16; ++l) t[l] = w;
        }
    }
    if (tid < 16) {
        const __half one = __float2half_rn(1.f), mone = __float2half_rn(-1.f);
        auto pm = [&](int bit) { return ((tid >> bit) & 1) ? one : mone; };
        reinterpret_cast<uint2*>(smem + L::kOffS)[tid] = make_uint2(h2bits(pm(0), pm(1)), h2bits(pm(2), pm(3)));
        const __half lo = cb_half(a.cbk, 0), hi = cb_half(a.cbk, 1);
        auto pk = [&](int bit) { return ((tid >> bit) & 1) ? hi : lo; };
        reinterpret_cast<uint2*>(smem + L::kOffK1)[tid] = make_uint2(h2bits(pk(0), pk(1)), h2bits(pk(2), pk(3)));
    }
}

// byte k (0..3) of w, times `scale` (a power of two), as a shared-memory byte offset
template <int K, int LOG2SCALE>
__device__ __forceinline__ uint32_t byte_off(uint32_t w) {
    constexpr int sh = 8 * K - LOG2SCALE;
    const uint32_t x = sh >= 0 ? (w >> sh) : (w << (-sh));
    return x & (0xffu << LOG2SCALE);
}
// nibble k (0..7) of w, times 8 (a uint2 table index as a byte offset)
template <int K>
__device__ __forceinline__ uint32_t nib_off8(uint32_t w) {
    constexpr int sh = 4 * K - 3;
    const uint32_t x = sh >= 0 ? (w >> sh) : (w << (-sh));
    return x & 0x78u;
}

// Lazy softmax rescaling: the running maximum only moves when a page exceeds it by
// more than 2^kSlack (log2 units), so exponentials stay <= 2^kSlack in fp32 / fp16.
constexpr float kSlack = 8.f;

// ------------------------------------------------------------------ split
template <int KM, int VM, bool PROD, int NT>
struct SplitCtx {
    uint32_t klo0, klo1, khi0, khi1;
    const uint8_t* smem;
    int lane, lane4, g, c;
};

template <int KM, int VM, bool PROD, int NT>
__device__ __forceinline__ void process_page(const PageRegs<KM, VM, PROD>& cur, int ntok,
                                             const SplitCtx<KM, VM, PROD, NT>& x, const uint32_t (&bq)[NT][8][2],
                                             const uint32_t (&bs)[NT][8][2], float (&m)[NT][2], float (&l)[NT][2],
                                             float (&acc)[NT][8][4]) {
    using L = SmemLayout<KM, VM, PROD>;
    const int g = x.g, c = x.c;
    const bool valid0 = g < ntok, valid1 = g + 8 < ntok;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        // ---- scores: 8 K-steps of 16 coordinates, even and odd K-steps in separate
        // accumulators (two independent MMA chains)
        float d1[2][4] = {}, d2[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            uint32_t ak[2][2];  // [row g / g+8][coords (4ks,4ks+1) / (4ks+2,4ks+3)]
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                if (KM == kKPrmt) {
                    const uint32_t w = cur.k[i][ks >> 1];
                    const uint32_t sel = (ks & 1) ? (w >> 16) : w;
                    const uint32_t lo = __byte_perm(x.klo0, x.klo1, sel);
                    const uint32_t hi = __byte_perm(x.khi0, x.khi1, sel);
                    ak[i][0] = __byte_perm(lo, hi, 0x5140);
                    ak[i][1] = __byte_perm(lo, hi, 0x7362);
                } else if (KM == kKByte4) {
                    const uint32_t w = cur.k[i][ks >> 1];
                    const uint32_t o0 = (ks & 1) ? byte_off<2, 7>(w) : byte_off<0, 7>(w);
                    const uint32_t o1 = (ks & 1) ? byte_off<3, 7>(w) : byte_off<1, 7>(w);
                    ak[i][0] = *reinterpret_cast<const uint32_t*>(x.smem + L::kOffK + (o0 | x.lane4));
                    ak[i][1] = *reinterpret_cast<const uint32_t*>(x.smem + L::kOffK + (o1 | x.lane4));
                } else if (KM == kKByte2) {
                    const uint32_t w = cur.k[i][ks >> 2];
                    uint32_t o;
                    switch (ks & 3) {
                        case 0: o = byte_off<0, 7>(w); break;
                        case 1: o = byte_off<1, 7>(w); break;
                        case 2: o = byte_off<2, 7>(w); break;
                        default: o = byte_off<3, 7>(w); break;
                    }
                    const uint2 e = *reinterpret_cast<const uint2*>(x.smem + L::kOffK + (o | ((x.lane & 15) << 3)));
                    ak[i][0] = e.x;
                    ak[i][1] = e.y;
                } else {
                    const uint2 e = reinterpret_cast<const uint2*>(x.smem + L::kOffK1)[(cur.k[i][0] >> (4 * ks)) & 0xfu];
                    ak[i][0] = e.x;
                    ak[i][1] = e.y;
                }
            }
            mma16816(d1[ks & 1], ak[0][0], ak[1][0], ak[0][1], ak[1][1], bq[nt][ks][0], bq[nt][ks][1]);
            if (PROD) {
                const uint32_t oa = nib_off8<0>(cur.s[0] >> (4 * ks));
                const uint32_t ob = nib_off8<0>(cur.s[1] >> (4 * ks));
                const uint2 s0 = *reinterpret_cast<const uint2*>(x.smem + L::kOffS + oa);
                const uint2 s1 = *reinterpret_cast<const uint2*>(x.smem + L::kOffS + ob);
                mma16816(d2[ks & 1], s0.x, s1.x, s0.y, s1.y, bs[nt][ks][0], bs[nt][ks][1]);
            }
        }
        // ---- base-2 logits of tokens g, g+8 for heads nt*8 + 2c + e
        float sc[2][2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float s = cur.kn[i] * (d1[0][2 * i + e] + d1[1][2 * i + e]);
                if (PROD) s = fmaf(cur.kg[i], d2[0][2 * i + e] + d2[1][2 * i + e], s);
                sc[i][e] = (i == 0 ? valid0 : valid1) ? s : -INFINITY;
            }
        // Lazy maximum: each lane checks its own two logits per column against
        // m + kSlack; only when one exceeds it is the page maximum reduced over the
        // column's lanes and the state rescaled.  l holds this lane's partial sum
        // (its rows), reduced over the column's lanes once per item.
        float pw[2][2];
        bool over = false;
#pragma unroll
        for (int e = 0; e < 2; ++e) over |= fmaxf(sc[0][e], sc[1][e]) > m[nt][e] + kSlack;
        if (__any_sync(0xffffffffu, over)) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float mx = fmaxf(sc[0][e], sc[1][e]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float mnew = mx > m[nt][e] + kSlack ? mx : m[nt][e];
                const float corr = exp2f(m[nt][e] - mnew);  // 1 when unchanged, 0 from -inf
                l[nt][e] *= corr;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    acc[nt][mt][e] *= corr;
                    acc[nt][mt][2 + e] *= corr;
                }
                m[nt][e] = mnew;
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float p0v = exp2f(sc[0][e] - m[nt][e]), p1v = exp2f(sc[1][e] - m[nt][e]);
            l[nt][e] += p0v + p1v;
            pw[0][e] = valid0 ? p0v * cur.vn[0] : 0.f;
            pw[1][e] = valid1 ? p1v * cur.vn[1] : 0.f;
        }
        // ---- P' to the B-operand layout: each 8-token half of the C fragment
        // (token row g, heads 2c, 2c + 1) transposed in registers to (tokens 2c,
        // 2c + 1, head g)
        const uint32_t pb0 = movmatrix_trans(h2bits(__float2half_rn(pw[0][0]), __float2half_rn(pw[0][1])));
        const uint32_t pb1 = movmatrix_trans(h2bits(__float2half_rn(pw[1][0]), __float2half_rn(pw[1][1])));
        // ---- values: m-tile mt, row g -> coord 16g + 2mt (nibbles), row g+8 -> +1
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t av[4];
            if (VM == kVByte4) {
                uint32_t t[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w = cur.v[i][mt >> 2];
                    uint32_t o;
                    switch (mt & 3) {
                        case 0: o = byte_off<0, 7>(w); break;
                        case 1: o = byte_off<1, 7>(w); break;
                        case 2: o = byte_off<2, 7>(w); break;
                        default: o = byte_off<3, 7>(w); break;
                    }
                    t[i] = *reinterpret_cast<const uint32_t*>(x.smem + L::kOffV + (o | x.lane4));
                }
                av[0] = __byte_perm(t[0], t[1], 0x5410);  // lower coord, tokens 2c, 2c+1
                av[1] = __byte_perm(t[0], t[1], 0x7632);  // upper coord
                av[2] = __byte_perm(t[2], t[3], 0x5410);  // tokens 2c+8, 2c+9
                av[3] = __byte_perm(t[2], t[3], 0x7632);
            } else {
                uint2 t[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t w = cur.v[i][0];
                    uint32_t o;
                    switch (mt >> 1) {
                        case 0: o = byte_off<0, 7>(w); break;
                        case 1: o = byte_off<1, 7>(w); break;
                        case 2: o = byte_off<2, 7>(w); break;
                        default: o = byte_off<3, 7>(w); break;
                    }
                    t[i] = *reinterpret_cast<const uint2*>(x.smem + L::kOffV + (o | ((x.lane & 15) << 3)));
                }
                const uint32_t x0 = (mt & 1) ? t[0].y : t[0].x, x1 = (mt & 1) ? t[1].y : t[1].x;
                const uint32_t x2 = (mt & 1) ? t[2].y : t[2].x, x3 = (mt & 1) ? t[3].y : t[3].x;
                av[0] = __byte_perm(x0, x1, 0x5410);
                av[1] = __byte_perm(x0, x1, 0x7632);
                av[2] = __byte_perm(x2, x3, 0x5410);
                av[3] = __byte_perm(x2, x3, 0x7632);
            }
            mma16816(acc[nt][mt], av[0], av[1], av[2], av[3], pb0, pb1);
        }
    }
}

template <int KM, int VM, bool PROD, int NT>
__global__ void __launch_bounds__(kThreads) decode_split_kernel(DecodeArgs a) {
    using L = SmemLayout<KM, VM, PROD>;
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    build_tables<KM, VM, PROD>(smem, a);
    SplitCtx<KM, VM, PROD, NT> x{};
    x.smem = smem;
    x.lane = lane;
    x.lane4 = lane << 2;
    x.g = g;
    x.c = c;
    if (KM == kKPrmt) {  // 8-entry key tables: low / high bytes of the fp16 levels
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t hb = __half_as_ushort(cb_half(a.cbk, k));
            if (k < 4) {
                x.klo0 |= (hb & 0xffu) << (8 * k);
                x.khi0 |= (hb >> 8) << (8 * k);
            } else {
                x.klo1 |= (hb & 0xffu) << (8 * (k - 4));
                x.khi1 |= (hb >> 8) << (8 * (k - 4));
            }
        }
    }
    const uint32_t ring = sm100::smem_u32(smem + L::kOffRing) + warp * kStagesD * kStageBytes;
    const uint32_t bars = sm100::smem_u32(smem + L::kOffBar) + warp * kStagesD * 8;
    if (lane == 0) {
        for (int st = 0; st < kStagesD; ++st) sm100::mbar_init(bars + 8 * st, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();  // q', s and the page prefix sums from the prep kernel; the caller's inputs
    griddep_launch_dependents();  // the merge kernel may stage its rotation meanwhile
    float* wm = reinterpret_cast<float*>(smem + L::kOffM);      // [warp][2][16]: m then l
    float* wacc = reinterpret_cast<float*>(smem + L::kOffAcc);  // [warp][16 heads][128]
    const volatile int never = 0;
    uint32_t issued = 0, consumed = 0;  // pages this warp has requested / processed (all items)
    bool dead = false;                  // a page copy never arrived: this warp stops working

    // this CTA's range [pos, end) of the pages of all units in order (unit
    // u = b Hkv + h holds the pages of sequence b), cut into pieces by unit
    const long total = (long)a.Hkv * a.prefix[a.B];
    long pos = total * (long)blockIdx.x / gridDim.x;
    const long end = total * (long)(blockIdx.x + 1) / gridDim.x;
    int b = 0;
    if (pos < end) {  // the last sequence b with Hkv * prefix[b] <= pos
        int lo = 0, hi = a.B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((long)a.Hkv * a.prefix[mid] <= pos) lo = mid;
            else hi = mid - 1;
        }
        b = lo;
    }
    while (pos < end && b < a.B) {
        const int np = a.prefix[b + 1] - a.prefix[b];  // pages of sequence b (the same for each kv head)
        const long off = pos - (long)a.Hkv * a.prefix[b];
        if (np == 0 || off >= (long)a.Hkv * np) {  // past sequence b
            ++b;
            continue;
        }
        const int hk = (int)(off / np);
        const int p0 = (int)(off - (long)hk * np);
        const int p1 = (int)min((long)np, p0 + (end - pos));
        pos += p1 - p0;
        const int unit = b * a.Hkv + hk;
        const int Ls = a.seq_lens[b];  // valid: np > 0

        // query fragments (B operand): head nt*8 + g, coords 32c .. 32c+31; K-step ks
        // uses coords 32c + 4ks + {0,1} (b0) and {2,3} (b1)
        uint32_t bq[NT][8][2], bs[NT][8][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = nt * 8 + g;
            if (h < a.G) {
                const uint4* src =
                    reinterpret_cast<const uint4*>(a.qf + (((size_t)unit * a.G + h) * 2) * kDim + 32 * c);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 w = src[i];
                    bq[nt][2 * i][0] = w.x, bq[nt][2 * i][1] = w.y;
                    bq[nt][2 * i + 1][0] = w.z, bq[nt][2 * i + 1][1] = w.w;
                    if (PROD) {
                        const uint4 u = src[i + kDim / 8];
                        bs[nt][2 * i][0] = u.x, bs[nt][2 * i][1] = u.y;
                        bs[nt][2 * i + 1][0] = u.z, bs[nt][2 * i + 1][1] = u.w;
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) bq[nt][i][0] = bq[nt][i][1] = bs[nt][i][0] = bs[nt][i][1] = 0u;
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

        // ---- page loop: the warp takes pages first, first + 4, ...; a ring of
        // kStagesD shared-memory stages keeps the next pages' bulk copies in flight
        const int first = p0 + warp;
        const int nj = first < p1 ? (p1 - first + kWarps - 1) / kWarps : 0;
        const int* btab = a.block_table + (size_t)b * a.max_blocks + first;
        const int win = (lane < nj) ? btab[lane * kWarps] : -1;  // block ids of the first 32 pages
        auto blk_of = [&](int j) -> int {
            int v = __shfl_sync(0xffffffffu, win, j & 31);
            if (j >= 32) {
                v = lane == 0 ? btab[j * kWarps] : 0;
                v = __shfl_sync(0xffffffffu, v, 0);
            }
            return v;
        };
        const uint32_t kb = (uint32_t)a.lk.bytes, vb = (uint32_t)a.lv.bytes;
        auto issue = [&](int j) {
            const int blk = blk_of(j);
            const uint32_t st = ring + (issued % kStagesD) * kStageBytes;
            const uint32_t bar = bars + 8 * (issued % kStagesD);
            if (lane == 0) {
                if (blk >= 0 && blk < a.num_blocks) {
                    const size_t chunk = (size_t)blk * a.Hkv + hk;
                    sm100::mbar_arrive_expect_tx(bar, kb + vb);
                    sm100::bulk_g2s(st, a.kc + chunk * kb, kb, bar);
                    sm100::bulk_g2s(st + kb, a.vc + chunk * vb, vb, bar);
                } else {
                    sm100::mbar_arrive(bar);  // nothing to copy: the stage completes at once
                }
            }
            ++issued;
        };
        if (!dead)
            for (int j = 0; j < nj && j < kStagesD; ++j) issue(j);
        for (int j = 0; j < nj && !dead; ++j) {
            const uint32_t sidx = consumed % kStagesD;
            const bool ok = sm100::mbar_wait_warp(bars + 8 * sidx, (consumed / kStagesD) & 1u, &never, 2000000000ull);
            const int blk = blk_of(j);
            if (!ok) {
                if (lane == 0) atomicOr(a.err, TQ_DEVERR_TIMEOUT);
                dead = true;
                break;
            }
            ++consumed;
            const int page = first + j * kWarps;
            if (blk < 0 || blk >= a.num_blocks) {
                if (lane == 0) atomicOr(a.err, TQ_DEVERR_BLOCK);
            } else {
                const uint8_t* st = smem + L::kOffRing + (size_t)(warp * kStagesD + sidx) * kStageBytes;
                PageRegs<KM, VM, PROD> r;
                load_page<KM, VM, PROD>(r, st, st + kb, a, g, c);
                process_page<KM, VM, PROD, NT>(r, min(kPage, Ls - page * kPage), x, bq, bs, m, l, acc);
            }
            sm100::fence_proxy_async_shared();  // this lane's reads before the refill's bulk copy
            __syncwarp();  // every lane is done with the stage before it is refilled
            if (j + kStagesD < nj) issue(j + kStagesD);
        }
        if (dead) {  // let copies already in flight land before the stages are reused
            while (consumed < issued) {
                sm100::mbar_wait(bars + 8 * (consumed % kStagesD), (consumed / kStagesD) & 1u, &never, 2000000000ull);
                ++consumed;
            }
        }

        // ---- merge the warps of the CTA (coordinates back in natural order)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {  // l over the column's lanes
                l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], 4);
                l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], 8);
                l[nt][e] += __shfl_xor_sync(0xffffffffu, l[nt][e], 16);
            }
        __syncthreads();
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h = nt * 8 + 2 * c + e;
                if (g == 0) {
                    wm[(warp * 2 + 0) * kMaxG + h] = m[nt][e];
                    wm[(warp * 2 + 1) * kMaxG + h] = l[nt][e];
                }
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    const int c0 = (VM == kVByte4) ? 16 * g + 2 * mt : 16 * g + 4 * (mt >> 1) + 2 * (mt & 1);
                    wacc[(warp * kMaxG + h) * kDim + c0] = acc[nt][mt][e];
                    wacc[(warp * kMaxG + h) * kDim + c0 + 1] = acc[nt][mt][2 + e];
                }
            }
        __syncthreads();
        for (int h = 0; h < a.G; ++h) {  // thread = coordinate
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[(w * 2) * kMaxG + h]);
            float Lsum = 0.f, A = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float mw = wm[(w * 2) * kMaxG + h];
                const float wt = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
                Lsum = fmaf(wt, wm[(w * 2 + 1) * kMaxG + h], Lsum);
                A = fmaf(wt, wacc[(w * kMaxG + h) * kDim + tid], A);
            }
            float* part = a.partial + (((size_t)unit + blockIdx.x) * a.G + h) * kPartStride;
            if (tid == 0) {
                part[0] = M;
                part[1] = Lsum;
            }
            part[2 + tid] = A;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ merge
// Persistent: with n items per CTA (chosen at launch so that the CTAs cover the
// SMs), CTA i takes the (unit, group of kMergeHeads heads) items i n .. i n + n - 1,
// then + grid n, ...; thread = coordinate, computing all the group's heads so that
// each element of R is read once per item.  An item has sg groups of 128 threads
// (sg > 1 when a unit spans many split CTAs, as in one long sequence): group g
// folds every sg-th slot from the g-th, and the first group combines the sg
// partial states and un-rotates.  R^T is staged once per CTA (while the split
// kernel runs).  Unit u's pieces sit in slots u + c for the split CTAs c whose
// page range meets it: c(p) = ((p + 1) grid - 1) / total is the CTA of page p.
constexpr int kMergeHeads = 4;
constexpr int kMergeItems = 4;  // most items per CTA
constexpr int kMergeGroups = 8; // most slot groups per item
constexpr int kMergeThreads = 1024;
size_t merge_smem(int ipc, int sg) {
    return sizeof(float) * (kDim * kDim + (size_t)ipc * kDim * kMergeHeads +
                            (sg > 1 ? (size_t)ipc * sg * (kDim * kMergeHeads + 2 * kMergeHeads) : 0));
}
__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(DecodeArgs a) {
    // RT [128*128] | orot [items][128][kMergeHeads] | group states A [items][sg][128][kMergeHeads],
    // (M, L) [items][sg][kMergeHeads][2]
    extern __shared__ __align__(16) float sm[];
    const int sg = a.merge_sg;
    const int ipc = (int)blockDim.x / (kDim * sg);
    const int i = threadIdx.x % kDim, gi = (threadIdx.x / kDim) % sg, il = threadIdx.x / (kDim * sg);
    float* rts = sm;
    float4* orot = reinterpret_cast<float4*>(sm + kDim * kDim) + il * kDim;  // this item's [j] of 4 heads
    float4* gA = reinterpret_cast<float4*>(sm + kDim * kDim + ipc * kDim * kMergeHeads) + (il * sg) * kDim;
    float* gML = sm + kDim * kDim + ipc * kDim * kMergeHeads + ipc * sg * kDim * kMergeHeads +
                 (il * sg) * 2 * kMergeHeads;
    {
        const float4* src = reinterpret_cast<const float4*>(a.RT);
        float4* dst = reinterpret_cast<float4*>(rts);
        for (int k = threadIdx.x; k < kDim * kDim / 4; k += blockDim.x) dst[k] = src[k];
    }
    // The items' units and slot ranges depend on the page prefix sums only, which the
    // prep kernel wrote before the split kernel could start (and so before this
    // kernel was launched): they are read before waiting for the split partials.
    const long total = (long)a.Hkv * a.prefix[a.B];
    const long grid = a.split_grid;
    const int groups = (a.G + kMergeHeads - 1) / kMergeHeads;
    const int items = a.B * a.Hkv * groups;
    auto item_info = [&](int item, int& unit, int& h0, int& c_lo, int& c_hi) {
        unit = 0, h0 = 0, c_lo = 0, c_hi = -1;
        if (item >= items) return;
        unit = item / groups;
        h0 = (item - unit * groups) * kMergeHeads;
        const int b = unit / a.Hkv, hk = unit - b * a.Hkv;
        const int np = a.prefix[b + 1] - a.prefix[b];
        if (np > 0) {
            const long first = (long)a.Hkv * a.prefix[b] + (long)hk * np, last = first + np - 1;
            c_lo = (int)(((first + 1) * grid - 1) / total);
            c_hi = (int)(((last + 1) * grid - 1) / total);
        }
    };
    int n_unit, n_h0, n_clo, n_chi;  // the first item's
    item_info(blockIdx.x * ipc + il, n_unit, n_h0, n_clo, n_chi);
    griddep_wait();  // the split partials
    for (int base = blockIdx.x * ipc; base < items; base += gridDim.x * ipc) {
        const int item = base + il;
        const bool live = item < items;
        int unit = n_unit, h0 = n_h0, c_lo = n_clo, c_hi = n_chi;
        if (base + gridDim.x * ipc < items) item_info(item + gridDim.x * ipc, n_unit, n_h0, n_clo, n_chi);
        // online log-sum-exp over the slots, all heads at once: the loads of several
        // slots are in flight together
        float M[kMergeHeads], Lsum[kMergeHeads], A[kMergeHeads];
#pragma unroll
        for (int e = 0; e < kMergeHeads; ++e) M[e] = -INFINITY, Lsum[e] = 0.f, A[e] = 0.f;
        const int nh = a.G - h0 < kMergeHeads ? a.G - h0 : kMergeHeads;
#pragma unroll 4
        for (int c = c_lo + gi; c <= c_hi; c += sg) {
            const float* pp = a.partial + (((size_t)unit + c) * a.G + h0) * kPartStride;
            float ms[kMergeHeads], ls[kMergeHeads], as[kMergeHeads];
#pragma unroll
            for (int e = 0; e < kMergeHeads; ++e) {
                const bool on = e < nh;
                ms[e] = on ? pp[e * kPartStride] : -INFINITY;
                ls[e] = on ? pp[e * kPartStride + 1] : 0.f;
                as[e] = on ? pp[e * kPartStride + 2 + i] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < kMergeHeads; ++e) {
                const float mn = fmaxf(M[e], ms[e]);
                const float sa = (M[e] == -INFINITY) ? 0.f : exp2f(M[e] - mn);
                const float sb = (ms[e] == -INFINITY) ? 0.f : exp2f(ms[e] - mn);
                Lsum[e] = fmaf(Lsum[e], sa, ls[e] * sb);
                A[e] = fmaf(A[e], sa, as[e] * sb);
                M[e] = mn;
            }
        }
        __syncthreads();  // the previous items' un-rotation is done with orot and the group states
        if (sg > 1) {  // the first group combines the groups' states
            if (i == 0)
#pragma unroll
                for (int e = 0; e < kMergeHeads; ++e) gML[gi * 2 * kMergeHeads + 2 * e] = M[e], gML[gi * 2 * kMergeHeads + 2 * e + 1] = Lsum[e];
            gA[gi * kDim + i] = make_float4(A[0], A[1], A[2], A[3]);
            __syncthreads();
            if (gi == 0) {
#pragma unroll
                for (int e = 0; e < kMergeHeads; ++e) {
                    float Mx = -INFINITY;
                    for (int g = 0; g < sg; ++g) Mx = fmaxf(Mx, gML[g * 2 * kMergeHeads + 2 * e]);
                    float L2 = 0.f, A2 = 0.f;
                    for (int g = 0; g < sg; ++g) {
                        const float mg = gML[g * 2 * kMergeHeads + 2 * e];
                        if (mg == -INFINITY) continue;
                        const float w = exp2f(mg - Mx);
                        const float4 ag = gA[g * kDim + i];
                        L2 = fmaf(gML[g * 2 * kMergeHeads + 2 * e + 1], w, L2);
                        A2 = fmaf(e == 0 ? ag.x : e == 1 ? ag.y : e == 2 ? ag.z : ag.w, w, A2);
                    }
                    M[e] = Mx, Lsum[e] = L2, A[e] = A2;
                }
            }
        }
        float o[kMergeHeads];
#pragma unroll
        for (int e = 0; e < kMergeHeads; ++e) o[e] = (live && Lsum[e] > 0.f) ? A[e] / Lsum[e] : 0.f;
        if (gi == 0) orot[i] = make_float4(o[0], o[1], o[2], o[3]);
        __syncthreads();
        if (!live || gi != 0) continue;
        float y[kMergeHeads] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int j = 0; j < kDim; ++j) {  // o_i = sum_j R[i][j] orot_j, for the 4 heads at once
            const float r = rts[j * kDim + i];
            const float4 v = orot[j];
            y[0] = fmaf(r, v.x, y[0]);
            y[1] = fmaf(r, v.y, y[1]);
            y[2] = fmaf(r, v.z, y[2]);
            y[3] = fmaf(r, v.w, y[3]);
        }
#pragma unroll
        for (int e = 0; e < kMergeHeads; ++e) {
            const int h = h0 + e;
            if (h >= a.G) break;
            const size_t oi = ((size_t)unit * a.G + h) * kDim + i;
            if (a.out_fp32)
                static_cast<float*>(a.out)[oi] = y[e];
            else
                static_cast<__half*>(a.out)[oi] = __float2half_rn(y[e]);
        }
    }
}

int kmode_of(const tq_ctx* ctx) {
    const int w = ctx->cb_key.width;
    if (w == 4) return ctx->cb_key.levels <= 8 ? kKPrmt : kKByte4;
    if (w == 2) return kKByte2;
    return kKBit1;
}

size_t split_smem(int km) {
    return (km == kKByte4 || km == kKByte2) ? SmemLayout<kKByte4, kVByte4, true>::kBytes
                                            : SmemLayout<kKPrmt, kVByte4, true>::kBytes;
}

int ctas_per_sm_for(size_t smem) {
    int n = (int)(233472 / (smem + 1024));  // 228 KB of shared memory per SM, 1 KB reserved per CTA
    if (n > 4) n = 4;
    return n < 1 ? 1 : n;
}


// Launch with programmatic stream serialization (see griddep_wait).
template <typename K>
cudaError_t launch_dependent(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, const DecodeArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

template <int KM, int VM, bool PROD, int NT>
cudaError_t launch_split(const DecodeArgs& a, int grid, cudaStream_t stream) {
    using L = SmemLayout<KM, VM, PROD>;
    auto k = decode_split_kernel<KM, VM, PROD, NT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (e != cudaSuccess) return e;
    return launch_dependent(k, dim3(grid), dim3(kThreads), L::kBytes, stream, a);
}

}  // namespace

DecodePlan plan_decode(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_seq_len) {
    DecodePlan p{};
    p.max_pages = (max_seq_len + kPage - 1) / kPage;
    const long resident = (long)ctx->sm_count * ctas_per_sm_for(split_smem(kmode_of(ctx)));
    const long units = (long)B * Hkv;
    // every resident CTA, but at least 16 pages (4 per warp) per CTA for small batches
    long grid = (units * p.max_pages + 4 * kWarps - 1) / (4 * kWarps);
    if (grid > resident) grid = resident;
    if (grid < 1) grid = 1;
    p.grid = (int)grid;
    p.slots = (int)(units + grid);
    const int G = Hkv > 0 ? Hq / Hkv : 0;
    size_t off = 0;
    p.qprep_off = off;
    off += (size_t)B * Hq * 2 * kDim * sizeof(__half);
    off = (off + 255) & ~size_t(255);
    p.partial_off = off;
    off += (size_t)p.slots * G * kPartStride * sizeof(float);
    off = (off + 255) & ~size_t(255);
    p.prefix_off = off;
    off += (size_t)(B + 1) * sizeof(int);
    off = (off + 255) & ~size_t(255);
    p.bytes = off;
    return p;
}

cudaError_t launch_decode(const tq_ctx* ctx, const DecodePlan& plan, const uint16_t* q, const uint8_t* kc,
                          const uint8_t* vc, int num_blocks, const int32_t* block_table, int max_blocks,
                          const int32_t* seq_lens, int B, int Hq, int Hkv, int max_seq_len, float scale, void* out,
                          int out_fp32, void* workspace, cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecodeArgs a{};
    a.q = q;
    a.qf = reinterpret_cast<__half*>(ws + plan.qprep_off);
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
    a.scale_log2 = scale * 1.4426950408889634f;
    a.qscale = a.scale_log2 / sqrtf((float)kDim);
    a.sscale = a.scale_log2 * 1.2533141373155003f / (float)kDim;
    a.partial = reinterpret_cast<float*>(ws + plan.partial_off);
    a.prefix = reinterpret_cast<int*>(ws + plan.prefix_off);
    a.split_grid = plan.grid;
    a.RT = ctx->dev.RT;
    a.RTh = ctx->dev.RTh;
    a.RTl = ctx->dev.RTl;
    a.Sh = ctx->dev.Sh;
    a.cbk = ctx->cb_key;
    a.cbv = ctx->cb_value;
    a.lk = ctx->lay_key;
    a.lv = ctx->lay_value;
    a.out = out;
    a.out_fp32 = out_fp32;
    a.err = ctx->dev_error;

    cudaError_t e = launch_dependent(decode_prep_kernel, dim3((B * Hq + 15) / 16, 4), dim3(kPrepThreads), 0, stream, a);
    if (e != cudaSuccess) return e;
    const int KM = kmode_of(ctx);
    const int VM = ctx->cb_value.width == 4 ? kVByte4 : kVByte2;
    const bool prod = ctx->lay_key.prod;
    const int NT = a.G <= 8 ? 1 : 2;
    const int grid = plan.grid;
    e = cudaErrorInvalidValue;
#define TQ_DEC_CASE(K_, V_, P_, N_) \
    if (KM == K_ && VM == V_ && prod == P_ && NT == N_) e = launch_split<K_, V_, P_, N_>(a, grid, stream);
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
    const int mitems = B * Hkv * ((a.G + kMergeHeads - 1) / kMergeHeads);
    // slot groups per item: a unit of the longest sequence meets about grid / units
    // + 1 split CTAs when all sequences are that long; one group per 4 such slots
    const long units = (long)B * Hkv;
    const long est_slots = units > 0 ? (grid + units - 1) / units + 1 : 1;
    int sg = (int)(est_slots / 4);
    sg = sg < 1 ? 1 : (sg > kMergeGroups ? kMergeGroups : sg);
    // items per CTA: as few as keep the CTAs within one per SM (at most kMergeItems; one
    // when an item has several groups)
    int ipc = 1;
    if (sg == 1) {
        ipc = (mitems + ctx->sm_count - 1) / ctx->sm_count;
        ipc = ipc < 1 ? 1 : (ipc > kMergeItems ? kMergeItems : ipc);
    }
    a.merge_sg = sg;
    const int mctas = (mitems + ipc - 1) / ipc;
    const dim3 mgrid(mctas < ctx->sm_count ? mctas : ctx->sm_count);
    const size_t msmem = merge_smem(ipc, sg);
    e = cudaFuncSetAttribute(decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)std::max(merge_smem(kMergeItems, 1), merge_smem(1, kMergeGroups)));
    if (e != cudaSuccess) return e;
    e = launch_dependent(decode_merge_kernel, mgrid, dim3(kDim * ipc * sg), msmem, stream, a);
    if (e != cudaSuccess) return e;
    count_launches(3);
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
