// Split-K decode attention over the paged compressed cache.
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…":
//   - section "注意力计算的特殊挑战与QJL校正": score estimator
//       <q,k> ~ <q,k_hat> + gamma sqrt(pi/2)/d <S q, sign(S r)>
//   - section "架构设计" / "关键工程改进": Paged Decode as split-K FlashDecoding.
// Scores are taken in the rotated domain: <q, k_hat> = n/sqrt(d) <R^T q, c[idx]>,
// values are accumulated as sum_t p_t n_t c[idx_t]/sqrt(d) and un-rotated once
// per query head (o = R acc).
//
// Three stages: (1) prep: q' = R^T q and s = S q per (sequence, query head);
// (2) split: each CTA scans a contiguous range of pages of one (sequence, kv
// head) for all of its G query heads with an online softmax; (3) merge: the
// log-sum-exp combination of the splits, the division by the softmax
// denominator and the un-rotation.
#include <cmath>

#include "device_util.cuh"

namespace tq {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxG = 16;
constexpr int kPartStride = kDim + 2;  // m, l, acc[128]

struct DecodeArgs {
    const uint16_t* q;
    const uint8_t* kc;
    const uint8_t* vc;
    int num_blocks;
    const int32_t* block_table;
    int max_blocks;
    const int32_t* seq_lens;
    int B, Hq, Hkv, G, max_seq_len;
    float scale;
    void* out;
    int out_fp32;
    float* qprep;     // [B*Hq][2][128]: R^T q, S q
    float* partial;   // [B*Hq][splits][130]
    int splits, pages_per_split;
    const float* R;   // row-major
    const float* RT;  // row-major R^T
    const float* ST;  // row-major S^T
    Codebook cbk, cbv;
    ChunkLayout lk, lv;
    uint32_t* err;
};

__global__ void __launch_bounds__(kThreads) decode_prep_kernel(DecodeArgs a) {
    __shared__ float qs[kDim];
    const int bh = blockIdx.x, j = threadIdx.x;
    qs[j] = half_bits_to_float(a.q[(size_t)bh * kDim + j]);
    __syncthreads();
    float qr = 0.f, sq = 0.f;
    for (int i = 0; i < kDim; ++i) {
        qr = fmaf(a.R[i * kDim + j], qs[i], qr);    // (R^T q)_j = sum_i R[i][j] q_i
        sq = fmaf(a.ST[i * kDim + j], qs[i], sq);   // (S q)_j = sum_i S[j][i] q_i
    }
    a.qprep[(size_t)bh * 2 * kDim + j] = qr;
    a.qprep[(size_t)bh * 2 * kDim + kDim + j] = sq;
}

__device__ __forceinline__ bool seq_len_ok(const DecodeArgs& a, int L) {
    return L >= 0 && L <= a.max_blocks * kPage && L <= a.max_seq_len;
}

__global__ void __launch_bounds__(kThreads) decode_split_kernel(DecodeArgs a) {
    __shared__ float qp[kMaxG][kDim];
    __shared__ float sq[kMaxG][kDim];
    __shared__ __align__(16) uint8_t kchunk[1536];
    __shared__ __align__(16) uint8_t vchunk[1152];
    __shared__ float sc[kMaxG][kPage];
    __shared__ float corr[kMaxG];
    __shared__ float msh[kMaxG], lsh[kMaxG];
    const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = a.G;
    int L = a.seq_lens[b];
    if (!seq_len_ok(a, L)) {
        if (tid == 0 && split == 0 && hk == 0) atomicOr(a.err, TQ_DEVERR_SEQLEN);
        L = 0;
    }
    const int npages = (L + kPage - 1) / kPage;
    const int p0 = split * a.pages_per_split;
    const int p1 = min(p0 + a.pages_per_split, npages);
    for (int g = 0; g < G; ++g) {
        const size_t bh = (size_t)b * a.Hq + hk * G + g;
        qp[g][tid] = a.qprep[bh * 2 * kDim + tid];
        sq[g][tid] = a.qprep[bh * 2 * kDim + kDim + tid];
    }
    if (tid < kMaxG) {
        msh[tid] = -INFINITY;
        lsh[tid] = 0.f;
    }
    float acc[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) acc[g] = 0.f;
    const float sqrt_d = sqrtf((float)kDim);
    const float qjl = sqrtf(3.14159265358979f / 2.f) / kDim;
    __syncthreads();

    for (int p = p0; p < p1; ++p) {
        const int blk = a.block_table[(size_t)b * a.max_blocks + p];
        if (blk < 0 || blk >= a.num_blocks) {
            if (tid == 0) atomicOr(a.err, TQ_DEVERR_BLOCK);
            continue;  // uniform across the CTA
        }
        const int ntok = min(kPage, L - p * kPage);
        const uint4* ksrc = reinterpret_cast<const uint4*>(a.kc + ((size_t)blk * a.Hkv + hk) * a.lk.bytes);
        const uint4* vsrc = reinterpret_cast<const uint4*>(a.vc + ((size_t)blk * a.Hkv + hk) * a.lv.bytes);
        for (int i = tid; i < a.lk.bytes / 16; i += kThreads) reinterpret_cast<uint4*>(kchunk)[i] = ksrc[i];
        for (int i = tid; i < a.lv.bytes / 16; i += kThreads) reinterpret_cast<uint4*>(vchunk)[i] = vsrc[i];
        __syncthreads();
        // scores: warp w takes tokens w, w+4, w+8, w+12; lane covers coordinates 4*lane .. 4*lane+3
        for (int t = warp; t < ntok; t += kThreads / 32) {
            const uint8_t* crow = kchunk + t * a.lk.code_row;
            float cval[4], sg[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = 4 * lane + e;
                const int c = extract_code(crow, j, a.cbk.width);
                float cv = 0.f;
#pragma unroll
                for (int k = 0; k < kMaxLevels; ++k) cv = (k == c) ? a.cbk.c[k] : cv;
                cval[e] = cv;
                sg[e] = a.lk.prod ? (extract_code(kchunk + a.lk.signs_off + t * (kDim / 8), j, 1) ? 1.f : -1.f) : 0.f;
            }
            const float n = reinterpret_cast<const float*>(kchunk + a.lk.norm_off)[t];
            const float gm = a.lk.prod ? reinterpret_cast<const float*>(kchunk + a.lk.gamma_off)[t] : 0.f;
            for (int g = 0; g < G; ++g) {
                float d1 = 0.f, d2 = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    d1 = fmaf(qp[g][4 * lane + e], cval[e], d1);
                    d2 = fmaf(sq[g][4 * lane + e], sg[e], d2);
                }
                d1 = warp_sum(d1);
                d2 = warp_sum(d2);
                if (lane == 0) sc[g][t] = a.scale * (n / sqrt_d * d1 + gm * qjl * d2);
            }
        }
        __syncthreads();
        // online softmax, one thread per query head
        if (tid < G) {
            const int g = tid;
            float mnew = msh[g];
            for (int t = 0; t < ntok; ++t) mnew = fmaxf(mnew, sc[g][t]);
            const float c = __expf(msh[g] - mnew);
            float l = lsh[g] * c;
            for (int t = 0; t < ntok; ++t) {
                const float e = __expf(sc[g][t] - mnew);
                sc[g][t] = e;
                l += e;
            }
            corr[g] = c;
            msh[g] = mnew;
            lsh[g] = l;
        }
        __syncthreads();
        // values: thread owns rotated coordinate tid
        {
            const int j = tid;
#pragma unroll
            for (int g = 0; g < kMaxG; ++g)
                if (g < G) acc[g] *= corr[g];
            for (int t = 0; t < ntok; ++t) {
                const int c = extract_code(vchunk + t * a.lv.code_row, j, a.cbv.width);
                float cv = 0.f;
#pragma unroll
                for (int k = 0; k < kMaxLevels; ++k) cv = (k == c) ? a.cbv.c[k] : cv;
                const float vh = reinterpret_cast<const float*>(vchunk + a.lv.norm_off)[t] / sqrt_d * cv;
#pragma unroll
                for (int g = 0; g < kMaxG; ++g)
                    if (g < G) acc[g] = fmaf(sc[g][t], vh, acc[g]);
            }
        }
        __syncthreads();
    }
    for (int g = 0; g < G; ++g) {
        float* part = a.partial + (((size_t)b * a.Hq + hk * G + g) * a.splits + split) * kPartStride;
        if (tid == 0) {
            part[0] = msh[g];
            part[1] = lsh[g];
        }
        float av = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxG; ++k) av = (k == g) ? acc[k] : av;
        part[2 + tid] = av;
    }
}

__global__ void __launch_bounds__(kThreads) decode_merge_kernel(DecodeArgs a) {
    __shared__ float orot[kDim];
    const int bh = blockIdx.x, i = threadIdx.x;
    const float* part = a.partial + (size_t)bh * a.splits * kPartStride;
    float M = -INFINITY;
    for (int s = 0; s < a.splits; ++s) M = fmaxf(M, part[s * kPartStride]);
    float l = 0.f, acc = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < a.splits; ++s) {
            const float w = __expf(part[s * kPartStride] - M);  // exp(-inf) = 0 for empty splits
            l = fmaf(w, part[s * kPartStride + 1], l);
            acc = fmaf(w, part[s * kPartStride + 2 + i], acc);
        }
    }
    orot[i] = (l > 0.f) ? acc / l : 0.f;
    __syncthreads();
    float o = 0.f;
    for (int j = 0; j < kDim; ++j) o = fmaf(a.RT[j * kDim + i], orot[j], o);  // o_i = sum_j R[i][j] orot_j
    if (a.out_fp32)
        static_cast<float*>(a.out)[(size_t)bh * kDim + i] = o;
    else
        static_cast<__half*>(a.out)[(size_t)bh * kDim + i] = __float2half_rn(o);
}

}  // namespace

DecodePlan plan_decode(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_seq_len) {
    DecodePlan p{};
    p.max_pages = (max_seq_len + kPage - 1) / kPage;
    // enough splits that (B * Hkv) * splits CTAs cover two waves of the SMs
    long work = (long)B * Hkv;
    if (work < 1) work = 1;
    long splits = (2L * ctx->sm_count + work - 1) / work;
    if (splits > p.max_pages) splits = p.max_pages;
    if (splits < 1) splits = 1;
    p.splits = (int)splits;
    p.pages_per_split = p.max_pages > 0 ? (p.max_pages + p.splits - 1) / p.splits : 0;
    size_t off = 0;
    p.qprep_off = off;
    off += (size_t)B * Hq * 2 * kDim * sizeof(float);
    p.partial_off = off;
    off += (size_t)B * Hq * p.splits * kPartStride * sizeof(float);
    off = (off + 255) & ~size_t(255);
    p.ticket_off = off;
    off += (size_t)B * Hq * sizeof(uint32_t);
    p.bytes = (off + 255) & ~size_t(255);
    return p;
}

cudaError_t launch_decode(const tq_ctx* ctx, const DecodePlan& plan, const uint16_t* q, const uint8_t* kc,
                          const uint8_t* vc, int num_blocks, const int32_t* block_table, int max_blocks,
                          const int32_t* seq_lens, int B, int Hq, int Hkv, int max_seq_len, float scale, void* out,
                          int out_fp32, void* workspace, cudaStream_t stream) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    DecodeArgs a{q, kc, vc, num_blocks, block_table, max_blocks, seq_lens, B, Hq, Hkv, Hq / Hkv, max_seq_len, scale,
                 out, out_fp32, reinterpret_cast<float*>(ws + plan.qprep_off),
                 reinterpret_cast<float*>(ws + plan.partial_off), plan.splits, plan.pages_per_split, ctx->dev.R,
                 ctx->dev.RT, ctx->dev.ST, ctx->cb_key, ctx->cb_value, ctx->lay_key, ctx->lay_value, ctx->dev_error};
    decode_prep_kernel<<<B * Hq, kThreads, 0, stream>>>(a);
    decode_split_kernel<<<dim3(plan.splits, Hkv, B), kThreads, 0, stream>>>(a);
    decode_merge_kernel<<<B * Hq, kThreads, 0, stream>>>(a);
    count_launches(3);
    return cudaGetLastError();
}

}  // namespace tq
