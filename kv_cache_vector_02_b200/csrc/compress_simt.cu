// Compress step on CUDA cores (fp32), one thread per output coordinate.
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…", section "TurboQuant" steps 1-4 and
// section "注意力计算的特殊挑战与QJL校正":
//   n = ||x||, y = R^T x, code_j = #{k : t_k < sqrt(d) y_j / n}, store (codes, n);
//   prod keys: r = y - n c[code]/sqrt(d) (the residual in the rotated domain),
//   sign_j = [(S R r)_j >= 0], gamma = ||r||.
// Working in the rotated domain is exact algebra: R is orthogonal, so
// ||x - x_hat|| = ||y - y_hat|| and S (x - x_hat) = (S R)(y - y_hat).
//
// This is the plain CUDA-core form of the step: it serves the small
// launches (a decode step appending a few tokens) and is the reference layout
// for the tensor-core kernel.
#include "device_util.cuh"

namespace tq {
namespace {

constexpr int kGroup = 128;  // threads per vector group (one per coordinate)
constexpr int kGroups = 2;   // groups per CTA
constexpr int kVB = 8;       // vectors per group iteration

struct CompressArgs {
    const uint16_t* x;
    int T, H;
    const int32_t* slots;
    uint8_t* cache;
    int num_blocks;
    const float* R;   // row-major R[i][j]
    const float* MT;  // row-major M^T, M = S R (prod keys)
    Codebook cb;
    ChunkLayout lay;
    uint32_t* err;
};

template <bool kProd>
__global__ void __launch_bounds__(kGroup * kGroups) compress_simt_kernel(CompressArgs a) {
    extern __shared__ float4 smem_raw[];
    float* Rs = reinterpret_cast<float*>(smem_raw);
    float* Ms = Rs + kDim * kDim;
    float* gbase = Ms + (kProd ? kDim * kDim : 0);
    constexpr int kGroupFloats = 2 * kVB * kDim + 8 * kVB + 32;
    const int tid = threadIdx.x, g = tid / kGroup, j = tid % kGroup, lane = tid & 31, wg = j >> 5;
    float* xs = gbase + g * kGroupFloats;     // [kVB][128]
    float* rs = xs + kVB * kDim;              // [kVB][128]
    float* red = rs + kVB * kDim;             // [4][kVB] norm partials
    float* red2 = red + 4 * kVB;              // [4][kVB] gamma partials
    float* cs = red2 + 4 * kVB;               // [16] levels

    for (int i = tid; i < kDim * kDim / 4; i += blockDim.x) {
        reinterpret_cast<float4*>(Rs)[i] = reinterpret_cast<const float4*>(a.R)[i];
        if (kProd) reinterpret_cast<float4*>(Ms)[i] = reinterpret_cast<const float4*>(a.MT)[i];
    }
    if (j < kMaxLevels) cs[j] = a.cb.c[j];
    __syncthreads();

    const long N = (long)a.T * a.H;
    const long nbatch = (N + kVB - 1) / kVB;
    const float sqrt_d = sqrtf((float)kDim);
    const int w = a.cb.width;
    const long max_slot = (long)a.num_blocks * kPage;

    for (long bi = (long)blockIdx.x * kGroups + g; bi < nbatch; bi += (long)gridDim.x * kGroups) {
        const long v0 = bi * kVB;
        float sq[kVB];
#pragma unroll
        for (int v = 0; v < kVB; ++v) {
            const long vi = v0 + v;
            const float xv = vi < N ? half_bits_to_float(a.x[vi * kDim + j]) : 0.f;
            xs[v * kDim + j] = xv;
            sq[v] = warp_sum(xv * xv);
        }
        if (lane == 0)
#pragma unroll
            for (int v = 0; v < kVB; ++v) red[wg * kVB + v] = sq[v];
        named_barrier(1 + g, kGroup);

        float nrm[kVB], acc[kVB];
#pragma unroll
        for (int v = 0; v < kVB; ++v) {
            nrm[v] = sqrtf(((red[v] + red[kVB + v]) + red[2 * kVB + v]) + red[3 * kVB + v]);
            acc[v] = 0.f;
        }
        // y_j = sum_i R[i][j] x_i
#pragma unroll 2
        for (int i = 0; i < kDim; i += 4) {
            const float r0 = Rs[(i + 0) * kDim + j], r1 = Rs[(i + 1) * kDim + j];
            const float r2 = Rs[(i + 2) * kDim + j], r3 = Rs[(i + 3) * kDim + j];
#pragma unroll
            for (int v = 0; v < kVB; ++v) {
                const float4 xv = *reinterpret_cast<const float4*>(&xs[v * kDim + i]);
                acc[v] = fmaf(r0, xv.x, acc[v]);
                acc[v] = fmaf(r1, xv.y, acc[v]);
                acc[v] = fmaf(r2, xv.z, acc[v]);
                acc[v] = fmaf(r3, xv.w, acc[v]);
            }
        }
        int code[kVB];
#pragma unroll
        for (int v = 0; v < kVB; ++v) {
            if (nrm[v] > 0.f) {
                const float val = acc[v] * (sqrt_d / nrm[v]);
                int idx = 0;
#pragma unroll
                for (int k = 0; k < kMaxLevels - 1; ++k) idx += (a.cb.t[k] < val) ? 1 : 0;
                code[v] = idx;
            } else {
                code[v] = a.cb.levels / 2 - 1;
            }
        }
        float gam[kVB];
        uint32_t sign_word[kVB];
        if (kProd) {
#pragma unroll
            for (int v = 0; v < kVB; ++v) {
                const float r = acc[v] - cs[code[v]] * (nrm[v] / sqrt_d);
                rs[v * kDim + j] = r;
                sq[v] = warp_sum(r * r);
            }
            if (lane == 0)
#pragma unroll
                for (int v = 0; v < kVB; ++v) red2[wg * kVB + v] = sq[v];
            named_barrier(1 + g, kGroup);
            float sk[kVB];
#pragma unroll
            for (int v = 0; v < kVB; ++v) {
                gam[v] = sqrtf(((red2[v] + red2[kVB + v]) + red2[2 * kVB + v]) + red2[3 * kVB + v]);
                sk[v] = 0.f;
            }
            // (S r)_j = sum_i M[j][i] r_i, M^T stored row-major
#pragma unroll 2
            for (int i = 0; i < kDim; i += 4) {
                const float m0 = Ms[(i + 0) * kDim + j], m1 = Ms[(i + 1) * kDim + j];
                const float m2 = Ms[(i + 2) * kDim + j], m3 = Ms[(i + 3) * kDim + j];
#pragma unroll
                for (int v = 0; v < kVB; ++v) {
                    const float4 rv = *reinterpret_cast<const float4*>(&rs[v * kDim + i]);
                    sk[v] = fmaf(m0, rv.x, sk[v]);
                    sk[v] = fmaf(m1, rv.y, sk[v]);
                    sk[v] = fmaf(m2, rv.z, sk[v]);
                    sk[v] = fmaf(m3, rv.w, sk[v]);
                }
            }
#pragma unroll
            for (int v = 0; v < kVB; ++v) sign_word[v] = __ballot_sync(0xffffffffu, sk[v] >= 0.f);
        }
        // pack and store
#pragma unroll
        for (int v = 0; v < kVB; ++v) {
            const long vi = v0 + v;
            if (vi >= N) break;
            const int t = (int)(vi / a.H), h = (int)(vi % a.H);
            const long s = a.slots[t];
            if (s < 0) continue;
            if (s >= max_slot) {
                if (j == 0) atomicOr(a.err, TQ_DEVERR_SLOT);
                continue;
            }
            uint8_t* chunk = a.cache + ((size_t)(s / kPage) * a.H + h) * (size_t)a.lay.bytes;
            const int row = (int)(s % kPage);
            const int per_word = 32 / w;  // codes per 32-bit word
            uint32_t word = (uint32_t)code[v] << (w * (lane % per_word));
            word = warp_or_within(word, per_word);
            if (lane % per_word == 0)
                *reinterpret_cast<uint32_t*>(chunk + row * a.lay.code_row + (j / per_word) * 4) = word;
            if (kProd && lane == 0)
                *reinterpret_cast<uint32_t*>(chunk + a.lay.signs_off + row * (kDim / 8) + wg * 4) = sign_word[v];
            if (j == 0) {
                reinterpret_cast<float*>(chunk + a.lay.norm_off)[row] = nrm[v];
                if (kProd) reinterpret_cast<float*>(chunk + a.lay.gamma_off)[row] = gam[v];
            }
        }
        named_barrier(1 + g, kGroup);
    }
}

size_t smem_bytes(bool prod) {
    return sizeof(float) * ((prod ? 2 : 1) * kDim * kDim + kGroups * (2 * kVB * kDim + 8 * kVB + 32));
}

}  // namespace

cudaError_t launch_compress_simt(const tq_ctx* ctx, int kind, const uint16_t* x, int T, int H,
                                 const int32_t* slots, uint8_t* cache, int num_blocks, cudaStream_t stream) {
    const bool value = (kind == TQ_KIND_VALUE);
    const ChunkLayout& lay = value ? ctx->lay_value : ctx->lay_key;
    CompressArgs a{x, T, H, slots, cache, num_blocks, ctx->dev.R, ctx->dev.MT,
                   value ? ctx->cb_value : ctx->cb_key, lay, ctx->dev_error};
    const long N = (long)T * H;
    const long nbatch = (N + kVB - 1) / kVB;
    const bool prod = lay.prod;
    const size_t smem = smem_bytes(prod);
    const int per_sm = prod ? 1 : 2;
    long grid = (nbatch + kGroups - 1) / kGroups;
    if (grid > (long)ctx->sm_count * per_sm) grid = (long)ctx->sm_count * per_sm;
    if (grid < 1) grid = 1;
    cudaError_t e;
    if (prod) {
        e = cudaFuncSetAttribute(compress_simt_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        compress_simt_kernel<true><<<(unsigned)grid, kGroup * kGroups, smem, stream>>>(a);
    } else {
        e = cudaFuncSetAttribute(compress_simt_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        compress_simt_kernel<false><<<(unsigned)grid, kGroup * kGroups, smem, stream>>>(a);
    }
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_compress(const tq_ctx* ctx, int kind, const uint16_t* x, int T, int H, const int32_t* slots,
                            uint8_t* cache, int num_blocks, cudaStream_t stream) {
    return launch_compress_simt(ctx, kind, x, T, H, slots, cache, num_blocks, stream);
}

}  // namespace tq
