// Decompress step (not on the timed path).
//
// [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…", section "架构设计" (Decompress:
// unpack + dequantize).  MSE: x_hat = n R c[idx] / sqrt(d).  Prod keys add the
// QJL term gamma sqrt(pi/2)/d S^T (2 sigma - 1), which makes <q, x_tilde> equal to
// the estimator of section "注意力计算的特殊挑战与QJL校正" for every q.
#include "device_util.cuh"

namespace tq {
namespace {

constexpr int kVB = 4;  // vectors per CTA iteration

struct DecompressArgs {
    const uint8_t* cache;
    int num_blocks;
    const int32_t* slots;
    int T, H;
    void* out;
    int out_fp32;
    const float* RT;  // R^T row-major: RT[j][i] = R[i][j]
    const float* S;   // S row-major as +-1.0f
    Codebook cb;
    ChunkLayout lay;
    uint32_t* err;
};

__global__ void __launch_bounds__(kDim) decompress_kernel(DecompressArgs a) {
    __shared__ float chat[kVB][kDim];
    __shared__ float sgn[kVB][kDim];
    __shared__ float nrm[kVB], gam[kVB];
    __shared__ int valid[kVB];
    const int i = threadIdx.x;
    const long N = (long)a.T * a.H;
    const long max_slot = (long)a.num_blocks * kPage;
    const float sqrt_d = sqrtf((float)kDim);
    const float qjl = sqrtf(3.14159265358979f / 2.f) / kDim;
    for (long v0 = (long)blockIdx.x * kVB; v0 < N; v0 += (long)gridDim.x * kVB) {
#pragma unroll
        for (int v = 0; v < kVB; ++v) {
            const long vi = v0 + v;
            int ok = 0;
            const uint8_t* chunk = nullptr;
            int row = 0;
            if (vi < N) {
                const long s = a.slots[vi / a.H];
                if (s >= max_slot) {
                    if (i == 0) atomicOr(a.err, TQ_DEVERR_SLOT);
                } else if (s >= 0) {
                    ok = 1;
                    chunk = a.cache + ((size_t)(s / kPage) * a.H + vi % a.H) * (size_t)a.lay.bytes;
                    row = (int)(s % kPage);
                }
            }
            if (ok) {
                const int c = extract_code(chunk + row * a.lay.code_row, i, a.cb.width);
                float cval = 0.f;
#pragma unroll
                for (int k = 0; k < kMaxLevels; ++k) cval = (k == c) ? a.cb.c[k] : cval;
                chat[v][i] = cval;
                if (a.lay.prod) sgn[v][i] = extract_code(chunk + a.lay.signs_off + row * (kDim / 8), i, 1) ? 1.f : -1.f;
                if (i == 0) {
                    nrm[v] = reinterpret_cast<const float*>(chunk + a.lay.norm_off)[row];
                    gam[v] = a.lay.prod ? reinterpret_cast<const float*>(chunk + a.lay.gamma_off)[row] : 0.f;
                }
            }
            if (i == 0) valid[v] = ok;
        }
        __syncthreads();
#pragma unroll
        for (int v = 0; v < kVB; ++v) {
            if (!valid[v]) continue;
            float s = 0.f, q = 0.f;
            for (int jj = 0; jj < kDim; ++jj) {
                s = fmaf(a.RT[jj * kDim + i], chat[v][jj], s);
                if (a.lay.prod) q = fmaf(a.S[jj * kDim + i], sgn[v][jj], q);
            }
            float xv = nrm[v] / sqrt_d * s;
            if (a.lay.prod) xv = fmaf(gam[v] * qjl, q, xv);
            const long o = (v0 + v) * kDim + i;
            if (a.out_fp32)
                static_cast<float*>(a.out)[o] = xv;
            else
                static_cast<__half*>(a.out)[o] = __float2half_rn(xv);
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_decompress(const tq_ctx* ctx, int kind, const uint8_t* cache, int num_blocks,
                              const int32_t* slots, int T, int H, void* out, int out_fp32, cudaStream_t stream) {
    const bool value = (kind == TQ_KIND_VALUE);
    DecompressArgs a{cache, num_blocks, slots, T, H, out, out_fp32, ctx->dev.RT, ctx->dev.S,
                     value ? ctx->cb_value : ctx->cb_key, value ? ctx->lay_value : ctx->lay_key, ctx->dev_error};
    const long N = (long)T * H;
    long grid = (N + kVB - 1) / kVB;
    if (grid > (long)ctx->sm_count * 8) grid = (long)ctx->sm_count * 8;
    if (grid < 1) grid = 1;
    decompress_kernel<<<(unsigned)grid, kDim, 0, stream>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace tq
