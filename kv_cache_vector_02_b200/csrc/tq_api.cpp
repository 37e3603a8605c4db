// C ABI of libtq: validation, parameter upload, dispatch.  The arithmetic of
// the hot path runs in the CUDA translation units; this file only checks
// arguments, owns the context and launches.
#include <nvtx3/nvToolsExt.h>
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_fp16.h>

#include "tq_internal.h"

using tq::kDim;

namespace {
std::atomic<uint64_t> g_launches{0};
}

void tq::count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

bool tq::take_stall(const tq_ctx* ctx) {
    int n = ctx->debug_stall.load(std::memory_order_relaxed);
    while (n > 0)
        if (ctx->debug_stall.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) return true;
    return false;
}

namespace {

tq::ChunkLayout make_layout(int code_bits, bool prod) {
    tq::ChunkLayout L{};
    L.prod = prod;
    L.code_row = kDim * tq::container_width(code_bits) / 8;
    int off = tq::kPage * L.code_row;
    if (prod) {
        L.signs_off = off;
        off += tq::kPage * (kDim / 8);
    } else {
        L.signs_off = -1;
    }
    L.norm_off = off;
    off += tq::kPage * 4;
    if (prod) {
        L.gamma_off = off;
        off += tq::kPage * 4;
    } else {
        L.gamma_off = -1;
    }
    L.bytes = off;
    return L;
}

tq::Codebook make_codebook(const std::vector<double>& c, const std::vector<double>& t, int bits) {
    tq::Codebook cb{};
    cb.bits = bits;
    cb.levels = 1 << bits;
    cb.width = tq::container_width(bits);
    for (int j = 0; j < tq::kMaxLevels; ++j) {
        cb.c[j] = j < cb.levels ? float(c[j]) : 0.f;
        cb.t[j] = j < cb.levels - 1 ? float(t[j]) : INFINITY;
    }
    return cb;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around each device entry point, named after it, for Nsight timelines;
// with no tool attached a push / pop costs a pointer test.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Records that ctx's parameters are in use by work queued on `stream` up to now.
// Returns false if the event could not be created or recorded.
bool note_use(const tq_ctx* ctx, cudaStream_t stream) {
    std::lock_guard<std::mutex> lock(ctx->use_mu);
    for (auto& u : ctx->uses)
        if (u.stream == stream) return cudaEventRecord(u.done, stream) == cudaSuccess;
    if (ctx->uses.size() >= 32) {  // many streams: the oldest one's work is waited for and its slot reused
        tq_ctx::StreamUse& old = ctx->uses.front();
        if (cudaEventSynchronize(old.done) != cudaSuccess) return false;
        old.stream = stream;
        std::rotate(ctx->uses.begin(), ctx->uses.begin() + 1, ctx->uses.end());
        return cudaEventRecord(ctx->uses.back().done, stream) == cudaSuccess;
    }
    tq_ctx::StreamUse u{stream, nullptr};
    if (cudaEventCreateWithFlags(&u.done, cudaEventDisableTiming) != cudaSuccess) return false;
    if (cudaEventRecord(u.done, stream) != cudaSuccess) {
        cudaEventDestroy(u.done);
        return false;
    }
    ctx->uses.push_back(u);
    return true;
}

}  // namespace

extern "C" {

uint64_t tq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

tq_status tq_debug_stall(tq_ctx* ctx, int launches) {
    if (!ctx || ctx->host_only || launches < 0) return TQ_ERR_INVALID_ARG;
    ctx->debug_stall.store(launches, std::memory_order_relaxed);
    return TQ_OK;
}

const char* tq_status_string(tq_status s) {
    switch (s) {
        case TQ_OK: return "TQ_OK";
        case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
        case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
        case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
        case TQ_ERR_OOM: return "TQ_ERR_OOM";
        case TQ_ERR_DEVICE: return "TQ_ERR_DEVICE";
    }
    return "TQ_ERR_UNKNOWN";
}

static tq_status validate_init(int head_dim, int bits, int rotation, int key_mode, int flags) {
    if (head_dim != kDim) return TQ_ERR_UNSUPPORTED;
    if (bits < 2 || bits > 4) return TQ_ERR_UNSUPPORTED;
    if (rotation != TQ_ROT_HAAR && rotation != TQ_ROT_HADAMARD) return TQ_ERR_UNSUPPORTED;
    if (key_mode != TQ_KEY_PROD && key_mode != TQ_KEY_MSE) return TQ_ERR_UNSUPPORTED;
    if (flags & ~(TQ_FLAG_SPHERE_CODEBOOK | TQ_FLAG_HOST_ONLY)) return TQ_ERR_UNSUPPORTED;
    return TQ_OK;
}

static void fill_host(tq_ctx* ctx, int head_dim, int bits, uint64_t seed, int rotation, int key_mode, int flags) {
    ctx->host = tq::make_host_params(head_dim, bits, seed, rotation, key_mode, flags & TQ_FLAG_SPHERE_CODEBOOK);
    const tq::HostParams& H = ctx->host;
    ctx->cb_value = make_codebook(H.cv, H.tv, H.vbits);
    ctx->cb_key = make_codebook(H.ck, H.tk, H.kbits);
    ctx->lay_value = make_layout(H.vbits, false);
    ctx->lay_key = make_layout(H.kbits, key_mode == TQ_KEY_PROD);
}

static tq_status init_host_only(int head_dim, int bits, uint64_t seed, int rotation, int key_mode, int flags,
                                tq_ctx** out) {
    tq_ctx* ctx = new (std::nothrow) tq_ctx();
    if (!ctx) return TQ_ERR_OOM;
    ctx->host_only = true;
    fill_host(ctx, head_dim, bits, seed, rotation, key_mode, flags);
    tq::TcBlob tcb;  // same tables as a device context, built to surface any failure here too
    if (!tq::build_tc_blob(ctx->host, tcb)) {
        delete ctx;
        return TQ_ERR_UNSUPPORTED;
    }
    *out = ctx;
    return TQ_OK;
}

tq_status tq_init_host(int head_dim, int bits, uint64_t seed, int rotation, int key_mode, tq_ctx** out) {
    return tq_init_ex(head_dim, bits, seed, rotation, key_mode, TQ_FLAG_HOST_ONLY, out);
}

tq_status tq_init(int head_dim, int bits, uint64_t seed, int rotation, int key_mode, tq_ctx** out) {
    return tq_init_ex(head_dim, bits, seed, rotation, key_mode, 0, out);
}

tq_status tq_init_ex(int head_dim, int bits, uint64_t seed, int rotation, int key_mode, int flags, tq_ctx** out) {
    if (!out) return TQ_ERR_INVALID_ARG;
    *out = nullptr;
    const tq_status v = validate_init(head_dim, bits, rotation, key_mode, flags);
    if (v != TQ_OK) return v;
    if (flags & TQ_FLAG_HOST_ONLY) return init_host_only(head_dim, bits, seed, rotation, key_mode, flags, out);

    tq_ctx* ctx = new (std::nothrow) tq_ctx();
    if (!ctx) return TQ_ERR_OOM;
    if (cudaGetDevice(&ctx->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&ctx->sm_count, cudaDevAttrMultiProcessorCount, ctx->device) != cudaSuccess) {
        delete ctx;
        cudaGetLastError();
        return TQ_ERR_CUDA;
    }
    fill_host(ctx, head_dim, bits, seed, rotation, key_mode, flags);
    const tq::HostParams& H = ctx->host;

    // device copies: R^T and S (fp32; decompress), R^T hi / lo and S (fp16; decode prep),
    // R hi / lo (fp16; decode merge); then the tensor-core blob
    const size_t n = size_t(kDim) * kDim;
    std::vector<float> blob(2 * n);
    std::vector<__half> blob16(5 * n);
    float* RT = blob.data();
    float* S = RT + n;
    for (int i = 0; i < kDim; ++i)
        for (int j = 0; j < kDim; ++j) {
            const double r = H.R[size_t(i) * kDim + j];
            RT[j * kDim + i] = float(r);
            S[i * kDim + j] = float(H.S[size_t(i) * kDim + j]);
            const __half hi = __double2half(r);
            blob16[size_t(j) * kDim + i] = hi;
            blob16[n + size_t(j) * kDim + i] = __double2half(r - double(__half2float(hi)));
            blob16[2 * n + size_t(i) * kDim + j] = __double2half(double(H.S[size_t(i) * kDim + j]));
            blob16[3 * n + size_t(i) * kDim + j] = hi;  // R row-major, hi / lo (decode merge)
            blob16[4 * n + size_t(i) * kDim + j] = blob16[n + size_t(j) * kDim + i];
        }
    tq::TcBlob tcb;
    if (!tq::build_tc_blob(H, tcb)) {
        delete ctx;
        return TQ_ERR_UNSUPPORTED;
    }
    const size_t f32_bytes = blob.size() * sizeof(float);
    const size_t f16_off = f32_bytes;
    const size_t f16_bytes = blob16.size() * sizeof(__half);
    const size_t tc_off = (f16_off + f16_bytes + 1023) & ~size_t(1023);
    const size_t bytes = tc_off + tcb.bytes.size();
    if (cudaMalloc(&ctx->dev_block, bytes) != cudaSuccess) {
        cudaGetLastError();
        delete ctx;
        return TQ_ERR_OOM;
    }
    if (cudaMalloc(reinterpret_cast<void**>(&ctx->dev_error), sizeof(uint32_t)) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(ctx->dev_block);
        delete ctx;
        return TQ_ERR_OOM;
    }
    uint8_t* base8 = static_cast<uint8_t*>(ctx->dev_block);
    if (cudaMemcpy(base8, blob.data(), f32_bytes, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base8 + f16_off, blob16.data(), f16_bytes, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base8 + tc_off, tcb.bytes.data(), tcb.bytes.size(), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemset(ctx->dev_error, 0, sizeof(uint32_t)) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(ctx->dev_block);
        cudaFree(ctx->dev_error);
        delete ctx;
        return TQ_ERR_CUDA;
    }
    const float* base = static_cast<const float*>(ctx->dev_block);
    ctx->dev.RT = base;
    ctx->dev.S = base + n;
    const uint16_t* base16 = reinterpret_cast<const uint16_t*>(base8 + f16_off);
    ctx->dev.RTh = base16;
    ctx->dev.RTl = base16 + n;
    ctx->dev.Sh = base16 + 2 * n;
    ctx->dev.Rh = base16 + 3 * n;
    ctx->dev.Rl = base16 + 4 * n;
    ctx->tc.images = base8 + tc_off + tcb.off_images;
    ctx->tc.lut_value = base8 + tc_off + tcb.off_lut_value;
    ctx->tc.lut_key = base8 + tc_off + tcb.off_lut_key;
    ctx->tc.lp_value = tcb.lp_value;
    ctx->tc.lp_key = tcb.lp_key;
    *out = ctx;
    return TQ_OK;
}

tq_status tq_destroy(tq_ctx* ctx) {
    if (!ctx) return TQ_OK;
    if (ctx->host_only) {
        delete ctx;
        return TQ_OK;
    }
    // the context's own work: every stream it launched on, up to its latest launch
    // (cudaFree below may still wait for the device as the runtime sees fit)
    {
        std::lock_guard<std::mutex> lock(ctx->use_mu);
        for (auto& u : ctx->uses) {
            cudaEventSynchronize(u.done);
            cudaEventDestroy(u.done);
        }
        ctx->uses.clear();
    }
    cudaFree(ctx->dev_block);
    cudaFree(ctx->dev_error);
    cudaGetLastError();
    delete ctx;
    return TQ_OK;
}

size_t tq_chunk_bytes(const tq_ctx* ctx, int kind) {
    if (!ctx) return 0;
    if (kind == TQ_KIND_KEY) return size_t(ctx->lay_key.bytes);
    if (kind == TQ_KIND_VALUE) return size_t(ctx->lay_value.bytes);
    return 0;
}

int tq_code_bits(const tq_ctx* ctx, int kind) {
    if (!ctx) return -1;
    if (kind == TQ_KIND_KEY) return ctx->host.kbits;
    if (kind == TQ_KIND_VALUE) return ctx->host.vbits;
    return -1;
}

tq_status tq_export_params(const tq_ctx* ctx, double* R, int8_t* S, int8_t* hsigns, double* cv, double* tv,
                           double* ck, double* tk) {
    if (!ctx) return TQ_ERR_INVALID_ARG;
    const tq::HostParams& H = ctx->host;
    if (R) std::memcpy(R, H.R.data(), H.R.size() * sizeof(double));
    if (S) std::memcpy(S, H.S.data(), H.S.size());
    if (hsigns && !H.hsigns.empty()) std::memcpy(hsigns, H.hsigns.data(), H.hsigns.size());
    if (cv) std::memcpy(cv, H.cv.data(), H.cv.size() * sizeof(double));
    if (tv) std::memcpy(tv, H.tv.data(), H.tv.size() * sizeof(double));
    if (ck) std::memcpy(ck, H.ck.data(), H.ck.size() * sizeof(double));
    if (tk) std::memcpy(tk, H.tk.data(), H.tk.size() * sizeof(double));
    return TQ_OK;
}

tq_status tq_compress(const tq_ctx* ctx, const uint16_t* k, const uint16_t* v, int T, int Hkv,
                      const int32_t* slot_mapping, uint8_t* k_cache, uint8_t* v_cache, int num_blocks,
                      void* stream) {
    NvtxRange nvtx("tq_compress");
    if (!ctx || ctx->host_only || T < 0 || Hkv < 1 || num_blocks < 0) return TQ_ERR_INVALID_ARG;
    if (T == 0) return TQ_OK;
    if (!slot_mapping || (!k && !v)) return TQ_ERR_INVALID_ARG;
    if ((k && !k_cache) || (v && !v_cache)) return TQ_ERR_INVALID_ARG;
    if ((k && (!aligned16(k) || !aligned16(k_cache))) || (v && (!aligned16(v) || !aligned16(v_cache))))
        return TQ_ERR_INVALID_ARG;
    if ((long long)T * Hkv > (1ll << 31) - 1) return TQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (k && tq::launch_compress(ctx, TQ_KIND_KEY, k, T, Hkv, slot_mapping, k_cache, num_blocks, s) != cudaSuccess)
        return TQ_ERR_CUDA;
    if (v && tq::launch_compress(ctx, TQ_KIND_VALUE, v, T, Hkv, slot_mapping, v_cache, num_blocks, s) != cudaSuccess)
        return TQ_ERR_CUDA;
    return note_use(ctx, s) ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_decompress(const tq_ctx* ctx, int kind, const uint8_t* cache, int num_blocks,
                        const int32_t* slot_mapping, int T, int Hkv, void* out, int out_fp32, void* stream) {
    NvtxRange nvtx("tq_decompress");
    if (!ctx || ctx->host_only || T < 0 || Hkv < 1 || num_blocks < 0) return TQ_ERR_INVALID_ARG;
    if (kind != TQ_KIND_KEY && kind != TQ_KIND_VALUE) return TQ_ERR_INVALID_ARG;
    if (T == 0) return TQ_OK;
    if (!cache || !slot_mapping || !out) return TQ_ERR_INVALID_ARG;
    if (!aligned16(cache) || !aligned16(out)) return TQ_ERR_INVALID_ARG;
    if (tq::launch_decompress(ctx, kind, cache, num_blocks, slot_mapping, T, Hkv, out, out_fp32,
                              static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return TQ_ERR_CUDA;
    return note_use(ctx, static_cast<cudaStream_t>(stream)) ? TQ_OK : TQ_ERR_CUDA;
}

size_t tq_decode_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_seq_len) {
    if (!ctx || ctx->host_only || B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || max_seq_len < 0) return 0;
    return tq::plan_decode(ctx, B, Hq, Hkv, max_seq_len).bytes;
}

namespace {
tq_status decode_common(const tq_ctx* ctx, const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                        int num_blocks, const int32_t* block_table, int max_blocks, const int32_t* seq_lens, int B,
                        int Hq, int Hkv, int max_seq_len, const tq::DecodeTail& tail, float scale, void* out,
                        int out_fp32, void* workspace, size_t workspace_bytes, void* stream) {
    NvtxRange nvtx("tq_decode_attention");
    if (!ctx || ctx->host_only || B < 0 || Hq < 1 || Hkv < 1 || max_blocks < 0 || num_blocks < 0 || max_seq_len < 0)
        return TQ_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || Hq / Hkv > 16) return TQ_ERR_INVALID_ARG;
    if (B == 0) return TQ_OK;
    if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out || !workspace) return TQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace))
        return TQ_ERR_INVALID_ARG;
    if (tail.k) {
        if (!tail.v || !tail.lens || tail.cap < 1 || tail.cap > tq::kDecodeTailMax) return TQ_ERR_INVALID_ARG;
        if (!aligned16(tail.k) || !aligned16(tail.v)) return TQ_ERR_INVALID_ARG;
    }
    if (!(scale >= 0.f) || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
    const tq::DecodePlan plan = tq::plan_decode(ctx, B, Hq, Hkv, max_seq_len);
    if (workspace_bytes < plan.bytes) return TQ_ERR_INVALID_ARG;
    if (scale == 0.f) scale = 1.0f / std::sqrt(float(kDim));
    if (tq::launch_decode(ctx, plan, q, k_cache, v_cache, num_blocks, block_table, max_blocks, seq_lens, B, Hq, Hkv,
                          max_seq_len, tail, scale, out, out_fp32, workspace, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return TQ_ERR_CUDA;
    return note_use(ctx, static_cast<cudaStream_t>(stream)) ? TQ_OK : TQ_ERR_CUDA;
}
}  // namespace

tq_status tq_decode_attention(const tq_ctx* ctx, const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                              int num_blocks, const int32_t* block_table, int max_blocks, const int32_t* seq_lens,
                              int B, int Hq, int Hkv, int max_seq_len, float scale, void* out, int out_fp32,
                              void* workspace, size_t workspace_bytes, void* stream) {
    return decode_common(ctx, q, k_cache, v_cache, num_blocks, block_table, max_blocks, seq_lens, B, Hq, Hkv,
                         max_seq_len, tq::DecodeTail{}, scale, out, out_fp32, workspace, workspace_bytes, stream);
}

tq_status tq_prefill_attention(const tq_ctx* ctx, const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                               int num_blocks, const int32_t* block_table, int max_blocks, int q_start, int Tq, int Hq,
                               int Hkv, float scale, void* out, int out_fp32, void* stream) {
    NvtxRange nvtx("tq_prefill_attention");
    if (!ctx || ctx->host_only || Tq < 0 || q_start < 0 || Hq < 1 || Hkv < 1 || max_blocks < 0 || num_blocks < 0)
        return TQ_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || Hq > 65535) return TQ_ERR_INVALID_ARG;  // one grid row per query head
    if (Tq == 0) return TQ_OK;
    if ((long long)q_start + Tq > (long long)max_blocks * tq::kPage) return TQ_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !block_table || !out) return TQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return TQ_ERR_INVALID_ARG;
    if (!(scale >= 0.f) || !std::isfinite(scale)) return TQ_ERR_INVALID_ARG;
    if (scale == 0.f) scale = 1.0f / std::sqrt(float(kDim));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tq::launch_prefill(ctx, q, k_cache, v_cache, num_blocks, block_table, max_blocks, q_start, Tq, Hq, Hkv, scale,
                           out, out_fp32, s) != cudaSuccess)
        return TQ_ERR_CUDA;
    return note_use(ctx, s) ? TQ_OK : TQ_ERR_CUDA;
}

tq_status tq_decode_attention_window(const tq_ctx* ctx, const uint16_t* q, const uint8_t* k_cache,
                                     const uint8_t* v_cache, int num_blocks, const int32_t* block_table,
                                     int max_blocks, const int32_t* seq_lens, int B, int Hq, int Hkv,
                                     int max_seq_len, const uint16_t* tail_k, const uint16_t* tail_v,
                                     const int32_t* tail_lens, int tail_cap, float scale, void* out, int out_fp32,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    if (!tail_k) return TQ_ERR_INVALID_ARG;
    tq::DecodeTail tail;
    tail.k = tail_k;
    tail.v = tail_v;
    tail.lens = tail_lens;
    tail.cap = tail_cap;
    return decode_common(ctx, q, k_cache, v_cache, num_blocks, block_table, max_blocks, seq_lens, B, Hq, Hkv,
                         max_seq_len, tail, scale, out, out_fp32, workspace, workspace_bytes, stream);
}

tq_status tq_get_device_error(const tq_ctx* ctx, void* stream, uint32_t* code) {
    if (!ctx || ctx->host_only || !code) return TQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t h = 0;
    if (cudaMemcpyAsync(&h, ctx->dev_error, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return TQ_ERR_CUDA;
    }
    if (h && (cudaMemsetAsync(ctx->dev_error, 0, sizeof(uint32_t), s) != cudaSuccess ||
              cudaStreamSynchronize(s) != cudaSuccess)) {
        cudaGetLastError();
        return TQ_ERR_CUDA;
    }
    *code = h;
    return h ? TQ_ERR_DEVICE : TQ_OK;
}

}  // extern "C"
