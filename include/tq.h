/*
 * libtq -- TurboQuant-style KV-cache compression and decode attention for
 * NVIDIA B200 (sm_100a).  C ABI.
 *
 * Method sources (cited by page title and section):
 *   [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案，让大模型推理显存占用降低7.5倍"
 *           (zingnex.cn, thread flashquant-kv-7-5):
 *           - "TurboQuant：Google Research的突破性算法": the four compress steps
 *             (1 normalize, 2 rotate by a Haar orthogonal R^T, 3 Gaussian
 *             Lloyd-Max scalar quantization, 4 nibble packing + fp32 norm);
 *           - "注意力计算的特殊挑战与QJL校正": the QJL key estimator
 *             <q,k> ~ <q,k_mse> + gamma*sqrt(pi/2)/d*<Sq, sign(Sr)>;
 *           - "架构设计": Compress / Decompress / Paged Decode (split-K
 *             FlashDecoding) kernels; Quantizer in MSE and Prod modes.
 *   [TQ-RS] "TurboQuant : compresser le KV-cache des LLM par 7x sans perdre en
 *           qualité" (patricehuetz.fr): "Couche 1" randomized Walsh-Hadamard
 *           rotation, "Couche 3" packing, "Couche 4" fp32 norms.
 *   [FQ-I4] "FlashQuant : Compression KV-Cache 7.5x CUDA pour LLM"
 *           (ayinedjimi-consultants.fr), "Architecture": 16-token PagedAttention
 *           blocks.
 *
 * Conventions shared by every call
 *   - d (head_dim) = 128.  Vectors are fp16, passed as uint16_t bit patterns.
 *   - Pointers named *_dev are device pointers; the caller allocates and owns
 *     every device buffer and stream.  The context owns only its parameters.
 *   - stream is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream.  Every call that takes a stream is asynchronous on it.
 *   - Errors are reported only through the returned tq_status; nothing aborts,
 *     traps or throws across the ABI.  Host-side validation runs before any
 *     launch.  Conditions that only the device can see (a slot or block id out
 *     of range, a sequence longer than its block table) make the kernel skip
 *     that item and set a bit in the context's device error word, read with
 *     tq_get_device_error.
 *   - A context is immutable after tq_init; calls on different streams may run
 *     concurrently (they share only the device error word).
 *
 * Paged cache layout (one "chunk" = one physical block x one kv head, 16 tokens):
 *   cache[num_blocks][Hkv][chunk_bytes], slot = block * 16 + row.
 *   container width w(b) = 4 bits for b in {3,4}, 2 for b = 2, 1 for b = 1.
 *   MSE chunk  (values; keys in TQ_KEY_MSE):
 *       codes[16][d*w/8] | norm f32[16]
 *   prod chunk (keys in TQ_KEY_PROD, code bits b-1):
 *       codes[16][d*w/8] | signs[16][d/8] | norm f32[16] | gamma f32[16]
 *   nibble: byte i = c[2i] | c[2i+1] << 4;  crumb: byte i = sum_k c[4i+k] << 2k;
 *   bit:    byte i = sum_k s[8i+k] << k, s_j = 1 iff (S r)_j >= 0.
 *   TQ4 (bits = 4, prod keys): 68 B per value vector, 88 B per key vector.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tq_ctx tq_ctx;

typedef enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, Hq % Hkv != 0, small workspace */
    TQ_ERR_UNSUPPORTED = 2,  /* head_dim != 128, bits outside {2,3,4}, unknown mode */
    TQ_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed */
    TQ_ERR_OOM = 4,          /* tq_init could not allocate its parameters */
    TQ_ERR_DEVICE = 5        /* the device error word was non-zero */
} tq_status;

typedef enum { TQ_ROT_HAAR = 0, TQ_ROT_HADAMARD = 1 } tq_rotation;
typedef enum { TQ_KEY_PROD = 0, TQ_KEY_MSE = 1 } tq_key_mode;
typedef enum { TQ_KIND_KEY = 0, TQ_KIND_VALUE = 1 } tq_kind;

/* Device error word bits (tq_get_device_error). */
#define TQ_DEVERR_SLOT      0x1u  /* compress/decompress: slot >= num_blocks*16 (item skipped) */
#define TQ_DEVERR_BLOCK     0x2u  /* decode: block id outside [0, num_blocks) (page skipped)   */
#define TQ_DEVERR_SEQLEN    0x4u  /* decode: seq_len < 0 or > min(max_blocks*16, max_seq_len)  */
#define TQ_DEVERR_TIMEOUT   0x8u  /* a bounded wait inside a kernel gave up (work abandoned)   */
#define TQ_DEVERR_INTERNAL  0x10u /* a kernel found its launch set-up unusable (nothing done)   */

/*
 * tq_init -- build the compressor parameters from one seed
 * [FQ-TQ "TurboQuant" steps 2-3 and "架构设计" (Codebook, Rotation); [TQ-RS]
 * "Couche 1"; [FQ-TQ] "QJL校正" (S)].
 *   head_dim : must be 128.
 *   bits     : 2, 3 or 4.  Values use a b-bit Gaussian Lloyd-Max codebook; keys
 *              use b-1 bits plus 1 QJL sign bit per dimension (TQ_KEY_PROD) or
 *              b bits (TQ_KEY_MSE).
 *   seed     : every random draw (Haar Gaussian matrix, S, Hadamard signs)
 *              comes from SplitMix64 streams of this seed (stream (seed, tag)
 *              starts at state seed + tag*2^48; tag 0 Haar, 1 S, 2 Hadamard).
 *   rotation : TQ_ROT_HAAR: R = Q of the QR of a d x d N(0,1) matrix with a
 *              positive-diagonal triangular factor; y = R^T x.
 *              TQ_ROT_HADAMARD: R^T = H D / sqrt(d) (Sylvester H, random D).
 *   key_mode : TQ_KEY_PROD or TQ_KEY_MSE.
 *   out      : receives the new context (set to NULL on failure).
 * Allocates device memory on the current device (the context is bound to it).
 */
TQ_API tq_status tq_init(int head_dim, int bits, uint64_t seed, int rotation, int key_mode, tq_ctx** out);

/* tq_init_ex flags. */
#define TQ_FLAG_SPHERE_CODEBOOK 0x1  /* exact-d Lloyd-Max codebooks instead of the Gaussian ones */
#define TQ_FLAG_HOST_ONLY       0x4  /* build the parameters on the host only (as tq_init_host) */

/*
 * tq_init_ex -- tq_init with options (tq_init = tq_init_ex with flags 0).
 *   TQ_FLAG_SPHERE_CODEBOOK: both codebooks are the Lloyd-Max quantizers of the
 *     exact law of a rotated unit vector's coordinate, v = sqrt(d) u_1 with u uniform
 *     on the sphere ((u_1 + 1)/2 ~ Beta((d-1)/2, (d-1)/2)), instead of its large-d
 *     limit N(0, 1) [TQ-RS "Étape 2" and "Couche 2": the spherical Beta law].  Only
 *     the codebooks and bucketize tables change; every call works as with tq_init.
 *   TQ_FLAG_HOST_ONLY: as tq_init_host.
 * Unknown flags give TQ_ERR_UNSUPPORTED.
 */
TQ_API tq_status tq_init_ex(int head_dim, int bits, uint64_t seed, int rotation, int key_mode, int flags,
                            tq_ctx** out);

/*
 * tq_init_host -- the same parameters as tq_init, built on the host only: no
 * device is touched and nothing is allocated on one.  Such a context serves
 * tq_chunk_bytes, tq_code_bits and tq_export_params; every call that launches
 * work returns TQ_ERR_INVALID_ARG for it.
 */
TQ_API tq_status tq_init_host(int head_dim, int bits, uint64_t seed, int rotation, int key_mode, tq_ctx** out);

/* tq_destroy -- free a context (NULL is accepted).  First waits for the work this
 * context has queued (on every stream it was given, up to each stream's latest
 * call), not for the whole device; the CUDA runtime's free may still wait for more. */
TQ_API tq_status tq_destroy(tq_ctx* ctx);

/* Bytes of one chunk (16 tokens, one kv head) for kind (tq_kind); 0 on error. */
TQ_API size_t tq_chunk_bytes(const tq_ctx* ctx, int kind);

/* Code bits of kind's scalar quantizer (b for values, b-1 or b for keys); -1 on error. */
TQ_API int tq_code_bits(const tq_ctx* ctx, int kind);

/*
 * tq_export_params -- copy the fp64 host parameters out, for cross-checking.
 * Any output pointer may be NULL.  Host pointers:
 *   R        [d*d] row-major, y = R^T x                 (fp64)
 *   S        [d*d] row-major, (S r)_j = sum_i S[j*d+i] r_i (int8, +-1)
 *   hsigns   [d]   Hadamard signs D (int8); left untouched for Haar
 *   cv, tv   value codebook [2^bv] and interior boundaries [2^bv - 1]
 *   ck, tk   key codebook   [2^bk] and interior boundaries [2^bk - 1]
 */
TQ_API tq_status tq_export_params(const tq_ctx* ctx, double* R, int8_t* S, int8_t* hsigns, double* cv, double* tv,
                           double* ck, double* tk);

/*
 * tq_compress -- the compress step [FQ-TQ "TurboQuant" steps 1-4; "QJL校正" for
 * keys; "架构设计" Compress kernel].  For every token t < T and kv head h the
 * fp16 vector x = k_dev[t][h][:] (resp. v_dev) is normalised (fp32 norm),
 * rotated (y = R^T x), bucketized against the Lloyd-Max boundaries in units of
 * ||x||/sqrt(d) and packed into row slot_mapping[t] % 16 of chunk
 * (slot_mapping[t] / 16, h).  Keys in prod mode also store sign(S r) and
 * gamma = ||r||, r = x - ||x|| R c[idx] / sqrt(d).
 *   k_dev, v_dev      : [T][Hkv][128] fp16, device; either may be NULL to skip it.
 *   slot_mapping_dev  : [T] int32, device.  A negative slot skips the token; a slot
 *                       >= num_blocks*16 is skipped and sets TQ_DEVERR_SLOT.
 *   k_cache_dev, v_cache_dev : [num_blocks][Hkv][chunk_bytes] bytes, device.
 * T = 0 is a no-op.  Returns TQ_ERR_INVALID_ARG on T < 0, Hkv < 1, a missing
 * cache for a given input, or mis-aligned (non 16-byte) pointers.
 */
TQ_API tq_status tq_compress(const tq_ctx* ctx, const uint16_t* k_dev, const uint16_t* v_dev, int T, int Hkv,
                      const int32_t* slot_mapping_dev, uint8_t* k_cache_dev, uint8_t* v_cache_dev, int num_blocks,
                      void* stream);

/*
 * tq_decompress -- unpack and dequantize [FQ-TQ "架构设计" Decompress kernel].
 * MSE: x_hat = ||x|| R c[idx] / sqrt(d).  Prod keys: x_hat + gamma*sqrt(pi/2)/d *
 * S^T (2 sigma - 1), the vector whose inner product with any q equals the QJL
 * estimator.  out_dev: [T][Hkv][128], fp16 (out_fp32 = 0) or fp32 (out_fp32 = 1).
 * Tokens with a negative slot are skipped (their rows are left untouched).
 */
TQ_API tq_status tq_decompress(const tq_ctx* ctx, int kind, const uint8_t* cache_dev, int num_blocks,
                        const int32_t* slot_mapping_dev, int T, int Hkv, void* out_dev, int out_fp32, void* stream);

/*
 * tq_decode_workspace_bytes -- device scratch needed by tq_decode_attention for
 * B sequences, Hq query heads over Hkv kv heads and sequences of at most
 * max_seq_len tokens (0 on invalid arguments).
 * Nothing in the workspace has to start at zero and it needs no clearing between
 * calls: every byte a decode reads is written earlier in the same call, except the
 * per-slot flags, which are compared against a 64-bit tag that no other launch in
 * the process uses.  Two decodes that run at the same time need separate
 * workspaces.
 */
TQ_API size_t tq_decode_workspace_bytes(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_seq_len);

/*
 * tq_decode_attention -- one decode step over the paged compressed cache
 * [FQ-TQ "注意力计算的特殊挑战与QJL校正" (estimator), "架构设计" Paged Decode
 * (split-K FlashDecoding)].  For sequence b and query head h (kv head h / (Hq/Hkv)):
 *   s_t = scale * ( <q, k_hat_t> + gamma_t*sqrt(pi/2)/d * <S q, 2 sigma_t - 1> ),
 *   o = sum_{t < seq_lens[b]} softmax(s)_t * v_hat_t.
 * Scores are taken in the rotated domain (<R^T q, c[idx]>), the value sum is
 * accumulated in the rotated domain and un-rotated once per head.
 * One kernel launch, cooperative: a CTA per SM (at most), all resident at once,
 * each over an equal share of the pages; the CTA that holds a (sequence, kv head)
 * unit's first page merges the unit's partial results from the CTAs after it
 * (waiting for them, bounded).  A device that cannot hold the grid at once (SMs
 * taken by other work) makes the launch fail: TQ_ERR_CUDA.
 *   q_dev          : [B][Hq][128] fp16, device.
 *   block_table_dev: [B][max_blocks] int32, device; page p of sequence b lives in
 *                    physical block block_table[b][p].
 *   seq_lens_dev   : [B] int32, device; each must be <= max_seq_len and <=
 *                    max_blocks*16 (else the sequence is skipped, its output
 *                    zeroed and TQ_DEVERR_SEQLEN set).  A length of 0 gives a
 *                    zero output row.
 *   max_seq_len    : host-side upper bound of seq_lens, sizes the split-K grid.
 *   scale          : softmax scale; pass 0 for the default 1/sqrt(d).
 *   out_dev        : [B][Hq][128], fp16 (out_fp32 = 0) or fp32 (out_fp32 = 1).
 *   workspace_dev  : >= tq_decode_workspace_bytes(ctx, B, Hq, Hkv, max_seq_len) bytes,
 *                    any contents (see above).
 */
TQ_API tq_status tq_decode_attention(const tq_ctx* ctx, const uint16_t* q_dev, const uint8_t* k_cache_dev,
                              const uint8_t* v_cache_dev, int num_blocks, const int32_t* block_table_dev,
                              int max_blocks, const int32_t* seq_lens_dev, int B, int Hq, int Hkv, int max_seq_len,
                              float scale, void* out_dev, int out_fp32, void* workspace_dev, size_t workspace_bytes,
                              void* stream);

/*
 * tq_decode_attention_window -- tq_decode_attention with an fp16 residual window
 * [TQ-RS "Couche 5 — Fenêtre résiduelle" and "Couche 7" (residual_window=128); the
 * KIVI page's FP16 residual of the most recent tokens].  The last tail_lens[b]
 * tokens of sequence b are kept uncompressed; they join the same softmax as its
 * seq_lens[b] compressed tokens:
 *   s_u = scale * <q, k_u>,   o = sum_t p_t v_hat_t + sum_u p_u v_u,
 * p the softmax over both sets (reading: one softmax over the compressed and the
 * window tokens; the pages give only the window's name and size).
 *   tail_k_dev, tail_v_dev : [B][tail_cap][Hkv][128] fp16, device, 16-byte aligned;
 *                            row u < tail_lens[b] of sequence b is window token u.
 *   tail_lens_dev          : [B] int32, device; a length outside [0, tail_cap] is
 *                            taken as 0 and sets TQ_DEVERR_SEQLEN.
 *   tail_cap               : 1 .. 256 (TQ_ERR_INVALID_ARG otherwise).
 * Every other argument, the workspace size and the results are those of
 * tq_decode_attention (which is this call without a window).
 */
TQ_API tq_status tq_decode_attention_window(const tq_ctx* ctx, const uint16_t* q_dev, const uint8_t* k_cache_dev,
                                            const uint8_t* v_cache_dev, int num_blocks,
                                            const int32_t* block_table_dev, int max_blocks,
                                            const int32_t* seq_lens_dev, int B, int Hq, int Hkv, int max_seq_len,
                                            const uint16_t* tail_k_dev, const uint16_t* tail_v_dev,
                                            const int32_t* tail_lens_dev, int tail_cap, float scale, void* out_dev,
                                            int out_fp32, void* workspace_dev, size_t workspace_bytes, void* stream);

/*
 * tq_prefill_attention -- causal attention of a chunk of queries of one sequence over
 * the sequence's compressed, paged cache [FQ-TQ "架构设计": the fused prefill attention
 * kernel, the compressed keys dequantized inline; estimator of "注意力计算的特殊挑战与
 * QJL校正"].  Query i (position q_start + i) attends to the tokens 0 .. q_start + i,
 * whose keys and values must already be in the cache (compress the chunk first):
 *   s_t = scale * ( <q_i, k_hat_t> + gamma_t*sqrt(pi/2)/d * <S q_i, 2 sigma_t - 1> ),
 *   o_i = sum_{t <= q_start + i} softmax(s)_t * v_hat_t.
 * (Reading: the pages name the kernel and its inline decompression; the causal
 * prefix and the decode's estimator are the plainest reading.)
 *   q_dev          : [Tq][Hq][128] fp16, device, 16-byte aligned; Hq 1 .. 65535, a
 *                    multiple of Hkv (TQ_ERR_INVALID_ARG otherwise).
 *   block_table_dev: [max_blocks] int32, device; page p of the sequence lives in
 *                    physical block block_table[p].  A block id outside
 *                    [0, num_blocks) skips the page and sets TQ_DEVERR_BLOCK.
 *   q_start + Tq   : <= max_blocks * 16 (TQ_ERR_INVALID_ARG otherwise).
 *   scale          : softmax scale; 0 for the default 1/sqrt(d).
 *   out_dev        : [Tq][Hq][128], fp16 (out_fp32 = 0) or fp32 (out_fp32 = 1).
 * No workspace.  One kernel launch; Tq = 0 launches nothing.
 */
TQ_API tq_status tq_prefill_attention(const tq_ctx* ctx, const uint16_t* q_dev, const uint8_t* k_cache_dev,
                                      const uint8_t* v_cache_dev, int num_blocks, const int32_t* block_table_dev,
                                      int max_blocks, int q_start, int Tq, int Hq, int Hkv, float scale, void* out_dev,
                                      int out_fp32, void* stream);

/*
 * Size of the device array behind tq_decode_attention_noalloc.  Every GPU that
 * loads libtq reserves this much device memory for it until the process exits.
 */
#define TQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * tq_decode_attention_noalloc -- tq_decode_attention without a workspace
 * argument, for callers that cannot allocate device memory at the call site:
 * code whose device memory is all owned by another allocator (for example a
 * serving runtime that reserves nearly all HBM for its KV cache at start-up,
 * so a fresh cudaMalloc would fail), and code that must not risk the device-wide
 * synchronisation a cudaMalloc / cudaFree may cause.  The pages describe no such
 * variant; it is an addition of this library.
 * The scratch is one file-scope device array of TQ_NOALLOC_SCRATCH_BYTES per
 * device, shared by every call: the decode needs
 * tq_decode_workspace_bytes(ctx, B, Hq, Hkv, max_seq_len) of it, and a larger
 * request is refused with TQ_ERR_INVALID_ARG before anything is launched.
 * Nothing in the scratch has to start at zero (every byte read is written
 * earlier in the same call).  Calls that overlap on the GPU (other streams, other
 * threads, the same device) race on the array and must be serialised by the
 * caller.  The first call on a device looks up the array's device address (with
 * that device current); make that first call before any stream capture.  The
 * current device must be the context's.  Arguments and results are otherwise
 * those of tq_decode_attention.  Allocates nothing.
 */
TQ_API tq_status tq_decode_attention_noalloc(const tq_ctx* ctx, const uint16_t* q_dev, const uint8_t* k_cache_dev,
                                             const uint8_t* v_cache_dev, int num_blocks,
                                             const int32_t* block_table_dev, int max_blocks,
                                             const int32_t* seq_lens_dev, int B, int Hq, int Hkv, int max_seq_len,
                                             float scale, void* out_dev, int out_fp32, void* stream);

/*
 * tq_get_device_error -- synchronize stream, return the device error word in
 * *code (TQ_DEVERR_* bits, 0 if clean) and clear it.  Returns TQ_ERR_DEVICE when
 * the word was non-zero, TQ_OK otherwise.
 */
TQ_API tq_status tq_get_device_error(const tq_ctx* ctx, void* stream, uint32_t* code);

/*
 * tq_debug_stall -- test hook for the failure-detection path (no counterpart on
 * the pages).  The next `launches` kernels of this context that wait for other
 * threads' work do not get it: the compress kernels skip issuing their input
 * copies; the decode kernel's CTAs do not publish the partial results of units
 * that another CTA merges.  The waits that expect them run out after their
 * bounded limit (about 2 s): the kernel sets TQ_DEVERR_TIMEOUT in the device error
 * word (its outputs are then undefined), releases what it holds and returns.
 * Nothing faults or hangs, and the context stays usable.  (A decode whose units
 * all fit one CTA each waits for nothing and is not affected.)
 * launches = 0 cancels a pending stall.  Returns TQ_ERR_INVALID_ARG for a null or
 * host-only context or a negative count.
 */
TQ_API tq_status tq_debug_stall(tq_ctx* ctx, int launches);

/* Number of kernels libtq has launched in this process so far (all contexts,
 * all devices).  Lets a caller count the library's launches in a region. */
TQ_API uint64_t tq_launch_count(void);

/* Human-readable name of a status code (static string). */
TQ_API const char* tq_status_string(tq_status status);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
