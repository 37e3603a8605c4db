// Internal declarations shared by the host API and the CUDA launchers of libtq.
#pragma once

#include <cstddef>
#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/tq.h"
#include "tc_params.h"

namespace tq {

constexpr int kDim = 128;       // head_dim supported on the device
constexpr int kPage = 16;       // tokens per page chunk
constexpr int kMaxLevels = 16;  // up to 4-bit codebooks

// fp64 parameters built on the host by tq_init.
struct HostParams {
    int d = 0, bits = 0, rotation = 0, key_mode = 0;
    int vbits = 0, kbits = 0;
    int flags = 0;                // TQ_FLAG_* of tq_init_ex
    std::vector<double> R;        // [d*d] row-major, y = R^T x
    std::vector<int8_t> S;        // [d*d] row-major, (S r)_j = sum_i S[j][i] r_i
    std::vector<int8_t> hsigns;   // [d] Hadamard signs (rotation == 1)
    std::vector<double> M;        // [d*d] row-major, M = S R
    std::vector<double> cv, tv;   // value codebook / interior boundaries
    std::vector<double> ck, tk;   // key codebook / interior boundaries
};

HostParams make_host_params(int d, int bits, uint64_t seed, int rotation, int key_mode, int flags);

// Codebook of one kind as the kernels see it (by value, kernel parameter space).
struct Codebook {
    float c[kMaxLevels];      // levels (unit variance)
    float t[kMaxLevels];      // interior boundaries t[0..L-2]
    int bits;                 // code bits
    int width;                // container width (4, 2 or 1)
    int levels;               // 2^bits
};

// Byte geometry of one 16-token chunk.
struct ChunkLayout {
    int code_row;     // bytes of packed codes per token (d * width / 8)
    int signs_off;    // offset of signs[16][d/8] (prod keys), else -1
    int norm_off;     // offset of norm f32[16]
    int gamma_off;    // offset of gamma f32[16] (prod keys), else -1
    int bytes;        // chunk size
    bool prod;        // QJL key chunk
};

// Device copies of the parameters (one allocation owned by the context).
struct DeviceParams {
    const float* RT;      // [d*d] R^T row-major
    const float* S;       // [d*d] S row-major as +-1.0f
    const uint16_t* RTh;  // [d*d] fp16 R^T, high part
    const uint16_t* RTl;  // [d*d] fp16 R^T - RTh
    const uint16_t* Sh;   // [d*d] fp16 S (+-1, exact)
    const uint16_t* Rh;   // [d*d] fp16 R row-major, high part
    const uint16_t* Rl;   // [d*d] fp16 R - Rh
};

inline int container_width(int b) { return b >= 3 ? 4 : (b == 2 ? 2 : 1); }

}  // namespace tq

struct tq_ctx {
    // Streams this context has launched work on, each with an event recorded after
    // its latest launches; tq_destroy waits for these (not for the whole device).
    struct StreamUse {
        cudaStream_t stream;
        cudaEvent_t done;
    };
    mutable std::mutex use_mu;
    mutable std::vector<StreamUse> uses;

    // Test hook (tq_debug_stall): launches left that skip their input copies.
    mutable std::atomic<int> debug_stall{0};

    bool host_only = false;         // built by tq_init_host: no device state
    int device = 0;
    int sm_count = 0;
    tq::HostParams host;
    tq::Codebook cb_value{}, cb_key{};
    tq::ChunkLayout lay_value{}, lay_key{};
    tq::DeviceParams dev{};
    tq::TcTables tc{};              // tensor-core compress operands and tables (in dev_block)
    void* dev_block = nullptr;      // all device parameters
    uint32_t* dev_error = nullptr;  // device error word
};

namespace tq {

// Adds n to the process-wide launch counter (tq_launch_count).
void count_launches(unsigned n);

// Test hook: true (once per pending stall) if this launch must skip its input
// copies so that its bounded waits run out (tq_debug_stall).
bool take_stall(const tq_ctx* ctx);

// Kernel launchers (CUDA translation units).  Each returns cudaSuccess or the
// launch error.
cudaError_t launch_compress_tc(const tq_ctx* ctx, int kind, const uint16_t* x, int T, int H, const int32_t* slots,
                               uint8_t* cache, int num_blocks, cudaStream_t stream);
cudaError_t launch_compress(const tq_ctx* ctx, int kind, const uint16_t* x, int T, int H, const int32_t* slots,
                            uint8_t* cache, int num_blocks, cudaStream_t stream);
cudaError_t launch_decompress(const tq_ctx* ctx, int kind, const uint8_t* cache, int num_blocks,
                              const int32_t* slots, int T, int H, void* out, int out_fp32, cudaStream_t stream);

// Split-K decode: the pages of all (sequence, kv head) units, in order, are cut
// into `grid` equal ranges, one per CTA of the decode kernel; the piece of unit u
// in CTA c leaves its partial softmax state in slot u + c (unique: each slot index
// counts the unit and CTA boundaries before the piece).
struct DecodePlan {
    int grid;            // CTAs of the decode kernel
    int slots;           // units + grid: unit u's slot in CTA c is u + c
    int max_pages;       // ceil(max_seq_len / 16)
    size_t qprep_off;    // workspace offsets (bytes): fp32 [slots][G][2][128] q' and s
    size_t partial_off;  // fp32 [slots][G][130] m, l, acc
    size_t flags_off;    // u64 [slots] launch tags of the published slots
    size_t prefix_off;   // int32 [grid][B + 1]: each CTA's page prefix sums
    size_t bytes;        // total workspace
};
DecodePlan plan_decode(const tq_ctx* ctx, int B, int Hq, int Hkv, int max_seq_len);
// Residual window of the decode: fp16 [B][cap][Hkv][128] keys and values, lengths [B]
// (k == nullptr: none).
struct DecodeTail {
    const uint16_t* k = nullptr;
    const uint16_t* v = nullptr;
    const int32_t* lens = nullptr;
    int cap = 0;
};
constexpr int kDecodeTailMax = 256;
// Causal prefill attention of one sequence (queries at q_start .. q_start + Tq - 1).
cudaError_t launch_prefill(const tq_ctx* ctx, const uint16_t* q, const uint8_t* kc, const uint8_t* vc, int num_blocks,
                           const int32_t* block_table, int max_blocks, int q_start, int Tq, int Hq, int Hkv, float scale,
                           void* out, int out_fp32, cudaStream_t stream);
cudaError_t launch_decode(const tq_ctx* ctx, const DecodePlan& plan, const uint16_t* q, const uint8_t* kc,
                          const uint8_t* vc, int num_blocks, const int32_t* block_table, int max_blocks,
                          const int32_t* seq_lens, int B, int Hq, int Hkv, int max_seq_len, const DecodeTail& tail,
                          float scale, void* out, int out_fp32, void* workspace, cudaStream_t stream);

}  // namespace tq
