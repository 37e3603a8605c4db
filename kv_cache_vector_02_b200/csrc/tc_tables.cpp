// Host preparation for the tensor-core compress kernel: fp16 operand images in
// the exact shared-memory layout the MMA reads (K-major, 128-byte swizzle), the
// bucketize tables, and the TMA descriptor of the input rows.
#include <cmath>
#include <cstring>
#include <mutex>

#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "tc_params.h"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kD = 128;
constexpr size_t kImageBytes = size_t(kD) * kD * 2;

uint16_t to_half_bits(double v) { return __half_as_ushort(__double2half(v)); }
double half_value(uint16_t b) { return (double)__half2float(__ushort_as_half(b)); }

// Operand B[n][k] (n = output column, k = contraction index), fp16, K-major with
// the 128-byte swizzle: two K-halves of 16 KB; row n of a half at n * 128 bytes,
// 16-byte chunk c of the row stored at chunk c ^ (n % 8).
void put_image(const std::vector<uint16_t>& B, uint8_t* dst) {
    for (int n = 0; n < kD; ++n)
        for (int k = 0; k < kD; ++k) {
            const int kb = k >> 6, c = (k & 63) >> 3, e = k & 7;
            const size_t off = size_t(kb) * 16384 + size_t(n) * 128 + size_t((c ^ (n & 7)) << 4) + size_t(e << 1);
            std::memcpy(dst + off, &B[size_t(n) * kD + k], 2);
        }
}

// Split a real matrix into fp16 hi + lo parts.
void split(const std::vector<double>& A, std::vector<uint16_t>& hi, std::vector<uint16_t>& lo) {
    hi.resize(A.size());
    lo.resize(A.size());
    for (size_t i = 0; i < A.size(); ++i) {
        hi[i] = to_half_bits(A[i]);
        lo[i] = to_half_bits(A[i] - half_value(hi[i]));
    }
}

inline int hadamard_sign(int i, int j) { return (__builtin_popcount(unsigned(i & j)) & 1) ? -1 : 1; }

// Bucketize table for boundaries t (L-1) and levels c (L).  The cell width w is
// chosen so that [-sqrt(d), sqrt(d)] maps inside [0, cells) and every boundary
// sits at least 5% of a cell away from a cell edge.  Boundaries and levels are
// stored in cell units (value * scale), the unit the kernel compares in.
bool build_lut(const std::vector<double>& t, const std::vector<double>& c, int cells, bool prod, uint8_t* dst,
               LutParams& lp) {
    const double vmax = std::sqrt(double(kD));
    for (int attempt = 0; attempt < 4000; ++attempt) {
        const double V = vmax + 0.15 + 0.0005 * attempt;
        const double w = 2.0 * V / cells;
        const float scale = float(1.0 / w);
        // positions in cell units as the kernel computes them (fp32 scale)
        bool good = true;
        for (double tk : t) {
            const double u = double(float(tk)) * double(scale);
            const double frac = u - std::floor(u);
            if (std::fabs(frac - 0.5) < 0.05) {
                good = false;
                break;
            }
        }
        if (!good) continue;
        // the extreme |v| must stay inside the table
        if (vmax * double(scale) + cells / 2 + 0.5 >= cells - 0.5) continue;
        lp.scale = scale;
        lp.magic = float(12582912.0 + cells / 2);
        const int L = int(c.size());
        for (int cell = 0; cell < cells; ++cell) {
            // cell covers u in [r - 0.5, r + 0.5), r = cell - cells/2
            const int r = cell - cells / 2;
            int base = 0;
            float bnd = INFINITY;  // the boundary inside the cell, as the kernel compares it
            for (double tk : t) {
                const float ub = float(tk * double(scale));
                if (double(ub) < r - 0.5) ++base;
                else if (double(ub) < r + 0.5) bnd = ub;
            }
            if (base > L - 1) base = L - 1;
            if (prod) {
                const float clo = float(c[base] * double(scale));
                const float chi = float(c[base + 1 < L ? base + 1 : base] * double(scale));
                for (int l = 0; l < kLutReplProd; ++l) {
                    uint8_t* e = dst + 128 * cell + 16 * l;
                    std::memcpy(e + 0, &bnd, 4);
                    std::memcpy(e + 4, &base, 4);
                    std::memcpy(e + 8, &clo, 4);
                    std::memcpy(e + 12, &chi, 4);
                }
                continue;
            }
            // offset in the cell (exact: |bnd - r| < 1/2); none: 1.0 > any u - r
            const float f = std::isfinite(bnd) ? bnd - float(r) : 1.0f;
            // the smallest float >= f whose 4 low mantissa bits are base
            uint32_t fb;
            std::memcpy(&fb, &f, 4);
            float best = INFINITY;
            for (int k = -2; k <= 2; ++k) {
                const uint32_t cand = uint32_t(int64_t(fb & ~15u) + 16 * k) | uint32_t(base);
                float cf;
                std::memcpy(&cf, &cand, 4);
                if (std::isfinite(cf) && cf >= f && cf < best && std::signbit(cf) == std::signbit(f)) best = cf;
            }
            if (!std::isfinite(best)) return false;
            for (int l = 0; l < kLutReplMse; ++l) std::memcpy(dst + 128 * cell + 4 * l, &best, 4);
        }
        return true;
    }
    return false;
}

}  // namespace

bool build_tc_blob(const HostParams& H, TcBlob& out) {
    const bool haar = (H.rotation == 0);
    const bool prod = (H.key_mode == 0);
    std::vector<std::vector<uint16_t>> images;
    if (haar) {
        // rotation: B[n][k] = 16 R[k][n], split hi + lo
        std::vector<double> B(size_t(kD) * kD);
        for (int n = 0; n < kD; ++n)
            for (int k = 0; k < kD; ++k) B[size_t(n) * kD + k] = 16.0 * H.R[size_t(k) * kD + n];
        std::vector<uint16_t> hi, lo;
        split(B, hi, lo);
        images.push_back(hi);
        images.push_back(lo);
        // sketch: B[j][i] = M[j][i], M = S R, split hi + lo
        split(H.M, hi, lo);
        images.push_back(hi);
        images.push_back(lo);
    } else {
        // rotation: B[n][k] = (H D)[n][k] = H[n][k] D[k], exact +-1
        std::vector<uint16_t> B(size_t(kD) * kD);
        for (int n = 0; n < kD; ++n)
            for (int k = 0; k < kD; ++k) B[size_t(n) * kD + k] = to_half_bits(double(hadamard_sign(n, k) * H.hsigns[k]));
        images.push_back(B);
        // sketch: M' = S D H (integers, |.| <= 128, exact in fp16)
        std::vector<int> DH(size_t(kD) * kD);
        for (int k = 0; k < kD; ++k)
            for (int i = 0; i < kD; ++i) DH[size_t(k) * kD + i] = H.hsigns[k] * hadamard_sign(k, i);
        for (int j = 0; j < kD; ++j)
            for (int i = 0; i < kD; ++i) {
                int s = 0;
                for (int k = 0; k < kD; ++k) s += int(H.S[size_t(j) * kD + k]) * DH[size_t(k) * kD + i];
                B[size_t(j) * kD + i] = to_half_bits(double(s));
            }
        images.push_back(B);
    }
    const size_t n_img = images.size();
    out.off_images = 0;
    out.off_lut_value = n_img * kImageBytes;
    out.off_lut_key = out.off_lut_value + kLutBytesMse;
    out.bytes.assign(out.off_lut_key + (prod ? kLutBytesProd : kLutBytesMse), 0);
    for (size_t i = 0; i < n_img; ++i) put_image(images[i], out.bytes.data() + i * kImageBytes);
    if (!build_lut(H.tv, H.cv, kLutCellsMse, false, out.bytes.data() + out.off_lut_value, out.lp_value)) return false;
    if (prod) {
        if (!build_lut(H.tk, H.ck, kLutCellsProd, true, out.bytes.data() + out.off_lut_key, out.lp_key)) return false;
    } else {
        if (!build_lut(H.tk, H.ck, kLutCellsMse, false, out.bytes.data() + out.off_lut_key, out.lp_key)) return false;
    }
    return true;
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

bool encode_rows_tmap(CUtensorMap* map, const void* x, int rows) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        cudaGetLastError();
    });
    if (!g_encode || rows < 1) return false;
    cuuint64_t dims[2] = {cuuint64_t(kD), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(kD) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(x), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tq
