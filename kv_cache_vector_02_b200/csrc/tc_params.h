// Parameters of the tensor-core compress kernel prepared on the host by tq_init.
#pragma once

#include <cstdint>
#include <vector>

#include <cuda.h>

namespace tq {

struct HostParams;

// Bucketize tables: uniform cells over v = sqrt(d) y / ||x|| in [-V, V]; a cell
// holds at most one interior boundary, at least 5% of a cell from its edges.  In
// cell units u = v * scale, cell r covers [r - 1/2, r + 1/2).
//   MSE (values and MSE keys): a 32-bit entry per cell, the fp32 offset
//     f = bnd - r of the boundary (1.0 if none) whose 4 low mantissa bits are
//     replaced by the code of the cell's lower side (base), the value rounded up
//     so that it never falls below f: code = base + [u - r > f'].  Stored once
//     per lane (32 copies, interleaved: byte offset = cell * 128 + lane * 4), so
//     a warp's 32 lookups never share a bank.
//   Product keys: a 16-byte entry {float bnd; int base; float c_lo; float c_hi}
//     (bnd = +inf if none; levels in cell units), one read gives the code and its
//     level: code = base + [u > bnd].  Stored once per 8 lanes (byte offset =
//     cell * 128 + (lane % 8) * 16), so a quarter-warp phase never shares a bank.
constexpr int kLutCellsMse = 256;
constexpr int kLutCellsProd = 128;
constexpr int kLutReplMse = 32;
constexpr int kLutReplProd = 8;
constexpr int kLutBytesMse = kLutCellsMse * 4 * kLutReplMse;
constexpr int kLutBytesProd = kLutCellsProd * 16 * kLutReplProd;

// u = v * scale; cell = bits(u + magic) - bits(1.5 * 2^23), magic = 1.5 * 2^23 + cells / 2
struct LutParams {
    float scale = 0.f, magic = 0.f;
};

struct TcTables {
    const uint8_t* images = nullptr;    // device: rotation operand(s), then sketch operand(s), 32 KB each
    const uint8_t* lut_value = nullptr; // device
    const uint8_t* lut_key = nullptr;   // device
    LutParams lp_value, lp_key;
};

// Host images of the device blob: [images | lut_value | lut_key].
struct TcBlob {
    std::vector<uint8_t> bytes;
    size_t off_images = 0, off_lut_value = 0, off_lut_key = 0;
    LutParams lp_value, lp_key;
};

// Builds the operand images and tables; returns false if no table geometry
// keeps every boundary away from the cell edges (never for Gaussian codebooks).
bool build_tc_blob(const HostParams& H, TcBlob& out);

// TMA descriptor of a [rows, 128] fp16 row-major matrix, boxes of 128 rows x 64
// columns with the 128-byte swizzle.  False if the driver entry point is missing
// or rejects the arguments.
bool encode_rows_tmap(CUtensorMap* map, const void* x, int rows);

}  // namespace tq
