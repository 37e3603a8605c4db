// Parameters of the tensor-core compress kernel prepared on the host by tq_init.
#pragma once

#include <cstdint>
#include <vector>

#include <cuda.h>

namespace tq {

struct HostParams;

// Bucketize tables: uniform cells over v = sqrt(d) y / ||x|| in [-V, V]; a cell
// holds at most one interior boundary, far from its edges.  Entries hold the
// boundary (+inf if none) and the levels in cell units u = v * scale.
// Each entry is stored once per lane group, interleaved, so that the lanes of
// one shared-memory phase (16 for 8-byte loads, 8 for 16-byte loads) always hit
// distinct banks: byte offset = cell * 128 + replica * entry_size.
constexpr int kLutCellsMse = 256;   // entry {float bnd; int base}
constexpr int kLutCellsProd = 128;  // entry {float bnd; int base; float c_lo; float c_hi}
constexpr int kLutReplMse = 16;
constexpr int kLutReplProd = 8;
constexpr int kLutBytesMse = kLutCellsMse * 8 * kLutReplMse;
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
