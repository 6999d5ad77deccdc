// Host interface of the quantizer kernels (not part of the C ABI).
#pragma once

#include "common.cuh"

namespace qat {

// One export descriptor as the kernel sees it.  Quantized tensors use one
// warp per row; fp16 passthrough tensors are cut into "rows" of `cols`
// elements of a flat array of `numel` elements.
struct ExportDescDev {
  const float* src;
  void* dst;
  __half* scales;
  int64_t rows, cols, numel;
  int64_t unit_begin;  // first global work unit of this descriptor
  int64_t unit_rows;   // rows per work unit
  int mode;           // 5, 6, 8 or QAT_EXPORT_FP16
  int m;              // quantile order statistic from the top (1 or 2)
  float frac;         // quantile interpolation fraction
  int pack6;          // codes stored as 6-bit fields, 4 codes in 3 bytes
  int search;         // per-row clip search over kClipCandidates
  int pad;
};

// Clip-search candidates (quantiles of |w|): the row maximum, the export's
// 99.99984 percentile, then four tighter clips.  Only the top four order
// statistics of a row are needed for rows of up to kExportMaxStagedCols.
constexpr int kClipCandidates = 6;
constexpr int kClipSearchTop = 4;

#ifndef QAT_EXPORT_BATCH_CAP
#define QAT_EXPORT_BATCH_CAP QAT_EXPORT_MAX_DESCS
#endif
// A batch as the kernel receives it (a __grid_constant__ parameter).  The
// launch passes the smallest capacity that holds the batch's descriptors: a
// launch uploads its whole parameter block, and the largest one is 22 KB.
template <int CAP>
struct ExportBatchT {
  int n;
  int buf_bytes;  // bytes of one row buffer (longest staged row, rounded to 128)
  int64_t total_units;
  ExportDescDev d[CAP];
};
using ExportBatch = ExportBatchT<QAT_EXPORT_BATCH_CAP>;

// Chunk length of the fp16 passthrough "rows" (6 KB of fp32, like a staged unit).
constexpr int64_t kFp16Chunk = 1536;

// Export kernel staging: row buffers per warp, the longest row staged in
// shared memory (longer rows are read from global memory), the shared memory
// a block may use and the most warps per block.  Buffers are sized for the
// longest staged row of the batch, so short-row state dicts get more warps.
#ifndef QAT_EXPORT_BUFS
#define QAT_EXPORT_BUFS 2
#endif
constexpr int kExportBufs = QAT_EXPORT_BUFS;
constexpr int64_t kExportUnitBytes = 6144;  // staged bytes per work unit (whole rows)
constexpr int64_t kExportMaxStagedCols = 2048;
constexpr int kExportSmemBudget = 224 * 1024;
constexpr int kExportMaxWarps = 16;

// Training-time quantization of several weights in one launch (a warp per row
// over the rows of all of them).
constexpr int kQuantMaxDescs = QAT_QUANT_MAX_DESCS;
struct QuantDescDev {
  const float* W;
  int8_t* codes;
  float* scales;
  __nv_bfloat16* operand;
  int N, K, bits, pad;
};
constexpr int kQuantTileRows = 8;  // warps per thread block (rows of up to 512 columns)
// Thread blocks for N rows of K columns: min(S, 8) warps per row, S = the
// row's 512-column segments, 8 / min(S, 8) rows per block.
inline int64_t quant_tiles(int64_t N, int64_t K) {
  const int64_t S = ((K >> 2) + 127) >> 7;
  const int64_t rpb = kQuantTileRows / (S < kQuantTileRows ? S : kQuantTileRows);
  return (N + rpb - 1) / rpb;
}
struct QuantBatch {
  int n;
  int64_t tile_begin[kQuantMaxDescs + 1];  // first tile of each weight; [n] = total
  QuantDescDev d[kQuantMaxDescs];
};
int launch_quantize_batch(const QuantBatch& b, cudaStream_t s);
int launch_quantize_weights(const float* W, int N, int K, int bits, int8_t* codes, float* scales,
                            __nv_bfloat16* operand, cudaStream_t s);
int launch_noisy_operand(const float* W, int N, int K, int bits, uint64_t seed, uint64_t offset,
                         float* scales, __nv_bfloat16* operand, cudaStream_t s);
int export_quantile_params(int64_t cols, int* m, float* frac);
int clip_search_supported(int64_t cols);
int launch_export_batch(ExportBatch& b, cudaStream_t s);
int launch_dequant(const int8_t* codes, const __half* scales, int64_t rows, int64_t cols,
                   int out_bf16, void* out, cudaStream_t s);

// Grouped dequantize: descriptor k covers tiles [tile_begin[k],
// tile_begin[k + 1]) of kDequantTile 4-element groups (items) each, the last
// one partial; one thread block per tile.  The row of group
// l is l / (cols / 4) = the high 64 bits of l * row_magic, row_magic =
// ceil(2^64 / (cols / 4)) (exact for l < 2^46: the product's error,
// l (row_magic - 2^64 / (cols / 4)) / 2^64 < l / 2^64, stays below the gap
// 1 / (cols / 4) between l / (cols / 4) and the next integer).
struct DequantDescDev {
  const int8_t* codes;
  const __half* scales;
  void* out;
  int64_t items;  // rows * cols / 4
  uint64_t row_magic;
  int out_bf16, pad;
};
constexpr int kDequantPerThread = 4;                 // items per thread
constexpr int kDequantTile = 256 * kDequantPerThread;  // items per block
// ceil(2^64 / c4) for c4 >= 2.
inline uint64_t dequant_row_magic(int64_t c4) {
  return ~0ull / static_cast<uint64_t>(c4) + 1ull;
}
constexpr int kDequantMaxDescs = QAT_DEQUANT_MAX_DESCS;
// As ExportBatchT: the launch passes the smallest capacity that holds it.
template <int CAP>
struct DequantBatchT {
  int n;
  int64_t tile_begin[CAP + 1];
  DequantDescDev d[CAP];
};
using DequantBatch = DequantBatchT<kDequantMaxDescs>;
int launch_dequant_batch(const DequantBatch& b, cudaStream_t s);
int launch_unpack6(const uint8_t* packed, int64_t n, int bits, int8_t* codes, cudaStream_t s);

}  // namespace qat
