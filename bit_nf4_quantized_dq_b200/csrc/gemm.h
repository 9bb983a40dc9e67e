// Host-side description of one launch of the tcgen05 GEMM engine.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "codebook.h"

namespace qnf4 {

// Source of the A operand (the 128-row UMMA "M" side) for one stretch of the K loop.
enum ASrc : int32_t {
  kATmaK = 0,    // bf16 tile loaded by TMA, K-major
  kATmaMN = 1,   // bf16 tile loaded by TMA, MN-major (two 64-wide boxes)
  kANf4K = 2,    // dequantized on chip from NF4 codes, W rows are the M side (forward)
  kANf4MN = 3,   // dequantized on chip from NF4 codes, W columns are the M side (dX)
};

enum Epi : int32_t {
  kEpiBf16T = 0,    // out_bf16[col * ld + row] = bf16(D[row][col])
  kEpiF32T = 1,     // ws[split * split_stride + col * ld + row] = D[row][col]
};

struct GemmSeg {
  int32_t kblocks;    // 64-wide k-blocks in this stretch
  int32_t k16_last;   // 16-wide MMA steps in its last k-block (1..4)
  int32_t a_src;      // ASrc
  int32_t a_map;      // tensor map index for A (codes map for NF4 sources)
  int32_t b_map;      // tensor map index for B (always K-major bf16)
  int32_t a_k0;       // first k coordinate of this stretch for A (elements, or W row for kANf4MN)
  int32_t b_k0;       // first k coordinate of this stretch for B (elements)
  int32_t pad;
};

constexpr int kMaxMaps = 5;
constexpr int kMaxSegs = 3;

struct GemmParams {
  CUtensorMap maps[kMaxMaps];
  GemmSeg seg[kMaxSegs];
  int32_t nseg;
  int32_t rows, cols;            // valid extent of D: rows on the UMMA M side, cols on the N side
  int32_t splits, kb_per_split;  // segment 0 is split over blockIdx.z; later segments run in split 0
  int32_t has_nf4, nf4_generic;  // NF4 producer present; codes fetched without TMA (K % 64 != 0)
  int32_t b_box_rows;            // rows of every B-operand TMA box (checked against the kernel's tile)
  // A operand in tensor memory (forward, 256-token tiles): the producers write the dequantized
  // tile, and the rows of kATmaK stretches from a_glob ([a_glob_rows][a_glob_cols] bf16, row
  // pitch a_glob_ld elements), straight into TMEM; shared memory holds only B and the codes.
  int32_t a_tmem;
  const uint16_t* a_glob;
  int64_t a_glob_ld, a_glob_rows, a_glob_cols;
  // 4-bit operand: codes / scale codes / group constants / mean of W [nw][kw], its 16 levels,
  // and the scale format (scale_fp32 = 1: c2 holds one fp32 scale per block of 64, the
  // single-level format without double quantization; scale_codes and mean are unused)
  const uint8_t* codes;
  const uint8_t* scale_codes;
  const float* c2;
  const float* mean;
  int64_t nw, kw;
  Codebook cb;
  int32_t scale_fp32;
  // epilogue
  int32_t epi;
  float alpha;
  void* out;
  int64_t ld_out;
  int64_t split_stride;
};

// Launch with tile width bn in {16, 32, 64, 128, 256}; grid = (ceil(rows/128), ceil(cols/bn), splits).
cudaError_t launch_gemm(const GemmParams& p, int bn, cudaStream_t st);

// Small helpers of the low-rank path.
cudaError_t launch_transpose_bf16(const uint16_t* in, int64_t rows, int64_t cols, uint16_t* out, int64_t ld_out,
                                  cudaStream_t st);
cudaError_t launch_reduce_splits_bf16(const float* ws, int splits, int64_t split_stride, int64_t cols, int64_t rows,
                                      int64_t ld, uint16_t* out, int64_t ld_out, cudaStream_t st);

}  // namespace qnf4
