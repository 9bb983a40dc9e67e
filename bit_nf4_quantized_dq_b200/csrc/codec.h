// Host-side launchers of the NF4 + double-quantization codec kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "codebook.h"

namespace qnf4 {

// w_map: W viewed as [numel / 64][64] bf16 (box 64 x 256, 128-byte swizzle), or NULL when
// numel < 64 (no whole block).
// gsum_ws == NULL: single-level quantization (no group sums, no double quantization; the
// absmax values written to absmax_ws are the scales).
cudaError_t launch_quantize(const CUtensorMap* w_map, const uint16_t* W, int64_t numel, const Codebook& cb,
                            uint8_t* codes, uint8_t* scale_codes, float* c2, float* mean, float* absmax_ws,
                            double* gsum_ws, cudaStream_t st, int sw_encode);
// scale_fp32: c2 holds one fp32 scale per block (single-level quantization).
cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scale_codes, const float* c2, const float* mean,
                           int64_t numel, uint16_t* out, const Codebook& cb, int scale_fp32, cudaStream_t st);
cudaError_t launch_e4m3_encode(const float* v, int64_t n, uint8_t* out, int sw, cudaStream_t st);
cudaError_t read_and_clear_error_word(uint32_t* word, cudaStream_t st);

}  // namespace qnf4
