// Adapter merge: W'' = bf16( W' + s * B A ) for the frozen 4-bit base W' [N][K] and the LoRA
// adapters A [r][K], B [N][r]; the result is then quantized again by the quantizer.
//
// "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged
// Optimizers" (fullstackaihub), "Engineering Limitations": full-rank updates need the
// adapters dequantized and merged into 16-bit precision; "QLoRA Explained ... Part 2/6"
// (video description): adapter merging / re-quantization at deployment.
//
// Arithmetic (fixed so that the result is reproducible bit for bit): the rank-r sum
// sum_j B[n][j] A[j][k] is formed in float64 term by term in index order j = 0 .. r-1 (each
// bf16 x bf16 product is exact in float64, so each fused multiply-add is one float64 rounding
// of the running sum); t = float64(s * sum); v = float64(W'[n][k] + t); W'' = bf16 of v, rounded
// once to nearest even.  W' is the dequantized base, bf16(fp32(level[code] * block scale)).
#pragma once

#include "nf4_device.cuh"

namespace qnf4 {

struct MergeParams {
  Codebook cb;
  const uint8_t* codes;
  const uint8_t* scale_codes;
  const float* scales;    // c2 per group (double quantization) or the fp32 scale per block
  const float* mean;
  int32_t scale_fp32;
  int64_t N, K;
  const uint16_t* A;      // [r][K] bf16
  const uint16_t* B;      // [N][r] bf16
  int32_t r;
  double s;
  uint16_t* out;          // [N][K] bf16
};

// bf16 nearest-even rounding of a float64, once: the significand keeps 8 bits.  Below 2^-126
// (the bf16 subnormals) the grid is 2^-133.
__device__ __forceinline__ uint16_t bf16_rn_from_f64(double v) {
  const double a = fabs(v);
  if (a < 1.1754943508222875e-38) {                       // 2^-126: subnormal grid
    const double m = rint(a * 1.0889035741470030e+40);    // a * 2^133, rounded to nearest even
    const uint32_t sign = (__double_as_longlong(v) < 0) ? 0x8000u : 0u;
    return (uint16_t)(sign | (uint32_t)m);                 // m <= 128 (128 carries into the normals)
  }
  uint64_t b = (uint64_t)__double_as_longlong(v);
  const uint64_t lsb = (b >> 45) & 1ull;
  b = (b + ((1ull << 44) - 1ull) + lsb) & ~((1ull << 45) - 1ull);
  const float f = (float)__longlong_as_double((long long)b);   // exact: 8 significant bits
  return (uint16_t)(__float_as_uint(f) >> 16);
}

// W' [n][k] of the stored base, as the dequant computes it.
__device__ __forceinline__ float base_weight(const MergeParams& p, int64_t n, int64_t k) {
  const int64_t e = n * p.K + k;
  const uint32_t byte = __ldg(p.codes + (e >> 1));
  const uint32_t code = (byte >> (4 * (e & 1))) & 15u;
  const int64_t blk = e >> 6;
  const float s = p.scale_fp32 ? __ldg(p.scales + blk)
                               : dq_block_scale(__ldg(p.scale_codes + blk), __ldg(p.scales + (blk >> 8)), __ldg(p.mean));
  const float w = __fmul_rn(p.cb.q[code], s);
  return __bfloat162float(__float2bfloat16_rn(w));
}

// One CTA per tile of 128 rows x 64 columns; thread t owns the 8 columns 8 (t % 8) .. + 7 of
// the four rows t / 8 + 32 i (i = 0..3), so that each pair of shared-memory loads of A feeds 32
// float64 fused multiply-adds.  The rank dimension goes through shared memory in chunks of 16,
// converted to float64 (exactly) on the way in.  Each accumulator still runs over j = 0 .. r-1
// in order.
constexpr int kMergeRows = 128, kMergeCols = 64, kMergeJ = 16, kMergeRowsPerThread = 4;

__global__ void __launch_bounds__(256) merge_dense_kernel(const __grid_constant__ MergeParams p) {
  __shared__ __align__(16) double As[kMergeJ][kMergeCols];    // 8 KB
  __shared__ double Bs[kMergeRows][kMergeJ + 1];               // 17 KB
  const int t = threadIdx.x;
  const int64_t n0 = (int64_t)blockIdx.y * kMergeRows, k0 = (int64_t)blockIdx.x * kMergeCols;
  const int rr = t >> 3, cc = (t & 7) * 8;
  double acc[kMergeRowsPerThread][8];
#pragma unroll
  for (int i = 0; i < kMergeRowsPerThread; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.0;
  for (int j0 = 0; j0 < p.r; j0 += kMergeJ) {
    const int jn = (p.r - j0) < kMergeJ ? (p.r - j0) : kMergeJ;
    __syncthreads();
    for (int i = t; i < kMergeJ * kMergeCols; i += 256) {
      const int j = i / kMergeCols, k = i % kMergeCols;
      double v = 0.0;
      if (j < jn && k0 + k < p.K) v = (double)__bfloat162float(__ushort_as_bfloat16(p.A[(int64_t)(j0 + j) * p.K + k0 + k]));
      As[j][k] = v;
    }
    for (int i = t; i < kMergeRows * kMergeJ; i += 256) {
      const int rrow = i / kMergeJ, j = i % kMergeJ;
      double v = 0.0;
      if (j < jn && n0 + rrow < p.N) v = (double)__bfloat162float(__ushort_as_bfloat16(p.B[(n0 + rrow) * p.r + j0 + j]));
      Bs[rrow][j] = v;
    }
    __syncthreads();
    for (int j = 0; j < jn; ++j) {
      double a[8];
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        const double2 a2 = *reinterpret_cast<const double2*>(&As[j][cc + c]);
        a[c] = a2.x;
        a[c + 1] = a2.y;
      }
#pragma unroll
      for (int i = 0; i < kMergeRowsPerThread; ++i) {
        const double b = Bs[rr + 32 * i][j];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = __fma_rn(b, a[c], acc[i][c]);   // b * a is exact
      }
    }
  }
  if (k0 + cc >= p.K) return;                              // K % 8 == 0: whole groups of 8 in or out
#pragma unroll
  for (int i = 0; i < kMergeRowsPerThread; ++i) {
    const int64_t n = n0 + rr + 32 * i;
    if (n >= p.N) break;
    uint32_t packed[4];
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      uint32_t h[2];
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        const int64_t k = k0 + cc + c + d;
        const double tterm = __dmul_rn(p.s, acc[i][c + d]);
        const double v = __dadd_rn((double)base_weight(p, n, k), tterm);
        h[d] = bf16_rn_from_f64(v);
      }
      packed[c / 2] = h[0] | (h[1] << 16);
    }
    *reinterpret_cast<uint4*>(p.out + n * p.K + k0 + cc) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
}

static cudaError_t launch_merge_dense(const MergeParams& p, cudaStream_t st) {
  dim3 grid((unsigned)((p.K + kMergeCols - 1) / kMergeCols), (unsigned)((p.N + kMergeRows - 1) / kMergeRows));
  merge_dense_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace qnf4
