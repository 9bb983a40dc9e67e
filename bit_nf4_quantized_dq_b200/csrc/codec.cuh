// NF4 + double quantization: quantize (three kernels) and the standalone dequant stream.
//
// "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged
// Optimizers" (fullstackaihub), section 3: level 1 (absmax per contiguous block of 64, the
// index of the nearest code-book level per weight) and level 2 (the fp32 absmax values,
// centred by their mean, coded as 8-bit floats in groups of 256 with one fp32 constant per
// group); section 4: the dequantization helper.  "QLoRA, explained." (vibeengines), method
// steps 2-4.
#pragma once

#include "nf4_device.cuh"
#include "codec.h"

namespace qnf4 {


// ---------------------------------------------------------------------------------------
// Q-A: absmax per block of 64, normalise, nearest level, pack two codes per byte.
// One thread per 8 consecutive weights (one 16-byte load), 8 threads per block.
// ---------------------------------------------------------------------------------------
// The nearest level is found through 33 buckets of width 1/16 over [-1, 1]: the midpoints
// between neighbouring levels are at least 0.085 apart, so each bucket holds at most one
// of them.  code = (#midpoints below the bucket) + (n > the bucket's midpoint).  The
// midpoint test uses theta_j = the largest fp32 not above the exact midpoint, which makes
// n > theta_j equivalent to n > midpoint for every fp32 n (ties go to the lower level).
struct BucketEntry {
  uint32_t base;
  float thr;
};

// Thread b < 33 computes bucket b once and fills its 32 per-lane copies (one copy per lane
// keeps the lookups of a warp free of bank conflicts).
__device__ __forceinline__ void build_bucket_table(BucketEntry (*tab)[32]) {
  constexpr float q[16] = QNF4_LEVELS;
  const int b = threadIdx.x;
  if (b >= 33) return;
  // bucket b holds the fp32 n with round(16 n + 16) == b
  const double lo = (b - 16.5) / 16.0, hi = (b - 15.5) / 16.0;
  uint32_t base = 0;
  float thr = __int_as_float(0x7F800000);  // +inf: no midpoint inside
  for (int j = 0; j < 15; ++j) {
    const double m = 0.5 * ((double)q[j] + (double)q[j + 1]);   // exact in float64
    const float theta = __double2float_rd(m);
    if ((double)theta < lo) ++base;
    else if ((double)theta < hi) thr = theta;
  }
  const BucketEntry e{base, thr};
  for (int l = 0; l < 32; ++l) tab[b][l] = e;
}

__device__ __forceinline__ uint32_t nearest_code(float n, const BucketEntry (*tab)[32], int lane) {
  const float t = __fmaf_rn(n, 16.0f, 12582928.0f);      // 1.5*2^23 + 16: integer rounding
  const uint32_t b = __float_as_uint(t) & 63u;
  const BucketEntry e = tab[b][lane];
  return e.base + (n > e.thr ? 1u : 0u);
}

__global__ void __launch_bounds__(256) nf4_quant_blocks_kernel(const uint16_t* __restrict__ W, int64_t numel,
                                                               int64_t nchunks, uint32_t* __restrict__ codes32,
                                                               float* __restrict__ absmax) {
  __shared__ BucketEntry tab[33][32];
  build_bucket_table(tab);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c - lane < nchunks; c += stride) {
    // all lanes of a warp take part in the shuffles; chunks past the end contribute zeros
    float w[8];
    const int64_t e0 = c * 8;
    if (c < nchunks && e0 + 8 <= numel) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(W) + c);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        w[2 * i] = __uint_as_float(u[i] << 16);
        w[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        w[i] = (c < nchunks && e0 + i < numel) ? __uint_as_float((uint32_t)W[e0 + i] << 16) : 0.0f;
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(w[i]));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
    if (c >= nchunks) continue;
    if ((lane & 7) == 0) absmax[c >> 3] = m;
    uint32_t packed = 0;
    if (m > 0.0f) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float n = __fdiv_rn(w[i], m);
        packed |= nearest_code(n, tab, lane) << (4 * i);
      }
    } else {
      packed = 0x77777777u;                       // all-zero block: every weight is level 7
    }
    codes32[c] = packed;
  }
}

// ---------------------------------------------------------------------------------------
// Q-B: float64 sum of the absmax values by a fixed binary tree over adjacent pairs, then
// the mean.  Stage 1: one warp per group of 256 (lane l owns blocks 8l..8l+7; the xor
// butterfly pairs lanes (0,1),(2,3),... which is the same adjacent-pair tree).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dq_group_sums_kernel(const float* __restrict__ absmax, int64_t nb,
                                                            int64_t ng, double* __restrict__ gsum) {
  const int lane = threadIdx.x & 31;
  const int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (g >= ng) return;                                   // whole warps exit together
  double v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t b = g * kB2 + lane * 8 + i;
    v[i] = (b < nb) ? (double)absmax[b] : 0.0;
  }
  double s = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) s = s + __shfl_xor_sync(0xFFFFFFFFu, s, off);
  if (lane == 0) gsum[g] = s;
}

// Stage 2: one CTA of 1024 threads reduces the group sums in aligned chunks of 2048 by the
// same adjacent-pair tree (zero padding is exact), then the chunk sums, then divides.
__global__ void __launch_bounds__(1024) dq_mean_kernel(const double* __restrict__ gsum, int64_t ng, int64_t nb,
                                                       float* __restrict__ mean) {
  __shared__ double buf[2048];
  __shared__ double chunk_sums[1024];
  const int t = threadIdx.x;
  const int64_t nchunks = (ng + 2047) / 2048;
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int64_t i0 = ch * 2048 + 2 * t;
    buf[2 * t] = (i0 < ng) ? gsum[i0] : 0.0;
    buf[2 * t + 1] = (i0 + 1 < ng) ? gsum[i0 + 1] : 0.0;
    __syncthreads();
    for (int n = 1024; n >= 1; n >>= 1) {
      double r = 0.0;
      if (t < n) r = buf[2 * t] + buf[2 * t + 1];
      __syncthreads();
      if (t < n) buf[t] = r;
      __syncthreads();
    }
    if (t == 0) chunk_sums[ch] = buf[0];
    __syncthreads();
  }
  // tree over the chunk sums, padded to 1024 with zeros
  buf[t] = (t < nchunks) ? chunk_sums[t] : 0.0;
  __syncthreads();
  for (int n = 512; n >= 1; n >>= 1) {
    double r = 0.0;
    if (t < n) r = buf[2 * t] + buf[2 * t + 1];
    __syncthreads();
    if (t < n) buf[t] = r;
    __syncthreads();
  }
  if (t == 0) mean[0] = __double2float_rn(buf[0] / (double)nb);
}

// ---------------------------------------------------------------------------------------
// Q-C: per group of 256 absmax values: d = fp32(c - mean), c2 = max |d|, code = E4M3(d/c2).
// One warp per group, lane l owns blocks 8l..8l+7.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dq_groups_kernel(const float* __restrict__ absmax, int64_t nb, int64_t ng,
                                                        const float* __restrict__ mean_p,
                                                        uint8_t* __restrict__ scale_codes, float* __restrict__ c2,
                                                        int sw_encode) {
  const int lane = threadIdx.x & 31;
  const int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (g >= ng) return;
  const float mean = *mean_p;
  float d[8];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t b = g * kB2 + lane * 8 + i;
    d[i] = (b < nb) ? __fsub_rn(absmax[b], mean) : 0.0f;
    m = fmaxf(m, fabsf(d[i]));
  }
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  uint32_t e[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = 0;
  if (m > 0.0f) {
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float v0 = __fdiv_rn(d[i], m), v1 = __fdiv_rn(d[i + 1], m);
      if (sw_encode) {
        e[i] = e4m3_encode_sw(v0);
        e[i + 1] = e4m3_encode_sw(v1);
      } else {
        const uint32_t p = e4m3x2_encode_hw(v0, v1);
        e[i] = p & 0xFFu;
        e[i + 1] = p >> 8;
      }
    }
  }
  const int64_t b0 = g * kB2 + lane * 8;
  if (b0 + 8 <= nb) {
    uint2 out;
    out.x = e[0] | (e[1] << 8) | (e[2] << 16) | (e[3] << 24);
    out.y = e[4] | (e[5] << 8) | (e[6] << 16) | (e[7] << 24);
    *reinterpret_cast<uint2*>(scale_codes + b0) = out;
  } else {
    for (int i = 0; i < 8; ++i)
      if (b0 + i < nb) scale_codes[b0 + i] = (uint8_t)e[i];
  }
  if (lane == 0) c2[g] = m;
}

// ---------------------------------------------------------------------------------------
// D: standalone dequant, one thread per block of 64 (two 16-byte code loads, the block's bf16
// table).  A warp's 32 blocks are one contiguous 4 KB of output: the expanded rows go to
// shared memory first (16-byte chunk j of block l at chunk position j ^ (l & 7), so that
// neither the writes nor the reads conflict), then the warp stores 512 contiguous bytes per
// instruction.  Warps whose blocks reach past the end use per-thread stores.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint8_t* __restrict__ codes,
                                                          const uint8_t* __restrict__ scale_codes,
                                                          const float* __restrict__ c2,
                                                          const float* __restrict__ mean_p, int64_t numel,
                                                          int64_t nb, uint16_t* __restrict__ out) {
  __shared__ uint4 stage[8][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b0 = (int64_t)blockIdx.x * blockDim.x + warp * 32;   // first block of this warp
  const int64_t b = b0 + lane;
  if (b0 >= nb) return;                                             // whole warps leave together
  const bool whole = (b0 + 32) * kB1 <= numel;                      // implies b0 + 32 <= nb
  uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  Nf4Lut L{};
  if (b < nb) {
    const float scale = dq_block_scale(__ldg(scale_codes + b), __ldg(c2 + (b >> 8)), __ldg(mean_p));
    nf4_lut_build(scale, L);
    const uint4* src = reinterpret_cast<const uint4*>(codes + b * 32);
    const uint4 c0 = __ldg(src), c1 = __ldg(src + 1);
    w[0] = c0.x; w[1] = c0.y; w[2] = c0.z; w[3] = c0.w;
    w[4] = c1.x; w[5] = c1.y; w[6] = c1.z; w[7] = c1.w;
  }
  if (whole) {
    uint4* row = stage[warp];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t o[4];
      nf4_expand8(w[j], L, o);
      row[lane * 8 + (j ^ (lane & 7))] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(out + b0 * kB1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = i * 32 + lane, lb = q >> 3, j = q & 7;
      dst[q] = row[lb * 8 + (j ^ (lb & 7))];
    }
    return;
  }
  if (b >= nb) return;
  const int64_t e0 = b * kB1;
  for (int j = 0; j < 8; ++j) {
    uint32_t o[4];
    nf4_expand8(w[j], L, o);
    if (e0 + 8 * j + 8 <= numel) {
      *reinterpret_cast<uint4*>(out + e0 + 8 * j) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
      for (int i = 0; i < 8; ++i) {
        const int64_t e = e0 + 8 * j + i;
        if (e < numel) out[e] = (uint16_t)((o[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
      }
    }
  }
}

// E4M3 encode of an fp32 array (hardware or software conversion); a utility for checking
// the scale-code format against other implementations.
__global__ void e4m3_encode_kernel(const float* __restrict__ v, int64_t n, uint8_t* __restrict__ out, int sw) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  out[i] = (uint8_t)(sw ? e4m3_encode_sw(v[i]) : (e4m3x2_encode_hw(v[i], 0.0f) & 0xFFu));
}

// ---------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------
static int grid_for(int64_t threads, int per_block, int cap) {
  int64_t g = (threads + per_block - 1) / per_block;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (int)g;
}

cudaError_t launch_quantize(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* scale_codes, float* c2,
                            float* mean, float* absmax_ws, double* gsum_ws, cudaStream_t st, int sw_encode) {
  const int64_t nb = (numel + kB1 - 1) / kB1;
  const int64_t ng = (nb + kB2 - 1) / kB2;
  const int64_t nchunks = nb * 8;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  nf4_quant_blocks_kernel<<<grid_for(nchunks, 256, sms * 8), 256, 0, st>>>(
      W, numel, nchunks, reinterpret_cast<uint32_t*>(codes), absmax_ws);
  dq_group_sums_kernel<<<grid_for(ng * 32, 256, 1 << 30), 256, 0, st>>>(absmax_ws, nb, ng, gsum_ws);
  dq_mean_kernel<<<1, 1024, 0, st>>>(gsum_ws, ng, nb, mean);
  dq_groups_kernel<<<grid_for(ng * 32, 256, 1 << 30), 256, 0, st>>>(absmax_ws, nb, ng, mean, scale_codes, c2,
                                                                     sw_encode);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* codes, const uint8_t* scale_codes, const float* c2, const float* mean,
                           int64_t numel, uint16_t* out, cudaStream_t st) {
  const int64_t nb = (numel + kB1 - 1) / kB1;
  nf4_dequant_kernel<<<grid_for(nb, 256, 1 << 30), 256, 0, st>>>(codes, scale_codes, c2, mean, numel, nb, out);
  return cudaGetLastError();
}

cudaError_t launch_e4m3_encode(const float* v, int64_t n, uint8_t* out, int sw, cudaStream_t st) {
  e4m3_encode_kernel<<<grid_for(n, 256, 1 << 30), 256, 0, st>>>(v, n, out, sw);
  return cudaGetLastError();
}

cudaError_t read_and_clear_error_word(uint32_t* word, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(word, g_error_word, sizeof(uint32_t), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

}  // namespace qnf4
