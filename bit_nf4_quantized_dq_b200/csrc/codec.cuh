// NF4 + double quantization: quantize (two kernels) and the standalone dequant stream.
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

// Correctly rounded quotient w / c from y = RN(1/c): q0 = RN(w y), the remainder w - c q0 is
// exact by one fused multiply-add, and RN(q0 + remainder * y) is RN(w / c).  This is
// Markstein's correction step (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990; the theorem on Markstein's
// iteration in Muller et al., "Handbook of Floating-Point Arithmetic"): with y within half an
// ulp of 1/c and q0 within one ulp of w/c, the corrected quotient is the correctly rounded one,
// as long as no intermediate leaves the normal range.  Callers keep 2^-100 <= c <= 2^100 and
// |w| <= c, which guarantees that (a tiny quotient may be subnormal, and such an n is far
// below every midpoint, so its code does not depend on the last bits).
__device__ __forceinline__ float div_rn_by_recip(float w, float c, float y) {
  const float q0 = __fmul_rn(w, y);
  const float r = __fmaf_rn(-c, q0, w);
  return __fmaf_rn(r, y, q0);
}

__device__ __forceinline__ bool recip_path_ok(float c) {
  return c >= 7.888609052210118e-31f && c <= 1.2676506002282294e+30f;   // 2^-100 .. 2^100
}

// Q-A: one group of 256 blocks (16384 weights, 32 KB of bf16) per CTA iteration.  Thread t
// handles chunk it * 256 + t of the group for it = 0..7 (one 16-byte load each, all eight
// issued before any is used); the eight lanes of a chunk's block reduce its absmax with
// three xor shuffles.  Per weight: the correctly rounded n = w / absmax (one reciprocal per
// block, three fp32 operations per weight), the nearest level, nibble packing.  The group's
// float64 absmax sum follows the adjacent-pair tree: each warp-iteration covers blocks
// 4m .. 4m + 3 (m = it * 8 + warp), summed as ((a0 + a1) + (a2 + a3)) by two shuffles, and
// the 64 four-block sums of the group are reduced by one warp in index order.
constexpr int kQuantThreads = 256;
constexpr int kGroupChunks = kB2 * 8;          // 16-byte chunks per group of 256 blocks

__global__ void __launch_bounds__(kQuantThreads) nf4_quant_groups_kernel(const uint16_t* __restrict__ W,
                                                                         int64_t numel, int64_t ng,
                                                                         uint32_t* __restrict__ codes32,
                                                                         float* __restrict__ absmax,
                                                                         double* __restrict__ gsum) {
  __shared__ BucketEntry tab[33][32];
  __shared__ double sum4[64];
  build_bucket_table(tab);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nchunks = 8 * ((numel + kB1 - 1) / kB1);   // chunks of whole blocks: the padded tail codes to level 7
  for (int64_t g = blockIdx.x; g < ng; g += gridDim.x) {
    const int64_t c0 = g * kGroupChunks + threadIdx.x;
    uint4 v[8];
    const bool whole = (g + 1) * kGroupChunks * 8 <= numel;   // every chunk of the group is full
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int64_t c = c0 + it * kQuantThreads;
      if (whole || (c + 1) * 8 <= numel) {
        v[it] = __ldg(reinterpret_cast<const uint4*>(W) + c);
      } else {
        uint32_t u[4] = {0u, 0u, 0u, 0u};
        for (int i = 0; i < 8; ++i)
          if (c * 8 + i < numel) u[i >> 1] |= (uint32_t)W[c * 8 + i] << (16 * (i & 1));
        v[it] = make_uint4(u[0], u[1], u[2], u[3]);
      }
    }
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int64_t c = c0 + it * kQuantThreads;
      const uint32_t u[4] = {v[it].x, v[it].y, v[it].z, v[it].w};
      float w[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        w[2 * i] = __uint_as_float(u[i] << 16);
        w[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(w[i]));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
      // four-block subtree sum of this warp-iteration (lanes 0, 8, 16, 24 hold blocks 4m..4m+3)
      double s = (double)m;
      s = s + __shfl_xor_sync(0xFFFFFFFFu, s, 8);
      s = s + __shfl_xor_sync(0xFFFFFFFFu, s, 16);
      if (lane == 0) sum4[it * 8 + warp] = s;
      if (c >= nchunks) continue;
      if ((lane & 7) == 0) absmax[c >> 3] = m;
      uint32_t packed = 0x77777777u;             // all-zero block: every weight is level 7
      if (m > 0.0f) {
        packed = 0u;
        if (recip_path_ok(m)) {
          const float y = __frcp_rn(m);
#pragma unroll
          for (int i = 0; i < 8; ++i) packed |= nearest_code(div_rn_by_recip(w[i], m, y), tab, lane) << (4 * i);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) packed |= nearest_code(__fdiv_rn(w[i], m), tab, lane) << (4 * i);
        }
      }
      codes32[c] = packed;
    }
    __syncthreads();
    if (warp == 0) {
      double t = sum4[2 * lane] + sum4[2 * lane + 1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) t = t + __shfl_xor_sync(0xFFFFFFFFu, t, off);
      if (lane == 0) gsum[g] = t;
    }
    __syncthreads();
  }
  // let the dependent double-quantization kernel start its launch while this grid drains
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// Q-B: double quantization.  Every CTA first forms the mean itself (so no other launch or
// grid-wide wait is needed): the float64 group sums, zero-padded, are reduced by the same
// adjacent-pair tree in aligned chunks of 2048 (eight per thread in registers, then the warp
// butterfly, then the eight warp sums), then the chunk sums (zero-padded to a power of two)
// by one warp.  Zero padding leaves every partial sum unchanged, so this equals the tree over
// the sums padded to the next power of two.  mean = fp32(sum / nb).  Then one warp per group
// of 256 absmax values: d = fp32(c - mean), c2 = max |d|, code = E4M3(fp32(d / c2)).
// ---------------------------------------------------------------------------------------
constexpr int kMaxMeanChunks = 1024;           // 2^21 groups: numel up to 2^35

__global__ void __launch_bounds__(256) dq_mean_groups_kernel(const float* __restrict__ absmax,
                                                             const double* __restrict__ gsum, int64_t nb,
                                                             int64_t ng, float* __restrict__ mean_out,
                                                             uint8_t* __restrict__ scale_codes,
                                                             float* __restrict__ c2, int sw_encode) {
  __shared__ double warp_sum[8];
  __shared__ double chunk_sum[kMaxMeanChunks];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the quantize kernel's absmax values and group sums are complete and visible after this
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t nchunks = (ng + 2047) / 2048;
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int64_t i0 = ch * 2048 + 8 * (int64_t)threadIdx.x;
    double x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = (i0 + i < ng) ? gsum[i0 + i] : 0.0;
    double s = ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) s = s + __shfl_xor_sync(0xFFFFFFFFu, s, off);
    if (lane == 0) warp_sum[warp] = s;
    __syncthreads();
    if (threadIdx.x == 0)
      chunk_sum[ch] = ((warp_sum[0] + warp_sum[1]) + (warp_sum[2] + warp_sum[3])) +
                      ((warp_sum[4] + warp_sum[5]) + (warp_sum[6] + warp_sum[7]));
    __syncthreads();
  }
  float mean;
  {
    int64_t p2 = 1;
    while (p2 < nchunks) p2 <<= 1;
    if (warp == 0) {
      // lane l reduces chunk sums [l q, (l + 1) q) by the adjacent-pair tree (q a power of two)
      const int64_t q = p2 >= 32 ? p2 / 32 : 1;
      double part = 0.0;
      if ((int64_t)lane * q < p2) {
        double* b = chunk_sum + lane * q;
        for (int64_t i = 0; i < q; ++i)
          if (lane * q + i >= nchunks) b[i] = 0.0;
        for (int64_t h = 1; h < q; h <<= 1)
          for (int64_t i = 0; i < q; i += 2 * h) b[i] = b[i] + b[i + h];
        part = b[0];
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) part = part + __shfl_xor_sync(0xFFFFFFFFu, part, off);
      if (lane == 0) warp_sum[0] = part;
    }
    __syncthreads();
    mean = __double2float_rn(warp_sum[0] / (double)nb);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) mean_out[0] = mean;
  for (int64_t g = (int64_t)blockIdx.x * 8 + warp; g < ng; g += (int64_t)gridDim.x * 8) {
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
          const uint32_t pk = e4m3x2_encode_hw(v0, v1);
          e[i] = pk & 0xFFu;
          e[i + 1] = pk >> 8;
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
  if (ng > (int64_t)kMaxMeanChunks * 2048) return cudaErrorInvalidValue;
  int sms = 148, per_sm = 4;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // a grid-stride loop over groups: as many CTAs as fit on the device at once
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, nf4_quant_groups_kernel, kQuantThreads, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  nf4_quant_groups_kernel<<<grid_for(ng, 1, sms * per_sm), kQuantThreads, 0, st>>>(
      W, numel, ng, reinterpret_cast<uint32_t*>(codes), absmax_ws, gsum_ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // The double-quantization kernel may launch while the quantize grid drains (programmatic
  // dependent launch); it waits for that grid's results before reading them.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid_for((ng + 7) / 8, 1, 2 * sms));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, dq_mean_groups_kernel, (const float*)absmax_ws, (const double*)gsum_ws, nb, ng,
                         mean, scale_codes, c2, sw_encode);
  if (e == cudaErrorNotSupported) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, dq_mean_groups_kernel, (const float*)absmax_ws, (const double*)gsum_ws, nb, ng,
                           mean, scale_codes, c2, sw_encode);
  }
  if (e != cudaSuccess) return e;
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
