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
struct __align__(8) BucketEntry {
  uint32_t base;
  float thr;
};

// Thread b < 33 computes bucket b once and fills its 32 per-lane copies (one copy per lane
// keeps the lookups of a warp free of bank conflicts).
__device__ __forceinline__ void build_bucket_table(BucketEntry (*tab)[32], const Codebook& cb) {
  const float* q = cb.q;
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

// Correctly rounded n = fp32(w / c) for bf16 w and c without a division per weight.
//
// w / c = (mw / mc) 2^k with 8-bit integer significands mw, mc.  Such a quotient is never an
// fp32 rounding midpoint, and is at least 2^-32 (relative) away from every one: the gap to
// a midpoint (2M + 1) 2^(E - 24) is 2^(E - 24) |mw 2^j - mc (2M + 1)| / mc, a nonzero integer
// over mc <= 255.  So any approximation of w / c within 2^-40 (relative) rounds to the same
// fp32 value.  With the reciprocal as an unevaluated sum y_hi + y_lo (y_hi = RN(1/c), the
// remainder 1 - c y_hi exact by a fused multiply-add, y_lo = RN(remainder * y_hi)), y_hi + y_lo
// is within about 2^-46 of 1/c, and fma(w, y_hi, RN(w y_lo)) rounds a value within about
// 2^-45 of w / c, once: the result is RN(w / c).  Valid while c, 1/c and y_lo stay normal;
// callers keep 2^-100 <= c <= 2^100 and |w| <= c (a subnormal n can only be a tiny one, far
// below every midpoint between levels, whose code cannot change).
struct Recip2 {
  float hi, lo;
};
__device__ __forceinline__ Recip2 recip2(float c) {
  const float hi = __frcp_rn(c);
  const float rem = __fmaf_rn(-c, hi, 1.0f);
  return Recip2{hi, __fmul_rn(rem, hi)};
}
__device__ __forceinline__ float div_rn_recip2(float w, Recip2 y) {
  return __fmaf_rn(w, y.hi, __fmul_rn(w, y.lo));
}
__device__ __forceinline__ bool recip_path_ok(float c) {
  return c >= 7.888609052210118e-31f && c <= 1.2676506002282294e+30f;   // 2^-100 .. 2^100
}

// Two fp32 lanes in one 64-bit register pair, for the sm_100 paired fp32 instructions (each
// lane is rounded exactly as the scalar instruction would round it).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// Packed bf16 pair -> its two fp32 values (exact), as one register pair.
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t u) {
  return f2_pack(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// max(|a|, |b|) of each bf16 lane (the sign of the result, the xor of the inputs', is
// discarded by the caller).  A NaN input gives NaN, so that a block holding one never takes
// the table path below (whose bucket address is only in range for |n| <= 1).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// One bucket-table entry by its 32-bit shared-memory address.
__device__ __forceinline__ uint2 lds_entry(uint32_t addr) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// Codes of one packed word (two weights) given n for both: bucket index from one fused
// multiply-add each (1.5 * 2^23 + 16 + 16 n rounds to the integer 16 + round(16 n) in the low
// mantissa bits, so (bits << 8) is 256 * bucket plus a constant that lane_bias cancels: one
// shift-add forms the entry's address), then code = base + (n > threshold), the comparison
// taken from the sign of the correctly rounded threshold - n (zero only when they are equal).
__device__ __forceinline__ uint32_t codes_of_pair(uint64_t n2, uint32_t lane_bias) {
  const uint64_t t2 = f2_fma(n2, f2_pack(16.0f, 16.0f), f2_pack(12582928.0f, 12582928.0f));
  const uint2 e0 = lds_entry(((uint32_t)t2 << 8) + lane_bias);
  const uint2 e1 = lds_entry(((uint32_t)(t2 >> 32) << 8) + lane_bias);
  const uint32_t c0 = e0.x + (__float_as_uint(__fsub_rn(__uint_as_float(e0.y), f2_lo(n2))) >> 31);
  const uint32_t c1 = e1.x + (__float_as_uint(__fsub_rn(__uint_as_float(e1.y), f2_hi(n2))) >> 31);
  return c0 + (c1 << 4);
}

// Q-A: one group of 256 blocks (16384 weights, 32 KB of bf16) per CTA iteration; thread t
// takes block t of the group: eight 16-byte loads (128 contiguous bytes, all in flight before
// any is used), absmax over its 64 weights, the correctly rounded n = w / absmax, the nearest
// level, 32 bytes of packed codes.  The group's float64 sum of its 256 absmax values follows
// the adjacent-pair tree: the xor butterfly over the 32 lanes of each warp (blocks
// 32 w .. 32 w + 31), then the eight warp sums in order.
constexpr int kQuantThreads = kB2;             // one block of 64 weights per thread

// Codes of a block whose absmax lies outside [2^-100, 2^100] (or of a ragged last block):
// one correctly rounded division per weight, the weights re-read from W (zero past numel).
__device__ __noinline__ void codes_by_division(const uint16_t* __restrict__ W, int64_t e0, int64_t numel, float m,
                                               const BucketEntry (*tab)[32], int lane, uint32_t* __restrict__ dst) {
  for (int i = 0; i < 8; ++i) {
    uint32_t p = 0u;
    for (int j = 0; j < 8; ++j) {
      const int64_t e = e0 + 8 * i + j;
      const float w = e < numel ? __uint_as_float((uint32_t)W[e] << 16) : 0.0f;
      p |= nearest_code(__fdiv_rn(w, m), tab, lane) << (4 * j);
    }
    dst[i] = p;
  }
}

// The ragged last block (zero-padded past numel), or any block when W holds no whole block:
// absmax and codes straight from global memory, one correctly rounded division per weight.
// Returns the block's absmax.
__device__ __noinline__ float quant_block_global(const uint16_t* __restrict__ W, int64_t b, int64_t numel,
                                                 const BucketEntry (*tab)[32], int lane, uint32_t* __restrict__ codes32,
                                                 float* __restrict__ absmax) {
  const int64_t e0 = b * kB1;
  float m = 0.0f;
  for (int64_t e = e0; e < e0 + kB1 && e < numel; ++e) m = fmaxf(m, fabsf(__uint_as_float((uint32_t)W[e] << 16)));
  absmax[b] = m;
  if (m > 0.0f) {
    codes_by_division(W, e0, numel, m, tab, lane, codes32 + b * 8);
  } else {
    for (int i = 0; i < 8; ++i) codes32[b * 8 + i] = 0x77777777u;
  }
  return m;
}

// Q-A, streaming form.  Persistent CTAs, two per SM: one thread of the last warp streams
// groups of 256 blocks (32 KB) into a ring of kQStages shared-memory stages with TMA tile loads
// of a [blocks][64] bf16 view of W (128-byte swizzle: chunk j of block row r sits at chunk
// position j ^ (r % 8), so the warps read their blocks without bank conflicts); sixteen
// warps code the stages in order.  Threads 2r and 2r + 1 own block r of the group, 32
// weights each: their chunks come from shared memory, then absmax (one shuffle
// joins the halves), the correctly rounded n = w / absmax, the nearest level and 16 bytes of
// packed codes each.  The group's float64 absmax sum follows the adjacent-pair tree: the xor
// butterfly over each warp's 16 blocks, then the sixteen warp sums in order.
constexpr int kQStages = 3;
constexpr int kQStageBytes = kB2 * kB1 * 2;           // 32 KB
constexpr int kQGroupWarps = 16;                      // warps coding one group (two threads per block)
constexpr int kQConsumerWarps = kQGroupWarps;
constexpr int kQThreads = 32 * (kQConsumerWarps + 1);
constexpr int kQSmemBytes = kQStages * kQStageBytes + 1024;
// Warp sums of a group are handed to thread 0 through a ring of kQSumSlots slots, each with an
// mbarrier that the group's warps arrive on; thread 0 forms a group's float64 sum one group
// later, so no warp waits for the others.  A warp can run at most kQStages groups ahead of the
// slowest one (a stage is reloaded only after every warp released it), so slot i % kQSumSlots
// is not rewritten, and its barrier not two phases ahead, while thread 0 still reads group i.
constexpr int kQSumSlots = 6;
static_assert(kQSumSlots >= kQStages + 3 && kQSumSlots <= 8, "sum ring too short for the pipeline depth");

struct QuantParams {
  CUtensorMap w_map;          // W as [nb_full][64] bf16, box 64 x 256, 128-byte swizzle
  Codebook cb;
  const uint16_t* W;
  int64_t numel, nb, nb_full, ng;
  uint32_t* codes32;
  float* absmax;
  double* gsum;
};

__global__ void __launch_bounds__(kQThreads, 2) nf4_quant_stream_kernel(const __grid_constant__ QuantParams p) {
  extern __shared__ uint8_t qsmem_dyn[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_dyn) + 1023) & ~uintptr_t(1023));
  __shared__ BucketEntry tab[33][32];
  __shared__ uint64_t full[kQStages], empty[kQStages], psum[kQSumSlots];
  __shared__ double warp_sum[kQSumSlots][kQGroupWarps];
  __shared__ uint32_t abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kQGroupWarps);
    }
    for (int s = 0; s < kQSumSlots; ++s) mbar_init(&psum[s], kQGroupWarps);
    abort_flag = 0u;
    mbar_fence_init();
  }
  build_bucket_table(tab, p.cb);
  __syncthreads();
  volatile uint32_t* abort_word = &abort_flag;
  const int64_t n_local = p.ng > blockIdx.x ? (p.ng - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == kQConsumerWarps) {
    // ------------------------------------------------------------------ producer
    if (lane == 0 && p.nb_full > 0) {
      tma_prefetch_desc(&p.w_map);
      int64_t issued = 0;
      for (int64_t i = 0; i < n_local; ++i) {
        const int s = (int)(i % kQStages);
        const uint32_t ph = (uint32_t)(i / kQStages) & 1u;
        if (!mbar_wait_thread(&empty[s], ph ^ 1u, abort_word, kErrWaitEmpty)) break;
        const int64_t g = blockIdx.x + i * gridDim.x;
        mbar_arrive_expect_tx(&full[s], kQStageBytes);
        tma_load_2d(ring + s * kQStageBytes, &p.w_map, 0, (int32_t)(g * kB2), &full[s]);
        issued = i + 1;
      }
      // drain copies still in flight before the CTA's shared memory goes away
      for (int64_t i = issued > kQStages ? issued - kQStages : 0; i < issued; ++i) {
        const int s = (int)(i % kQStages);
        const uint32_t ph = (uint32_t)(i / kQStages) & 1u;
        for (int k = 0; k < (1 << 22) && !mbar_try_wait(&full[s], ph); ++k) {}
      }
    }
  } else {
    // ------------------------------------------------------------------ consumers
    const int t = threadIdx.x;
    const int r = t >> 1, h = t & 1;          // block of the group, and which half of it
    // tab[v][lane] sits at tab + 256 v + 8 lane; the bucket's float bits shifted left by 8
    // carry 256 v plus 0x40000000 (mod 2^32), which the bias removes
    const uint32_t lane_bias = smem_u32(&tab[0][lane]) - 0x40000000u;
    int s = 0;
    uint32_t ph = 0;
    // sum-ring position: slot in bits 0-2, phase parity in bit 3
    uint32_t sp = 0, prev_sp = 0;
    // thread 0: the float64 sum of group i from its sixteen warp sums (adjacent-pair tree)
    auto group_sum = [&](int64_t i, uint32_t at) -> bool {
      const int sl = (int)(at & 7u);
      if (!mbar_wait_thread(&psum[sl], at >> 3, abort_word, kErrWaitGroup)) return false;
      const double* w = warp_sum[sl];
      const double q0 = ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
      const double q1 = ((w[8] + w[9]) + (w[10] + w[11])) + ((w[12] + w[13]) + (w[14] + w[15]));
      p.gsum[blockIdx.x + i * gridDim.x] = q0 + q1;
      return true;
    };
    const bool sums = warp == 0 && p.gsum != nullptr;   // no group sums without double quantization
    int64_t i = 0;
    for (; i < n_local; ++i) {
      const int64_t g = blockIdx.x + i * gridDim.x;
      const int64_t b = g * kB2 + r;
      // a warp whose wait gave up still hands in its (zero) warp sum below, so that thread 0
      // is not left waiting for it; all warps leave at the abort check after that
      bool ok = true;
      uint4 v[4];
      if (p.nb_full > 0) {
        ok = mbar_wait(&full[s], ph, abort_word, kErrWaitTma);
        if (ok) {
          const uint8_t* row = ring + s * kQStageBytes + r * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4*>(row + (((4 * h + j) ^ (r & 7)) << 4));
        }
      }
      const bool whole = ok && b < p.nb_full;
      float m = 0.0f;
      if (ok && p.nb_full > 0) {
        // every loaded word enters the absmax (bf16 pairs, max of magnitudes, exact), so the
        // stage's data are in registers before the stage is handed back for the next load
        uint32_t a2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) a2[j] = bf16x2_absmax(bf16x2_absmax(v[j].x, v[j].y), bf16x2_absmax(v[j].z, v[j].w));
        const uint32_t am = bf16x2_absmax(bf16x2_absmax(a2[0], a2[1]), bf16x2_absmax(a2[2], a2[3]));
        m = fmax_nan(__uint_as_float((am << 16) & 0x7FFF0000u), __uint_as_float(am & 0x7FFF0000u));
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (!whole) m = 0.0f;
      }
      if (++s == kQStages) {
        s = 0;
        ph ^= 1u;
      }
      if (!whole && ok && b < p.nb && h == 0) {
        m = quant_block_global(p.W, b, p.numel, tab, lane, p.codes32, p.absmax);
      }
      // join the two halves of each block (a NaN in either half reaches both)
      m = fmax_nan(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      double sum = (double)m;
#pragma unroll
      for (int off = 2; off < 32; off <<= 1) sum = sum + __shfl_xor_sync(0xFFFFFFFFu, sum, off);
      if (lane == 0) {
        warp_sum[sp & 7u][warp] = sum;
        mbar_arrive(&psum[sp & 7u]);   // release: the sum is visible to thread 0 after its wait
      }
      if (whole) {
        if (h == 0) p.absmax[b] = m;
        uint4* dst = reinterpret_cast<uint4*>(p.codes32 + b * 8) + h;
        // table path: 2^-100 <= m <= 2^100 and no NaN in the block, so every |n| <= 1
        if (m > 0.0f && recip_path_ok(m)) {
          const Recip2 y = recip2(m);
          const uint64_t yhi = f2_pack(y.hi, y.hi), ylo = f2_pack(y.lo, y.lo);
          uint32_t packed[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
            uint32_t pk = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              // n = RN(w / m) for both weights of the word (the reciprocal-pair quotient)
              const uint64_t w2 = bf16x2_to_f2(u[k]);
              const uint64_t n2 = f2_fma(w2, yhi, f2_mul(w2, ylo));
              pk += codes_of_pair(n2, lane_bias) << (8 * k);
            }
            packed[j] = pk;
          }
          *dst = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        } else if (m > 0.0f) {
          if (h == 0) codes_by_division(p.W, b * kB1, p.numel, m, tab, lane, p.codes32 + b * 8);
        } else {
          *dst = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);   // all-zero block: level 7
        }
      }
      if (sums && i > 0) {
        // lane 0 waits; the whole warp takes the outcome, so it stays converged
        bool done = true;
        if (lane == 0) done = group_sum(i - 1, prev_sp);
        if (!__shfl_sync(0xFFFFFFFFu, (int)done, 0)) break;
      }
      prev_sp = sp;
      sp = (sp & 7u) == kQSumSlots - 1 ? (sp & 8u) ^ 8u : sp + 1u;
      if (__any_sync(0xFFFFFFFFu, *abort_word != 0u)) break;
    }
    if (sums && lane == 0 && i == n_local && n_local > 0) group_sum(n_local - 1, prev_sp);
  }
  // let the dependent double-quantization kernel start its launch while this grid drains
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// Q-B: double quantization.  Every CTA first forms the mean itself (so no other launch or
// grid-wide wait is needed): the float64 group sums, zero-padded, are reduced by the same
// adjacent-pair tree in aligned chunks of 8192 (eight per thread in registers, then the warp
// butterfly, then the 32 warp sums by one more butterfly), then the chunk sums (zero-padded to
// a power of two) by one warp.  Zero padding leaves every partial sum unchanged, so this
// equals the tree over the sums padded to the next power of two.  mean = fp32(sum / nb).  A
// group count up to 8192 (numel up to 2^27) takes one pass, so one round trip to memory.
// Then one warp per group of 256 absmax values: d = fp32(c - mean), c2 = max |d|,
// code = E4M3(fp32(d / c2)).
// ---------------------------------------------------------------------------------------
constexpr int kDqThreads = 1024;
constexpr int kDqWarps = kDqThreads / 32;
constexpr int kDqChunk = 8 * kDqThreads;       // group sums per pass
constexpr int kMaxMeanChunks = 1024;           // 2^23 groups: numel up to 2^37

__global__ void __launch_bounds__(kDqThreads, 1) dq_mean_groups_kernel(const float* __restrict__ absmax,
                                                                    const double* __restrict__ gsum, int64_t nb,
                                                                    int64_t ng, float* __restrict__ mean_out,
                                                                    uint8_t* __restrict__ scale_codes,
                                                                    float* __restrict__ c2, int sw_encode) {
  __shared__ double warp_sum[kDqWarps];
  __shared__ double chunk_sum[kMaxMeanChunks];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the quantize kernel's absmax values and group sums are complete and visible after this
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // this warp's first group: its absmax values are in flight while the mean is formed
  int64_t g = (int64_t)blockIdx.x * kDqWarps + warp;
  float a[8];
  auto load_group = [&](int64_t gg) {
    const int64_t b0 = gg * kB2 + lane * 8;
    if (b0 + 8 <= nb) {
      const float4* src = reinterpret_cast<const float4*>(absmax + b0);
      const float4 x0 = src[0], x1 = src[1];
      a[0] = x0.x; a[1] = x0.y; a[2] = x0.z; a[3] = x0.w;
      a[4] = x1.x; a[5] = x1.y; a[6] = x1.z; a[7] = x1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = (b0 + i < nb) ? absmax[b0 + i] : 0.0f;
    }
  };
  if (g < ng) load_group(g);
  const int64_t nchunks = (ng + kDqChunk - 1) / kDqChunk;
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int64_t i0 = ch * kDqChunk + 8 * (int64_t)threadIdx.x;
    double x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = (i0 + i < ng) ? gsum[i0 + i] : 0.0;
    double s = ((x[0] + x[1]) + (x[2] + x[3])) + ((x[4] + x[5]) + (x[6] + x[7]));
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) s = s + __shfl_xor_sync(0xFFFFFFFFu, s, off);
    if (lane == 0) warp_sum[warp] = s;
    __syncthreads();
    if (warp == 0) {
      // the 32 warp sums, in order, by the same butterfly
      double w = warp_sum[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) w = w + __shfl_xor_sync(0xFFFFFFFFu, w, off);
      if (lane == 0) chunk_sum[ch] = w;
    }
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
  for (; g < ng; g += (int64_t)gridDim.x * kDqWarps) {
    float d[8];
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g * kB2 + lane * 8 + i;
      d[i] = (b < nb) ? __fsub_rn(a[i], mean) : 0.0f;
      m = fmaxf(m, fabsf(d[i]));
    }
    if (g + (int64_t)gridDim.x * kDqWarps < ng) load_group(g + (int64_t)gridDim.x * kDqWarps);
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
                                                          int64_t nb, uint16_t* __restrict__ out, const Codebook cb,
                                                          int scale_fp32) {
  __shared__ uint4 stage[8][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b0 = (int64_t)blockIdx.x * blockDim.x + warp * 32;   // first block of this warp
  const int64_t b = b0 + lane;
  if (b0 >= nb) return;                                             // whole warps leave together
  const bool whole = (b0 + 32) * kB1 <= numel;                      // implies b0 + 32 <= nb
  uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  Nf4Lut L{};
  if (b < nb) {
    // scale_fp32: c2 holds the fp32 absmax of every block (single-level quantization)
    const float scale = scale_fp32 ? __ldg(c2 + b) : dq_block_scale(__ldg(scale_codes + b), __ldg(c2 + (b >> 8)), __ldg(mean_p));
    nf4_lut_build(scale, L, cb);
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

cudaError_t launch_quantize(const CUtensorMap* w_map, const uint16_t* W, int64_t numel, const Codebook& cb,
                            uint8_t* codes, uint8_t* scale_codes, float* c2, float* mean, float* absmax_ws,
                            double* gsum_ws, cudaStream_t st, int sw_encode) {
  const int64_t nb = (numel + kB1 - 1) / kB1;
  const int64_t ng = (nb + kB2 - 1) / kB2;
  if (ng > (int64_t)kMaxMeanChunks * kDqChunk) return cudaErrorInvalidValue;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = enable_smem_once(nf4_quant_stream_kernel, kQSmemBytes, configured);
  if (e != cudaSuccess) return e;
  QuantParams qp;
  memset(&qp, 0, sizeof(qp));
  if (w_map) qp.w_map = *w_map;
  qp.cb = cb;
  qp.W = W;
  qp.numel = numel;
  qp.nb = nb;
  qp.nb_full = w_map ? numel / kB1 : 0;
  qp.ng = ng;
  qp.codes32 = reinterpret_cast<uint32_t*>(codes);
  qp.absmax = absmax_ws;
  qp.gsum = gsum_ws;
  nf4_quant_stream_kernel<<<grid_for(ng, 1, 2 * sms), kQThreads, kQSmemBytes, st>>>(qp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (!gsum_ws) return cudaSuccess;   // single-level quantization: the absmax values are the scales
  // The double-quantization kernel may launch while the quantize grid drains (programmatic
  // dependent launch); it waits for that grid's results before reading them.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid_for((ng + kDqWarps - 1) / kDqWarps, 1, sms));
  cfg.blockDim = dim3(kDqThreads);
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
                           int64_t numel, uint16_t* out, const Codebook& cb, int scale_fp32, cudaStream_t st) {
  const int64_t nb = (numel + kB1 - 1) / kB1;
  nf4_dequant_kernel<<<grid_for(nb, 256, 1 << 30), 256, 0, st>>>(codes, scale_codes, c2, mean, numel, nb, out, cb,
                                                                  scale_fp32);
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
