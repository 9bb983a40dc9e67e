// Low-rank products of the QLoRA linear with float64-accurate accumulation:
//   t  = s x A^T        (rows = tokens,   cols = rank; reduction over in-features)
//   u  = s dY B         (rows = tokens,   cols = rank; reduction over out-features)
//   dA^T = x^T u        (rows = in-features,  cols = rank; reduction over tokens)
//   dB   = dY^T t       (rows = out-features, cols = rank; reduction over tokens)
//
// "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged
// Optimizers" (fullstackaihub), section 4: the adapter term (alpha/r) X L1 L2 of the forward
// pass and the adapter-only gradients of the backward; "QLoRA, explained." step 5.
//
// The tensor cores multiply exact bf16 values (x, dY, A, B, or an exact three-term bf16
// split of an fp32 t or u: fp32 = t1 + t2 + t3 with 8 significant bits each) and accumulate
// one 64-wide k-block at a time in TMEM (fp32), one column group per split term.  After every
// k-block eight flush warps add the block sums into a running sum held as an unevaluated pair
// of fp32 values (hi + lo, about 48 significant bits: each block sum enters hi by an exact
// two-sum and the rounding error goes to lo), with up to four TMEM accumulator buffers so
// that the next k-blocks' MMAs overlap the flush.  The three split terms' block sums of a
// column are first added in fp32, smallest first: one more rounding of the block sum's size,
// the same order as the block's own fp32 accumulation.  (A float64 running sum did the same,
// but the fp32 -> fp64 conversions run on a quarter-rate unit and paced the kernel.)  The
// partial (hi + lo in float64) of each K split goes to the workspace; a finalize kernel sums
// the splits.  With
// the long reductions here (thousands of tokens), plain fp32 accumulation leaves errors far
// above the elementwise absolute floor at outputs that cancel to near zero; this keeps the
// error at the level of one fp32 rounding per 64-wide block.
#pragma once

#include "nf4_device.cuh"

namespace qnf4 {

struct LowRankParams {
  CUtensorMap a_map;      // A operand (K-major: rows x k, or MN-major: k x rows)
  CUtensorMap b_map[3];   // B operand terms, each K-major [cols][k]
  int32_t a_mn;           // A operand is MN-major (two 64-row boxes per k-block)
  int32_t kblocks, k16_last;
  int32_t splits, kb_per_split;
  int32_t rows, cols;     // valid extent: rows on the UMMA M side, cols = rank columns
  double* partial;        // [splits][cols][rows] float64
};

// Warps: 0 and 6 issue TMA loads (alternate k-blocks), 1 issues MMAs, 2-5 and 7-10 flush to
// float64 (two groups, each draining half of the columns).
constexpr int kLrThreads = 352;
// The accumulator hand-offs between the MMA issuer and the flush warps poll without a
// suspend hint: each k-block crosses them twice, and a suspended waiter wakes late.
constexpr bool kLrSpin = true;

template <int BJ, int TERMS>
struct LrCfg {
  static constexpr int BN = BJ * TERMS;            // UMMA N
  static constexpr int kABytes = 128 * 64 * 2;
  static constexpr int kBTermBytes = BJ * 64 * 2;
  static constexpr int kBBytes = TERMS * kBTermBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStagesRaw = (200 * 1024) / kStageBytes;
  static constexpr int kStages = (kStagesRaw > 8 ? 8 : kStagesRaw) & ~1;   // even: two TMA warps own alternate stages
  // Accumulator buffers in TMEM: the MMA of k-block it writes buffer it % kBufs while the
  // flush warps drain older ones; four where they fit in the 512 columns, else two.
  static constexpr int kBufs = (4 * BN <= 512) ? 4 : 2;
  static constexpr int kTmemCols = (kBufs * BN <= 32) ? 32 : (kBufs * BN <= 64) ? 64 : (kBufs * BN <= 128) ? 128
                                   : (kBufs * BN <= 256) ? 256 : 512;
  static constexpr int kSmemBytes = kStages * kStageBytes + 256 + 1024;
  static_assert(BN % 16 == 0 && BN <= 256, "UMMA N");
  static_assert(kBTermBytes % 1024 == 0, "term boxes keep the swizzle atom alignment");
};

__device__ __forceinline__ void tmem_ld_32x32b_x16_lr(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// One 64-deep k-block into a fresh accumulator: four unrolled 16-deep MMAs whose
// descriptors differ only in the start address field.
template <int BN, bool A_MN>
__device__ __forceinline__ void lr_kblock(uint32_t d, uint32_t a_addr, uint32_t b_addr) {
  constexpr uint32_t idesc = umma_idesc_bf16(128, BN, A_MN ? 1u : 0u, 0u);
  const uint64_t a0 = A_MN ? umma_sdesc_sw128(a_addr, 8192u, 1024u) : umma_sdesc_sw128(a_addr, 16u, 1024u);
  const uint64_t b0 = umma_sdesc_sw128(b_addr, 16u, 1024u);
#pragma unroll
  for (int k16 = 0; k16 < 4; ++k16) {
    const uint64_t ad = a0 + (uint64_t)((A_MN ? 2048u : 32u) * (uint32_t)k16 >> 4);
    const uint64_t bd = b0 + (uint64_t)(32u * (uint32_t)k16 >> 4);
    umma_bf16(d, ad, bd, idesc, k16 > 0 ? 1u : 0u);
  }
}

// Two fp32 lanes as one register pair, for the sm_100 paired fp32 instructions (each lane is
// rounded to nearest exactly as the scalar instruction would round it).
__device__ __forceinline__ uint64_t pair_of(uint32_t lo_bits, uint32_t hi_bits) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo_bits), "r"(hi_bits));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// (hi, lo) += v for both lanes: s = hi + v and its exact error e (the two-sum: e = (hi - (s -
// b)) + (v - b) with b = s - hi, exact in round-to-nearest without overflow), then hi = s and
// lo = lo + e.  hi + lo carries about 48 significant bits over the whole reduction.
__device__ __forceinline__ void two_sum_acc(uint64_t& hi, uint64_t& lo, uint64_t v) {
  const uint64_t s = f2_add(hi, v);
  const uint64_t b = f2_sub(s, hi);
  const uint64_t e = f2_add(f2_sub(hi, f2_sub(s, b)), f2_sub(v, b));
  hi = s;
  lo = f2_add(lo, e);
}

template <int BJ, int TERMS>
__global__ void __launch_bounds__(kLrThreads, 1) lowrank_kernel(const __grid_constant__ LowRankParams p) {
  using C = LrCfg<BJ, TERMS>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* empty = full + S;
  constexpr int NB = C::kBufs;
  uint64_t* accfull = empty + S;      // [NB]
  uint64_t* accempty = accfull + NB;  // [NB]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + NB);
  volatile uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * 128, col0 = blockIdx.y * BJ, split = blockIdx.z;
  const int kb_begin = split * p.kb_per_split;
  int kb_end = kb_begin + p.kb_per_split;
  if (kb_end > p.kblocks) kb_end = p.kblocks;
  const int n_iters = kb_end > kb_begin ? kb_end - kb_begin : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 8);
    }
    *abort_word = 0u;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.a_map);
    for (int t = 0; t < TERMS; ++t) tma_prefetch_desc(&p.b_map[t]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------------ TMA
    // A bulk-tensor load holds its issuing thread for a few hundred cycles whatever its size,
    // while loads of different warps, and of different lanes of one instruction, proceed side
    // by side: two warps take alternate k-blocks, and each k-block's boxes (A, or two halves
    // of an MN-major A, then one per B term) go out as one instruction from lanes 0..4.
    const int tw = (warp == 0) ? 0 : 1;
    int last_issue[8];
    for (int s = 0; s < 8; ++s) last_issue[s] = -1;
    bool ok = true;
    for (int it = tw; it < n_iters; it += 2) {
      const int s = it % S;
      const uint32_t ph = (uint32_t)(it / S) & 1u;
      if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, kErrWaitEmpty)) { ok = false; break; }
      uint8_t* A = smem + s * C::kStageBytes;
      uint8_t* B = A + C::kABytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], C::kABytes + C::kBBytes);
        last_issue[s] = it;
      }
      __syncwarp();
      const int k = (kb_begin + it) * 64;
      const int na = p.a_mn ? 2 : 1;
      const CUtensorMap* map = nullptr;
      uint8_t* dst = nullptr;
      int cx = 0, cy = 0;
      if (lane < na) {
        map = &p.a_map;
        if (p.a_mn) { dst = A + lane * 8192; cx = row0 + 64 * lane; cy = k; }
        else { dst = A; cx = k; cy = row0; }
      } else if (lane < na + TERMS) {
        const int t = lane - na;
        map = &p.b_map[t]; dst = B + t * C::kBTermBytes; cx = k; cy = col0;
      }
      if (map) tma_load_2d(dst, map, cx, cy, &full[s]);
      __syncwarp();
    }
    if (!ok && lane == 0) {
      for (int s = 0; s < S; ++s)
        if (last_issue[s] >= 0) {
          const uint32_t ph = (uint32_t)(last_issue[s] / S) & 1u;
          for (int i = 0; i < (1 << 20) && !mbar_try_wait(&full[s], ph); ++i) {}
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    // Lane 0 alone: the tensor pipe queues only about one MMA ahead, so the issuer keeps
    // warp-collective instructions out of its loop and issues each k-block unrolled.
    if (lane == 0) {
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % S;
        const uint32_t ph = (uint32_t)(it / S) & 1u;
        const int buf = it % NB;
        const uint32_t bph = (uint32_t)(it / NB) & 1u;
        if (!mbar_wait_thread<false, kLrSpin>(&accempty[buf], bph ^ 1u, abort_word, kErrWaitMma)) break;
        if (!mbar_wait_thread(&full[s], ph, abort_word, kErrWaitTma)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * C::kStageBytes);
        const uint32_t b_addr = a_addr + C::kABytes;
        const uint32_t d = tmem_base + (uint32_t)(buf * C::BN);
        if (kb_begin + it != p.kblocks - 1 || p.k16_last == 4) {
          if (p.a_mn) lr_kblock<C::BN, true>(d, a_addr, b_addr);
          else lr_kblock<C::BN, false>(d, a_addr, b_addr);
        } else {
          const uint32_t idesc = umma_idesc_bf16(128, C::BN, p.a_mn ? 1u : 0u, 0u);
          for (int k16 = 0; k16 < p.k16_last; ++k16) {
            const uint64_t ad = p.a_mn ? umma_sdesc_sw128(a_addr + (uint32_t)k16 * 2048u, 8192u, 1024u)
                                       : umma_sdesc_sw128(a_addr + (uint32_t)k16 * 32u, 16u, 1024u);
            const uint64_t bd = umma_sdesc_sw128(b_addr + (uint32_t)k16 * 32u, 16u, 1024u);
            umma_bf16(d, ad, bd, idesc, k16 > 0 ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
        umma_commit(&accfull[buf]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ flush to float64
    // Group g (warps 2-5, then 7-10) drains columns [g * HALF, (g + 1) * HALF) of each
    // k-block's accumulator; warp w reads TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31.  With
    // BJ = 16 the second group only keeps the hand-off count.
    constexpr int HALF = BJ >= 32 ? BJ / 2 : BJ;
    const int c0 = (warp >= 7) ? HALF : 0;
    const bool active = c0 < BJ;
    const int q = warp & 3;
    const int row = row0 + 32 * q + lane;
    // running sums of columns (2i, 2i + 1) as paired fp32 hi and lo parts
    uint64_t hi[HALF / 2], lo[HALF / 2];
#pragma unroll
    for (int j = 0; j < HALF / 2; ++j) hi[j] = lo[j] = 0ull;
    bool ok = true;
    for (int it = 0; it < n_iters; ++it) {
      const int buf = it % NB;
      const uint32_t bph = (uint32_t)(it / NB) & 1u;
      if (!mbar_wait<false, kLrSpin>(&accfull[buf], bph, abort_word, kErrWaitMma)) { ok = false; break; }
      tc_fence_after();
      if (active) {
        const uint32_t tb = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * C::BN + c0);
#pragma unroll
        for (int j0 = 0; j0 < HALF; j0 += 16) {
          uint32_t r[TERMS][16];
#pragma unroll
          for (int t = 0; t < TERMS; ++t) tmem_ld_32x32b_x16_lr(tb + (uint32_t)(t * BJ + j0), r[t]);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            uint64_t v = pair_of(r[0][j], r[0][j + 1]);
            if constexpr (TERMS == 3) v = f2_add(v, f2_add(pair_of(r[2][j], r[2][j + 1]), pair_of(r[1][j], r[1][j + 1])));
            two_sum_acc(hi[(j0 + j) / 2], lo[(j0 + j) / 2], v);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[buf]);
    }
    if (ok && active && row < p.rows) {
      double* out = p.partial + (int64_t)split * p.cols * p.rows;
#pragma unroll
      for (int j = 0; j < HALF; ++j) {
        const int col = col0 + c0 + j;
        const uint64_t h = hi[j / 2], l = lo[j / 2];
        const float hj = __uint_as_float((uint32_t)(j & 1 ? h >> 32 : h));
        const float lj = __uint_as_float((uint32_t)(j & 1 ? l >> 32 : l));
        if (col < p.cols) out[(int64_t)col * p.rows + row] = (double)hj + (double)lj;
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BJ, int TERMS>
static cudaError_t launch_lowrank_t(const LowRankParams& p, cudaStream_t st) {
  using C = LrCfg<BJ, TERMS>;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = enable_smem_once(lowrank_kernel<BJ, TERMS>, C::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  dim3 grid((p.rows + 127) / 128, (p.cols + BJ - 1) / BJ, p.splits);
  lowrank_kernel<BJ, TERMS><<<grid, kLrThreads, C::kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

// bj in {16, 32, 64}, terms in {1, 3}
static cudaError_t launch_lowrank(const LowRankParams& p, int bj, int terms, cudaStream_t st) {
  if (terms == 1) {
    if (bj == 16) return launch_lowrank_t<16, 1>(p, st);
    if (bj == 32) return launch_lowrank_t<32, 1>(p, st);
    if (bj == 64) return launch_lowrank_t<64, 1>(p, st);
  } else if (terms == 3) {
    if (bj == 16) return launch_lowrank_t<16, 3>(p, st);
    if (bj == 32) return launch_lowrank_t<32, 3>(p, st);
    if (bj == 64) return launch_lowrank_t<64, 3>(p, st);
  }
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------------------
// finalize kernels
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint16_t bf16_bits_rn(double v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn((float)v));
}

// Three bf16 terms of v: t1 = bf16(v), t2 = bf16(v - t1), t3 = bf16(v - t1 - t2), each
// difference formed in float64.  For an fp32 v the three terms are exact (8 + 8 + 8 bits).
__device__ __forceinline__ void split3(double v, uint16_t& a, uint16_t& b, uint16_t& c) {
  const __nv_bfloat16 h1 = __float2bfloat16_rn((float)v);
  const double r1 = v - (double)__bfloat162float(h1);
  const __nv_bfloat16 h2 = __float2bfloat16_rn((float)r1);
  const double r2 = r1 - (double)__bfloat162float(h2);
  a = __bfloat16_as_ushort(h1);
  b = __bfloat16_as_ushort(h2);
  c = __bfloat16_as_ushort(__float2bfloat16_rn((float)r2));
}

// sum_z p[z * stride] for z = 0 .. splits-1, added in that order; the loads of up to eight
// splits are issued before their sum, so the splits' memory latencies overlap.
__device__ __forceinline__ double sum_splits(const double* __restrict__ p, int splits, int64_t stride) {
  double v = 0.0;
  for (int z0 = 0; z0 < splits; z0 += 8) {
    double x[8];
#pragma unroll
    for (int z = 0; z < 8; ++z) x[z] = (z0 + z < splits) ? p[(int64_t)(z0 + z) * stride] : 0.0;
#pragma unroll
    for (int z = 0; z < 8; ++z)
      if (z0 + z < splits) v += x[z];
  }
  return v;
}

// Token-side result (t or u): v = alpha * sum_z partial[z][j][m].  Optional outputs:
// fp32 [M][r]; bf16 hi / lo [M][r] (two-term split, for the fused GEMMs' adapter k-blocks);
// the three-term split transposed, T3[term][j][m] with row pitch ldT (for dA / dB).
// One 32 x 32 tile (m0.., j0..) per block of 32 x 8 threads: the partials are read along m,
// the [M][r] outputs written along j through a shared-memory transpose.
__global__ void finalize_tokens_kernel(const double* __restrict__ partial, int splits, int64_t M, int64_t r,
                                       double alpha, float* __restrict__ f32, uint16_t* __restrict__ hi,
                                       uint16_t* __restrict__ lo, uint16_t* __restrict__ T3, int64_t ldT) {
  __shared__ double tile[32][33];
  const int64_t m0 = (int64_t)blockIdx.x * 32, j0 = (int64_t)blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t j = j0 + i, m = m0 + threadIdx.x;
    double v = 0.0;
    if (m < M && j < r) {
      v = sum_splits(partial + j * M + m, splits, r * M);
      v *= alpha;
      if (T3) {
        uint16_t a, b, c;
        split3(v, a, b, c);
        T3[j * ldT + m] = a;
        T3[(r + j) * ldT + m] = b;
        T3[(2 * r + j) * ldT + m] = c;
      }
    }
    tile[i][threadIdx.x] = v;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t m = m0 + i, j = j0 + threadIdx.x;
    if (m >= M || j >= r) continue;
    const double v = tile[threadIdx.x][i];
    if (f32) f32[m * r + j] = (float)v;
    if (hi) {
      const __nv_bfloat16 h = __float2bfloat16_rn((float)v);
      hi[m * r + j] = __bfloat16_as_ushort(h);
      lo[m * r + j] = bf16_bits_rn(v - (double)__bfloat162float(h));
    }
  }
}

// fp32 t [M][r] -> exact three-term split, transposed: T3[term][j][m].
__global__ void split3_T_kernel(const float* __restrict__ t, int64_t M, int64_t r, uint16_t* __restrict__ T3,
                                int64_t ldT) {
  __shared__ float tile[32][33];
  const int64_t m0 = (int64_t)blockIdx.y * 32, j0 = (int64_t)blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t m = m0 + i, j = j0 + threadIdx.x;
    tile[i][threadIdx.x] = (m < M && j < r) ? t[m * r + j] : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t j = j0 + i, m = m0 + threadIdx.x;
    if (m < M && j < r) {
      uint16_t a, b, c;
      split3((double)tile[threadIdx.x][i], a, b, c);
      T3[j * ldT + m] = a;
      T3[(r + j) * ldT + m] = b;
      T3[(2 * r + j) * ldT + m] = c;
    }
  }
}

// Feature-side gradient: g[j][i] = bf16(sum_z partial[z][j][i]); transpose_out = 0 writes
// out[j * n + i] (dA, [r][K]), 1 writes out[i * r + j] (dB, [N][r]).  One 32 x 32 tile
// (i0.., j0..) per block of 32 x 8 threads; the transposed case goes through shared memory so
// that both the partials and the output are accessed along their rows.
__global__ void finalize_grad_kernel(const double* __restrict__ partial, int splits, int64_t r, int64_t n,
                                     uint16_t* __restrict__ out, int transpose_out) {
  __shared__ uint16_t tile[32][34];
  const int64_t i0 = (int64_t)blockIdx.x * 32, j0 = (int64_t)blockIdx.y * 32;
  for (int a = threadIdx.y; a < 32; a += blockDim.y) {
    const int64_t j = j0 + a, i = i0 + threadIdx.x;
    uint16_t g = 0;
    if (i < n && j < r) {
      const double v = sum_splits(partial + j * n + i, splits, r * n);
      g = bf16_bits_rn(v);
      if (!transpose_out) out[j * n + i] = g;
    }
    tile[a][threadIdx.x] = g;
  }
  if (!transpose_out) return;
  __syncthreads();
  for (int a = threadIdx.y; a < 32; a += blockDim.y) {
    const int64_t i = i0 + a, j = j0 + threadIdx.x;
    if (i < n && j < r) out[i * r + j] = tile[threadIdx.x][a];
  }
}

static cudaError_t launch_finalize_tokens(const double* partial, int splits, int64_t M, int64_t r, double alpha,
                                          float* f32, uint16_t* hi, uint16_t* lo, uint16_t* T3, int64_t ldT,
                                          cudaStream_t st) {
  dim3 grid((unsigned)((M + 31) / 32), (unsigned)((r + 31) / 32));
  finalize_tokens_kernel<<<grid, dim3(32, 8), 0, st>>>(partial, splits, M, r, alpha, f32, hi, lo, T3, ldT);
  return cudaGetLastError();
}

static cudaError_t launch_split3_T(const float* t, int64_t M, int64_t r, uint16_t* T3, int64_t ldT,
                                   cudaStream_t st) {
  dim3 grid((unsigned)((r + 31) / 32), (unsigned)((M + 31) / 32));
  split3_T_kernel<<<grid, dim3(32, 8), 0, st>>>(t, M, r, T3, ldT);
  return cudaGetLastError();
}

static cudaError_t launch_finalize_grad(const double* partial, int splits, int64_t r, int64_t n, uint16_t* out,
                                        int transpose_out, cudaStream_t st) {
  dim3 grid((unsigned)((n + 31) / 32), (unsigned)((r + 31) / 32));
  finalize_grad_kernel<<<grid, dim3(32, 8), 0, st>>>(partial, splits, r, n, out, transpose_out);
  return cudaGetLastError();
}

}  // namespace qnf4
