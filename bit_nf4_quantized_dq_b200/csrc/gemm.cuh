// tcgen05 GEMM engine with an on-chip NF4 -> bf16 dequant producer.
//
// D[rows x cols] (fp32, in TMEM) = sum over K-loop stretches of A[rows x k] * B[cols x k]^T.
// The 128-row A side is either loaded by TMA or produced on chip from packed NF4 codes; the
// dequantized 16-bit weights exist only in shared memory or, with A_TMEM, in tensor memory,
// never in HBM.  The B side is a K-major bf16 tile loaded by TMA.  Lane 0 of warp 1 issues
// tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) into the TMEM accumulator.
//
// The method's forward and backward ("QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double
// Quantization, and Paged Optimizers" (fullstackaihub), section 4) use this engine for
//   y^T  = W' x^T + B t^T            (rows = out features, cols = tokens)
//   dX^T = W'^T dY^T + A^T u^T       (rows = in features,  cols = tokens)
// with the fp32 t = s x A^T and u = s dY B (computed in lowrank.cuh) split into bf16 hi + lo
// parts, run as extra k-blocks of the same accumulator, so that the adapter terms keep close
// to fp32 accuracy through bf16 tensor-core inputs.
//
// The kernel is persistent: one CTA per SM walks the tiles blockIdx.x, blockIdx.x + gridDim.x,
// ... (row tiles fastest).  Ring stages and their phases are counted over the CTA's whole
// sequence of k-blocks, so the loads and the dequant production of the next tile proceed
// while the current one finishes.  Warp roles: warps 0 and 10 issue the TMA loads of
// alternate k-blocks, warp 1 allocates TMEM and (lane 0) issues the MMAs, warps 2-9 run the
// dequant producer (two groups of four warps on alternate k-blocks), warps 11.. drain the
// accumulator (the epilogue).  With A in shared memory the accumulator is double-buffered in
// TMEM, so a tile's epilogue overlaps the next tile's MMAs; with A in TMEM (which then holds
// the A slots beside one accumulator) eight epilogue warps drain it, and the next tile's
// MMAs start once they are done.  Per stage s:
//   full[s]   the B tile (and a TMA-loaded A tile) has landed;
//   cfull[s]  the codes have landed (shared-memory A), or a plain arrive: producers may start;
//   prod[s]   the producers wrote the A tile, after they also saw full[s];
//   empty[s]  the MMAs that read stage s completed (tcgen05.commit);
// per accumulator buffer b: accfull[b] (its MMAs completed), accempty[b] (drained).
#pragma once

#include "nf4_device.cuh"
#include "gemm.h"

namespace qnf4 {

constexpr int kBM = 128;
constexpr int kBK = 64;
// A bulk-tensor load holds the thread that issues it for a few hundred cycles, whatever the box
// size, while loads from different warps proceed side by side: kTmaWarps warps share the loads,
// warp w (warp 0, then warp 10) taking the k-blocks whose global index i has i % kTmaWarps == w.
constexpr int kTmaWarps = 2;
constexpr int kEpiWarp0 = 11;       // first epilogue warp
constexpr int kCodesBytes = 4096;   // packed codes of one 128 x 64 weight tile

// A_TMEM: the A tile lives in tensor memory (slot s at column kATmemCol0 + 32 s), so a stage
// holds only B and the codes and more stages fit.
constexpr uint32_t kATmemCol0 = 256;

template <int BN, bool A_TMEM = false>
struct Cfg {
  static constexpr int kABytes = A_TMEM ? 0 : kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes + kCodesBytes;
  static constexpr int kStagesRaw = (220 * 1024 - 2048) / kStageBytes;
  // Even: the two producer groups take alternate k-blocks, so each group must own whole
  // stages and wait on every phase of their barriers (a parity wait that skips a phase can
  // pass early).
  static constexpr int kStages = (kStagesRaw > 8 ? 8 : kStagesRaw) & ~1;
  // Accumulator buffers: two when TMEM has room (A in shared memory), else one.
  static constexpr int kAccBufs = A_TMEM ? 1 : 2;
  static constexpr int kEpiWarps = A_TMEM ? 8 : 4;
  static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
  // accumulator buffer b starts at TMEM column b * kAccStride (at least 32 columns apart)
  static constexpr int kAccStride = BN < 32 ? 32 : BN;
  static constexpr int kTmemCols = A_TMEM ? 512 : 2 * kAccStride;
  static_assert(!A_TMEM || (BN == 256 && kStages <= 8), "A in TMEM: 256-column accumulator + 8 slots of 32 columns");
  static constexpr int kBarrierBytes = 512;
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;
  static_assert(kStages >= 2 && kStages % 2 == 0, "pipeline too shallow, or odd");
  static_assert(kStages % kTmaWarps == 0, "each TMA warp must own whole stages");
  static_assert(kBBytes % 1024 == 0, "B tile must keep 1024-byte alignment");
  static_assert(4 * kStages * 8 + 5 * 8 + 8 <= kBarrierBytes, "barrier area");
};

struct IterPos {
  int seg;
  int kb;    // k-block within the stretch
  bool last; // last k-block of the stretch
};

// Stretch/k-block of iteration `it` for this CTA: segment 0 restricted to [kb_begin, kb_end),
// then (split 0 only) every later segment in full.
__device__ __forceinline__ IterPos iter_pos(const GemmParams& p, int it, int kb_begin, int kb_end, bool first_split) {
  const int n0 = kb_end - kb_begin;
  if (it < n0) return IterPos{0, kb_begin + it, kb_begin + it == p.seg[0].kblocks - 1};
  int rem = it - n0;
  for (int s = 1; s < p.nseg; ++s) {
    if (rem < p.seg[s].kblocks) return IterPos{s, rem, rem == p.seg[s].kblocks - 1};
    rem -= p.seg[s].kblocks;
  }
  return IterPos{0, 0, false};
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// ---------------------------------------------------------------------------------------
// the dequant producer: one 64-weight unit per thread per k-block
// ---------------------------------------------------------------------------------------
// A unit is one (W row n, 64 consecutive W columns) stretch.  It becomes one 128-byte row of
// the A tile: row t of a K-major tile (forward), or row n_local of MN-major chunk `half`
// (dX).  16-byte chunk j of the row lands at chunk j ^ (row & 7) (128-byte swizzle).
struct UnitGeom {
  int64_t n;      // W row
  int64_t kcol;   // first W column of the unit
  uint32_t dst;   // byte offset of the unit's 128-byte row inside the A tile
  uint32_t swz;   // row & 7
  uint32_t coff;  // byte offset of the unit's 32 code bytes inside the stage's codes tile
};

__device__ __forceinline__ UnitGeom unit_geom(int a_src, int t, int row0, int64_t k) {
  UnitGeom u;
  if (a_src == kANf4K) {            // forward: rows of W, k-block k of its columns
    u.n = row0 + t;
    u.kcol = k;
    u.dst = (uint32_t)t * 128u;
    u.swz = (uint32_t)t & 7u;
    u.coff = (uint32_t)t * 32u;     // codes tile [128 W rows][32 bytes]
  } else {                          // dX: columns row0.. of W, k-block k of its rows
    // Thread t = 8 g + l takes W row nl = 8 (g / 2) + l and column half ((l / 2) & 1) ^ (g & 1):
    // every 8 lanes then write 8 different rows (their swizzled 16-byte chunks never share a
    // bank), and their code loads (codes tile [64 W rows][64 bytes]) meet at most 2-way.
    const int g = t >> 3, l = t & 7;
    const int nl = 8 * (g >> 1) + l, half = ((l >> 1) & 1) ^ (g & 1);
    u.n = k + nl;
    u.kcol = (int64_t)row0 + 64 * half;
    u.dst = (uint32_t)half * 8192u + (uint32_t)nl * 128u;
    u.swz = (uint32_t)nl & 7u;
    u.coff = (uint32_t)nl * 64u + (uint32_t)half * 32u;
  }
  return u;
}

// Per-unit block scales, fetched (and formed) one iteration ahead of their use.
struct UnitScale {
  float s0, s1;      // scale of the unit's block and (generic path) of the next block
  int32_t split;     // words before the block boundary (8 = one block), generic path only
  int32_t valid;     // valid 8-code words (0 = unit outside the weight)
};

__device__ __forceinline__ float block_scale_of(const GemmParams& p, int64_t blk, float mean) {
  if (p.scale_fp32) return __ldg(p.c2 + blk);
  return dq_block_scale(__ldg(p.scale_codes + blk), __ldg(p.c2 + (blk >> 8)), mean);
}

template <bool GENERIC>
__device__ __forceinline__ UnitScale fetch_scale(const GemmParams& p, const UnitGeom& u, int64_t nb, float mean) {
  UnitScale r{0.0f, 0.0f, 8, 0};
  if (u.n >= p.nw || u.kcol >= p.kw) return r;
  const int64_t f0 = u.n * p.kw + u.kcol;
  const int64_t blk = f0 >> 6;
  r.s0 = block_scale_of(p, blk, mean);
  r.valid = 8;
  if constexpr (GENERIC) {
    r.split = (int32_t)((64 - (f0 & 63)) >> 3);
    if (r.split < 8 && blk + 1 < nb) r.s1 = block_scale_of(p, blk + 1, mean);
    const int64_t vw = (p.kw - u.kcol) >> 3;
    r.valid = (int32_t)(vw < 8 ? vw : 8);
  }
  return r;
}

// tcgen05.mma with the A operand in tensor memory (kind::f16, bf16 x bf16 -> fp32): row i of A
// is TMEM lane i, two consecutive K elements per 32-bit column.
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive 32-bit columns of this warp's 32 TMEM lanes (one lane per thread).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// One k-block with A in TMEM: four 16-deep MMAs, A advancing 8 columns per slice.
template <int BN>
__device__ __forceinline__ void umma_kblock_ts(uint32_t tmem_acc, uint32_t a_tmem, uint32_t b_addr, uint32_t acc,
                                               int nk16) {
  constexpr uint32_t idesc = umma_idesc_bf16(kBM, BN, 0u, 0u);
  const uint64_t b0 = umma_sdesc_sw128(b_addr, 16u, 1024u);
  if (nk16 == 4) {
#pragma unroll
    for (int k16 = 0; k16 < 4; ++k16)
      umma_bf16_ts(tmem_acc, a_tmem + 8u * (uint32_t)k16, b0 + (uint64_t)(32u * (uint32_t)k16 >> 4), idesc,
                   k16 == 0 ? acc : 1u);
  } else {
    for (int k16 = 0; k16 < nk16; ++k16)
      umma_bf16_ts(tmem_acc, a_tmem + 8u * (uint32_t)k16, b0 + (uint64_t)(32u * (uint32_t)k16 >> 4), idesc,
                   (acc || k16 > 0) ? 1u : 0u);
  }
}

// One k-block (64 deep) of MMAs: four 16-deep tcgen05.mma into the accumulator.  The
// descriptors of consecutive 16-deep slices differ only in their start address (bits 0-13,
// 16-byte units): 32 bytes along a K-major row, 2048 bytes (16 K rows of 128 bytes) down an
// MN-major chunk.  Start addresses stay below 2^18, so the field never carries.
template <int BN, bool A_MN>
__device__ __forceinline__ void umma_kblock(uint32_t tmem_acc, uint32_t a_addr, uint32_t b_addr, uint32_t acc) {
  constexpr uint32_t idesc = umma_idesc_bf16(kBM, BN, A_MN ? 1u : 0u, 0u);
  const uint64_t a0 = A_MN ? umma_sdesc_sw128(a_addr, 8192u, 1024u) : umma_sdesc_sw128(a_addr, 16u, 1024u);
  const uint64_t b0 = umma_sdesc_sw128(b_addr, 16u, 1024u);
#pragma unroll
  for (int k16 = 0; k16 < 4; ++k16) {
    const uint64_t ad = a0 + (uint64_t)((A_MN ? 2048u : 32u) * (uint32_t)k16 >> 4);
    const uint64_t bd = b0 + (uint64_t)(32u * (uint32_t)k16 >> 4);
    umma_bf16(tmem_acc, ad, bd, idesc, k16 == 0 ? acc : 1u);
  }
}

// The last k-block of a stretch whose depth is not a multiple of 64: nk16 < 4 slices.
template <int BN>
__device__ __noinline__ void umma_kblock_ragged(uint32_t tmem_acc, uint32_t a_addr, uint32_t b_addr, uint32_t acc,
                                                bool a_mn, int nk16) {
  const uint32_t idesc = umma_idesc_bf16(kBM, BN, a_mn ? 1u : 0u, 0u);
  for (int k16 = 0; k16 < nk16; ++k16) {
    const uint64_t ad = a_mn ? umma_sdesc_sw128(a_addr + (uint32_t)k16 * 2048u, 8192u, 1024u)
                             : umma_sdesc_sw128(a_addr + (uint32_t)k16 * 32u, 16u, 1024u);
    const uint64_t bd = umma_sdesc_sw128(b_addr + (uint32_t)k16 * 32u, 16u, 1024u);
    umma_bf16(tmem_acc, ad, bd, idesc, (acc || k16 > 0) ? 1u : 0u);
  }
}

// One tile of the persistent schedule: tile t -> (row tile, column tile, K split), row tiles
// fastest; its k-block range of segment 0 and its number of k-blocks (later segments run in
// split 0 only).
struct TileInfo {
  int row0, col0, split, kb_begin, kb_end, n_iters;
};

template <int BN>
__device__ __forceinline__ TileInfo tile_info(const GemmParams& p, int tiles_m, int tiles_n, int64_t t) {
  TileInfo ti;
  const int64_t per_split = (int64_t)tiles_m * tiles_n;
  ti.split = (int)(t / per_split);
  const int64_t rem = t - (int64_t)ti.split * per_split;
  ti.row0 = (int)(rem % tiles_m) * kBM;
  ti.col0 = (int)(rem / tiles_m) * BN;
  ti.kb_begin = ti.split * p.kb_per_split;
  ti.kb_end = ti.kb_begin + p.kb_per_split;
  if (ti.kb_end > p.seg[0].kblocks) ti.kb_end = p.seg[0].kblocks;
  ti.n_iters = ti.kb_end - ti.kb_begin;
  if (ti.split == 0)
    for (int s = 1; s < p.nseg; ++s) ti.n_iters += p.seg[s].kblocks;
  return ti;
}

// Walks this CTA's k-blocks (tile by tile) in steps of 1 or 2 from `first`; stage and phase
// are the ring position of the current k-block, counted over the CTA's whole sequence (32-bit
// and incremental: they sit on the issuing threads' critical path).
template <int BN, int S>
struct KIter {
  int tiles_m, tiles_n;
  int64_t ntiles, t;
  TileInfo ti;
  int it;
  int stage;
  uint32_t phase;
  bool done;

  __device__ __forceinline__ void init(const GemmParams& p, int first) {
    tiles_m = (p.rows + kBM - 1) / kBM;
    tiles_n = (p.cols + BN - 1) / BN;
    ntiles = (int64_t)tiles_m * tiles_n * p.splits;
    t = blockIdx.x;
    done = t >= ntiles;
    it = 0;
    stage = 0;
    phase = 0u;
    if (!done) ti = tile_info<BN>(p, tiles_m, tiles_n, t);
    advance(p, first);
  }
  __device__ __forceinline__ void advance(const GemmParams& p, int k) {
    it += k;
    stage += k;
    if (stage >= S) {
      stage -= S;
      phase ^= 1u;
    }
    while (!done && it >= ti.n_iters) {
      it -= ti.n_iters;
      t += gridDim.x;
      if (t >= ntiles) {
        done = true;
      } else {
        ti = tile_info<BN>(p, tiles_m, tiles_n, t);
      }
    }
  }
};

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// TMA tile load with an L2 cache-eviction hint (no multicast).
__device__ __forceinline__ void tma_load_2d_hint(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, "
      "{%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// In-warp transpose of 8 x 8 bf16 values within each group of 8 lanes: on entry lane j holds
// elements (j, 0..7) as four packed pairs x0..x3, on exit elements (0..7, j).  Three exchange
// stages swap the off-diagonal blocks of 4, 2 and 1 elements with the lane at xor distance
// 4, 2 and 1.
__device__ __forceinline__ void transpose8x8_bf16(uint32_t& x0, uint32_t& x1, uint32_t& x2, uint32_t& x3, int lane) {
  const bool b2 = lane & 4, b1 = lane & 2, b0 = lane & 1;
  {
    const uint32_t s0 = b2 ? x0 : x2, s1 = b2 ? x1 : x3;
    const uint32_t r0 = __shfl_xor_sync(0xFFFFFFFFu, s0, 4), r1 = __shfl_xor_sync(0xFFFFFFFFu, s1, 4);
    if (b2) { x0 = r0; x1 = r1; } else { x2 = r0; x3 = r1; }
  }
  {
    const uint32_t s0 = b1 ? x0 : x1, s1 = b1 ? x2 : x3;
    const uint32_t r0 = __shfl_xor_sync(0xFFFFFFFFu, s0, 2), r1 = __shfl_xor_sync(0xFFFFFFFFu, s1, 2);
    if (b1) { x0 = r0; x2 = r1; } else { x1 = r0; x3 = r1; }
  }
  uint32_t* x[4] = {&x0, &x1, &x2, &x3};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t v = *x[k];
    const uint32_t send = b0 ? (v & 0xFFFFu) : (v >> 16);
    const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
    *x[k] = b0 ? ((v & 0xFFFF0000u) | recv) : ((v & 0xFFFFu) | (recv << 16));
  }
}

// The MMA issuer's inner loop over `count` k-blocks of one stretch (one A layout).  The tensor
// pipe queues only about one MMA ahead of the issuing thread, so the time this thread spends
// between two k-blocks is pipe idle time: the ready barrier is polled inline (the bounded
// wait only when the phase is not complete yet), ring positions and descriptors come from
// incremental 32-bit counters, and the last k-block of a stretch is ragged only when
// `k16_tail` < 4.  Returns false if a wait gave up.
template <int BN, bool A_TMEM, bool A_MN, int S>
__device__ __forceinline__ bool mma_run(int count, int k16_tail, uint64_t* ready, uint64_t* empty, uint32_t ready_err,
                                        volatile uint32_t* abort_word, uint32_t smem_base, uint32_t tmem_base,
                                        uint32_t tmem_acc, bool first, int& s, uint32_t& ph) {
  using C = Cfg<BN, A_TMEM>;
  for (int j = 0; j < count; ++j) {
    if (!mbar_try_wait(&ready[s], ph))
      if (!mbar_wait_thread(&ready[s], ph, abort_word, ready_err)) return false;
    tc_fence_after();
    const uint32_t a_addr = smem_base + (uint32_t)s * (uint32_t)C::kStageBytes;
    const uint32_t b_addr = a_addr + (uint32_t)C::kABytes;
    const uint32_t acc = (first && j == 0) ? 0u : 1u;
    const int nk16 = (j == count - 1) ? k16_tail : 4;
    if constexpr (A_TMEM) {
      umma_kblock_ts<BN>(tmem_acc, tmem_base + kATmemCol0 + 32u * (uint32_t)s, b_addr, acc, nk16);
    } else if (nk16 == 4) {
      umma_kblock<BN, A_MN>(tmem_acc, a_addr, b_addr, acc);
    } else {
      umma_kblock_ragged<BN>(tmem_acc, a_addr, b_addr, acc, A_MN, nk16);
    }
    umma_commit(&empty[s]);
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
  }
  return true;
}

template <int BN, bool GENERIC, bool A_TMEM>
__global__ void __launch_bounds__(Cfg<BN, A_TMEM>::kThreads, 1) qlora_gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<BN, A_TMEM>;
  constexpr int S = C::kStages;
  constexpr int NB = C::kAccBufs;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes);
  uint64_t* cfull = full + S;   // the stage's codes have landed (or a plain arrive): producers may start
  uint64_t* prod = cfull + S;
  uint64_t* empty = prod + S;
  uint64_t* accfull = empty + S;      // [2]
  uint64_t* accempty = accfull + 2;   // [2]
  uint64_t* mma_done = accempty + 2;  // the MMA thread's final commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&cfull[s], 1);
      mbar_init(&prod[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], C::kEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_word = 0u;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    for (int m = 0; m < kMaxMaps; ++m) tma_prefetch_desc(&p.maps[m]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto stage_a = [&](int s) { return smem + s * C::kStageBytes; };
  auto stage_b = [&](int s) { return smem + s * C::kStageBytes + C::kABytes; };
  auto stage_c = [&](int s) { return smem + s * C::kStageBytes + C::kABytes + C::kBBytes; };

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------------ TMA producers
    const int tw = (warp == 0) ? 0 : 1;
    const uint64_t codes_policy = l2_policy_evict_last();   // the codes are re-read by every column tile
    int last_issue[8];            // phase of the last load issued into each stage (-1: none)
    for (int s = 0; s < 8; ++s) last_issue[s] = -1;
    bool ok = true;
    KIter<BN, S> ki;
    ki.init(p, tw);
    for (; !ki.done; ki.advance(p, kTmaWarps)) {
      const int s = ki.stage;
      const uint32_t ph = ki.phase;
      if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, kErrWaitEmpty)) { ok = false; break; }
      const IterPos ip = iter_pos(p, ki.it, ki.ti.kb_begin, ki.ti.kb_end, ki.ti.split == 0);
      const GemmSeg& sg = p.seg[ip.seg];
      const bool nf4 = (sg.a_src == kANf4K || sg.a_src == kANf4MN);
      if (lane == 0) {
        // With A in shared memory the codes complete on cfull[s], so the producers can
        // dequantize while the (larger) B tile is still landing on full[s].  With A in tensor
        // memory the codes complete on full[s].
        const bool codes_tma = nf4 && !GENERIC;
        mbar_arrive_expect_tx(&full[s], C::kBBytes + (nf4 ? 0u : (uint32_t)C::kABytes) +
                                            ((A_TMEM && codes_tma) ? (uint32_t)kCodesBytes : 0u));
        if (!A_TMEM && codes_tma) mbar_arrive_expect_tx(&cfull[s], kCodesBytes);
        else mbar_arrive(&cfull[s]);
        last_issue[s] = (int)ph;
      }
      __syncwarp();
      // Lanes 0..2 each take one load and issue them as a single instruction: lane 0 the B
      // tile, lanes 1 and 2 the A side.
      const int row0 = ki.ti.row0, col0 = ki.ti.col0;
      const int k = sg.a_k0 + ip.kb * kBK;
      int map = -1, cx = 0, cy = 0;
      bool codes = false;
      uint8_t* dst = nullptr;
      uint64_t* bar = &full[s];
      if (lane == 0) {
        map = sg.b_map; dst = stage_b(s); cx = sg.b_k0 + ip.kb * kBK; cy = col0;
      } else if (lane == 1) {
        if (sg.a_src == kANf4K) {
          if (!GENERIC) { map = sg.a_map; dst = stage_c(s); cx = k / 2; cy = row0; bar = A_TMEM ? &full[s] : &cfull[s]; codes = true; }
        } else if (sg.a_src == kANf4MN) {
          if (!GENERIC) { map = sg.a_map; dst = stage_c(s); cx = row0 / 2; cy = k; bar = A_TMEM ? &full[s] : &cfull[s]; codes = true; }
        } else if (sg.a_src == kATmaK) {
          if (!A_TMEM) { map = sg.a_map; dst = stage_a(s); cx = k; cy = row0; }
        } else {
          map = sg.a_map; dst = stage_a(s); cx = row0; cy = k;
        }
      } else if (lane == 2 && sg.a_src == kATmaMN) {
        map = sg.a_map; dst = stage_a(s) + 8192; cx = row0 + 64; cy = k;
      }
      if (map >= 0) {
        if (codes) tma_load_2d_hint(dst, &p.maps[map], cx, cy, bar, codes_policy);
        else tma_load_2d(dst, &p.maps[map], cx, cy, bar);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      // drain copies still in flight before the CTA's shared memory goes away
      for (int s = 0; s < S; ++s)
        if (last_issue[s] >= 0) {
          const uint32_t ph = (uint32_t)last_issue[s];
          for (int i = 0; i < (1 << 20) && !mbar_try_wait(&full[s], ph); ++i) {}
          for (int i = 0; i < (1 << 20) && !mbar_try_wait(&cfull[s], ph); ++i) {}
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // Lane 0 alone runs this loop.  The tensor pipe queues only about one MMA ahead, so every
    // cycle the issuer spends between k-blocks shows up as pipe idle time: no warp-collective
    // instruction here, one barrier wait per k-block, and a fully unrolled MMA sequence.
    // The producers arrive on prod[s] only after they saw full[s] complete, so with a
    // producer present prod[s] alone orders the MMAs after both the TMA data and the
    // dequantized tile.
    if (lane == 0) {
      uint64_t* const ready = p.has_nf4 ? prod : full;
      const uint32_t ready_err = p.has_nf4 ? kErrWaitProducer : kErrWaitTma;
      const int tiles_m = (p.rows + kBM - 1) / kBM;
      const int tiles_n = (p.cols + BN - 1) / BN;
      const int64_t ntiles = (int64_t)tiles_m * tiles_n * p.splits;
      int s = 0;
      uint32_t ph = 0u;
      int64_t tc = 0;           // tiles started
      bool ok = true;
      for (int64_t tt = blockIdx.x; tt < ntiles && ok; tt += gridDim.x, ++tc) {
        const TileInfo ti = tile_info<BN>(p, tiles_m, tiles_n, tt);
        const int buf = (int)(tc % NB);
        const uint32_t use = (uint32_t)(tc / NB) & 1u;
        if (!mbar_wait_thread(&accempty[buf], use ^ 1u, abort_word, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tmem_acc = tmem_base + (uint32_t)(buf * C::kAccStride);
        const uint32_t smem_base = smem_u32(smem);
        // segment 0 over this tile's K range, then (split 0) the adapter stretches
        bool first = true;
        for (int sgi = 0; sgi < p.nseg && ok; ++sgi) {
          if (sgi > 0 && ti.split != 0) break;
          const GemmSeg sg = p.seg[sgi];
          const int count = sgi == 0 ? ti.kb_end - ti.kb_begin : sg.kblocks;
          if (count <= 0) continue;
          const bool ends = sgi > 0 || ti.kb_end == sg.kblocks;   // the stretch's last k-block is in this run
          const int k16_tail = ends ? sg.k16_last : 4;
          const bool a_mn = (sg.a_src == kANf4MN || sg.a_src == kATmaMN);
          ok = a_mn ? mma_run<BN, A_TMEM, true, S>(count, k16_tail, ready, empty, ready_err, abort_word, smem_base,
                                                    tmem_base, tmem_acc, first, s, ph)
                    : mma_run<BN, A_TMEM, false, S>(count, k16_tail, ready, empty, ready_err, abort_word, smem_base,
                                                     tmem_base, tmem_acc, first, s, ph);
          first = false;
        }
        if (ok) umma_commit(&accfull[buf]);
      }
      // every MMA issued so far has completed before TMEM is released
      umma_commit(mma_done);
      for (int i = 0; i < (1 << 22) && !mbar_try_wait(mma_done, 0u); ++i) {}
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------------ dequant producer
    // Two groups of four warps take alternate k-blocks; within a group thread t owns one
    // 64-weight unit per k-block.
    const int grp = (warp - 2) >> 2;          // 0: warps 2-5, 1: warps 6-9
    const int t = 32 * (warp & 3) + lane;       // tile row t = TMEM lane t (warp w reaches lanes 32 (w % 4) ..)
    if (p.has_nf4) {
      const float mean = p.scale_fp32 ? 0.0f : __ldg(p.mean);
      const int64_t nb = (p.nw * p.kw + kB1 - 1) / kB1;
      const Codebook& cb = p.cb;
      auto geom = [&](const KIter<BN, S>& q, bool& nf4, UnitGeom& u) {
        const IterPos ip = iter_pos(p, q.it, q.ti.kb_begin, q.ti.kb_end, q.ti.split == 0);
        const GemmSeg& sg = p.seg[ip.seg];
        nf4 = (sg.a_src == kANf4K || sg.a_src == kANf4MN);
        if (nf4) u = unit_geom(sg.a_src, t, q.ti.row0, (int64_t)sg.a_k0 + (int64_t)ip.kb * kBK);
      };
      KIter<BN, S> cur;
      cur.init(p, grp);
      KIter<BN, S> nxt = cur;
      bool nf4_next = false;
      UnitGeom u_next{};
      UnitScale sc_next{};
      if (!nxt.done) {
        geom(nxt, nf4_next, u_next);
        if (nf4_next) sc_next = fetch_scale<GENERIC>(p, u_next, nb, mean);
      }
      for (; !cur.done; cur.advance(p, 2)) {
        const int s = cur.stage;
        const uint32_t ph = cur.phase;
        const bool nf4 = nf4_next;
        const UnitGeom u = u_next;
        const UnitScale sc = sc_next;
        nxt.advance(p, 2);                    // prefetch the next k-block's scales
        if (!nxt.done) {
          geom(nxt, nf4_next, u_next);
          if (nf4_next) sc_next = fetch_scale<GENERIC>(p, u_next, nb, mean);
        }
        Nf4Lut L0, L1;
        uint32_t words[8];
        if (nf4) {
          nf4_lut_build(sc.valid ? sc.s0 : 0.0f, L0, cb);
          if constexpr (GENERIC) {
            if (sc.split < 8) nf4_lut_build(sc.s1, L1, cb);
            const uint32_t* src = reinterpret_cast<const uint32_t*>(p.codes + ((u.n * p.kw + u.kcol) >> 1));
#pragma unroll
            for (int j = 0; j < 8; ++j) words[j] = (j < sc.valid) ? __ldg(src + j) : 0u;
          }
        }
        if (!mbar_wait(A_TMEM ? &full[s] : &cfull[s], ph, abort_word, kErrWaitTma)) break;
        if constexpr (A_TMEM) {
          // Row t of the A tile (64 bf16 = 32 columns) into TMEM slot s.  Slot s is free: full[s]
          // of this k-block follows the release of stage s by the MMAs that last read it.
          uint32_t v[32];
          if (nf4) {
            if constexpr (!GENERIC) {
              const uint4* src = reinterpret_cast<const uint4*>(stage_c(s) + u.coff);
              const uint4 c0 = src[0], c1 = src[1];
              words[0] = c0.x; words[1] = c0.y; words[2] = c0.z; words[3] = c0.w;
              words[4] = c1.x; words[5] = c1.y; words[6] = c1.z; words[7] = c1.w;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint32_t o[4] = {0u, 0u, 0u, 0u};
              if (!GENERIC || j < sc.valid) nf4_expand8(words[j], (GENERIC && j >= sc.split) ? L1 : L0, o);
              v[4 * j] = o[0]; v[4 * j + 1] = o[1]; v[4 * j + 2] = o[2]; v[4 * j + 3] = o[3];
            }
          } else {
            // a kATmaK stretch: row t of the adapter matrix, k-block kb, from global memory
            const IterPos ip = iter_pos(p, cur.it, cur.ti.kb_begin, cur.ti.kb_end, cur.ti.split == 0);
            const int64_t row = (int64_t)cur.ti.row0 + t;
            const int64_t kk = (int64_t)p.seg[ip.seg].a_k0 + (int64_t)ip.kb * kBK;
            const uint4* src = reinterpret_cast<const uint4*>(p.a_glob + row * p.a_glob_ld + kk);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              uint4 w4 = make_uint4(0u, 0u, 0u, 0u);
              if (row < p.a_glob_rows && kk + 8 * q + 8 <= p.a_glob_cols) w4 = __ldg(src + q);
              v[4 * q] = w4.x; v[4 * q + 1] = w4.y; v[4 * q + 2] = w4.z; v[4 * q + 3] = w4.w;
            }
          }
          tmem_st_32x32b_x32(tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + kATmemCol0 + 32u * (uint32_t)s, v);
          tmem_st_wait();
          tc_fence_before();
        } else if (nf4) {
          uint8_t* A = stage_a(s);
          if constexpr (!GENERIC) {
            const uint4* src = reinterpret_cast<const uint4*>(stage_c(s) + u.coff);
            const uint4 c0 = src[0], c1 = src[1];
            words[0] = c0.x; words[1] = c0.y; words[2] = c0.z; words[3] = c0.w;
            words[4] = c1.x; words[5] = c1.y; words[6] = c1.z; words[7] = c1.w;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint32_t o[4];
              nf4_expand8(words[j], L0, o);
              *reinterpret_cast<uint4*>(A + u.dst + (((uint32_t)j ^ u.swz) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint32_t o[4] = {0u, 0u, 0u, 0u};
              if (j < sc.valid) nf4_expand8(words[j], j < sc.split ? L0 : L1, o);
              *reinterpret_cast<uint4*>(A + u.dst + (((uint32_t)j ^ u.swz) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
          fence_proxy_async_smem();
        }
        // prod[s] is the MMA issuer's only wait, so it also vouches for the B tile
        if (!A_TMEM && !mbar_wait(&full[s], ph, abort_word, kErrWaitTma)) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&prod[s]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    // Warp w drains TMEM lanes 32 (w % 4) .. + 31 (one output row per thread), chunk by chunk.
    // With one accumulator (A in TMEM) eight warps each take half of the 256 columns and the
    // next tile's MMAs wait for the drain (its loads and dequant proceed meanwhile); with two
    // accumulators four warps drain all columns while the next tile's MMAs run in the other
    // buffer.
    const int e = warp - kEpiWarp0;
    const int q = warp & 3;
    constexpr int kChunk = BN < 32 ? BN : 32;
    constexpr int kCols = A_TMEM ? BN / 2 : BN;   // columns this warp drains
    const int c_base = A_TMEM ? (e >> 2) * (BN / 2) : 0;
    const int tiles_m = (p.rows + kBM - 1) / kBM;
    const int tiles_n = (p.cols + BN - 1) / BN;
    const int64_t ntiles = (int64_t)tiles_m * tiles_n * p.splits;
    int64_t tc = 0;
    for (int64_t tt = blockIdx.x; tt < ntiles; tt += gridDim.x, ++tc) {
      const TileInfo ti = tile_info<BN>(p, tiles_m, tiles_n, tt);
      const int buf = (int)(tc % NB);
      const uint32_t use = (uint32_t)(tc / NB) & 1u;
      if (!mbar_wait(&accfull[buf], use, abort_word, kErrWaitMma)) break;
      tc_fence_after();
      const int row = ti.row0 + 32 * q + lane;
      const bool row_ok = row < p.rows;
      const uint32_t taddr0 = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(buf * C::kAccStride + c_base);
      {
#pragma unroll 1
        for (int c0 = 0; c0 < kCols; c0 += kChunk) {
          uint32_t r[32];
          if constexpr (kChunk == 32) tmem_ld_32x32b_x32(taddr0 + (uint32_t)c0, r);
          else tmem_ld_32x32b_x16(taddr0 + (uint32_t)c0, r);
          tmem_ld_wait();
          if constexpr (kChunk == 32) {
            if (p.epi == kEpiBf16T) {
              // bf16 pairs, then an 8 x 8 transpose per group of 8 lanes: lane j of a group
              // ends up with 8 consecutive output features of token j of each 8-token block,
              // one 16-byte store instead of eight 2-byte ones
              uint32_t w[16];
#pragma unroll
              for (int k = 0; k < 16; ++k) w[k] = pack_bf16x2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
              const int fbase = ti.row0 + 32 * q + (lane & ~7);
              uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                uint32_t x0 = w[4 * b], x1 = w[4 * b + 1], x2 = w[4 * b + 2], x3 = w[4 * b + 3];
                transpose8x8_bf16(x0, x1, x2, x3, lane);
                const int col = ti.col0 + c_base + c0 + 8 * b + (lane & 7);
                if (col < p.cols && fbase < p.rows)
                  *reinterpret_cast<uint4*>(out + (int64_t)col * p.ld_out + fbase) = make_uint4(x0, x1, x2, x3);
              }
              continue;
            }
          }
          if (!row_ok) continue;
          if (p.epi == kEpiBf16T) {
            uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
#pragma unroll
            for (int j = 0; j < kChunk; ++j) {
              const int col = ti.col0 + c_base + c0 + j;
              if (col < p.cols) out[(int64_t)col * p.ld_out + row] = f32_to_bf16_bits(__uint_as_float(r[j]));
            }
          } else {
            float* out = reinterpret_cast<float*>(p.out) + (int64_t)ti.split * p.split_stride;
#pragma unroll
            for (int j = 0; j < kChunk; ++j) {
              const int col = ti.col0 + c_base + c0 + j;
              if (col < p.cols) out[(int64_t)col * p.ld_out + row] = __uint_as_float(r[j]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[buf]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BN, bool GENERIC, bool A_TMEM = false>
static cudaError_t launch_bn(const GemmParams& p, cudaStream_t st) {
  using C = Cfg<BN, A_TMEM>;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = enable_smem_once(qlora_gemm_kernel<BN, GENERIC, A_TMEM>, C::kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntiles = (int64_t)((p.rows + kBM - 1) / kBM) * ((p.cols + BN - 1) / BN) * p.splits;
  const int grid = (int)(ntiles < sms ? ntiles : sms);
  qlora_gemm_kernel<BN, GENERIC, A_TMEM><<<grid, C::kThreads, C::kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

template <bool GENERIC>
static cudaError_t launch_gemm_g(const GemmParams& p, int bn, cudaStream_t st) {
  if (p.b_box_rows != bn) return cudaErrorInvalidValue;   // each B box must fill exactly one B tile
  if (p.a_tmem) {                                         // A in tensor memory: 256-token tiles only
    if (bn != 256) return cudaErrorInvalidValue;
    return launch_bn<256, GENERIC, true>(p, st);
  }
  switch (bn) {
    case 16: return launch_bn<16, GENERIC>(p, st);
    case 32: return launch_bn<32, GENERIC>(p, st);
    case 64: return launch_bn<64, GENERIC>(p, st);
    case 128: return launch_bn<128, GENERIC>(p, st);
    case 256: return launch_bn<256, GENERIC>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(const GemmParams& p, int bn, cudaStream_t st) {
  return p.nf4_generic ? launch_gemm_g<true>(p, bn, st) : launch_gemm_g<false>(p, bn, st);
}

// ---------------------------------------------------------------------------------------
// small helpers of the low-rank path
// ---------------------------------------------------------------------------------------
// out[c][r] = in[r][c] (bf16), 32x32 tiles through shared memory.
__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ in, int64_t rows, int64_t cols,
                                      uint16_t* __restrict__ out, int64_t ld_out) {
  __shared__ uint16_t tile[32][33];
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[c * ld_out + r] = tile[threadIdx.x][i];
  }
}


// out[c * ld_out + r] = bf16(sum_z ws[z * split_stride + c * ld + r])
__global__ void reduce_splits_bf16_kernel(const float* __restrict__ ws, int splits, int64_t split_stride,
                                          int64_t cols, int64_t rows, int64_t ld, uint16_t* __restrict__ out,
                                          int64_t ld_out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= cols * rows) return;
  const int64_t c = i / rows, r = i % rows;
  float acc = 0.0f;
  for (int z = 0; z < splits; ++z) acc += ws[(int64_t)z * split_stride + c * ld + r];
  out[c * ld_out + r] = f32_to_bf16_bits(acc);
}


cudaError_t launch_transpose_bf16(const uint16_t* in, int64_t rows, int64_t cols, uint16_t* out, int64_t ld_out,
                                  cudaStream_t st) {
  dim3 grid((unsigned)((cols + 31) / 32), (unsigned)((rows + 31) / 32));
  transpose_bf16_kernel<<<grid, dim3(32, 8), 0, st>>>(in, rows, cols, out, ld_out);
  return cudaGetLastError();
}


cudaError_t launch_reduce_splits_bf16(const float* ws, int splits, int64_t split_stride, int64_t cols, int64_t rows,
                                      int64_t ld, uint16_t* out, int64_t ld_out, cudaStream_t st) {
  const int64_t n = cols * rows;
  reduce_splits_bf16_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(ws, splits, split_stride, cols, rows, ld,
                                                                          out, ld_out);
  return cudaGetLastError();
}


}  // namespace qnf4
