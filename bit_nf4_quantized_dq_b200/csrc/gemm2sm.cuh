// Two-SM (cta_group::2) version of the fused dequant GEMM for wide token tiles.
//
// A cluster of two CTAs computes a 256 x 256 tile of D = A * B^T: each CTA dequantizes (or
// TMA-loads) its own 128 rows of A, and TMA-loads half of the 256-token B tile; one thread of
// the even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256), which reads A from both
// CTAs and B from both halves, and accumulates rows 0-127 in the even CTA's TMEM and rows
// 128-255 in the odd CTA's.  Per SM this halves the bytes of B streamed from L2 and read
// from shared memory for the same tensor work, compared with one CTA computing 128 x 256.
//
// Two rings per CTA: a TMA ring of 8 stages (this CTA's half of the B tile + its packed
// codes, 20 KB) and a ring of 4 A slots written by the dequant producer (or by TMA for the
// adapter k-blocks).  Decoupling them keeps 160 KB of loads in flight per SM, enough to hide
// the load latency at the tensor cores' rate.  Barriers: the even CTA's full[s] counts the B
// (and TMA-loaded A) bytes of both CTAs (the loads carry .cta_group::2 and complete on the
// even CTA's barrier); every CTA's cfull[s] counts its own codes; every producer warp of the
// pair arrives on the even CTA's prod[a]; the MMA commits arrive on empty[s] and aempty[a],
// and at the end on accfull, of both CTAs.  No load uses cluster multicast.
#pragma once

#include "gemm.cuh"

namespace qnf4 {

// TMA warps 0 and 10.. (kTmaWarps2 of them, alternate k-blocks), MMA warp 1, producer / epilogue
// warps 2-9.  One warp's bulk loads complete one after another, so the ring is spread over
// several issuing warps.
constexpr int kTmaWarps2 = 2;
constexpr int kThreads2 = 320 + 32 * (kTmaWarps2 - 1);

struct Cfg2 {
  static constexpr int BN = 256;                    // UMMA N (tokens per pair)
  static constexpr int kABytes = 128 * 64 * 2;      // one A slot: this CTA's 128 rows x 64 k
  static constexpr int kBBytes = 128 * 64 * 2;      // this CTA's half of the B tile
  static constexpr int kTStageBytes = kBBytes + kCodesBytes;   // TMA ring stage: B half + codes
  static constexpr int kTStages = 8;
  static constexpr int kASlots = 4;
  // mbarrier parity waits are only safe while a waiter is never two phases ahead of, or
  // behind, the barrier it polls:
  //  - the two producer groups take alternate k-blocks, so each group must own whole rings
  //    (even stage and slot counts) and see every phase of the barriers it waits on;
  //  - the TMA thread waits on aempty[a] (adapter k-blocks only) while being at most
  //    kTStages k-blocks ahead of the MMA, so kTStages <= 2 * kASlots keeps that barrier at
  //    most one phase behind the phase it waits for.
  static_assert(kTStages % 2 == 0 && kASlots % 2 == 0, "rings must split evenly between the producer groups");
  static_assert(kTStages <= 2 * kASlots, "TMA run-ahead must not alias the A-slot barrier phases");
  static_assert(kTStages % kTmaWarps2 == 0 && kASlots % kTmaWarps2 == 0, "each TMA warp owns whole stages and A slots");
  static constexpr int kBarrierOffset = kTStages * kTStageBytes + kASlots * kABytes;
  static constexpr int kTmemCols = 256;
  static constexpr int kSmemBytes = kBarrierOffset + 512 + 1024;   // rings, barriers, alignment
  static_assert(kTStageBytes % 1024 == 0 && kABytes % 1024 == 0, "swizzle atoms stay 1024-aligned");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_cta(uint32_t smem_addr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(cta));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier of another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory whose completion is counted on the mbarrier at
// `bar_cluster_addr` (the even CTA's barrier); never multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 uint32_t bar_cluster_addr) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster_addr)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at this offset in both CTAs of the pair when the MMAs issued so
// far have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}

// One k-block (64 deep) of pair MMAs (M = 256 over the two CTAs, N = 256): the descriptors of
// consecutive 16-deep slices differ only in their start address field.
template <bool A_MN>
__device__ __forceinline__ void umma_kblock_pair(uint32_t tmem_acc, uint32_t a_addr, uint32_t b_addr, uint32_t acc) {
  constexpr uint32_t idesc = umma_idesc_bf16(256, Cfg2::BN, A_MN ? 1u : 0u, 0u);
  const uint64_t a0 = A_MN ? umma_sdesc_sw128(a_addr, 8192u, 1024u) : umma_sdesc_sw128(a_addr, 16u, 1024u);
  const uint64_t b0 = umma_sdesc_sw128(b_addr, 16u, 1024u);
#pragma unroll
  for (int k16 = 0; k16 < 4; ++k16) {
    const uint64_t ad = a0 + (uint64_t)((A_MN ? 2048u : 32u) * (uint32_t)k16 >> 4);
    const uint64_t bd = b0 + (uint64_t)(32u * (uint32_t)k16 >> 4);
    umma_bf16_pair(tmem_acc, ad, bd, idesc, k16 == 0 ? acc : 1u);
  }
}

template <bool GENERIC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
    qlora_gemm2_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg2;
  constexpr int ST = C::kTStages;
  constexpr int SA = C::kASlots;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarrierOffset);   // [ST] even CTA: B (+A) bytes of both CTAs
  uint64_t* cfull = full + ST;       // [ST] this CTA's codes (or a plain arrive)
  uint64_t* empty = cfull + ST;      // [ST] MMA done with TMA stage s (both CTAs)
  uint64_t* prod = empty + ST;       // [SA] even CTA: A slot written by all producer warps of the pair
  uint64_t* aempty = prod + SA;      // [SA] MMA done with A slot a (both CTAs)
  uint64_t* accfull = aempty + SA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
  volatile uint32_t* abort_word = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0: issues the MMAs
  const int row0 = blockIdx.x * 128;                // this CTA's 128 rows
  const int col0 = blockIdx.y * C::BN;              // the pair's 256 tokens
  const int split = blockIdx.z;
  const int kb_begin = split * p.kb_per_split;
  int kb_end = kb_begin + p.kb_per_split;
  if (kb_end > p.seg[0].kblocks) kb_end = p.seg[0].kblocks;
  const bool first_split = (split == 0);
  int n_iters = kb_end - kb_begin;
  if (first_split)
    for (int s = 1; s < p.nseg; ++s) n_iters += p.seg[s].kblocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&cfull[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < SA; ++a) {
      mbar_init(&prod[a], 8);       // four producer warps of each CTA
      mbar_init(&aempty[a], 1);
    }
    mbar_init(accfull, 1);
    *abort_word = 0u;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    for (int m = 0; m < kMaxMaps; ++m) tma_prefetch_desc(&p.maps[m]);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();        // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;
  const uint32_t full_leader0 = map_to_cta(smem_u32(&full[0]), 0);
  const uint32_t prod_leader0 = map_to_cta(smem_u32(&prod[0]), 0);

  auto tstage_b = [&](int s) { return smem + s * C::kTStageBytes; };
  auto tstage_c = [&](int s) { return smem + s * C::kTStageBytes + C::kBBytes; };
  auto aslot = [&](int a) { return smem + ST * C::kTStageBytes + a * C::kABytes; };

  if (warp == 0 || warp >= 10) {
    // ------------------------------------------------------------------ TMA (both CTAs)
    // kTmaWarps2 warps (0, 10, ..) take turns on k-blocks: a bulk-tensor load holds its issuing
    // thread for a few hundred cycles whatever its size, while loads of different warps, and
    // of different lanes of one instruction, proceed side by side.  Each k-block's loads go
    // out as one instruction: lane 0 this CTA's half of the B tile, lane 1 the codes (or the
    // A tile), lane 2 the second half of an MN-major A tile.  All use the pair form, which
    // completes on any mbarrier of the pair: the even CTA's full[s], or this CTA's cfull[s].
    const int tw = (warp == 0) ? 0 : warp - 9;
    int last_issue[ST];
    for (int s = 0; s < ST; ++s) last_issue[s] = -1;
    bool ok = true;
    for (int it = tw; it < n_iters && ok; it += kTmaWarps2) {
      const int s = it % ST, a = it % SA;
      const uint32_t ph = (uint32_t)(it / ST) & 1u, pa = (uint32_t)(it / SA) & 1u;
      if (!mbar_wait(&empty[s], ph ^ 1u, abort_word, kErrWaitEmpty)) { ok = false; break; }
      const IterPos ip = iter_pos(p, it, kb_begin, kb_end, first_split);
      const GemmSeg& sg = p.seg[ip.seg];
      const bool nf4 = (sg.a_src == kANf4K || sg.a_src == kANf4MN);
      if (!nf4 && !mbar_wait(&aempty[a], pa ^ 1u, abort_word, kErrWaitEmpty)) { ok = false; break; }
      const uint32_t fbar = full_leader0 + (uint32_t)s * 8u;
      if (lane == 0) {
        if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (C::kBBytes + (nf4 ? 0u : (uint32_t)C::kABytes)));
        if (nf4 && !GENERIC) mbar_arrive_expect_tx(&cfull[s], kCodesBytes);
        else mbar_arrive(&cfull[s]);      // keeps the producers in step with the stages
        last_issue[s] = it;
      }
      __syncwarp();
      const int k = sg.a_k0 + ip.kb * kBK;
      int map = -1, cx = 0, cy = 0;
      uint8_t* dst = nullptr;
      uint32_t bar = fbar;
      if (lane == 0) {
        map = sg.b_map; dst = tstage_b(s); cx = sg.b_k0 + ip.kb * kBK; cy = col0 + 128 * (int)rank;
      } else if (lane == 1) {
        if (nf4) {
          if (!GENERIC) {
            map = sg.a_map; dst = tstage_c(s); bar = smem_u32(&cfull[s]);
            if (sg.a_src == kANf4K) { cx = k / 2; cy = row0; } else { cx = row0 / 2; cy = k; }
          }
        } else if (sg.a_src == kATmaK) {
          map = sg.a_map; dst = aslot(a); cx = k; cy = row0;
        } else {
          map = sg.a_map; dst = aslot(a); cx = row0; cy = k;
        }
      } else if (lane == 2 && sg.a_src == kATmaMN) {
        map = sg.a_map; dst = aslot(a) + 8192; cx = row0 + 64; cy = k;
      }
      if (map >= 0) tma_load_2d_pair(dst, &p.maps[map], cx, cy, bar);
      __syncwarp();
    }
    if (!ok && lane == 0) {
      // drain this warp's copies still in flight (the pair's B copies complete on the even
      // CTA's barriers, which that CTA drains)
      for (int s = 0; s < ST; ++s)
        if (last_issue[s] >= 0) {
          const uint32_t ph = (uint32_t)(last_issue[s] / ST) & 1u;
          for (int i = 0; i < (1 << 20) && !mbar_try_wait(&cfull[s], ph); ++i) {}
          if (rank == 0)
            for (int i = 0; i < (1 << 20) && !mbar_try_wait(&full[s], ph); ++i) {}
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    // Lane 0 of the even CTA alone runs this loop: the tensor pipe queues only about one MMA
    // ahead, so the issuer keeps warp-collective instructions out of it and issues each
    // k-block as one unrolled sequence.
    if (rank == 0 && lane == 0) {
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % ST, a = it % SA;
        const uint32_t ph = (uint32_t)(it / ST) & 1u, pa = (uint32_t)(it / SA) & 1u;
        if (!mbar_wait_thread(&full[s], ph, abort_word, kErrWaitTma)) break;
        if (!mbar_wait_thread(&prod[a], pa, abort_word, kErrWaitProducer)) break;
        tc_fence_after();
        const IterPos ip = iter_pos(p, it, kb_begin, kb_end, first_split);
        const GemmSeg& sg = p.seg[ip.seg];
        const bool a_mn = (sg.a_src == kANf4MN || sg.a_src == kATmaMN);
        const uint32_t a_addr = smem_u32(aslot(a));
        const uint32_t b_addr = smem_u32(tstage_b(s));
        const uint32_t acc = it > 0 ? 1u : 0u;
        if (!ip.last || sg.k16_last == 4) {
          if (a_mn) umma_kblock_pair<true>(tmem_acc, a_addr, b_addr, acc);
          else umma_kblock_pair<false>(tmem_acc, a_addr, b_addr, acc);
        } else {
          const uint32_t idesc = umma_idesc_bf16(256, C::BN, a_mn ? 1u : 0u, 0u);
          for (int k16 = 0; k16 < sg.k16_last; ++k16) {
            const uint64_t ad = a_mn ? umma_sdesc_sw128(a_addr + (uint32_t)k16 * 2048u, 8192u, 1024u)
                                     : umma_sdesc_sw128(a_addr + (uint32_t)k16 * 32u, 16u, 1024u);
            const uint64_t bd = umma_sdesc_sw128(b_addr + (uint32_t)k16 * 32u, 16u, 1024u);
            umma_bf16_pair(tmem_acc, ad, bd, idesc, (acc || k16 > 0) ? 1u : 0u);
          }
        }
        umma_commit_pair(&empty[s]);
        umma_commit_pair(&aempty[a]);
      }
      umma_commit_pair(accfull);   // also on abort: in-flight MMAs drain first
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ dequant producer
    // Two groups of four warps take alternate k-blocks; within a group thread t owns one
    // 64-weight unit per k-block.
    const int grp = (warp - 2) >> 2;
    const int t = (threadIdx.x - 64) & 127;
    bool ok = true;
    const float mean = p.has_nf4 ? __ldg(p.mean) : 0.0f;
    const int64_t nb = (p.nw * p.kw + kB1 - 1) / kB1;
    auto geom = [&](int it, bool& nf4, UnitGeom& u) {
      const IterPos ip = iter_pos(p, it, kb_begin, kb_end, first_split);
      const GemmSeg& sg = p.seg[ip.seg];
      nf4 = (sg.a_src == kANf4K || sg.a_src == kANf4MN);
      if (nf4) u = unit_geom(sg.a_src, t, row0, (int64_t)sg.a_k0 + (int64_t)ip.kb * kBK);
    };
    bool nf4_next = false;
    UnitGeom u_next{};
    UnitScale sc_next{};
    if (grp < n_iters) {
      geom(grp, nf4_next, u_next);
      if (nf4_next) sc_next = fetch_scale<GENERIC>(p, u_next, nb);
    }
    for (int it = grp; it < n_iters; it += 2) {
      const int s = it % ST, a = it % SA;
      const uint32_t ph = (uint32_t)(it / ST) & 1u, pa = (uint32_t)(it / SA) & 1u;
      const bool nf4 = nf4_next;
      const UnitGeom u = u_next;
      const UnitScale sc = sc_next;
      if (it + 2 < n_iters) {
        geom(it + 2, nf4_next, u_next);
        if (nf4_next) sc_next = fetch_scale<GENERIC>(p, u_next, nb);
      }
      Nf4Lut L0, L1;
      uint32_t words[8];
      if (nf4) {
        nf4_lut_build(sc.valid ? dq_block_scale(sc.e0, sc.c20, mean) : 0.0f, L0);
        if constexpr (GENERIC) {
          if (sc.split < 8) nf4_lut_build(dq_block_scale(sc.e1, sc.c21, mean), L1);
          const uint32_t* src = reinterpret_cast<const uint32_t*>(p.codes + ((u.n * p.kw + u.kcol) >> 1));
#pragma unroll
          for (int j = 0; j < 8; ++j) words[j] = (j < sc.valid) ? __ldg(src + j) : 0u;
        }
      }
      if (!mbar_wait(&cfull[s], ph, abort_word, kErrWaitTma)) { ok = false; break; }
      if (!mbar_wait(&aempty[a], pa ^ 1u, abort_word, kErrWaitEmpty)) { ok = false; break; }
      if (nf4) {
        uint8_t* A = aslot(a);
        if constexpr (!GENERIC) {
          const uint4* src = reinterpret_cast<const uint4*>(tstage_c(s) + u.coff);
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
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(prod_leader0 + (uint32_t)a * 8u);
    }
    // ------------------------------------------------------------------ epilogue
    const int c_begin = grp * (C::BN / 2);
    const int c_end = c_begin + C::BN / 2;
    if (mbar_wait(accfull, 0u, abort_word, kErrWaitMma)) {
      tc_fence_after();
      const int q = warp & 3;
      const int row = row0 + 32 * q + lane;
      const bool row_ok = row < p.rows;
#pragma unroll 1
      for (int c0 = c_begin; c0 < c_end; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_acc + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, r);
        tmem_ld_wait();
        if (!row_ok) continue;
        if (p.epi == kEpiBf16T) {
          uint16_t* out = reinterpret_cast<uint16_t*>(p.out);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = col0 + c0 + j;
            if (col < p.cols) out[(int64_t)col * p.ld_out + row] = f32_to_bf16_bits(__uint_as_float(r[j]));
          }
        } else {
          float* out = reinterpret_cast<float*>(p.out) + (int64_t)split * p.split_stride;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = col0 + c0 + j;
            if (col < p.cols) out[(int64_t)col * p.ld_out + row] = __uint_as_float(r[j]);
          }
        }
      }
    }
    tc_fence_before();
    (void)ok;
  }

  tc_fence_before();
  cluster_sync_all();        // no CTA leaves while its pair may still use its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_acc, C::kTmemCols);
  }
}

template <bool GENERIC>
static cudaError_t launch_gemm2_g(const GemmParams& p, cudaStream_t st) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(qlora_gemm2_kernel<GENERIC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg2::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int pairs = (p.rows + 255) / 256;
  dim3 grid(2 * pairs, (p.cols + Cfg2::BN - 1) / Cfg2::BN, p.splits);
  qlora_gemm2_kernel<GENERIC><<<grid, kThreads2, Cfg2::kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

// 256 x 256 pair tiles; grid.x = 2 * ceil(rows / 256), grid.y = ceil(cols / 256).
static cudaError_t launch_gemm2(const GemmParams& p, cudaStream_t st) {
  if (p.b_box_rows != 128) return cudaErrorInvalidValue;  // each CTA loads a 128-row half of B
  return p.nf4_generic ? launch_gemm2_g<true>(p, st) : launch_gemm2_g<false>(p, st);
}

}  // namespace qnf4
