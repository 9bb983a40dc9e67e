// The library's single translation unit: the codec and GEMM kernels, and the C ABI
// (argument checks, workspace layout, TMA tensor maps, kernel sequencing).
#include <cstdarg>
#include <cstdio>
#include <cmath>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>

#include "qlora_nf4.h"
#include "codec.cuh"
#include "gemm.cuh"
#include "lowrank.cuh"
#include "merge.cuh"
#include "adamw.cuh"

namespace {

thread_local std::string g_last_error;
thread_local void* const* g_events = nullptr;
thread_local int g_n_events = 0;

void mark(int i, cudaStream_t st) {
  if (g_events && i < g_n_events && g_events[i]) cudaEventRecord(static_cast<cudaEvent_t>(g_events[i]), st);
}

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(QNF4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_arch() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  static int cached_dev = -1, cached_major = 0;
  if (cached_dev != dev) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    cached_dev = dev;
    cached_major = major;
  }
  if (cached_major != 10) return fail(QNF4_ERR_ARCH, "device %d is sm_%d0, this library targets sm_100a", dev,
                                      cached_major);
  return QNF4_OK;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ------------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over a row-major [outer][inner] array with row pitch `row_bytes`.
int make_map(CUtensorMap* m, const void* base, bool bf16, uint64_t inner, uint64_t outer, uint64_t row_bytes,
             uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(QNF4_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if (!aligned(base, 16) || row_bytes % 16 != 0)
    return fail(QNF4_ERR_UNSUPPORTED, "TMA operand needs a 16-byte aligned base and row pitch (pitch %llu)",
                (unsigned long long)row_bytes);
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QNF4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return QNF4_OK;
}

int bn_for(int64_t cols) {
  if (cols >= 256) return 256;
  if (cols > 64) return 128;   // 128 columns: fewer wasted MMA columns than 256
  if (cols > 32) return 64;
  if (cols > 16) return 32;
  return 16;
}

int kblocks(int64_t k) { return (int)((k + 63) / 64); }
int k16_last(int64_t k) {
  const int64_t rem = k - 64 * (int64_t)(kblocks(k) - 1);
  return (int)((rem + 15) / 16);
}

constexpr int kSms = 148;

// Split of the K loop over blockIdx.z so that small tile grids still cover the SMs.
// Every split gets at least one k-block: the count is re-derived from the per-split share.
int choose_splits(int64_t tiles, int kb) {
  // Every CTA of these kernels fills an SM (shared memory), so a launch with s splits runs in
  // ceil(tiles * s / kSms) waves; a wave costs its ceil(kb / s) k-blocks plus a fixed
  // kSplitOverhead k-blocks' worth of prologue, pipeline fill and partial stores.  Take the
  // split count with the lowest total (the smallest on ties), at least 4 k-blocks per split.
  constexpr int64_t kSplitOverhead = 4;
  if (tiles >= kSms) return 1;
  int best = 1;
  int64_t best_cost = ((tiles + kSms - 1) / kSms) * ((int64_t)kb + kSplitOverhead);
  const int cap = kb / 4 > 1 ? kb / 4 : 1;
  for (int s = 2; s <= cap; ++s) {
    const int64_t per = (kb + s - 1) / s;
    const int64_t used = (kb + per - 1) / per;   // splits that get k-blocks
    const int64_t cost = ((tiles * used + kSms - 1) / kSms) * (per + kSplitOverhead);
    if (cost < best_cost) {
      best_cost = cost;
      best = (int)used;
    }
  }
  return best;
}

// ------------------------------------------------------------------------ shapes
struct LinearShape {
  int64_t M, K, N;
  int r;
};

int check_linear_shape(const LinearShape& s) {
  if (s.M <= 0 || s.K <= 0 || s.N <= 0 || s.r <= 0) return fail(QNF4_ERR_INVALID, "sizes must be positive");
  if (s.K % 8 || s.N % 8) return fail(QNF4_ERR_UNSUPPORTED, "K and N must be multiples of 8 (K=%lld N=%lld)",
                                      (long long)s.K, (long long)s.N);
  if (s.r % 8 || s.r > 256) return fail(QNF4_ERR_UNSUPPORTED, "r must be a multiple of 8 in [8, 256] (r=%d)", s.r);
  if (s.M >= (1ll << 31) || s.K >= (1ll << 31) || s.N >= (1ll << 31) || s.N * s.K >= (1ll << 40))
    return fail(QNF4_ERR_INVALID, "sizes too large");
  return QNF4_OK;
}

int64_t ld8(int64_t m) { return (m + 7) / 8 * 8; }

// Workspace carving: every region 256-byte aligned.
struct Carver {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

// Column tile of the low-rank kernels (rank columns per CTA).
int bj_for(int r) { return r <= 16 ? 16 : (r <= 32 ? 32 : 64); }

struct LowRankPlan {
  int bj, splits;
};

LowRankPlan plan_lowrank(int64_t rows, int r, int64_t kdim) {
  LowRankPlan p;
  p.bj = bj_for(r);
  const int64_t tiles = ((rows + 127) / 128) * ((r + p.bj - 1) / p.bj);
  p.splits = choose_splits(tiles, kblocks(kdim));
  return p;
}

struct FwdPlan {
  int bn, splits;   // fused forward
  LowRankPlan t;    // t = s x A^T
};

FwdPlan plan_fwd(const LinearShape& s) {
  FwdPlan p;
  p.bn = bn_for(s.M);
  const int64_t tiles = ((s.N + 127) / 128) * ((s.M + p.bn - 1) / p.bn);
  p.splits = choose_splits(tiles, kblocks(s.K));
  p.t = plan_lowrank(s.M, s.r, s.K);
  return p;
}

struct BwdPlan {
  int bn, splits;      // fused dX
  LowRankPlan u, a, b; // u = s dY B, dA, dB
};

BwdPlan plan_bwd(const LinearShape& s) {
  BwdPlan p;
  p.bn = bn_for(s.M);
  const int64_t tiles = ((s.K + 127) / 128) * ((s.M + p.bn - 1) / p.bn);
  p.splits = choose_splits(tiles, kblocks(s.N));
  p.u = plan_lowrank(s.M, s.r, s.N);
  p.a = plan_lowrank(s.K, s.r, s.M);
  p.b = plan_lowrank(s.N, s.r, s.M);
  return p;
}

struct FwdWs {
  uint16_t *thi, *tlo;
  double* partial;
  float* part;
};

size_t fwd_carve(Carver& c, const LinearShape& s, const FwdPlan& p, FwdWs* w) {
  w->thi = c.take<uint16_t>((size_t)s.M * s.r);
  w->tlo = c.take<uint16_t>((size_t)s.M * s.r);
  w->partial = c.take<double>((size_t)p.t.splits * s.r * s.M);
  w->part = p.splits > 1 ? c.take<float>((size_t)p.splits * s.M * s.N) : nullptr;
  return c.off;
}

struct BwdWs {
  uint16_t *Bt, *uhi, *ulo, *uT3, *tT3;
  double* partial;
  float* partX;
};

size_t bwd_carve(Carver& c, const LinearShape& s, const BwdPlan& p, BwdWs* w) {
  const int64_t ldM = ld8(s.M);
  w->Bt = c.take<uint16_t>((size_t)s.r * s.N);
  w->uhi = c.take<uint16_t>((size_t)s.M * s.r);
  w->ulo = c.take<uint16_t>((size_t)s.M * s.r);
  w->uT3 = c.take<uint16_t>((size_t)3 * s.r * ldM);
  w->tT3 = c.take<uint16_t>((size_t)3 * s.r * ldM);
  size_t np = (size_t)p.u.splits * s.r * s.M;
  np = std::max(np, (size_t)p.a.splits * s.r * s.K);
  np = std::max(np, (size_t)p.b.splits * s.r * s.N);
  w->partial = c.take<double>(np);
  w->partX = p.splits > 1 ? c.take<float>((size_t)p.splits * s.M * s.K) : nullptr;
  return c.off;
}

// One low-rank product: A operand map (K-major over [rows][k] or MN-major over [k][rows]),
// `terms` B maps over [r][k] (K-major), fp64 partials into `partial`.
int run_lowrank(const void* a_base, bool a_mn, int64_t a_inner, int64_t a_outer, int64_t a_pitch_bytes,
                const uint16_t* const* b_terms, int terms, int64_t b_inner, int64_t b_pitch_bytes, int r,
                int64_t rows, int64_t kdim, const LowRankPlan& pl, double* partial, cudaStream_t st) {
  qnf4::LowRankParams lp;
  memset(&lp, 0, sizeof(lp));
  if (a_mn) {
    if (int rc = make_map(&lp.a_map, a_base, true, a_inner, a_outer, a_pitch_bytes, 64, 64)) return rc;
  } else {
    if (int rc = make_map(&lp.a_map, a_base, true, a_inner, a_outer, a_pitch_bytes, 64, 128)) return rc;
  }
  for (int t = 0; t < terms; ++t)
    if (int rc = make_map(&lp.b_map[t], b_terms[t], true, b_inner, r, b_pitch_bytes, 64, pl.bj)) return rc;
  lp.a_mn = a_mn ? 1 : 0;
  lp.kblocks = kblocks(kdim);
  lp.k16_last = k16_last(kdim);
  lp.splits = pl.splits;
  lp.kb_per_split = (lp.kblocks + pl.splits - 1) / pl.splits;
  lp.rows = (int32_t)rows;
  lp.cols = r;
  lp.partial = partial;
  cudaError_t e = qnf4::launch_lowrank(lp, pl.bj, terms, st);
  if (e != cudaSuccess) return cuda_fail(e, "low-rank launch");
  return QNF4_OK;
}

// The fused forward keeps its A operand in tensor memory (gemm.cuh, A_TMEM) on 256-token tiles.
constexpr bool kATmemForward = true;
// Rows of each B-operand TMA box: one box fills one token tile.
int b_box_rows(int bn) { return bn; }

cudaError_t launch_fused(const qnf4::GemmParams& gp, int bn, cudaStream_t st) { return qnf4::launch_gemm(gp, bn, st); }

// ------------------------------------------------------------------------ code books
// NF4: the 8-decimal levels of the code book table, each the nearest fp32 (the compiler rounds
// the literals).  FP4 E2M1: its 16 values 0, 0.5, 1, 1.5, 2, 3, 4, 6 (both signs, two zeros)
// over 6, sorted.  INT4: 16 levels equally spaced over [-1, 1], -1 + 2 i / 15.  The quotients
// are formed in double and rounded once to float; none of them lies near a float rounding
// midpoint (their binary expansions repeat), so that is the nearest float.
int get_codebook(int id, qnf4::Codebook* cb) {
  static const float nf4[16] = QNF4_LEVELS;
  switch (id) {
    case QNF4_CODEBOOK_NF4:
      for (int j = 0; j < 16; ++j) cb->q[j] = nf4[j];
      break;
    case QNF4_CODEBOOK_FP4_E2M1: {
      static const double mags[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
      for (int j = 0; j < 8; ++j) {
        cb->q[7 - j] = -(float)(mags[j] / 6.0);   // -0 at index 7
        cb->q[8 + j] = (float)(mags[j] / 6.0);
      }
      break;
    }
    case QNF4_CODEBOOK_INT4:
      for (int j = 0; j < 16; ++j) cb->q[j] = (float)((double)(2 * j - 15) / 15.0);
      break;
    default:
      return fail(QNF4_ERR_INVALID, "unknown code book %d", id);
  }
  // The quantizer finds the nearest level through 33 buckets of width 1/16 over [-1, 1] and
  // one threshold compare per bucket: every bucket may hold at most one threshold (the largest
  // float not above a midpoint between neighbouring levels).
  if (cb->q[0] != -1.0f || cb->q[15] != 1.0f) return fail(QNF4_ERR_INVALID, "code book must span [-1, 1]");
  int count[33] = {0};
  for (int j = 0; j < 15; ++j) {
    if (!(cb->q[j] <= cb->q[j + 1])) return fail(QNF4_ERR_INVALID, "code book levels must not decrease");
    const double m = 0.5 * ((double)cb->q[j] + (double)cb->q[j + 1]);
    float th = (float)m;
    if ((double)th > m) th = std::nextafter(th, -2.0f);
    for (int b = 0; b < 33; ++b)
      if ((double)th >= (b - 16.5) / 16.0 && (double)th < (b - 15.5) / 16.0) ++count[b];
  }
  for (int b = 0; b < 33; ++b)
    if (count[b] > 1) return fail(QNF4_ERR_UNSUPPORTED, "code book: two midpoints share a quantizer bucket");
  return QNF4_OK;
}

int nf4_operand(qnf4::GemmParams& gp, const qnf4::Codebook& cb, int double_quant, const uint8_t* codes,
                const uint8_t* scale_codes, const float* scales, const float* mean, int64_t N, int64_t K) {
  gp.has_nf4 = 1;
  gp.nf4_generic = (K % 64 != 0) ? 1 : 0;
  gp.codes = codes;
  gp.scale_codes = scale_codes;
  gp.c2 = scales;
  gp.mean = mean;
  gp.nw = N;
  gp.kw = K;
  gp.cb = cb;
  gp.scale_fp32 = double_quant ? 0 : 1;
  return QNF4_OK;
}

// Checks of the stored-format pointers: with double quantization scale codes, group constants
// and the mean; without it, one fp32 scale per block (scale_codes and mean unused).
int check_format(int double_quant, const uint8_t* codes, const uint8_t* scale_codes, const float* scales,
                 const float* mean) {
  if (double_quant != 0 && double_quant != 1) return fail(QNF4_ERR_INVALID, "double_quant must be 0 or 1");
  if (!codes || !scales || (double_quant && (!scale_codes || !mean))) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (!aligned(codes, 16)) return fail(QNF4_ERR_UNSUPPORTED, "codes need 16 B alignment");
  return QNF4_OK;
}

}  // namespace

// ---------------------------------------------------------------------------------------
// Library-owned quantization scratch (nf4_quantize_dq_noalloc)
// ---------------------------------------------------------------------------------------
// For callers that cannot allocate device memory when they quantize (a host program handed
// only the weight and output buffers, or a runtime whose device memory is all reserved for
// its own pool), the absmax and group-sum scratch of the quantizer lives in this static
// array: QNF4_NOALLOC_MAX_NUMEL / 64 fp32 absmax values, then the float64 group sums.  The
// CUDA runtime reserves it on each device when it loads this module there.
namespace {
constexpr int64_t kNoAllocBlocks = QNF4_NOALLOC_MAX_NUMEL / 64;
constexpr int64_t kNoAllocGroups = (kNoAllocBlocks + 255) / 256;
constexpr size_t kNoAllocAbsmaxBytes = (size_t)kNoAllocBlocks * 4;
constexpr size_t kNoAllocScratchBytes = kNoAllocAbsmaxBytes + (size_t)kNoAllocGroups * 8;
static_assert(QNF4_NOALLOC_MAX_NUMEL % 64 == 0 && kNoAllocAbsmaxBytes % 256 == 0, "scratch layout");
}  // namespace

static __device__ __align__(256) unsigned char g_quant_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
struct NoAllocSlot {
  CUcontext ctx;   // context the address was looked up in
  void* ptr;       // device address of g_quant_scratch in that context
};
NoAllocSlot g_noalloc_scratch[kNoAllocMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

// Set-up per device: with that device current, look up the scratch's device address.  The
// address belongs to the device's current context, so it is looked up again whenever that
// context differs from the one it was found in (after a cudaDeviceReset, for instance).
int noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(QNF4_ERR_UNSUPPORTED, "device ordinal %d: the static scratch supports devices 0..%d", dev,
                kNoAllocMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocSlot& slot = g_noalloc_scratch[dev];
  const CUcontext ctx = current_context();
  if (!slot.ptr || !ctx || slot.ctx != ctx) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_quant_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the quantization scratch");
    slot.ptr = ptr;
    slot.ctx = current_context();   // the lookup has made the device's context current
  }
  *out = slot.ptr;
  return QNF4_OK;
}
}  // namespace

extern "C" {

int qnf4_version(void) { return 100; }

int qnf4_set_timing_events(void* const* events, int n) {
  if (n < 0) return fail(QNF4_ERR_INVALID, "n must be >= 0");
  g_events = (n > 0) ? events : nullptr;
  g_n_events = (events && n > 0) ? n : 0;
  return QNF4_OK;
}

const char* qnf4_last_error(void) { return g_last_error.c_str(); }

int qnf4_device_error(void* stream, uint32_t* word) {
  if (!word) return fail(QNF4_ERR_INVALID, "word is NULL");
  cudaError_t e = qnf4::read_and_clear_error_word(word, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (*word) return fail(QNF4_ERR_DEVICE, "a kernel gave up waiting (flags 0x%x)", *word);
  return QNF4_OK;
}

namespace qnf4 {
// The bounded-wait self-test: one thread waits on an mbarrier that nothing arrives at, through
// the same helper every pipeline wait uses, so the wait must give up after `limit_ns`, raise its
// flag in the device error word and return.
__global__ void selftest_bounded_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile uint32_t* abort_word = &abort_flag;
    (void)mbar_wait_thread(&bar, 0u, abort_word, kErrWaitSelfTest, limit_ns);
  }
}
}  // namespace qnf4

int qnf4_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  g_last_error.clear();
  if (limit_ns < 1000000ull || limit_ns > 10000000000ull)
    return fail(QNF4_ERR_INVALID, "limit_ns must lie in [1 ms, 10 s]");
  if (int rc = check_arch()) return rc;
  qnf4::selftest_bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return QNF4_OK;
}

size_t nf4_quantize_workspace_bytes(int64_t numel) { return qnf4_quantize_workspace_bytes_ex(numel, 1); }

size_t qnf4_quantize_workspace_bytes_ex(int64_t numel, int double_quant) {
  if (numel <= 0) return 0;
  const int64_t nb = (numel + 63) / 64, ng = (nb + 255) / 256;
  if (!double_quant) return 256;   // the absmax values are the outputs; nothing else is needed
  return align_up((size_t)nb * 4, 256) + (size_t)ng * 8;
}

}  // extern "C"

namespace {

// Quantize into caller buffers; absmax / gsum are the scratch of double quantization (unused
// without it: the block absmax values go straight to `scales`).
int quantize_impl(const uint16_t* W, int64_t numel, int codebook, int double_quant, uint8_t* codes,
                  uint8_t* scale_codes, float* scales, float* mean, float* absmax, double* gsum, cudaStream_t st) {
  qnf4::Codebook cb;
  if (int rc = get_codebook(codebook, &cb)) return rc;
  CUtensorMap wmap;
  const bool has_map = numel >= 64;
  if (has_map)
    if (int rc = make_map(&wmap, W, true, 64, (uint64_t)(numel / 64), 128, 64, 256)) return rc;
  cudaError_t e = double_quant
                      ? qnf4::launch_quantize(has_map ? &wmap : nullptr, W, numel, cb, codes, scale_codes, scales, mean,
                                              absmax, gsum, st, 0)
                      : qnf4::launch_quantize(has_map ? &wmap : nullptr, W, numel, cb, codes, nullptr, nullptr,
                                              nullptr, scales, nullptr, st, 0);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return QNF4_OK;
}

int check_quantize_args(const uint16_t* W, int64_t numel, int double_quant, uint8_t* codes, uint8_t* scale_codes,
                        float* scales, float* mean) {
  if (!W) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (int rc = check_format(double_quant, codes, scale_codes, scales, mean)) return rc;
  if (numel <= 0) return fail(QNF4_ERR_INVALID, "numel must be positive");
  if (numel > (1ll << 35)) return fail(QNF4_ERR_UNSUPPORTED, "numel above 2^35");
  if (!aligned(W, 16) || (double_quant && !aligned(scale_codes, 8)))
    return fail(QNF4_ERR_UNSUPPORTED, "alignment: W and codes 16 B, scale_codes 8 B");
  return QNF4_OK;
}

}  // namespace

extern "C" {

int qnf4_quantize_ex(const uint16_t* W, int64_t numel, int codebook, int double_quant, uint8_t* codes,
                     uint8_t* scale_codes, float* scales, float* mean, void* workspace, size_t workspace_bytes,
                     void* stream) {
  g_last_error.clear();
  if (int rc = check_quantize_args(W, numel, double_quant, codes, scale_codes, scales, mean)) return rc;
  if (double_quant) {
    if (!workspace) return fail(QNF4_ERR_INVALID, "NULL pointer");
    if (!aligned(workspace, 256)) return fail(QNF4_ERR_UNSUPPORTED, "workspace needs 256-byte alignment");
    const size_t need = qnf4_quantize_workspace_bytes_ex(numel, 1);
    if (workspace_bytes < need) return fail(QNF4_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  }
  if (int rc = check_arch()) return rc;
  const int64_t nb = (numel + 63) / 64;
  float* absmax = double_quant ? static_cast<float*>(workspace) : nullptr;
  double* gsum = double_quant ? reinterpret_cast<double*>(static_cast<char*>(workspace) + align_up((size_t)nb * 4, 256))
                              : nullptr;
  return quantize_impl(W, numel, codebook, double_quant, codes, scale_codes, scales, mean, absmax, gsum,
                       static_cast<cudaStream_t>(stream));
}

int nf4_quantize_dq(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* scale_codes, float* c2, float* mean,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return qnf4_quantize_ex(W, numel, QNF4_CODEBOOK_NF4, 1, codes, scale_codes, c2, mean, workspace, workspace_bytes,
                          stream);
}

int nf4_quantize_dq_noalloc(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* scale_codes, float* c2,
                            float* mean, void* stream) {
  g_last_error.clear();
  if (numel > QNF4_NOALLOC_MAX_NUMEL)
    return fail(QNF4_ERR_UNSUPPORTED,
                "numel %lld is above the static scratch limit of %lld weights; use nf4_quantize_dq with a workspace",
                (long long)numel, (long long)QNF4_NOALLOC_MAX_NUMEL);
  if (int rc = check_quantize_args(W, numel, 1, codes, scale_codes, c2, mean)) return rc;
  if (int rc = check_arch()) return rc;
  void* scratch = nullptr;
  if (int rc = noalloc_scratch(&scratch)) return rc;
  // Same carving as nf4_quantize_dq's workspace; both parts are written before they are read.
  const int64_t nb = (numel + 63) / 64;
  float* absmax = static_cast<float*>(scratch);
  double* gsum = reinterpret_cast<double*>(static_cast<char*>(scratch) + align_up((size_t)nb * 4, 256));
  return quantize_impl(W, numel, QNF4_CODEBOOK_NF4, 1, codes, scale_codes, c2, mean, absmax, gsum,
                       static_cast<cudaStream_t>(stream));
}

int qnf4_dequant_ex(const uint8_t* codes, int codebook, int double_quant, const uint8_t* scale_codes,
                    const float* scales, const float* mean, int64_t numel, uint16_t* W_out, void* stream) {
  g_last_error.clear();
  if (!W_out) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (int rc = check_format(double_quant, codes, scale_codes, scales, mean)) return rc;
  if (numel <= 0) return fail(QNF4_ERR_INVALID, "numel must be positive");
  if (!aligned(W_out, 16)) return fail(QNF4_ERR_UNSUPPORTED, "codes and W_out need 16 B");
  qnf4::Codebook cb;
  if (int rc = get_codebook(codebook, &cb)) return rc;
  if (int rc = check_arch()) return rc;
  cudaError_t e = qnf4::launch_dequant(codes, scale_codes, scales, mean, numel, W_out, cb, double_quant ? 0 : 1,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
  return QNF4_OK;
}

int nf4_dequant(const uint8_t* codes, const uint8_t* scale_codes, const float* c2, const float* mean,
                int64_t numel, uint16_t* W_out, void* stream) {
  return qnf4_dequant_ex(codes, QNF4_CODEBOOK_NF4, 1, scale_codes, c2, mean, numel, W_out, stream);
}

int nf4_e4m3_encode(const float* v, int64_t n, uint8_t* out, int mode, void* stream) {
  g_last_error.clear();
  if (!v || !out) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (n <= 0) return fail(QNF4_ERR_INVALID, "n must be positive");
  if (mode != 0 && mode != 1) return fail(QNF4_ERR_INVALID, "mode must be 0 or 1");
  if (int rc = check_arch()) return rc;
  cudaError_t e = qnf4::launch_e4m3_encode(v, n, out, mode, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "e4m3 launch");
  return QNF4_OK;
}

int qnf4_paged_alloc(size_t bytes, void** ptr) {
  g_last_error.clear();
  if (!ptr) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (bytes == 0) return fail(QNF4_ERR_INVALID, "bytes must be positive");
  *ptr = nullptr;
  cudaError_t e = cudaMallocManaged(ptr, bytes, cudaMemAttachGlobal);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocManaged");
  return QNF4_OK;
}

int qnf4_paged_free(void* ptr) {
  g_last_error.clear();
  if (!ptr) return QNF4_OK;
  cudaError_t e = cudaFree(ptr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFree of managed memory");
  return QNF4_OK;
}

int qnf4_paged_prefetch(const void* ptr, size_t bytes, int to_device, void* stream) {
  g_last_error.clear();
  if (!ptr || bytes == 0) return fail(QNF4_ERR_INVALID, "NULL pointer or zero size");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaMemPrefetchAsync(ptr, bytes, to_device ? dev : cudaCpuDeviceId, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemPrefetchAsync");
  return QNF4_OK;
}

int qlora_adamw_step(float* param, const uint16_t* grad, float* m, float* v, uint16_t* param_bf16, int64_t n,
                     double lr, double beta1, double beta2, double eps, double weight_decay, int step,
                     void* stream) {
  g_last_error.clear();
  if (!param || !grad || !m || !v) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (n <= 0 || step <= 0) return fail(QNF4_ERR_INVALID, "n and step must be positive");
  if (!(beta1 >= 0.0 && beta1 < 1.0 && beta2 >= 0.0 && beta2 < 1.0))
    return fail(QNF4_ERR_INVALID, "betas must lie in [0, 1)");
  if (!aligned(param, 16) || !aligned(m, 16) || !aligned(v, 16) || !aligned(grad, 8) ||
      (param_bf16 && !aligned(param_bf16, 8)))
    return fail(QNF4_ERR_UNSUPPORTED, "alignment: param, m, v 16 B; grad and param_bf16 8 B");
  if (int rc = check_arch()) return rc;
  qnf4::AdamWArgs a;
  a.lr = (float)lr;
  a.b1 = (float)beta1;
  a.omb1 = (float)(1.0 - beta1);
  a.b2 = (float)beta2;
  a.omb2 = (float)(1.0 - beta2);
  a.eps = (float)eps;
  a.wd = (float)weight_decay;
  a.bc1 = (float)(1.0 - std::pow(beta1, (double)step));
  a.bc2 = (float)(1.0 - std::pow(beta2, (double)step));
  cudaError_t e = qnf4::launch_adamw(param, grad, m, v, param_bf16, n, a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "adamw launch");
  return QNF4_OK;
}

size_t qlora_merge_workspace_bytes(int64_t N, int64_t K, int double_quant, int merged_out_given) {
  if (N <= 0 || K <= 0) return 0;
  const size_t merged = merged_out_given ? 0 : align_up((size_t)N * (size_t)K * 2, 256);
  return merged + qnf4_quantize_workspace_bytes_ex(N * K, double_quant);
}

int qlora_merge_requantize(const uint8_t* codes, const uint8_t* scale_codes, const float* scales, const float* mean,
                           int64_t N, int64_t K, int codebook, int double_quant, const uint16_t* A, const uint16_t* B,
                           int r, float s, uint8_t* codes_out, uint8_t* scale_codes_out, float* scales_out,
                           float* mean_out, uint16_t* merged_out, void* workspace, size_t workspace_bytes,
                           void* stream) {
  g_last_error.clear();
  if (!A || !B || !workspace) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (int rc = check_format(double_quant, codes, scale_codes, scales, mean)) return rc;
  if (int rc = check_format(double_quant, codes_out, scale_codes_out, scales_out, mean_out)) return rc;
  if (N <= 0 || K <= 0 || r <= 0) return fail(QNF4_ERR_INVALID, "sizes must be positive");
  if (K % 8 || r > 1024) return fail(QNF4_ERR_UNSUPPORTED, "K must be a multiple of 8 and r <= 1024");
  if (N * K > (1ll << 35)) return fail(QNF4_ERR_UNSUPPORTED, "N * K above 2^35");
  if (!aligned(workspace, 256) || (merged_out && !aligned(merged_out, 16)) ||
      (double_quant && !aligned(scale_codes_out, 8)))
    return fail(QNF4_ERR_UNSUPPORTED, "alignment: workspace 256 B, merged_out and codes 16 B, scale codes 8 B");
  const size_t need = qlora_merge_workspace_bytes(N, K, double_quant, merged_out ? 1 : 0);
  if (workspace_bytes < need) return fail(QNF4_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  qnf4::Codebook cb;
  if (int rc = get_codebook(codebook, &cb)) return rc;
  if (int rc = check_arch()) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  uint16_t* merged = merged_out;
  if (!merged) {
    merged = reinterpret_cast<uint16_t*>(ws);
    ws += align_up((size_t)N * (size_t)K * 2, 256);
  }
  qnf4::MergeParams mp;
  memset(&mp, 0, sizeof(mp));
  mp.cb = cb;
  mp.codes = codes;
  mp.scale_codes = scale_codes;
  mp.scales = scales;
  mp.mean = mean;
  mp.scale_fp32 = double_quant ? 0 : 1;
  mp.N = N;
  mp.K = K;
  mp.A = A;
  mp.B = B;
  mp.r = r;
  mp.s = (double)s;
  mp.out = merged;
  cudaError_t e = qnf4::launch_merge_dense(mp, st);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  const int64_t numel = N * K, nb = (numel + 63) / 64;
  float* absmax = double_quant ? reinterpret_cast<float*>(ws) : nullptr;
  double* gsum = double_quant ? reinterpret_cast<double*>(ws + align_up((size_t)nb * 4, 256)) : nullptr;
  return quantize_impl(merged, numel, codebook, double_quant, codes_out, scale_codes_out, scales_out, mean_out, absmax,
                       gsum, st);
}

size_t qlora_linear_fwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r) {
  LinearShape s{M, K, N, r};
  if (M <= 0 || K <= 0 || N <= 0 || r <= 0) return 0;
  Carver c{nullptr};
  FwdWs w;
  return fwd_carve(c, s, plan_fwd(s), &w);
}

int qlora_linear_fwd(const uint16_t* x, int64_t M, int64_t K, int64_t N, const uint8_t* codes,
                     const uint8_t* scale_codes, const float* c2, const float* mean, const uint16_t* A,
                     const uint16_t* B, int r, float s, uint16_t* y, float* t_saved, void* workspace,
                     size_t workspace_bytes, void* stream) {
  return qlora_linear_fwd_ex(x, M, K, N, QNF4_CODEBOOK_NF4, 1, codes, scale_codes, c2, mean, A, B, r, s, y, t_saved,
                             workspace, workspace_bytes, stream);
}

int qlora_linear_fwd_ex(const uint16_t* x, int64_t M, int64_t K, int64_t N, int codebook, int double_quant,
                        const uint8_t* codes, const uint8_t* scale_codes, const float* c2, const float* mean,
                        const uint16_t* A, const uint16_t* B, int r, float s, uint16_t* y, float* t_saved,
                        void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  if (!x || !A || !B || !y || !t_saved || !workspace) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (int rc = check_format(double_quant, codes, scale_codes, c2, mean)) return rc;
  qnf4::Codebook cb;
  if (int rc = get_codebook(codebook, &cb)) return rc;
  LinearShape sh{M, K, N, r};
  if (int rc = check_linear_shape(sh)) return rc;
  if (!aligned(x, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(y, 16) || !aligned(codes, 16) ||
      !aligned(t_saved, 16) || !aligned(workspace, 256))
    return fail(QNF4_ERR_UNSUPPORTED, "alignment: operands 16 B, workspace 256 B");
  const FwdPlan plan = plan_fwd(sh);
  Carver c{static_cast<char*>(workspace)};
  FwdWs w;
  const size_t need = fwd_carve(c, sh, plan, &w);
  if (workspace_bytes < need) return fail(QNF4_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  if (int rc = check_arch()) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  mark(0, st);

  // 1) t = s x A^T: float64-accumulated partials, then t (fp32) and its bf16 hi / lo parts
  {
    const uint16_t* bt[1] = {A};
    if (int rc = run_lowrank(x, false, K, M, K * 2, bt, 1, K, K * 2, r, M, K, plan.t, w.partial, st)) return rc;
    cudaError_t e = qnf4::launch_finalize_tokens(w.partial, plan.t.splits, M, r, (double)s, t_saved, w.thi, w.tlo,
                                                 nullptr, 0, st);
    if (e != cudaSuccess) return cuda_fail(e, "finalize launch");
  }
  mark(1, st);
  // 2) y^T = W' x^T + B t_hi^T + B t_lo^T, W' dequantized on chip
  {
    qnf4::GemmParams gp;
    memset(&gp, 0, sizeof(gp));
    const bool generic = (K % 64 != 0);
    if (!generic) {
      if (int rc = make_map(&gp.maps[0], codes, false, K / 2, N, K / 2, 32, 128)) return rc;
    }
    const int bbox = b_box_rows(plan.bn);
    if (int rc = make_map(&gp.maps[1], x, true, K, M, K * 2, 64, bbox)) return rc;
    if (int rc = make_map(&gp.maps[2], B, true, r, N, (uint64_t)r * 2, 64, 128)) return rc;
    if (int rc = make_map(&gp.maps[3], w.thi, true, r, M, (uint64_t)r * 2, 64, bbox)) return rc;
    if (int rc = make_map(&gp.maps[4], w.tlo, true, r, M, (uint64_t)r * 2, 64, bbox)) return rc;
    gp.b_box_rows = bbox;
    nf4_operand(gp, cb, double_quant, codes, scale_codes, c2, mean, N, K);
    gp.nseg = 3;
    gp.seg[0] = qnf4::GemmSeg{kblocks(K), k16_last(K), qnf4::kANf4K, 0, 1, 0, 0, 0};
    gp.seg[1] = qnf4::GemmSeg{kblocks(r), k16_last(r), qnf4::kATmaK, 2, 3, 0, 0, 0};
    gp.seg[2] = qnf4::GemmSeg{kblocks(r), k16_last(r), qnf4::kATmaK, 2, 4, 0, 0, 0};
    if (kATmemForward && plan.bn == 256) {
      // 256-token tiles keep the dequantized W tile (and the adapter matrix rows) in tensor
      // memory, which leaves shared memory for 6 stages instead of 4
      gp.a_tmem = 1;
      gp.a_glob = B;
      gp.a_glob_ld = r;
      gp.a_glob_rows = N;
      gp.a_glob_cols = r;
    }
    gp.rows = (int32_t)N;
    gp.cols = (int32_t)M;
    gp.splits = plan.splits;
    gp.kb_per_split = (kblocks(K) + plan.splits - 1) / plan.splits;
    if (plan.splits > 1) {
      gp.epi = qnf4::kEpiF32T;
      gp.out = w.part;
      gp.ld_out = N;
      gp.split_stride = M * N;
    } else {
      gp.epi = qnf4::kEpiBf16T;
      gp.out = y;
      gp.ld_out = N;
    }
    cudaError_t e = launch_fused(gp, plan.bn, st);
    if (e != cudaSuccess) return cuda_fail(e, "fused forward launch");
    if (plan.splits > 1) {
      e = qnf4::launch_reduce_splits_bf16(w.part, plan.splits, M * N, M, N, N, y, N, st);
      if (e != cudaSuccess) return cuda_fail(e, "split reduce launch");
    }
  }
  mark(2, st);
  return QNF4_OK;
}

int qlora_linear_plan(int64_t M, int64_t K, int64_t N, int r, int* fwd_launches, int* bwd_launches,
                      int* fwd_splits, int* dx_splits) {
  g_last_error.clear();
  LinearShape sh{M, K, N, r};
  if (int rc = check_linear_shape(sh)) return rc;
  const FwdPlan f = plan_fwd(sh);
  const BwdPlan b = plan_bwd(sh);
  // forward: t, finalize, fused (+ split reduce); backward: B^T, t split, u, finalize,
  // fused dX (+ split reduce), dA, finalize, dB, finalize
  if (fwd_launches) *fwd_launches = 3 + (f.splits > 1 ? 1 : 0);
  if (bwd_launches) *bwd_launches = 9 + (b.splits > 1 ? 1 : 0);
  if (fwd_splits) *fwd_splits = f.splits;
  if (dx_splits) *dx_splits = b.splits;
  return QNF4_OK;
}

size_t qlora_linear_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r) {
  LinearShape s{M, K, N, r};
  if (M <= 0 || K <= 0 || N <= 0 || r <= 0) return 0;
  Carver c{nullptr};
  BwdWs w;
  return bwd_carve(c, s, plan_bwd(s), &w);
}

int qlora_linear_bwd(const uint16_t* dY, const uint16_t* x, const float* t_saved, int64_t M, int64_t K, int64_t N,
                     const uint8_t* codes, const uint8_t* scale_codes, const float* c2, const float* mean,
                     const uint16_t* A, const uint16_t* B, int r, float s, uint16_t* dX, uint16_t* dA,
                     uint16_t* dB, void* workspace, size_t workspace_bytes, void* stream) {
  return qlora_linear_bwd_ex(dY, x, t_saved, M, K, N, QNF4_CODEBOOK_NF4, 1, codes, scale_codes, c2, mean, A, B, r, s,
                             dX, dA, dB, workspace, workspace_bytes, stream);
}

int qlora_linear_bwd_ex(const uint16_t* dY, const uint16_t* x, const float* t_saved, int64_t M, int64_t K, int64_t N,
                        int codebook, int double_quant, const uint8_t* codes, const uint8_t* scale_codes,
                        const float* c2, const float* mean, const uint16_t* A, const uint16_t* B, int r, float s,
                        uint16_t* dX, uint16_t* dA, uint16_t* dB, void* workspace, size_t workspace_bytes,
                        void* stream) {
  g_last_error.clear();
  if (!dY || !x || !t_saved || !A || !B || !dA || !dB || !workspace) return fail(QNF4_ERR_INVALID, "NULL pointer");
  if (int rc = check_format(double_quant, codes, scale_codes, c2, mean)) return rc;
  qnf4::Codebook cb;
  if (int rc = get_codebook(codebook, &cb)) return rc;
  LinearShape sh{M, K, N, r};
  if (int rc = check_linear_shape(sh)) return rc;
  if (!aligned(dY, 16) || !aligned(x, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(codes, 16) ||
      !aligned(t_saved, 16) || !aligned(dA, 16) || !aligned(dB, 16) || (dX && !aligned(dX, 16)) ||
      !aligned(workspace, 256))
    return fail(QNF4_ERR_UNSUPPORTED, "alignment: operands 16 B, workspace 256 B");
  const BwdPlan plan = plan_bwd(sh);
  Carver c{static_cast<char*>(workspace)};
  BwdWs w;
  const size_t need = bwd_carve(c, sh, plan, &w);
  if (workspace_bytes < need) return fail(QNF4_ERR_WORKSPACE, "workspace needs %zu bytes", need);
  if (int rc = check_arch()) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t ldM = ld8(M);
  cudaError_t e;
  mark(0, st);

  // 1) B^T [r][N]; t split into three exact bf16 terms, transposed [3][r][M]
  e = qnf4::launch_transpose_bf16(B, N, r, w.Bt, N, st);
  if (e != cudaSuccess) return cuda_fail(e, "transpose launch");
  e = qnf4::launch_split3_T(t_saved, M, r, w.tT3, ldM, st);
  if (e != cudaSuccess) return cuda_fail(e, "split launch");
  mark(1, st);

  // 2) u = s dY B (float64-accumulated): hi / lo [M][r] for dX, three terms [3][r][M] for dA
  {
    const uint16_t* bt[1] = {w.Bt};
    if (int rc = run_lowrank(dY, false, N, M, N * 2, bt, 1, N, N * 2, r, M, N, plan.u, w.partial, st)) return rc;
    e = qnf4::launch_finalize_tokens(w.partial, plan.u.splits, M, r, (double)s, nullptr, w.uhi, w.ulo, w.uT3, ldM,
                                     st);
    if (e != cudaSuccess) return cuda_fail(e, "finalize launch");
  }
  mark(2, st);
  // 3) dX^T = W'^T dY^T + A^T u_hi^T + A^T u_lo^T
  if (dX) {
    qnf4::GemmParams gp;
    memset(&gp, 0, sizeof(gp));
    const bool generic = (K % 64 != 0);
    if (!generic) {
      if (int rc = make_map(&gp.maps[0], codes, false, K / 2, N, K / 2, 64, 64)) return rc;
    }
    const int bbox = b_box_rows(plan.bn);
    if (int rc = make_map(&gp.maps[1], dY, true, N, M, N * 2, 64, bbox)) return rc;
    if (int rc = make_map(&gp.maps[2], A, true, K, r, K * 2, 64, 64)) return rc;
    if (int rc = make_map(&gp.maps[3], w.uhi, true, r, M, (uint64_t)r * 2, 64, bbox)) return rc;
    if (int rc = make_map(&gp.maps[4], w.ulo, true, r, M, (uint64_t)r * 2, 64, bbox)) return rc;
    gp.b_box_rows = bbox;
    nf4_operand(gp, cb, double_quant, codes, scale_codes, c2, mean, N, K);
    gp.nseg = 3;
    gp.seg[0] = qnf4::GemmSeg{kblocks(N), k16_last(N), qnf4::kANf4MN, 0, 1, 0, 0, 0};
    gp.seg[1] = qnf4::GemmSeg{kblocks(r), k16_last(r), qnf4::kATmaMN, 2, 3, 0, 0, 0};
    gp.seg[2] = qnf4::GemmSeg{kblocks(r), k16_last(r), qnf4::kATmaMN, 2, 4, 0, 0, 0};
    gp.rows = (int32_t)K;
    gp.cols = (int32_t)M;
    gp.splits = plan.splits;
    gp.kb_per_split = (kblocks(N) + plan.splits - 1) / plan.splits;
    if (plan.splits > 1) {
      gp.epi = qnf4::kEpiF32T;
      gp.out = w.partX;
      gp.ld_out = K;
      gp.split_stride = M * K;
    } else {
      gp.epi = qnf4::kEpiBf16T;
      gp.out = dX;
      gp.ld_out = K;
    }
    e = launch_fused(gp, plan.bn, st);
    if (e != cudaSuccess) return cuda_fail(e, "fused dX launch");
    if (plan.splits > 1) {
      e = qnf4::launch_reduce_splits_bf16(w.partX, plan.splits, M * K, M, K, K, dX, K, st);
      if (e != cudaSuccess) return cuda_fail(e, "split reduce launch");
    }
  }
  mark(3, st);
  // 4) dA^T = x^T u (u as three terms), reduced over the M tokens
  {
    const uint16_t* bt[3] = {w.uT3, w.uT3 + (size_t)r * ldM, w.uT3 + (size_t)2 * r * ldM};
    if (int rc = run_lowrank(x, true, K, M, K * 2, bt, 3, M, ldM * 2, r, K, M, plan.a, w.partial, st)) return rc;
    e = qnf4::launch_finalize_grad(w.partial, plan.a.splits, r, K, dA, 0, st);
    if (e != cudaSuccess) return cuda_fail(e, "dA finalize launch");
  }
  mark(4, st);
  // 5) dB = dY^T t (t as three terms), reduced over the M tokens
  {
    const uint16_t* bt[3] = {w.tT3, w.tT3 + (size_t)r * ldM, w.tT3 + (size_t)2 * r * ldM};
    if (int rc = run_lowrank(dY, true, N, M, N * 2, bt, 3, M, ldM * 2, r, N, M, plan.b, w.partial, st)) return rc;
    e = qnf4::launch_finalize_grad(w.partial, plan.b.splits, r, N, dB, 1, st);
    if (e != cudaSuccess) return cuda_fail(e, "dB finalize launch");
  }
  mark(5, st);
  return QNF4_OK;
}

}  // extern "C"
