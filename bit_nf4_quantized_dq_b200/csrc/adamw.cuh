// AdamW step on the LoRA parameters (the optimizer whose states the paged optimizer keeps in
// unified memory).  "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and
// Paged Optimizers" (fullstackaihub), section 5; "QLoRA, explained." step 6.
//
// AdamW with decoupled weight decay, fp32 parameters and states, bf16 gradients:
//   m = b1 m + (1 - b1) g,  v = b2 v + (1 - b2) g^2,
//   p = p - lr ( (m / bc1) / (sqrt(v / bc2) + eps) + wd p ),  bc1 = 1 - b1^t, bc2 = 1 - b2^t.
// Optionally also writes the updated parameters as bf16 (the adapters' compute copy).
// An HBM stream: four elements per thread and iteration (16-byte loads of p, m, v).
#pragma once

#include "common.cuh"

namespace qnf4 {

// Every constant is the fp32 rounding of a value the host formed in double: in particular
// omb1 = 1 - b1 and omb2 = 1 - b2 (forming 1 - b2 in fp32 from an fp32 b2 = 0.999 would miss
// the true 0.001 by about 1.3e-5 relative).
struct AdamWArgs {
  float lr, b1, omb1, b2, omb2, eps, wd, bc1, bc2;
};

__device__ __forceinline__ void adamw_one(float& p, float g, float& m, float& v, const AdamWArgs& a) {
  m = __fmaf_rn(a.b1, m, __fmul_rn(a.omb1, g));
  v = __fmaf_rn(a.b2, v, __fmul_rn(a.omb2, __fmul_rn(g, g)));
  const float mhat = __fdiv_rn(m, a.bc1);
  const float vhat = __fdiv_rn(v, a.bc2);
  const float upd = __fadd_rn(__fdiv_rn(mhat, __fadd_rn(__fsqrt_rn(vhat), a.eps)), __fmul_rn(a.wd, p));
  p = __fsub_rn(p, __fmul_rn(a.lr, upd));
}

__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const uint16_t* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    uint16_t* __restrict__ p_bf16, int64_t n, const AdamWArgs a) {
  const int64_t n4 = n / 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 pp = reinterpret_cast<float4*>(p)[i];
    float4 mm = reinterpret_cast<float4*>(m)[i];
    float4 vv = reinterpret_cast<float4*>(v)[i];
    const uint2 gg = reinterpret_cast<const uint2*>(g)[i];
    adamw_one(pp.x, __uint_as_float(gg.x << 16), mm.x, vv.x, a);
    adamw_one(pp.y, __uint_as_float(gg.x & 0xFFFF0000u), mm.y, vv.y, a);
    adamw_one(pp.z, __uint_as_float(gg.y << 16), mm.z, vv.z, a);
    adamw_one(pp.w, __uint_as_float(gg.y & 0xFFFF0000u), mm.w, vv.w, a);
    reinterpret_cast<float4*>(p)[i] = pp;
    reinterpret_cast<float4*>(m)[i] = mm;
    reinterpret_cast<float4*>(v)[i] = vv;
    if (p_bf16) reinterpret_cast<uint2*>(p_bf16)[i] = make_uint2(pack_bf16x2(pp.x, pp.y), pack_bf16x2(pp.z, pp.w));
  }
  // the tail of n % 4 elements
  for (int64_t i = 4 * n4 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    float pp = p[i], mm = m[i], vv = v[i];
    adamw_one(pp, __uint_as_float((uint32_t)g[i] << 16), mm, vv, a);
    p[i] = pp;
    m[i] = mm;
    v[i] = vv;
    if (p_bf16) p_bf16[i] = __bfloat16_as_ushort(__float2bfloat16_rn(pp));
  }
}

static cudaError_t launch_adamw(float* p, const uint16_t* g, float* m, float* v, uint16_t* p_bf16, int64_t n,
                                const AdamWArgs& a, cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (n / 4 + 255) / 256;
  if (blocks > 8 * (int64_t)sms) blocks = 8 * (int64_t)sms;
  if (blocks < 1) blocks = 1;
  adamw_kernel<<<(unsigned)blocks, 256, 0, st>>>(p, g, m, v, p_bf16, n, a);
  return cudaGetLastError();
}

}  // namespace qnf4
