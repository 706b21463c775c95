// RMSNorm in front of the layer's first projection (the recipe takes its RMSNorm from Liger, Show HN: LoRA over
// GGUF, "Things involved in the training"): x_n = x r g with r = 1 / sqrt(mean(x^2) + eps) and a
// frozen gain g. One warp per token row, 16-byte loads: the forward reads x once for the sum of
// squares and once more (from L2) to write the projection's bf16 input x_n and r; the backward forms
// dL/dx = r g d - (r^3 x / K) sum(x g d) with d = dL/dx_n in one pass over the row.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "decode.cuh"
#include "lora.cuh"
#include "qlora.h"

namespace qlora {

__global__ void rmsnorm_fwd_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ g, int M,
                                   int K, float eps, __nv_bfloat16* __restrict__ Xn, float* __restrict__ rstd) {
  const int warp = (int)((blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (warp >= M) return;
  const uint4* x4 = reinterpret_cast<const uint4*>(X + (long)warp * K);
  const uint4* g4 = reinterpret_cast<const uint4*>(g);
  const int n8 = K / 8;
  float ss = 0.f;
  for (int c = lane; c < n8; c += 32) {
    float f[8];
    bf16x8_to_f32(__ldg(x4 + c), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = 1.0f / sqrtf(ss / (float)K + eps);
  if (lane == 0) rstd[warp] = r;
  uint4* o4 = reinterpret_cast<uint4*>(Xn + (long)warp * K);
  for (int c = lane; c < n8; c += 32) {
    float f[8], gg[8], y[8];
    bf16x8_to_f32(__ldg(x4 + c), f);
    bf16x8_to_f32(__ldg(g4 + c), gg);
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = f[i] * r * gg[i];
    o4[c] = pack_bf16x8(y);
  }
}

__global__ void rmsnorm_bwd_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ g,
                                   const float* __restrict__ rstd, const void* __restrict__ dXn, int dxn_dtype, int M,
                                   int K, void* __restrict__ dX, int dx_dtype) {
  const int warp = (int)((blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (warp >= M) return;
  const uint4* x4 = reinterpret_cast<const uint4*>(X + (long)warp * K);
  const uint4* g4 = reinterpret_cast<const uint4*>(g);
  const int n8 = K / 8;
  auto load_d = [&](int c, float (&d)[8]) {
    if (dxn_dtype == QL_F32) {
      const float4* d4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(dXn) + (long)warp * K) + 2 * c;
      const float4 a = __ldg(d4), b = __ldg(d4 + 1);
      d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w; d[4] = b.x; d[5] = b.y; d[6] = b.z; d[7] = b.w;
    } else {
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(dXn) +
                                                          (long)warp * K) + c), d);
    }
  };
  float s = 0.f;
  for (int c = lane; c < n8; c += 32) {
    float f[8], gg[8], d[8];
    bf16x8_to_f32(__ldg(x4 + c), f);
    bf16x8_to_f32(__ldg(g4 + c), gg);
    load_d(c, d);
#pragma unroll
    for (int i = 0; i < 8; ++i) s = fmaf(f[i] * gg[i], d[i], s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float r = rstd[warp];
  const float c3 = r * r * r * s / (float)K;
  for (int c = lane; c < n8; c += 32) {
    float f[8], gg[8], d[8], y[8];
    bf16x8_to_f32(__ldg(x4 + c), f);
    bf16x8_to_f32(__ldg(g4 + c), gg);
    load_d(c, d);
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = r * gg[i] * d[i] - c3 * f[i];
    if (dx_dtype == QL_F32) {
      float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(dX) + (long)warp * K) + 2 * c;
      o[0] = make_float4(y[0], y[1], y[2], y[3]);
      o[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else {
      reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dX) + (long)warp * K)[c] = pack_bf16x8(y);
    }
  }
}

}  // namespace qlora
