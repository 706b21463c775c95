// One AdamW step on the adapter parameters with 8-bit block-wise moments (the recipe's bitsandbytes
// 8-bit AdamW, Show HN: LoRA over GGUF, "Things involved in the training"; AdamW with decoupled
// weight decay, states block-wise quantized with dynamic tree codes as in the 8-bit optimizers
// paper). The layout and code tables are described with qlora_adamw8_step in qlora.h.
//
// One CTA of 256 threads per block of 256 values, one value per thread: decode m and v (absmax times
// the code's table entry), update them and the parameter in fp32, take the block's new absmax of |m|
// and of v by warp and CTA max-reductions, and store each value's nearest code. Every fp32 operation
// is written out with an explicit rounding mode (no fused multiply-add), so the arithmetic, and with
// it every code decision, is the same as any other fp32 evaluation in the same order.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace qlora {

constexpr int kAdamBlock = 256;

// Code tables, built on the host: dec[q] = table entry of code q; srt / cod = the distinct entries in
// ascending order and the code each stands for (n of them).
struct Adamw8Tables {
  float dec_s[256], dec_u[256];
  float srt_s[256], srt_u[256];
  uint8_t cod_s[256], cod_u[256];
  int ns, nu;
};

struct Adamw8Args {
  float lr, b1, b2, eps, wd, c1, c2;
};

// Nearest code of y: the entry minimizing |y - entry| in fp32, equal distances to the smaller entry.
__device__ __forceinline__ uint8_t adamw8_nearest(float y, const float* srt, const uint8_t* cod, int n) {
  int lo = 0, hi = n - 1;  // last index with srt[idx] <= y (0 if none)
  if (y <= srt[0]) return cod[0];
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (srt[mid] <= y) lo = mid; else hi = mid - 1;
  }
  if (lo + 1 < n) {
    const float dl = __fsub_rn(y, srt[lo]);
    const float dh = __fsub_rn(srt[lo + 1], y);
    if (dh < dl) return cod[lo + 1];
  }
  return cod[lo];
}

__device__ __forceinline__ float block_max256(float x, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = x;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kAdamBlock / 32; ++w) r = fmaxf(r, red[w]);
  return r;
}

__global__ void __launch_bounds__(kAdamBlock) adamw8_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                            uint8_t* __restrict__ mq, float* __restrict__ mabs,
                                                            uint8_t* __restrict__ vq, float* __restrict__ vabs,
                                                            long n, Adamw8Args a,
                                                            const __grid_constant__ Adamw8Tables T,
                                                            __nv_bfloat16* __restrict__ pb) {
  __shared__ float s_dec_s[256], s_dec_u[256], s_srt_s[256], s_srt_u[256];
  __shared__ uint8_t s_cod_s[256], s_cod_u[256];
  __shared__ float s_red[2][kAdamBlock / 32];
  const int tid = threadIdx.x;
  s_dec_s[tid] = T.dec_s[tid];
  s_dec_u[tid] = T.dec_u[tid];
  s_srt_s[tid] = T.srt_s[tid];
  s_srt_u[tid] = T.srt_u[tid];
  s_cod_s[tid] = T.cod_s[tid];
  s_cod_u[tid] = T.cod_u[tid];
  const long blk = blockIdx.x;
  const long i = blk * kAdamBlock + tid;
  const bool valid = i < n;
  const float am = mabs[blk], av = vabs[blk];
  __syncthreads();
  float m = 0.f, v = 0.f;
  if (valid) {
    m = __fmul_rn(am, s_dec_s[mq[i]]);
    v = __fmul_rn(av, s_dec_u[vq[i]]);
    const float gi = g[i], pi = p[i];
    m = __fadd_rn(__fmul_rn(a.b1, m), __fmul_rn(__fsub_rn(1.0f, a.b1), gi));
    v = __fadd_rn(__fmul_rn(a.b2, v), __fmul_rn(__fsub_rn(1.0f, a.b2), __fmul_rn(gi, gi)));
    const float mh = __fdiv_rn(m, a.c1);
    const float vh = __fdiv_rn(v, a.c2);
    const float den = __fadd_rn(__fsqrt_rn(vh), a.eps);
    const float upd = __fadd_rn(__fdiv_rn(mh, den), __fmul_rn(a.wd, pi));
    const float pn = __fsub_rn(pi, __fmul_rn(a.lr, upd));
    p[i] = pn;
    if (pb != nullptr) pb[i] = __float2bfloat16_rn(pn);
  }
  const float am2 = block_max256(fabsf(m), s_red[0]);
  const float av2 = block_max256(fabsf(v), s_red[1]);
  if (tid == 0) {
    mabs[blk] = am2;
    vabs[blk] = av2;
  }
  if (valid) {
    const float ym = am2 > 0.f ? __fdiv_rn(m, am2) : 0.f;
    const float yv = av2 > 0.f ? __fdiv_rn(v, av2) : 0.f;
    mq[i] = adamw8_nearest(ym, s_srt_s, s_cod_s, T.ns);
    vq[i] = adamw8_nearest(yv, s_srt_u, s_cod_u, T.nu);
  }
}

}  // namespace qlora
