// Cross-entropy over the vocabulary for one chunk of token rows of an lm_head's fp32 logits (the
// recipe's chunked cross-entropy over the quantized matmul's logits, in the Liger manner, Show HN: LoRA over
// GGUF, "Things involved in the training"). A CTA takes rows in turn: an online max / sum of
// exponentials over the row (float4 loads), lse = max + log(sum), loss = lse - logit[label]; then, if
// asked, the gradient of the summed loss times grad_scale, (softmax - onehot(label)) * grad_scale, in
// bf16 for the input-gradient GEMM. A negative label marks an ignored token: loss 0 and a zero
// gradient row. Given the logits GEMM's per-tile row statistics (max, sum exp per 256 columns),
// the first pass is a merge of those and the logits are read once. Otherwise, one CTA per SM
// keeps the rows in flight (one per SM, 4 bytes x V each) well inside L2, so the second pass over
// a row reads it from L2 rather than from DRAM.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace qlora {

constexpr int kCeThreads = 1024;
constexpr int kCeUnroll = 4;  // 16-byte loads per thread in flight (64 KB per SM)

__device__ __forceinline__ void ce_merge(float& m, float& s, float m2, float s2) {
  const float mm = fmaxf(m, m2);
  s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mm));
  m = mm;
}

__global__ void __launch_bounds__(kCeThreads, 1) lm_ce_kernel(const float* __restrict__ logits, int V, int rows,
                                                              const float2* __restrict__ stats, int ntiles,
                                                              const int32_t* __restrict__ labels, float grad_scale,
                                                              float* __restrict__ loss,
                                                              __nv_bfloat16* __restrict__ dlog) {
  __shared__ float s_m[kCeThreads / 32], s_s[kCeThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const float4* l4 = reinterpret_cast<const float4*>(logits + (long)row * V);
    const int lab = labels[row];
    float m = -INFINITY, s = 0.f;
    // with stats: the row's (max, sum exp) per column tile, merged in tile order per thread and
    // then across lanes and warps in a fixed order; without: one pass over the row
    if (stats != nullptr) {
      for (int i = tid; i < ntiles; i += kCeThreads) {
        const float2 t = __ldg(stats + (long)row * ntiles + i);
        ce_merge(m, s, t.x, t.y);
      }
    }
    // kCeUnroll independent 16-byte loads per thread in flight before any is used
    for (int c0 = tid; stats == nullptr && c0 < V / 4; c0 += kCeUnroll * kCeThreads) {
      float4 xv[kCeUnroll];
#pragma unroll
      for (int u = 0; u < kCeUnroll; ++u) {
        const int c = c0 + u * kCeThreads;
        xv[u] = c < V / 4 ? __ldg(l4 + c) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
#pragma unroll
      for (int u = 0; u < kCeUnroll; ++u) {
        const float xs[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (xs[i] > m) {
            s = (m == -INFINITY ? 0.f : s * expf(m - xs[i])) + 1.f;
            m = xs[i];
          } else if (xs[i] != -INFINITY) {
            s += expf(xs[i] - m);
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
      ce_merge(m, s, m2, s2);
    }
    __syncthreads();  // the previous row's readers of s_m / s_s are done
    if (lane == 0) {
      s_m[warp] = m;
      s_s[warp] = s;
    }
    __syncthreads();
    m = s_m[0];
    s = s_s[0];
    for (int w = 1; w < kCeThreads / 32; ++w) ce_merge(m, s, s_m[w], s_s[w]);
    const float lse = m + logf(s);
    if (tid == 0) loss[row] = lab >= 0 ? lse - logits[(long)row * V + lab] : 0.f;
    if (dlog == nullptr) continue;
    uint2* d2 = reinterpret_cast<uint2*>(dlog + (long)row * V);
    for (int c0 = tid; c0 < V / 4; c0 += kCeUnroll * kCeThreads) {
      float4 xv[kCeUnroll];
#pragma unroll
      for (int u = 0; u < kCeUnroll; ++u) {
        const int c = c0 + u * kCeThreads;
        xv[u] = c < V / 4 ? __ldg(l4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kCeUnroll; ++u) {
        const int c = c0 + u * kCeThreads;
        if (c >= V / 4) break;
        const float xs[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
        float d[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int v = 4 * c + i;
          d[i] = lab >= 0 ? (expf(xs[i] - lse) - (v == lab ? 1.f : 0.f)) * grad_scale : 0.f;
        }
        const __nv_bfloat162 a = __floats2bfloat162_rn(d[0], d[1]), b = __floats2bfloat162_rn(d[2], d[3]);
        d2[c] = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
      }
    }
  }
}

}  // namespace qlora
