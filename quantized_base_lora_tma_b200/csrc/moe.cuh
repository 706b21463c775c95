// Routed MoE helpers: routing (top-k, counts, scan, permutation), gathers and the slot-ordered
// combine. "MoE routing like OpenAI triton-kernels" (Show HN: LoRA over GGUF, "Things involved in
// the training"); only the selected experts' weights are read and their outputs are summed per
// token ("sparse reduce", ai-manual.ru, "Fused dequant-matmul и MoE kernels").
//
// Routing of token t over E experts: the k largest logits, equal logits going to the lower expert
// index, in descending order (slot 0 = largest); weight of slot j = softmax over the k selected
// logits. Pairs (t, j) are numbered t*k + j and sorted by (expert, token, slot): perm[pos] = pair,
// inv_perm[pair] = pos. counts[e], offsets[e] (exclusive scan, offsets[E] = T*k) and
// mblk[e] = sum_{e' < e} ceil(counts[e'] / 128) (the grouped GEMM's 128-row block list) follow.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace qlora {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 16;

// One warp per token. E <= 256, k <= 16.
__global__ void moe_topk_kernel(const __nv_bfloat16* __restrict__ logits, int T, int E, int k,
                                int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                int32_t* __restrict__ counts) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const __nv_bfloat16* l = logits + (long)warp * E;
  float v[kMaxExperts / 32];
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __bfloat162float(l[e]) : -INFINITY;
  }
  float sel_v[kMaxTopK];
  int sel_e[kMaxTopK];
  for (int j = 0; j < k; ++j) {
    // lane-local best: larger value, then lower index (indices increase with i)
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const int e = lane + 32 * i;
      if (e < E && (v[i] > bv || (v[i] == bv && e < be))) { bv = v[i]; be = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    sel_v[j] = bv;
    sel_e[j] = be;
    // a selected expert can never be selected again: mark it below every finite logit
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i)
      if (lane + 32 * i == be) v[i] = -INFINITY;
  }
  if (lane == 0) {
    const float vmax = sel_v[0];
    float w[kMaxTopK];
    float sum = 0.f;
    for (int j = 0; j < k; ++j) {
      w[j] = expf(sel_v[j] - vmax);
      sum += w[j];
    }
    const float inv = 1.0f / sum;
    for (int j = 0; j < k; ++j) {
      topk_idx[(long)warp * k + j] = sel_e[j];
      topk_w[(long)warp * k + j] = w[j] * inv;
      atomicAdd(counts + sel_e[j], 1);  // a count: the order of the additions does not matter
    }
  }
}

// One CTA (1024 threads) per expert e: offsets[e] and mblk[e] from the counts of the experts before
// it, then e's pairs in token order: perm[offsets[e] + rank] = t*k + j and its inverse, where rank
// counts the earlier tokens that selected e (block-wide ballot prefix sums over 1024 tokens at a
// time). CTA 0 also writes offsets[E] and mblk[E].
__global__ void __launch_bounds__(1024) moe_place_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                                                         const int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets, int32_t* __restrict__ mblk,
                                                         int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
  __shared__ int s_base;
  __shared__ int s_warp[32];
  const int e = blockIdx.x;
  if (threadIdx.x == 0) {
    int o = 0, mb = 0;
    for (int q = 0; q < e; ++q) {
      const int c = counts[q];
      o += c;
      mb += (c + 127) / 128;
    }
    offsets[e] = o;
    mblk[e] = mb;
    if (e == 0) {
      int ot = 0, mt = 0;
      for (int q = 0; q < E; ++q) {
        const int c = counts[q];
        ot += c;
        mt += (c + 127) / 128;
      }
      offsets[E] = ot;
      mblk[E] = mt;
    }
    s_base = o;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t0 = 0; t0 < T; t0 += 1024) {
    const int t = t0 + threadIdx.x;
    int slot = -1;
    if (t < T)
      for (int j = 0; j < k; ++j)
        if (topk_idx[(long)t * k + j] == e) slot = j;
    const uint32_t b = __ballot_sync(0xffffffffu, slot >= 0);
    if (lane == 0) s_warp[warp] = __popc(b);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = s_warp[w];
      if (w < warp) before += c;
      total += c;
    }
    if (slot >= 0) {
      const int pos = s_base + before + __popc(b & ((1u << lane) - 1u));
      perm[pos] = t * k + slot;
      inv_perm[t * k + slot] = pos;
    }
    __syncthreads();
    if (threadIdx.x == 0) s_base += total;
    __syncthreads();
  }
}

// Row gather in pair order: dst[p] = src[perm[p] / k] (bf16 rows of `cols`), and optionally the
// routing weight of each pair, row_w[p] = topk_w[perm[p]].
__global__ void moe_gather_rows_kernel(const __nv_bfloat16* __restrict__ src, int cols, const int32_t* __restrict__ perm,
                                       int P, int k, __nv_bfloat16* __restrict__ dst, const float* __restrict__ topk_w,
                                       float* __restrict__ row_w) {
  const int vec = cols / 8;
  const long total = (long)P * vec;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int p = (int)(i / vec), q = (int)(i % vec);
    const int pair = min(max(__ldg(perm + p), 0), P - 1);  // defensive: never leave the buffers
    const int t = pair / k;
    reinterpret_cast<uint4*>(dst + (long)p * cols)[q] = __ldg(reinterpret_cast<const uint4*>(src + (long)t * cols) + q);
    if (q == 0 && row_w != nullptr) row_w[p] = __ldg(topk_w + pair);
  }
}

// Slot-ordered combine: out[t] = sum_{j < k} rows[inv_perm[t*k + j]] (fp32 rows, fp32 sum in
// slot order).
__global__ void moe_combine_kernel(const float* __restrict__ rows, int cols, const int32_t* __restrict__ inv_perm,
                                   int T, int k, void* __restrict__ out, int out_dtype) {
  const int vec = cols / 4;
  const long total = (long)T * vec;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int t = (int)(i / vec), q = (int)(i % vec);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      const int p = min(max(__ldg(inv_perm + (long)t * k + j), 0), T * k - 1);
      const float4 v = __ldg(reinterpret_cast<const float4*>(rows + (long)p * cols) + q);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (out_dtype == QL_F32) {
      reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + (long)t * cols)[q] = acc;
    } else {
      const __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y);
      const __nv_bfloat162 b = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 r;
      r.x = *reinterpret_cast<const uint32_t*>(&a);
      r.y = *reinterpret_cast<const uint32_t*>(&b);
      reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + (long)t * cols)[q] = r;
    }
  }
}

// Per-pair dot products dw[p] = sum over the tiles of dw_part[p][tile]; and the router-logit
// gradient of the selected experts: for token t, d_l[t][e_j] = w_j (dw_j - sum_i w_i dw_i),
// zero for unselected experts (d_logits may be NULL).
__global__ void moe_dw_dlogits_kernel(const float* __restrict__ dw_part, int ntiles, const int32_t* __restrict__ inv_perm,
                                      const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int E,
                                      int k, float* __restrict__ dw_pair_out, float* __restrict__ d_logits) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float dw[kMaxTopK];
  float s = 0.f;
  for (int j = 0; j < k; ++j) {
    const int p = inv_perm[(long)t * k + j];
    float a = 0.f;
    for (int q = 0; q < ntiles; ++q) a += dw_part[(long)p * ntiles + q];
    dw[j] = a;
    if (dw_pair_out) dw_pair_out[(long)t * k + j] = a;
    s += topk_w[(long)t * k + j] * a;
  }
  if (d_logits != nullptr) {
    for (int e = 0; e < E; ++e) d_logits[(long)t * E + e] = 0.f;
    for (int j = 0; j < k; ++j) {
      const float w = topk_w[(long)t * k + j];
      d_logits[(long)t * E + topk_idx[(long)t * k + j]] = w * (dw[j] - s);
    }
  }
}

}  // namespace qlora
