// Routed MoE helpers: routing (top-k, counts, scan, permutation), gathers and the slot-ordered
// combine. The recipe's MoE routing, after OpenAI's Triton routing kernels (Show HN: LoRA over GGUF, "Things involved in
// the training"); only the selected experts' weights are read and their outputs are summed per
// token (a sparse reduction, ai-manual.ru, "Fused dequant-matmul и MoE kernels").
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

constexpr int kRouteRow = 32;  // tokens per histogram row: one warp's lanes

// Routing, first pass: one CTA of 32 warps per row of 32 tokens, one token per warp. The warp
// chooses the token's top-k (lane-local best of 8 logits, then a butterfly over the lanes: larger
// value wins, equal values go to the lower expert index); the weights are the softmax over the k
// selected logits. The row's per-expert histogram is built without atomics on global memory: for
// each slot, the lanes of warp 0 (one token each) that picked the same expert find each other with
// __match_any_sync and their leader adds the group's size to the shared histogram, which becomes
// row `blockIdx.x` of hist [rows x E].
__global__ void __launch_bounds__(1024) moe_route_select_kernel(const __nv_bfloat16* __restrict__ logits, int T,
                                                                int E, int k, int32_t* __restrict__ topk_idx,
                                                                float* __restrict__ topk_w,
                                                                int32_t* __restrict__ hist) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  __shared__ int s_hist[kMaxExperts];
  __shared__ uint8_t s_sel[kRouteRow][kMaxTopK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteRow + warp;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  if (t < T) {
    const __nv_bfloat16* l = logits + (long)t * E;
    float v[kMaxExperts / 32];
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < E ? __bfloat162float(l[e]) : -INFINITY;
    }
    float sel_v[kMaxTopK];
    int sel_e[kMaxTopK];
    for (int j = 0; j < k; ++j) {
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
#pragma unroll
      for (int i = 0; i < kMaxExperts / 32; ++i)  // never selected again
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
        topk_idx[(long)t * k + j] = sel_e[j];
        topk_w[(long)t * k + j] = w[j] * inv;
        s_sel[warp][j] = (uint8_t)sel_e[j];
      }
    }
  }
  __syncthreads();
  if (warp == 0) {  // lane = token of the row
    const bool has = blockIdx.x * kRouteRow + lane < T;
    for (int j = 0; j < k; ++j) {
      const int e = has ? (int)s_sel[lane][j] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (has && lane == __ffs(peers) - 1) atomicAdd(&s_hist[e], __popc(peers));
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(long)blockIdx.x * E + e] = s_hist[e];
}

// Routing, second pass (one CTA of 256 threads): thread e turns column e of the histogram table into
// its exclusive prefix over the rows (in place) and keeps the total; block scans over the experts
// give counts, offsets (offsets[E] = T k) and mblk.
__global__ void __launch_bounds__(kMaxExperts) moe_route_scan_kernel(int32_t* __restrict__ hist, int E, int nrow,
                                                                     int32_t* __restrict__ counts,
                                                                     int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ mblk) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  __shared__ int s_scan[kMaxExperts / 32 * 2];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int tot = 0;
  if (tid < E)
    for (int q0 = 0; q0 < nrow; q0 += 16) {  // 16 rows loaded together, then their prefixes stored
      int c[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) c[i] = q0 + i < nrow ? hist[(long)(q0 + i) * E + tid] : 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (q0 + i < nrow) hist[(long)(q0 + i) * E + tid] = tot;
        tot += c[i];
      }
    }
  // exclusive scans over e of tot and of ceil(tot / 128): warp scans, then over the 8 warps
  const int nb = (tot + 127) / 128;
  int x = tot, y = nb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xo = __shfl_up_sync(0xffffffffu, x, o), yo = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) { x += xo; y += yo; }
  }
  if (lane == 31) { s_scan[warp] = x; s_scan[kMaxExperts / 32 + warp] = y; }
  __syncthreads();
  int wx = 0, wy = 0;
  for (int w = 0; w < warp; ++w) { wx += s_scan[w]; wy += s_scan[kMaxExperts / 32 + w]; }
  if (tid < E) {
    const int off_e = wx + x - tot, mb_e = wy + y - nb;
    counts[tid] = tot;
    offsets[tid] = off_e;
    mblk[tid] = mb_e;
    if (tid == E - 1) {
      offsets[E] = off_e + tot;
      mblk[E] = mb_e + nb;
    }
  }
}

// Routing, third pass: 8 warps per CTA, warp = one row of 32 tokens (lane = token), placing the
// row's pairs in (expert, token, slot) order. A token picks an expert at most once, so the rank of
// pair (t, j) with expert e among e's pairs is the number of earlier tokens that picked e:
// offsets[e], plus e's pairs in the earlier rows (the scanned table), plus the earlier lanes of this
// row that picked e (the popcount of the row's lane mask of e, set by shared atomicOr).
__global__ void __launch_bounds__(256) moe_route_place_kernel(
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ hist, const int32_t* __restrict__ offsets,
    int T, int E, int k, int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  __shared__ uint32_t s_bits[8][kMaxExperts];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x * 8 + warp;
  const int t = row * kRouteRow + lane;
  const bool has = t < T;
  for (int i = lane; i < kMaxExperts; i += 32) s_bits[warp][i] = 0u;
  __syncwarp();
  int sel[kMaxTopK];
  for (int j = 0; j < k; ++j) {
    sel[j] = has ? __ldg(topk_idx + (long)t * k + j) : 0;
    if (has) atomicOr(&s_bits[warp][sel[j]], 1u << lane);
  }
  __syncwarp();
  if (!has) return;
  const uint32_t lt = (1u << lane) - 1u;
  for (int j = 0; j < k; ++j) {
    const int e = sel[j];
    const int r = __ldg(offsets + e) + __ldg(hist + (long)row * E + e) + __popc(s_bits[warp][e] & lt);
    perm[r] = t * k + j;
    inv_perm[(long)t * k + j] = r;
  }
}

// Row gather in pair order: dst[p] = src[perm[p] / k] (bf16 rows of `cols`), and optionally the
// routing weight of each pair, row_w[p] = topk_w[perm[p]].
__global__ void moe_gather_rows_kernel(const __nv_bfloat16* __restrict__ src, int cols, const int32_t* __restrict__ perm,
                                       int P, int k, __nv_bfloat16* __restrict__ dst, const float* __restrict__ topk_w,
                                       float* __restrict__ row_w) {
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
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
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
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
  pdl_wait();  // inputs come from earlier launches in the stream
  pdl_launch_dependents();
  // one warp per token: lane j < k takes slot j (its tile partials summed in tile order), the
  // weighted sum over slots is a fixed butterfly, and the lanes write the token's logit row
  const int t = (int)((blockIdx.x * (long)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float a = 0.f, w = 0.f;
  int sel = 0;
  if (lane < k) {
    const int p = inv_perm[(long)t * k + lane];
    for (int q = 0; q < ntiles; ++q) a += dw_part[(long)p * ntiles + q];
    w = topk_w[(long)t * k + lane];
    sel = topk_idx[(long)t * k + lane];
    if (dw_pair_out) dw_pair_out[(long)t * k + lane] = a;
  }
  float s = w * a;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (d_logits != nullptr) {
    for (int e = lane; e < E; e += 32) d_logits[(long)t * E + e] = 0.f;
    __syncwarp();  // the zeros are ordered before the selected entries
    if (lane < k) d_logits[(long)t * E + sel] = w * (a - s);
  }
}

}  // namespace qlora
