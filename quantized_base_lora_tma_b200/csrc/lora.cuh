// Adapter-side kernels of the layer (bandwidth-bound, CUDA cores, fp32 accumulation):
//
//   lora_rows      out[m, j] = oscale * sum_k Y[m, k] Z(j, k)        H = X A^T,  G = s dY B
//                  and the tensor-core operand LA[m] = [hi(v) | lo(v)], v = lscale * sum
//   lora_bop       LB[n] = [Z(n, :) | Z(n, :)]                        B (forward) or A^T (dX)
//   colred         part[slice, c, j] = sum_{m in slice} Y[m, c] Z[m, j]   then an ordered sum
//                  over slices: dB = s dY^T H, dA = G^T X (deterministic: no atomics)
//
// The fast LoRA backward these implement is the plain chain rule of the layer (Show HN: LoRA over
// GGUF, "Things involved in the training": "Fast LoRA bwd formula like Unsloth for linear layer
// and MoE layer"). Adapter gradients stay in fp32 end to end.
#pragma once
#include <cuda_bf16.h>

#include "decode.cuh"
#include "ptx.cuh"

namespace qlora {

__device__ __forceinline__ void bf16x8_to_f32(const uint4 q, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Row-wise reduction against a small [r x Kin] operand Z(j, k) = Z[j*zj + k*zk].
// One warp per row (ROWS rows per CTA of 8 warps); K in chunks of 256 staged in shared memory.
// Grouped use: zexp[row] picks the expert (Z advances by z_exp_stride per expert); NULL = dense.
// out: [M x r] fp32 (nullable); la: [M x 2RP] bf16 (nullable), RP = 32 * ceil(r / 32).
template <int RM>
__global__ void __launch_bounds__(256) lora_rows_kernel(const __nv_bfloat16* __restrict__ Y, long ldy, int M,
                                                        int Kin, const __nv_bfloat16* __restrict__ Z, long zj,
                                                        long zk, long z_exp_stride, const int* __restrict__ row_exp,
                                                        int r, float oscale, float lscale, float* __restrict__ out,
                                                        __nv_bfloat16* __restrict__ la, int RP) {
  __shared__ __align__(16) __nv_bfloat16 zs[RM * 256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  // rows of one CTA share an expert only in dense mode; grouped mode loads Z per warp
  const bool grouped = row_exp != nullptr;
  float acc[RM];
#pragma unroll
  for (int j = 0; j < RM; ++j) acc[j] = 0.f;
  const int e = (grouped && row < M) ? __ldg(row_exp + row) : 0;
  const __nv_bfloat16* Ze = Z + (long)e * z_exp_stride;
  for (int k0 = 0; k0 < Kin; k0 += 256) {
    if (!grouped) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < r * 256; idx += 256) {
        int j, kk;
        if (zk == 1) { j = idx / 256; kk = idx % 256; } else { j = idx % r; kk = idx / r; }
        const int k = k0 + kk;
        zs[j * 256 + kk] = (k < Kin) ? Z[(long)j * zj + (long)k * zk] : __float2bfloat16(0.f);
      }
      __syncthreads();
    }
    if (row < M) {
      const int k = k0 + 8 * lane;
      if (k < Kin) {
        float y[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(Y + (long)row * ldy + k), y);
#pragma unroll
        for (int j = 0; j < RM; ++j) {
          if (j < r) {
            float z[8];
            if (!grouped) {
              bf16x8_to_f32(*reinterpret_cast<const uint4*>(zs + j * 256 + 8 * lane), z);
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) z[i] = __bfloat162float(Ze[(long)j * zj + (long)(k + i) * zk]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[j] = fmaf(y[i], z[i], acc[j]);
          }
        }
      }
    }
  }
  if (row >= M) return;
#pragma unroll
  for (int j = 0; j < RM; ++j) {
    if (j < r) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
  }
  // lanes write distinct columns
  for (int j = lane; j < 2 * RP; j += 32) {
    float a = 0.f;
#pragma unroll
    for (int jj = 0; jj < RM; ++jj) if (jj == (j < RP ? j : j - RP)) a = acc[jj];
    const int jr = j < RP ? j : j - RP;
    if (out != nullptr && j < r) out[(long)row * r + j] = oscale * a;
    if (la != nullptr) {
      __nv_bfloat16 v = __float2bfloat16(0.f);
      if (jr < r) {
        const float x = lscale * a;
        const __nv_bfloat16 hi = __float2bfloat16_rn(x);
        v = (j < RP) ? hi : __float2bfloat16_rn(x - __bfloat162float(hi));
      }
      la[(long)row * 2 * RP + j] = v;
    }
  }
}

// LB[e*rows + n][j] = LB[..][RP + j] = Z(e, n, j) = Z[e*zes + n*zn + j*zjs] for j < r, else 0.
__global__ void lora_bop_kernel(const __nv_bfloat16* __restrict__ Z, long zn, long zjs, long zes, int rows,
                                int nexp, int r, int RP, __nv_bfloat16* __restrict__ LB) {
  const long total = (long)nexp * rows * 2 * RP;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int j2 = (int)(i % (2 * RP));
    const long rn = i / (2 * RP);
    const int n = (int)(rn % rows);
    const int e = (int)(rn / rows);
    const int j = j2 < RP ? j2 : j2 - RP;
    LB[i] = (j < r) ? Z[(long)e * zes + (long)n * zn + (long)j * zjs] : __float2bfloat16(0.f);
  }
}

// Partial column reductions over one slice of rows: part[slice][c][j] = sum_m Y[m][c] * Z[m][j]
// for m in [row_lo, row_hi) of the slice; 128 threads x 2 columns per CTA, grid (C/256, slices).
// Slices: dense mode slice s = rows [128 s, 128 s + 128); grouped mode slice s = m-block s of the
// routed batch (seg_off / mblk_off / E as in the GEMM), never crossing an expert boundary.
// zw (nullable) scales row m of Z by zw[m] (routing weight).
template <int RM>
__global__ void __launch_bounds__(128) colred_partial_kernel(const __nv_bfloat16* __restrict__ Y, long ldy, int Ccols,
                                                             const float* __restrict__ Z, int r, int M,
                                                             const float* __restrict__ zw, const int* __restrict__ seg_off,
                                                             const int* __restrict__ mblk_off, int E,
                                                             float* __restrict__ part) {
  __shared__ float zs[128 * RM];
  const int slice = blockIdx.y;
  int lo, hi;
  if (E == 0) {
    lo = slice * 128;
    hi = min(M, lo + 128);
  } else {
    const int total = __ldg(mblk_off + E);
    if (slice >= total) return;
    int a = 0, b = E - 1;
    while (a < b) {
      const int mid = (a + b + 1) >> 1;
      if (__ldg(mblk_off + mid) <= slice) a = mid; else b = mid - 1;
    }
    lo = __ldg(seg_off + a) + (slice - __ldg(mblk_off + a)) * 128;
    hi = min(__ldg(seg_off + a + 1), lo + 128);
  }
  const int n = hi - lo;
  for (int i = threadIdx.x; i < n * r; i += 128) {
    const int m = i / r, j = i % r;
    float z = Z[(long)(lo + m) * r + j];
    if (zw != nullptr) z *= zw[lo + m];
    zs[m * RM + j] = z;
  }
  __syncthreads();
  const int c = blockIdx.x * 256 + 2 * threadIdx.x;
  if (c >= Ccols) return;
  float a0[RM], a1[RM];
#pragma unroll
  for (int j = 0; j < RM; ++j) { a0[j] = 0.f; a1[j] = 0.f; }
  for (int m = 0; m < n; ++m) {
    const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Y + (long)(lo + m) * ldy + c));
#pragma unroll
    for (int j = 0; j < RM; ++j) {
      if (j < r) {
        const float z = zs[m * RM + j];
        a0[j] = fmaf(y.x, z, a0[j]);
        a1[j] = fmaf(y.y, z, a1[j]);
      }
    }
  }
  float* o = part + ((long)slice * Ccols + c) * r;
#pragma unroll
  for (int j = 0; j < RM; ++j) {
    if (j < r) {
      o[j] = a0[j];
      o[r + j] = a1[j];
    }
  }
}

// out = scale * ordered sum over the slices of each expert (dense: all slices, E = 1 output).
// transpose = 0: out[e][c][j]; transpose = 1: out[e][j][c].
__global__ void colred_reduce_kernel(const float* __restrict__ part, int Ccols, int r, int nslices_dense,
                                     const int* __restrict__ mblk_off, int E, float scale, int transpose,
                                     float* __restrict__ out) {
  const int nexp = E == 0 ? 1 : E;
  const long total = (long)nexp * Ccols * r;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const int e = (int)(i / ((long)Ccols * r));
    const long cj = i % ((long)Ccols * r);
    int s0, s1;
    if (E == 0) { s0 = 0; s1 = nslices_dense; }
    else { s0 = __ldg(mblk_off + e); s1 = __ldg(mblk_off + e + 1); }
    float acc = 0.f;
    for (int s = s0; s < s1; ++s) acc += part[(long)s * Ccols * r + cj];
    const int c = (int)(cj / r), j = (int)(cj % r);
    const long o = transpose ? ((long)e * r + j) * Ccols + c : ((long)e * Ccols + c) * r + j;
    out[o] = scale * acc;
  }
}

// Standalone dequant: one thread per 8 consecutive weights.
template <int QT>
__global__ void gguf_dequant_kernel(const uint8_t* __restrict__ wq, long rows, long cols, void* __restrict__ out,
                                    int out_dtype) {
  const long groups_per_row = cols / 256;
  const long row_bytes = groups_per_row * QTraits<QT>::kGroupBytes;
  const long total = rows * (cols / 8);
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const long row = i / (cols / 8);
    const long c8 = i % (cols / 8);  // chunk of 8 within the row
    const uint8_t* g = wq + row * row_bytes + (c8 / 32) * QTraits<QT>::kGroupBytes;
    float w[8];
    decode8<QT>(g, (int)(c8 % 32), w);
    if (out_dtype == QL_F32) {
      float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + row * cols + c8 * 8);
      o[0] = make_float4(w[0], w[1], w[2], w[3]);
      o[1] = make_float4(w[4], w[5], w[6], w[7]);
    } else {
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + row * cols + c8 * 8) = pack_bf16x8(w);
    }
  }
}

// A block that waits on a barrier no one arrives at (bounded-wait self-check).
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(smem_u32(&bar), 0, 99, true, limit_ns)) {
      // the wait recorded QL_ERR_TIMEOUT; nothing else to undo
    }
  }
  __syncthreads();
}

}  // namespace qlora
