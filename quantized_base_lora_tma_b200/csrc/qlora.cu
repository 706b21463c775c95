// C ABI of the layer library: argument checks, workspace carving, tensor maps and launch order.
// Declarations and their contracts live in include/qlora.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "qlora.h"
#include "lora.cuh"
#include "qgemm.cuh"

namespace qlora {

static std::atomic<uint64_t> g_launches{0};

// Optional timing events recorded around the tensor-core GEMM launches (slot 0: forward GEMM,
// 1: input-gradient GEMM, 2..5: grouped GEMMs of the MoE layer), on the launch stream.
constexpr int kEventSlots = 8;
static cudaEvent_t g_ev[kEventSlots][2] = {};

static void ev_record(int slot, int which, cudaStream_t st) {
  if (slot >= 0 && slot < kEventSlots && g_ev[slot][which]) cudaEventRecord(g_ev[slot][which], st);
}

// ------------------------------------------------------------------------------------------------
// Driver entry point for tensor-map encoding (no link-time dependency on libcuda).
// ------------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D row-major tensor [rows x inner] of elements of `esize` bytes; box [box_rows x box_inner].
static bool make_tmap(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int esize, uint64_t inner,
                      uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                      CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  (void)esize;
  CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool tmap_bf16_rows(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  return make_tmap(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cols, rows, cols * 2, 64, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

static bool tmap_packed(CUtensorMap* m, const void* ptr, uint64_t row_bytes, uint64_t rows, uint32_t group_bytes) {
  return make_tmap(m, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, row_bytes / 4, rows, row_bytes, group_bytes / 4, 64,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
}

static int num_sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int group_bytes(int qtype) {
  switch (qtype) {
    case QL_Q8_0: return 272;
    case QL_Q4_0: return 144;
    case QL_Q4_K: return 144;
    default: return 0;
  }
}

static int64_t packed_row_bytes(int qtype, int64_t cols) { return cols / 256 * group_bytes(qtype); }

static inline int lora_rp(int r) { return 32 * ((r + 31) / 32); }

static inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

// ------------------------------------------------------------------------------------------------
// Launch helpers
// ------------------------------------------------------------------------------------------------
template <int QT, bool TRANS, int EPI>
static int launch_qgemm(const CUtensorMap& tA, const CUtensorMap& tW, const CUtensorMap& tLA, const CUtensorMap& tLB,
                        const GemmParams& p, int grid, cudaStream_t st, int slot) {
  using C = GemmCfg<QT, TRANS>;
  auto k = qgemm_kernel<QT, TRANS, EPI>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return QL_ERR_CUDA;
  ev_record(slot, 0, st);
  k<<<grid, kGemmThreads, C::SMEM_BYTES, st>>>(tA, tW, tLA, tLB, p);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  ev_record(slot, 1, st);
  return launch_status();
}

template <bool TRANS, int EPI>
static int launch_qgemm_q(int qtype, const CUtensorMap& tA, const CUtensorMap& tW, const CUtensorMap& tLA,
                          const CUtensorMap& tLB, const GemmParams& p, int grid, cudaStream_t st, int slot) {
  switch (qtype) {
    case QL_Q8_0: return launch_qgemm<QL_Q8_0, TRANS, EPI>(tA, tW, tLA, tLB, p, grid, st, slot);
    case QL_Q4_0: return launch_qgemm<QL_Q4_0, TRANS, EPI>(tA, tW, tLA, tLB, p, grid, st, slot);
    case QL_Q4_K: return launch_qgemm<QL_Q4_K, TRANS, EPI>(tA, tW, tLA, tLB, p, grid, st, slot);
    default: return QL_ERR_UNSUPPORTED;
  }
}

static int launch_lora_rows(const __nv_bfloat16* Y, long ldy, int M, int Kin, const __nv_bfloat16* Z, long zj, long zk,
                            long zes, const int* row_exp, int r, float oscale, float lscale, float* out,
                            __nv_bfloat16* la, cudaStream_t st) {
  const int RP = lora_rp(r);
  const int grid = (M + 7) / 8;
  if (grid == 0) return QL_OK;
  if (r <= 16)
    lora_rows_kernel<16><<<grid, 256, 0, st>>>(Y, ldy, M, Kin, Z, zj, zk, zes, row_exp, r, oscale, lscale, out, la, RP);
  else if (r <= 32)
    lora_rows_kernel<32><<<grid, 256, 0, st>>>(Y, ldy, M, Kin, Z, zj, zk, zes, row_exp, r, oscale, lscale, out, la, RP);
  else
    lora_rows_kernel<64><<<grid, 256, 0, st>>>(Y, ldy, M, Kin, Z, zj, zk, zes, row_exp, r, oscale, lscale, out, la, RP);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

static int launch_lora_bop(const __nv_bfloat16* Z, long zn, long zjs, long zes, int rows, int nexp, int r,
                           __nv_bfloat16* LB, cudaStream_t st) {
  const int RP = lora_rp(r);
  const long total = (long)nexp * rows * 2 * RP;
  const int grid = (int)std::min<long>((total + 255) / 256, 148L * 16);
  lora_bop_kernel<<<grid, 256, 0, st>>>(Z, zn, zjs, zes, rows, nexp, r, RP, LB);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

// out = scale * sum over slices of Y[m, c] Z[m, j]
static int launch_colred(const __nv_bfloat16* Y, long ldy, int Ccols, const float* Z, int r, int M, const float* zw,
                         const int* seg_off, const int* mblk_off, int E, int max_slices, float* part, float scale,
                         int transpose, float* out, cudaStream_t st) {
  if (max_slices <= 0) return QL_OK;
  dim3 grid((Ccols + 255) / 256, max_slices);
  if (r <= 16)
    colred_partial_kernel<16><<<grid, 128, 0, st>>>(Y, ldy, Ccols, Z, r, M, zw, seg_off, mblk_off, E, part);
  else if (r <= 32)
    colred_partial_kernel<32><<<grid, 128, 0, st>>>(Y, ldy, Ccols, Z, r, M, zw, seg_off, mblk_off, E, part);
  else
    colred_partial_kernel<64><<<grid, 128, 0, st>>>(Y, ldy, Ccols, Z, r, M, zw, seg_off, mblk_off, E, part);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (launch_status() != QL_OK) return QL_ERR_CUDA;
  const long total = (long)(E == 0 ? 1 : E) * Ccols * r;
  const int g2 = (int)std::min<long>((total + 255) / 256, 148L * 16);
  colred_reduce_kernel<<<g2, 256, 0, st>>>(part, Ccols, r, max_slices, mblk_off, E, scale, transpose, out);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

// Workspace layout of the dense layer (byte offsets, 256-aligned).
struct LinearWs {
  size_t la, lb, g, part, total;
};
static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
static LinearWs linear_ws(int64_t M, int64_t N, int64_t K, int r) {
  LinearWs w;
  const int KL = 2 * lora_rp(r);
  const int64_t NK = N > K ? N : K;
  size_t o = 0;
  w.la = o; o = al256(o + (size_t)M * KL * 2);
  w.lb = o; o = al256(o + (size_t)NK * KL * 2);
  w.g = o; o = al256(o + (size_t)M * r * 4);
  w.part = o; o = al256(o + (size_t)((M + 127) / 128) * NK * r * 4);
  w.total = o;
  return w;
}

static int check_linear(int qtype, const void* wq, int64_t N, int64_t K, const void* X, int64_t M, const void* A,
                        const void* B, int r) {
  if (!wq || !X || !A || !B) return QL_ERR_INVALID_ARG;
  if (group_bytes(qtype) == 0) return QL_ERR_UNSUPPORTED;
  if (M < 1 || N < 1 || K < 1) return QL_ERR_INVALID_ARG;
  if (r < 1 || r > 64) return QL_ERR_UNSUPPORTED;
  if (K % 256 != 0 || N % 64 != 0) return QL_ERR_SHAPE;
  if (M > (1 << 30) || N > (1 << 24) || K > (1 << 24)) return QL_ERR_SHAPE;
  if (!aligned16(wq) || !aligned16(X) || !aligned16(A) || !aligned16(B)) return QL_ERR_ALIGNMENT;
  return QL_OK;
}

}  // namespace qlora

using namespace qlora;

extern "C" {

const char* qlora_status_string(int s) {
  switch (s) {
    case QL_OK: return "QL_OK";
    case QL_ERR_INVALID_ARG: return "QL_ERR_INVALID_ARG";
    case QL_ERR_UNSUPPORTED: return "QL_ERR_UNSUPPORTED";
    case QL_ERR_SHAPE: return "QL_ERR_SHAPE";
    case QL_ERR_ALIGNMENT: return "QL_ERR_ALIGNMENT";
    case QL_ERR_WORKSPACE: return "QL_ERR_WORKSPACE";
    case QL_ERR_CUDA: return "QL_ERR_CUDA";
    case QL_ERR_TIMEOUT: return "QL_ERR_TIMEOUT";
    default: return "QL_UNKNOWN_STATUS";
  }
}

uint64_t qlora_launch_count(void) { return g_launches.load(); }

int qlora_set_kernel_events(int slot, void* start, void* stop) {
  if (slot < 0 || slot >= kEventSlots) return QL_ERR_INVALID_ARG;
  if ((start == nullptr) != (stop == nullptr)) return QL_ERR_INVALID_ARG;
  g_ev[slot][0] = (cudaEvent_t)start;
  g_ev[slot][1] = (cudaEvent_t)stop;
  return QL_OK;
}

int qlora_device_status(int* site, int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return QL_ERR_CUDA;
  DeviceStatus h;
  if (cudaMemcpyFromSymbol(&h, g_dev_status, sizeof(h)) != cudaSuccess) return QL_ERR_CUDA;
  if (site) *site = h.site;
  if (reset) {
    DeviceStatus z = {0, 0, 0, 0};
    if (cudaMemcpyToSymbol(g_dev_status, &z, sizeof(z)) != cudaSuccess) return QL_ERR_CUDA;
  }
  return h.status;
}

int qlora_selftest_wait_timeout(int64_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 2000000) return QL_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

int gguf_dequant(int qtype, const void* wq, int64_t rows, int64_t cols, void* out, int out_dtype, void* stream) {
  if (!wq || !out) return QL_ERR_INVALID_ARG;
  if (group_bytes(qtype) == 0) return QL_ERR_UNSUPPORTED;
  if (out_dtype != QL_F32 && out_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return QL_ERR_INVALID_ARG;
  if (cols % 256 != 0) return QL_ERR_SHAPE;
  if (!aligned16(wq) || !aligned16(out)) return QL_ERR_ALIGNMENT;
  const long total = rows * (cols / 8);
  const int grid = (int)std::min<long>((total + 255) / 256, (long)num_sms() * 32);
  cudaStream_t st = (cudaStream_t)stream;
  switch (qtype) {
    case QL_Q8_0: gguf_dequant_kernel<QL_Q8_0><<<grid, 256, 0, st>>>((const uint8_t*)wq, rows, cols, out, out_dtype); break;
    case QL_Q4_0: gguf_dequant_kernel<QL_Q4_0><<<grid, 256, 0, st>>>((const uint8_t*)wq, rows, cols, out, out_dtype); break;
    case QL_Q4_K: gguf_dequant_kernel<QL_Q4_K><<<grid, 256, 0, st>>>((const uint8_t*)wq, rows, cols, out, out_dtype); break;
  }
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

size_t qlora_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 1 || N < 1 || K < 1 || r < 1 || r > 64) return 0;
  return linear_ws(M, N, K, r).total;
}

int qlora_linear_fwd(int qtype, const void* wq, int64_t N, int64_t K, const void* X, int64_t M, const void* A,
                     const void* B, int r, float scale, void* Y, int y_dtype, float* H, void* ws, size_t ws_bytes,
                     void* stream) {
  int rc = check_linear(qtype, wq, N, K, X, M, A, B, r);
  if (rc != QL_OK) return rc;
  if (!Y || !H) return QL_ERR_INVALID_ARG;
  if (y_dtype != QL_F32 && y_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (!aligned16(Y) || !aligned16(H)) return QL_ERR_ALIGNMENT;
  const LinearWs w = linear_ws(M, N, K, r);
  if (!ws || ws_bytes < w.total) return QL_ERR_WORKSPACE;
  if (!aligned16(ws)) return QL_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* wsb = (uint8_t*)ws;
  __nv_bfloat16* LA = (__nv_bfloat16*)(wsb + w.la);
  __nv_bfloat16* LB = (__nv_bfloat16*)(wsb + w.lb);
  const int KL = 2 * lora_rp(r);

  // H = X A^T (saved) and the split operand of s*H
  rc = launch_lora_rows((const __nv_bfloat16*)X, K, (int)M, (int)K, (const __nv_bfloat16*)A, K, 1, 0, nullptr, r,
                        1.0f, scale, H, LA, st);
  if (rc) return rc;
  rc = launch_lora_bop((const __nv_bfloat16*)B, r, 1, 0, (int)N, 1, r, LB, st);
  if (rc) return rc;

  CUtensorMap tA, tW, tLA, tLB;
  const int64_t rb = packed_row_bytes(qtype, K);
  if (!tmap_bf16_rows(&tA, X, K, M, 128) || !tmap_packed(&tW, wq, rb, N, group_bytes(qtype)) ||
      !tmap_bf16_rows(&tLA, LA, KL, M, 128) || !tmap_bf16_rows(&tLB, LB, KL, N, 64))
    return QL_ERR_CUDA;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = (int)M;
  p.Nd = (int)N;
  p.Kd = (int)K;
  p.n_lora_kb = KL / 64;
  p.num_n_tiles = (int)((N + 127) / 128);
  p.num_m_blocks = (int)((M + 127) / 128);
  p.out = Y;
  p.out_dtype = y_dtype;
  p.ldo = N;
  const int tiles = p.num_n_tiles * p.num_m_blocks;
  const int grid = std::min(tiles, num_sms());
  return launch_qgemm_q<false, EPI_STORE>(qtype, tA, tW, tLA, tLB, p, grid, st, 0);
}

int qlora_linear_bwd(int qtype, const void* wq, int64_t N, int64_t K, const void* X, const void* dY, int64_t M,
                     const void* A, const void* B, int r, float scale, const float* H, void* dX, int dx_dtype,
                     float* dA, float* dB, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_linear(qtype, wq, N, K, X, M, A, B, r);
  if (rc != QL_OK) return rc;
  if (!dY || !H || !dA || !dB) return QL_ERR_INVALID_ARG;
  if (dX && dx_dtype != QL_F32 && dx_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(H) || !aligned16(dA) || !aligned16(dB) || (dX && !aligned16(dX)))
    return QL_ERR_ALIGNMENT;
  const LinearWs w = linear_ws(M, N, K, r);
  if (!ws || ws_bytes < w.total) return QL_ERR_WORKSPACE;
  if (!aligned16(ws)) return QL_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* wsb = (uint8_t*)ws;
  __nv_bfloat16* LA = (__nv_bfloat16*)(wsb + w.la);
  __nv_bfloat16* LB = (__nv_bfloat16*)(wsb + w.lb);
  float* G = (float*)(wsb + w.g);
  float* part = (float*)(wsb + w.part);
  const int KL = 2 * lora_rp(r);
  const int slices = (int)((M + 127) / 128);

  // G = s dY B (kept in fp32) and its split operand
  rc = launch_lora_rows((const __nv_bfloat16*)dY, N, (int)M, (int)N, (const __nv_bfloat16*)B, 1, r, 0, nullptr, r,
                        scale, scale, G, LA, st);
  if (rc) return rc;
  if (dX) {
    // LB[k] = [A^T(k) | A^T(k)]
    rc = launch_lora_bop((const __nv_bfloat16*)A, 1, K, 0, (int)K, 1, r, LB, st);
    if (rc) return rc;
    CUtensorMap tA, tW, tLA, tLB;
    const int64_t rb = packed_row_bytes(qtype, K);
    if (!tmap_bf16_rows(&tA, dY, N, M, 128) || !tmap_packed(&tW, wq, rb, N, group_bytes(qtype)) ||
        !tmap_bf16_rows(&tLA, LA, KL, M, 128) || !tmap_bf16_rows(&tLB, LB, KL, K, 64))
      return QL_ERR_CUDA;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    p.M = (int)M;
    p.Nd = (int)K;
    p.Kd = (int)N;
    p.n_lora_kb = KL / 64;
    p.num_n_tiles = (int)(K / 256);
    p.num_m_blocks = slices;
    p.out = dX;
    p.out_dtype = dx_dtype;
    p.ldo = K;
    const int tiles = p.num_n_tiles * p.num_m_blocks;
    rc = launch_qgemm_q<true, EPI_STORE>(qtype, tA, tW, tLA, tLB, p, std::min(tiles, num_sms()), st, 1);
    if (rc) return rc;
  }
  // dB = s dY^T H ; dA = G^T X
  rc = launch_colred((const __nv_bfloat16*)dY, N, (int)N, H, r, (int)M, nullptr, nullptr, nullptr, 0, slices, part,
                     scale, 0, dB, st);
  if (rc) return rc;
  rc = launch_colred((const __nv_bfloat16*)X, K, (int)K, G, r, (int)M, nullptr, nullptr, nullptr, 0, slices, part,
                     1.0f, 1, dA, st);
  return rc;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Forward without any allocation: the adapter operands live in a static device array.
// ------------------------------------------------------------------------------------------------
namespace qlora {

// Scratch of qlora_linear_fwd_noalloc: LA [M x KL] then LB [N x KL], bf16 (KL = 64 for r <= 32,
// 128 for r <= 64). Every device that loads the library holds these 4 MiB until the process exits.
constexpr size_t kStaticScratchBytes = (size_t)4 << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
static std::mutex g_static_scratch_mu;
static void* g_static_scratch_dev[kMaxDevices] = {};

// Device address of g_static_scratch on the current device; looked up on the first use per device.
static int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return QL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (g_static_scratch_dev[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr) return QL_ERR_CUDA;
    g_static_scratch_dev[dev] = ptr;
  }
  *out = g_static_scratch_dev[dev];
  return QL_OK;
}

}  // namespace qlora

extern "C" int qlora_linear_fwd_noalloc(int qtype, const void* wq, int64_t N, int64_t K, const void* X, int64_t M,
                                        const void* A, const void* B, int r, float scale, void* Y, int y_dtype,
                                        float* H, void* stream) {
  int rc = check_linear(qtype, wq, N, K, X, M, A, B, r);
  if (rc != QL_OK) return rc;
  if (!Y || !H) return QL_ERR_INVALID_ARG;
  if (y_dtype != QL_F32 && y_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (!aligned16(Y) || !aligned16(H)) return QL_ERR_ALIGNMENT;
  const int KL = 2 * lora_rp(r);
  const size_t la_bytes = al256((size_t)M * KL * 2);
  const size_t need = la_bytes + (size_t)N * KL * 2;
  if (need > kStaticScratchBytes) return QL_ERR_WORKSPACE;
  void* base = nullptr;
  rc = static_scratch_address(&base);
  if (rc != QL_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  // Both operands are rewritten in full (padding included) before the GEMM reads them, so what
  // an earlier call left in the array does not matter.
  __nv_bfloat16* LA = (__nv_bfloat16*)base;
  __nv_bfloat16* LB = (__nv_bfloat16*)((uint8_t*)base + la_bytes);

  rc = launch_lora_rows((const __nv_bfloat16*)X, K, (int)M, (int)K, (const __nv_bfloat16*)A, K, 1, 0, nullptr, r,
                        1.0f, scale, H, LA, st);
  if (rc) return rc;
  rc = launch_lora_bop((const __nv_bfloat16*)B, r, 1, 0, (int)N, 1, r, LB, st);
  if (rc) return rc;
  CUtensorMap tA, tW, tLA, tLB;
  const int64_t rb = packed_row_bytes(qtype, K);
  if (!tmap_bf16_rows(&tA, X, K, M, 128) || !tmap_packed(&tW, wq, rb, N, group_bytes(qtype)) ||
      !tmap_bf16_rows(&tLA, LA, KL, M, 128) || !tmap_bf16_rows(&tLB, LB, KL, N, 64))
    return QL_ERR_CUDA;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = (int)M;
  p.Nd = (int)N;
  p.Kd = (int)K;
  p.n_lora_kb = KL / 64;
  p.num_n_tiles = (int)((N + 127) / 128);
  p.num_m_blocks = (int)((M + 127) / 128);
  p.out = Y;
  p.out_dtype = y_dtype;
  p.ldo = N;
  const int tiles = p.num_n_tiles * p.num_m_blocks;
  return launch_qgemm_q<false, EPI_STORE>(qtype, tA, tW, tLA, tLB, p, std::min(tiles, num_sms()), st, 0);
}
