// C ABI of the layer library: argument checks, workspace carving, tensor maps and launch order.
// Declarations and their contracts live in include/qlora.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <random>
#include <vector>

#include "qlora.h"
#include "lora.cuh"
#include "qgemm.cuh"
#include "qgemm2.cuh"
#include "gemv.cuh"
#include "moe.cuh"
#include "adamw8.cuh"
#include "rmsnorm.cuh"
#include "lmhead.cuh"

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

// bf16 rows [rows x cols] (cols a multiple of 64) seen as [rows][cols / 64][64]: box [box_rows][kc][64],
// 128-byte swizzled, landing as 128-byte lines (row y, chunk z) at line y kc + z.
static bool tmap_bf16_chunks(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows,
                             uint32_t kc) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, cols / 64, rows};
  cuuint64_t strides[2] = {128, cols * 2};
  cuuint32_t box[3] = {64, kc, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool tmap_bf16_rows(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  return make_tmap(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, cols, rows, cols * 2, 64, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_128B);
}

static bool tmap_packed(CUtensorMap* m, const void* ptr, uint64_t row_bytes, uint64_t rows, uint32_t group_bytes,
                        uint32_t box_rows = 64) {
  return make_tmap(m, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, row_bytes / 4, rows, row_bytes, group_bytes / 4, box_rows,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Per-device host state that launches look up on every call: the SM count and which kernels have
// had their dynamic shared-memory limit raised (cudaFuncSetAttribute costs microseconds).
constexpr int kHostDevices = 64;
static std::atomic<int> g_num_sms[kHostDevices];

static int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < kHostDevices) {
    const int c = g_num_sms[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = n > 0 ? n : 148;
  if (dev >= 0 && dev < kHostDevices) g_num_sms[dev].store(n, std::memory_order_relaxed);
  return n;
}

static std::mutex g_smem_attr_mu;
static std::vector<std::pair<std::pair<const void*, int>, int>> g_smem_attr;  // (kernel, device) -> bytes set

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel, device and size.
template <typename Kernel>
static cudaError_t set_smem(Kernel k, int bytes) {
  int dev = 0;
  cudaGetDevice(&dev);
  const void* key = reinterpret_cast<const void*>(k);
  {
    std::lock_guard<std::mutex> lock(g_smem_attr_mu);
    for (const auto& e : g_smem_attr)
      if (e.first.first == key && e.first.second == dev && e.second >= bytes) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_smem_attr_mu);
  for (auto& x : g_smem_attr)
    if (x.first.first == key && x.first.second == dev) {
      x.second = std::max(x.second, bytes);
      return cudaSuccess;
    }
  g_smem_attr.push_back({{key, dev}, bytes});
  return cudaSuccess;
}

static inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Packed bytes of 256 weights of a row, for the types the layer's GEMMs take (0 otherwise).
static int group_bytes(int qtype) {
  switch (qtype) {
    case QL_Q8_0: return 272;
    case QL_Q4_0: return 144;
    case QL_Q4_K: return 144;
    case QL_Q5_K: return 176;
    default: return 0;
  }
}

static int64_t packed_row_bytes(int qtype, int64_t cols) { return cols / 256 * group_bytes(qtype); }

static inline int lora_rp(int r) { return 32 * ((r + 31) / 32); }
static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

static inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? QL_OK : QL_ERR_CUDA;
}

// ------------------------------------------------------------------------------------------------
// Launch helpers
// ------------------------------------------------------------------------------------------------
// While a NoEarlyStart is alive on a thread, PdlLaunch launches from that thread without programmatic
// stream serialization: the kernel starts only once the previous kernel in the stream has completed
// (for a GEMM whose A operand the immediately preceding kernel writes: the unfused pair GEMM streams
// A before it waits for its predecessor).
static thread_local int t_no_early_start = 0;
struct NoEarlyStart {
  NoEarlyStart() { ++t_no_early_start; }
  ~NoEarlyStart() { --t_no_early_start; }
};

// Launch configuration with programmatic stream serialization (the kernel may start while the
// previous kernel in the stream finishes; the dense-path kernels wait on it in-kernel) and, when
// cluster_y > 0, a (1, cluster_y, 1) cluster shape.
struct PdlLaunch {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  PdlLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_y = 0) {
    cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = t_no_early_start ? 0 : 1;
    int n = 1;
    if (cluster_y > 0) {
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = 1;
      attr[1].val.clusterDim.y = (unsigned)cluster_y;
      attr[1].val.clusterDim.z = 1;
      n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
  }
};
// A launch that may start while the previous kernel in the stream finishes (the kernel itself
// waits for it with griddepcontrol.wait before touching memory).
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  PdlLaunch L(grid, block, smem, st);
  return cudaLaunchKernelEx(&L.cfg, kern, static_cast<KArgs>(args)...);
}
static int launch_result(cudaError_t e) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return launch_status();
}
template <int QT, bool TRANS, int EPI, int MS, int BN = 128>
static int launch_qgemm(const CUtensorMap& tA, const CUtensorMap& tW, const CUtensorMap& tLA, const CUtensorMap& tLB,
                        const GemmParams& p, int grid, cudaStream_t st, int slot) {
  using C = GemmCfg<QT, TRANS, MS, BN>;
  auto k = qgemm_kernel<QT, TRANS, EPI, MS, BN>;
  if (set_smem(k, C::SMEM_BYTES) != cudaSuccess)
    return QL_ERR_CUDA;
  PdlLaunch L(dim3(grid), dim3(kGemmThreads), C::SMEM_BYTES, st);
  ev_record(slot, 0, st);
  const cudaError_t e = cudaLaunchKernelEx(&L.cfg, k, tA, tW, tLA, tLB, p);
  ev_record(slot, 1, st);
  return launch_result(e);
}

template <bool TRANS, int EPI, int MS>
static int launch_qgemm_q(int qtype, const CUtensorMap& tA, const CUtensorMap& tW, const CUtensorMap& tLA,
                          const CUtensorMap& tLB, const GemmParams& p, int grid, cudaStream_t st, int slot,
                          int bn = 128) {
  switch (qtype) {
    case QL_Q8_0: return launch_qgemm<QL_Q8_0, TRANS, EPI, MS>(tA, tW, tLA, tLB, p, grid, st, slot);
    case QL_Q4_0:
      return bn == 256 ? launch_qgemm<QL_Q4_0, TRANS, EPI, MS, 256>(tA, tW, tLA, tLB, p, grid, st, slot)
                       : launch_qgemm<QL_Q4_0, TRANS, EPI, MS>(tA, tW, tLA, tLB, p, grid, st, slot);
    case QL_Q4_K:
      return bn == 256 ? launch_qgemm<QL_Q4_K, TRANS, EPI, MS, 256>(tA, tW, tLA, tLB, p, grid, st, slot)
                       : launch_qgemm<QL_Q4_K, TRANS, EPI, MS>(tA, tW, tLA, tLB, p, grid, st, slot);
    case QL_Q5_K: return launch_qgemm<QL_Q5_K, TRANS, EPI, MS>(tA, tW, tLA, tLB, p, grid, st, slot);
    default: return QL_ERR_UNSUPPORTED;
  }
}

// Tile width of a grouped GEMM: 256 columns where the 144-byte groups let the raw ring hold 256
// rows and the output width divides (div = the column count per tile unit), else 128.
static int grouped_bn(int qtype, int64_t cols, int64_t div256) {
  return group_bytes(qtype) == 144 && cols % div256 == 0 ? 256 : 128;
}

// Pair-tile dense GEMM: clusters of two CTAs, one cluster per pair tile slot. The grid is capped at
// the number of clusters that can be resident at once (a persistent kernel must never have CTAs
// waiting for a free SM pair).
// Clusters of the pair GEMM that are resident at once (cached per device; 0 on error).
template <int QT, bool TRANS, int MS>
static int qgemm2_max_clusters() {
  using C = Gemm2Cfg<QT, TRANS, MS>;
  auto k = qgemm2_kernel<QT, TRANS, MS>;
  if (set_smem(k, C::SMEM_BYTES) != cudaSuccess) return 0;
  static int max_clusters[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  int& mc = max_clusters[dev & 15];
  if (mc <= 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    cfg.blockDim = dim3(kGemm2Threads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess || n <= 0) return 0;
    mc = n;
  }
  return mc;
}

// With p.rx row clusters (fused adapter row products) in front of the tile clusters.
template <int QT, bool TRANS, int MS>
static int launch_qgemm2(const CUtensorMap& tA, const CUtensorMap& tW, const CUtensorMap& tLA, const CUtensorMap& tLB,
                         const CUtensorMap& tRY, const CUtensorMap& tZ, const GemmParams& p, int tiles, cudaStream_t st,
                         int slot) {
  using C = Gemm2Cfg<QT, TRANS, MS>;
  auto k = qgemm2_kernel<QT, TRANS, MS>;
  const int mc = qgemm2_max_clusters<QT, TRANS, MS>();
  if (mc <= p.rx) return QL_ERR_CUDA;
  const int clusters = p.rx + std::min(tiles, mc - p.rx);
  PdlLaunch L(dim3(2 * clusters), dim3(kGemm2Threads), C::SMEM_BYTES, st);  // cluster shape from the kernel
  ev_record(slot, 0, st);
  const cudaError_t e = cudaLaunchKernelEx(&L.cfg, k, tA, tW, tLA, tLB, tRY, tZ, p);
  ev_record(slot, 1, st);
  return launch_result(e);
}

template <bool TRANS, int MS>
static int launch_qgemm2_q(int qtype, const CUtensorMap& tA, const CUtensorMap& tW, const CUtensorMap& tLA,
                           const CUtensorMap& tLB, const CUtensorMap& tRY, const CUtensorMap& tZ, const GemmParams& p,
                           int tiles, cudaStream_t st, int slot) {
  switch (qtype) {
    case QL_Q8_0: return launch_qgemm2<QL_Q8_0, TRANS, MS>(tA, tW, tLA, tLB, tRY, tZ, p, tiles, st, slot);
    case QL_Q4_0: return launch_qgemm2<QL_Q4_0, TRANS, MS>(tA, tW, tLA, tLB, tRY, tZ, p, tiles, st, slot);
    case QL_Q4_K: return launch_qgemm2<QL_Q4_K, TRANS, MS>(tA, tW, tLA, tLB, tRY, tZ, p, tiles, st, slot);
    case QL_Q5_K: return launch_qgemm2<QL_Q5_K, TRANS, MS>(tA, tW, tLA, tLB, tRY, tZ, p, tiles, st, slot);
    default: return QL_ERR_UNSUPPORTED;
  }
}
template <bool TRANS, int MS>
static int qgemm2_max_clusters_q(int qtype) {
  switch (qtype) {
    case QL_Q8_0: return qgemm2_max_clusters<QL_Q8_0, TRANS, MS>();
    case QL_Q4_0: return qgemm2_max_clusters<QL_Q4_0, TRANS, MS>();
    case QL_Q4_K: return qgemm2_max_clusters<QL_Q4_K, TRANS, MS>();
    case QL_Q5_K: return qgemm2_max_clusters<QL_Q5_K, TRANS, MS>();
    default: return 0;
  }
}
template <bool TRANS, int MS>
static int qgemm2_smem_q(int qtype) {
  switch (qtype) {
    case QL_Q8_0: return Gemm2Cfg<QL_Q8_0, TRANS, MS>::SMEM_BYTES;
    case QL_Q4_0: return Gemm2Cfg<QL_Q4_0, TRANS, MS>::SMEM_BYTES;
    case QL_Q5_K: return Gemm2Cfg<QL_Q5_K, TRANS, MS>::SMEM_BYTES;
    default: return Gemm2Cfg<QL_Q4_K, TRANS, MS>::SMEM_BYTES;
  }
}

// Dense row reduction with the in-cluster split-K sum: out = oscale * Y Z^T, la = split(lscale *
// Y Z^T), optionally hs = split(hscale * hin) for the same rows, and, in the same launch,
// LB = [Zb | Zb] (bop).
template <int NT>
static cudaError_t launch_rows_nt(cudaLaunchConfig_t& cfg, const CUtensorMap& tmY, int M, int Kin, int kchunk,
                                  const __nv_bfloat16* Z, long zj, long zk, int r, float oscale, float lscale,
                                  float* out, __nv_bfloat16* la, int RP, BopArgs bop, __nv_bfloat16* LB,
                                  int row_blocks, const float* hin, float hscale, __nv_bfloat16* hs, int* zc, int zn) {
  auto k = lora_rows_cluster_kernel<NT>;
  cudaError_t e = set_smem(k, (int)cfg.dynamicSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k, tmY, M, Kin, kchunk, Z, zj, zk, r, oscale, lscale, out, la, RP, bop, LB,
                            row_blocks, hin, hscale, hs, zc, zn);
}

// Clusters of KS CTAs of the row kernel (NT, smem) that are resident at once (cached).
static int rows_cluster_capacity(int NT, size_t smem, int KS) {
  static std::mutex mu;
  static std::vector<std::pair<std::array<long, 4>, int>> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const std::array<long, 4> key{NT, (long)smem, KS, dev};
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const auto& e : cache)
      if (e.first == key) return e.second;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, KS, 1);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = KS;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  cudaError_t e;
  if (NT == 2) {
    set_smem(lora_rows_cluster_kernel<2>, (int)smem);
    e = cudaOccupancyMaxActiveClusters(&n, lora_rows_cluster_kernel<2>, &cfg);
  } else if (NT == 4) {
    set_smem(lora_rows_cluster_kernel<4>, (int)smem);
    e = cudaOccupancyMaxActiveClusters(&n, lora_rows_cluster_kernel<4>, &cfg);
  } else {
    set_smem(lora_rows_cluster_kernel<8>, (int)smem);
    e = cudaOccupancyMaxActiveClusters(&n, lora_rows_cluster_kernel<8>, &cfg);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  cache.push_back({key, n});
  return n;
}

static int launch_rows_dense(const __nv_bfloat16* Y, long ldy, int M, int Kin, const __nv_bfloat16* Z, long zj,
                             long zk, int r, float oscale, float lscale, float* out, __nv_bfloat16* la, BopArgs bop,
                             __nv_bfloat16* LB, cudaStream_t st, const float* hin = nullptr, float hscale = 0.f,
                             __nv_bfloat16* hs = nullptr, int* zc = nullptr, int zn = 0) {
  if (M <= 0) return QL_OK;
  const int RP = lora_rp(r);
  // k range per cluster rank: a multiple of the 128-wide streamed tile
  int KS = std::max(1, std::min(8, (Kin + 127) / 128));
  int kchunk = (Kin + KS - 1) / KS;
  kchunk = (kchunk + 127) / 128 * 128;
  KS = (Kin + kchunk - 1) / kchunk;
  const int NT = r <= 16 ? 2 : (r <= 32 ? 4 : 8);
  const size_t smem = rows_smem_bytes(NT, kchunk, zk != 1);
  CUtensorMap tmY;
  if (!make_tmap(&tmY, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Kin, M, ldy * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return QL_ERR_CUDA;
  if (smem > 232448) return QL_ERR_SHAPE;  // the staged adapter slice does not fit on chip
  // aux clusters beside the row clusters for the LB operand and hs (about 8 items per thread, at
  // most 32 CTAs) when they all fit in the same wave; otherwise the row CTAs share that work
  const int row_blocks = (M + 63) / 64;
  const long aux_items = (bop.Z ? (long)bop.rows * (2 * RP / 8) : 0) + (hs ? (long)M * RP / 4 : 0);
  const int aux_ctas = aux_items ? (int)std::min<long>(32, std::max<long>(1, (aux_items + 1023) / 1024)) : 0;
  int aux_blocks = (aux_ctas + KS - 1) / KS;
  if (aux_blocks > 0 && row_blocks + aux_blocks > rows_cluster_capacity(NT, smem, KS)) aux_blocks = 0;
  PdlLaunch L(dim3(row_blocks + aux_blocks, KS, 1), dim3(128), smem, st, KS);
  cudaLaunchConfig_t& cfg = L.cfg;
  cudaError_t e;
  if (NT == 2)
    e = launch_rows_nt<2>(cfg, tmY, M, Kin, kchunk, Z, zj, zk, r, oscale, lscale, out, la, RP, bop, LB, row_blocks,
                          hin, hscale, hs, zc, zn);
  else if (NT == 4)
    e = launch_rows_nt<4>(cfg, tmY, M, Kin, kchunk, Z, zj, zk, r, oscale, lscale, out, la, RP, bop, LB, row_blocks,
                          hin, hscale, hs, zc, zn);
  else
    e = launch_rows_nt<8>(cfg, tmY, M, Kin, kchunk, Z, zj, zk, r, oscale, lscale, out, la, RP, bop, LB, row_blocks,
                          hin, hscale, hs, zc, zn);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return launch_status();
}

// Two dense column reductions in one launch (dB and dA of the backward): out_p = scale_p *
// Y_p^T Z_p for Y_p [M x C_p] bf16 and the split operands Z_p [M x 2RP] bf16. Tiles of 256 rows
// (128 for r > 32, so that two stages still fit); rows go in chunks of at most 2048, so that a
// launch at the bench shape has one unit per column block and no partials.
struct ColredPlan {
  int nb0, nblk, csu, mchunk, tr;
};
static ColredPlan plan_colred(int64_t M, int64_t C0, int64_t C1, int r) {
  ColredPlan p;
  p.nb0 = (int)((C0 + 127) / 128);
  p.nblk = p.nb0 + (int)((C1 + 127) / 128);
  p.tr = lora_rp(r) <= 32 ? 256 : 128;
  const int csu = (int)std::max<int64_t>(1, std::min<int64_t>(8, (M + 2047) / 2048));
  int mchunk = (int)((M + csu - 1) / csu);
  mchunk = (mchunk + p.tr - 1) / p.tr * p.tr;
  p.mchunk = mchunk;
  p.csu = (int)((M + mchunk - 1) / mchunk);
  return p;
}
// Counters and partials of the column reduction, for the workspace.
static size_t colred_ctr_bytes(const ColredPlan& p) { return (size_t)(1 + p.nblk) * 4; }
static size_t colred_ws_bytes(const ColredPlan& p, int r) {
  const int JT = (r + 15) / 16;
  return al256(colred_ctr_bytes(p)) + (p.csu > 1 ? (size_t)p.nblk * p.csu * JT * 16 * 128 * 4 : 0);
}

template <int JT>
static cudaError_t launch_colred_jt(cudaLaunchConfig_t& cfg, const CUtensorMap* tm, const ColredFlow& P) {
  auto k = colred_flow_kernel<JT>;
  cudaError_t e = set_smem(k, (int)cfg.dynamicSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k, tm[0], tm[1], tm[2], tm[3], P);
}

// crws: the plan's workspace (counters zeroed by an earlier kernel of the same stream, then
// partials). defer_wait: the previous kernel in the stream waited for this launch's inputs itself.
// gate: with defer_wait, a count of the previous launch's that reaches gate_target once the inputs
// Z0 and Z1 (and the zeroed counters) are written; the producer waits for it before its first claim.
static int launch_colred_dense(const __nv_bfloat16* Y0, int C0, const __nv_bfloat16* Z0, const ColredOut& o0,
                               const __nv_bfloat16* Y1, int C1, const __nv_bfloat16* Z1, const ColredOut& o1, int M, int r,
                               uint8_t* crws, int defer_wait, cudaStream_t st,
                               const unsigned long long* gate = nullptr, unsigned gate_seq = 0, int gate_target = 0) {
  const int RP = lora_rp(r);
  const int JT = (r + 15) / 16;
  CUtensorMap tm[4];
  const ColredPlan pl = plan_colred(M, C0, C1, r);
  if (!tmap_bf16_rows(&tm[0], Y0, C0, M, pl.tr) || !tmap_bf16_rows(&tm[1], Y1, C1, M, pl.tr) ||
      !tmap_bf16_rows(&tm[2], Z0, 2 * RP, M, pl.tr) || !tmap_bf16_rows(&tm[3], Z1, 2 * RP, M, pl.tr))
    return QL_ERR_CUDA;
  ColredFlow P;
  P.o0 = o0;
  P.o1 = o1;
  P.nb0 = pl.nb0;
  P.nblk = pl.nblk;
  P.M = M;
  P.r = r;
  P.RP = RP;
  P.mchunk = pl.mchunk;
  P.tr = pl.tr;
  P.csu = pl.csu;
  P.defer_wait = defer_wait;
  P.ctr = reinterpret_cast<int*>(crws);
  P.part = reinterpret_cast<float*>(crws + al256(colred_ctr_bytes(pl)));
  P.gate = gate;
  P.gate_seq = gate_seq;
  P.gate_target = gate_target;
  const size_t smem = colred_smem_bytes(RP, JT, pl.tr);
  const int per_sm = std::max(1, (int)(233472 / (smem + 1024)));
  const int grid = std::min(pl.nblk * pl.csu, per_sm * num_sms());
  PdlLaunch L(dim3(grid), dim3(32 * kColWarps), smem, st);
  cudaLaunchConfig_t& cfg = L.cfg;
  cudaError_t e;
  if (JT == 1) e = launch_colred_jt<1>(cfg, tm, P);
  else if (JT == 2) e = launch_colred_jt<2>(cfg, tm, P);
  else if (JT == 3) e = launch_colred_jt<3>(cfg, tm, P);
  else e = launch_colred_jt<4>(cfg, tm, P);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  return launch_status();
}

static int launch_colred(const __nv_bfloat16* Y, long ldy, int Ccols, const float* Z, int r, int M, const float* zw,
                         const int* seg_off, const int* mblk_off, int E, int max_slices, float* part, float scale,
                         int transpose, float* out, cudaStream_t st, const __nv_bfloat16* Ylo = nullptr,
                         const int32_t* rowmap = nullptr, int rk = 1) {
  if (max_slices <= 0) return QL_OK;
  dim3 grid((Ccols + 127) / 128, max_slices);
  const int JT = (r + 15) / 16;
  const size_t sm = colred_mma_smem(JT, Ylo != nullptr);
  cudaError_t e;
  if (JT == 1) {
    e = set_smem(colred_mma_kernel<1>, (int)sm);
    if (e == cudaSuccess) e = launch_pdl(colred_mma_kernel<1>, grid, 128, sm, st, Y, ldy, Ccols, Z, r, M, zw, seg_off, mblk_off, E, part, Ylo, rowmap, rk);
  } else if (JT == 2) {
    e = set_smem(colred_mma_kernel<2>, (int)sm);
    if (e == cudaSuccess) e = launch_pdl(colred_mma_kernel<2>, grid, 128, sm, st, Y, ldy, Ccols, Z, r, M, zw, seg_off, mblk_off, E, part, Ylo, rowmap, rk);
  } else if (JT == 3) {
    e = set_smem(colred_mma_kernel<3>, (int)sm);
    if (e == cudaSuccess) e = launch_pdl(colred_mma_kernel<3>, grid, 128, sm, st, Y, ldy, Ccols, Z, r, M, zw, seg_off, mblk_off, E, part, Ylo, rowmap, rk);
  } else {
    e = set_smem(colred_mma_kernel<4>, (int)sm);
    if (e == cudaSuccess) e = launch_pdl(colred_mma_kernel<4>, grid, 128, sm, st, Y, ldy, Ccols, Z, r, M, zw, seg_off, mblk_off, E, part, Ylo, rowmap, rk);
  }
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QL_ERR_CUDA;
  }
  const long per_e = (long)Ccols * r;
  if (per_e >= (1L << 31) || per_e % 4 != 0) return QL_ERR_SHAPE;
  // per expert a few CTAs of 256 threads (about eight outputs per thread): most experts of a
  // skewed batch are empty, and their CTAs only store zeros
  const long per_cta = E == 0 ? 256 : 2048;
  const dim3 g2((unsigned)std::min<long>((per_e + per_cta - 1) / per_cta, 64L), E == 0 ? 1 : E);
  launch_pdl(colred_reduce_kernel, g2, 256, 0, st, part, Ccols, r, max_slices, mblk_off, E, scale, transpose, out);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

// Tile plan of a dense GEMM. More than 256 rows: 512 x 256 pair tiles (two CTAs, two 128-row A
// blocks each, ms = 2); 129 to 256 rows: 256 x 256 pair tiles (ms = 1); otherwise 128 x 128 tiles on
// one CTA (ms = 0). In that last, small-M, weight-streaming regime K is split into ksplit parts of
// kb_per_split k-blocks (a multiple of 4 in forward mode) when the output has fewer tiles than there
// are SMs.
struct DensePlan {
  int ms;
  int ksplit, kbs, mblocks, ntiles;
};
static DensePlan plan_dense(int64_t M, int64_t Nd, int64_t Kd, bool trans, bool allow_split) {
  DensePlan d;
  d.ms = M > 256 ? 2 : (M > 128 ? 1 : 0);
  const int tm = d.ms ? 256 * d.ms : 128, tn = d.ms ? 256 : 128;
  d.mblocks = (int)((M + tm - 1) / tm);
  d.ntiles = (int)((Nd + tn - 1) / tn);
  const int kb_main = (int)(Kd / 64);
  const int unit = trans ? 1 : 4;
  d.ksplit = 1;
  d.kbs = kb_main;
  const int tiles = d.mblocks * d.ntiles;
  const int slots = num_sms();
  int ks = 1;
  if (allow_split && d.ms == 0 && tiles < slots) {
    ks = std::min((4 * slots + tiles - 1) / tiles, std::min(kb_main / unit, 32));
  } else if (allow_split && d.ms > 0 && 2 * tiles <= slots / 2) {
    // pair tiles filling at most half of the SM pairs (e.g. a 2048 x 2048 input gradient over a
    // long reduction: 32 tiles on 74 pairs): split K so that one wave fills most pairs; the fp32
    // parts are summed in part order afterwards
    ks = std::min((slots / 2) / tiles, std::min(kb_main / unit / 8, 4));
  }
  if (ks > 1) {
    int kbs = (kb_main + ks - 1) / ks;
    kbs = (kbs + unit - 1) / unit * unit;
    d.kbs = kbs;
    d.ksplit = (kb_main + kbs - 1) / kbs;
  }
  return d;
}
static size_t split_bytes(const DensePlan& d, int64_t M, int64_t Nd) {
  return d.ksplit > 1 ? (size_t)d.ksplit * M * Nd * 4 : 0;
}

static int launch_split_reduce(const float* part, int ksplit, long stride, long count, void* out, int out_dtype,
                               cudaStream_t st) {
  const long vec = count / 4;
  const int grid = (int)std::min<long>((vec + 255) / 256, (long)num_sms() * 8);
  PdlLaunch L(dim3(grid), dim3(256), 0, st);
  return launch_result(cudaLaunchKernelEx(&L.cfg, split_reduce_kernel, part, ksplit, stride, count, out, out_dtype));
}


// Which dense pair GEMMs compute the adapter row products in their own launch when they can
// (qlora_set_rows_fusion): bit 0 the forward, bit 1 the input gradient. The input gradient is not
// fused by default: there the column reductions that follow need the SMs the row clusters hold.
static std::atomic<int> g_rows_fusion{1};

// Row clusters of a fused dense pair GEMM (0: the row kernel runs before the GEMM). The tiles take
// one wave of clusters and leave at least one idle; the row clusters take the idle ones, as many as
// give every CTA one 128-row block, and fusion is used only when no CTA gets more than three (so
// the row products end well before the tiles' main loops). The input-gradient direction stages the
// adapter B [N x r] by TMA, whose rows must be a multiple of 16 bytes: r % 8 == 0. Not while the
// stream is being captured into a graph: the launch's counter tag is a kernel argument, and every
// replay of the graph would reuse it.
static int dense_fuse_rx(int qtype, int64_t M, int64_t Nd, int64_t Kd, bool trans, int r, cudaStream_t st) {
  if (!(g_rows_fusion.load(std::memory_order_relaxed) & (trans ? 2 : 1))) return 0;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return 0;
  const DensePlan d = plan_dense(M, Nd, Kd, trans, true);
  if (d.ms == 0 || d.ksplit != 1) return 0;
  if (trans && r % 8 != 0) return 0;
  const int mc = trans ? (d.ms == 2 ? qgemm2_max_clusters_q<true, 2>(qtype) : qgemm2_max_clusters_q<true, 1>(qtype))
                       : (d.ms == 2 ? qgemm2_max_clusters_q<false, 2>(qtype) : qgemm2_max_clusters_q<false, 1>(qtype));
  const int idle = mc - d.mblocks * d.ntiles;
  const int nblk = (int)((M + 127) / 128);
  const int rx = std::min(idle, (nblk + 1) / 2);
  if (rx < 1 || (nblk + 2 * rx - 1) / (2 * rx) > 3) return 0;
  return rx;
}
// Tagged counters of a fused launch: [0], [1], then one per M block of the pair tiles (at most
// M / 256), 8 bytes each. Tags are launch sequence numbers, unique within the process (the start is
// random, so a reloaded library does not meet its predecessor's tags in a reused workspace).
static size_t fuse_ctr_bytes(int64_t M) { return (size_t)(2 + (M + 255) / 256) * 8; }
static unsigned fuse_seq_start() {
  try {
    return (unsigned)std::random_device{}();
  } catch (...) {  // no entropy source: the clock will do
    return (unsigned)std::chrono::steady_clock::now().time_since_epoch().count();
  }
}
static unsigned next_fuse_seq() {
  static std::atomic<unsigned> seq{fuse_seq_start()};
  return seq.fetch_add(1, std::memory_order_relaxed) + 1u;
}
static int lora_nt(int r) { return r <= 16 ? 2 : (r <= 32 ? 4 : 8); }
// The row clusters' ring in the pair GEMM's shared memory: two 64-wide k chunks per stage when at
// least three such stages fit, else one.
static void fuse_ring(int qtype, bool trans, int ms, int nt, int& kc, int& stages) {
  const int smem = trans ? (ms == 2 ? qgemm2_smem_q<true, 2>(qtype) : qgemm2_smem_q<true, 1>(qtype))
                         : (ms == 2 ? qgemm2_smem_q<false, 2>(qtype) : qgemm2_smem_q<false, 1>(qtype));
  for (kc = 2;; --kc) {
    const int sb = kc * (128 * 128 + 8 * nt * 128);
    stages = std::min(8, (smem - 1024) / (sb + 16));
    if (stages >= 3 || kc == 1) return;
  }
}

// One dense dequant GEMM (forward: TRANS = false, D = A deq(W)^T; input-gradient: TRANS = true,
// D = A deq(W)) with its LoRA k-blocks, planned by plan_dense; with a K split the fp32 partials go
// to split_buf and are summed in order into `out`. With rx > 0 (from dense_fuse_rx) the launch also
// computes the adapter row products (rf, the adapter's tensor map tZ; rf->ctr zeroed beforehand).
template <bool TRANS>
static int launch_dense_gemm(int qtype, const void* A, int64_t M, int64_t Kd, const void* wq, int64_t w_rows,
                             int64_t w_cols, const __nv_bfloat16* LA, const __nv_bfloat16* LB, int KL, int64_t Nd,
                             void* out, int out_dtype, float* split_buf, bool allow_split, cudaStream_t st, int slot,
                             int rx = 0, const RowsFuse* rf = nullptr, const CUtensorMap* tRY = nullptr,
                             const CUtensorMap* tZ = nullptr, bool* sum_pending = nullptr,
                             float2* row_stats = nullptr) {
  const DensePlan d = plan_dense(M, Nd, Kd, TRANS, allow_split && split_buf != nullptr);
  // per-row softmax statistics come from the pair GEMM's fp32 store epilogue, without a K split
  if (row_stats != nullptr && (d.ms == 0 || d.ksplit != 1 || out_dtype != QL_F32)) return QL_ERR_INVALID_ARG;
  const uint32_t box = 128u;
  CUtensorMap tA, tW, tLA, tLB;
  if (!tmap_bf16_rows(&tA, A, Kd, M, box) ||
      !tmap_packed(&tW, wq, packed_row_bytes(qtype, w_cols), w_rows, group_bytes(qtype)))
    return QL_ERR_CUDA;
  if (KL == 0) {  // no adapter k-blocks (the kernels never read these maps then)
    tLA = tA;
    tLB = tA;
  } else if (!tmap_bf16_rows(&tLA, LA, KL, M, box) || !tmap_bf16_rows(&tLB, LB, KL, Nd, 64)) {
    return QL_ERR_CUDA;
  }
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = (int)M;
  p.Nd = (int)Nd;
  p.Kd = (int)Kd;
  p.n_lora_kb = KL / 64;
  p.num_n_tiles = d.ntiles;
  p.num_m_blocks = d.mblocks;
  p.ksplit = d.ksplit;
  p.kb_per_split = d.kbs;
  p.ldo = Nd;
  p.row_stats = row_stats;
  if (d.ksplit > 1) {
    p.out = split_buf;
    p.out_dtype = QL_F32;
    p.split_stride = (long)M * Nd;
  } else {
    p.out = out;
    p.out_dtype = out_dtype;
  }
  const int tiles = d.mblocks * d.ntiles * d.ksplit;
  if (rx > 0) {
    if (d.ms == 0 || d.ksplit != 1 || rf == nullptr || tRY == nullptr || tZ == nullptr) return QL_ERR_INVALID_ARG;
    p.rx = rx;
    p.rf = *rf;
    if (p.rf.stages < 2) return QL_ERR_SHAPE;
  }
  const CUtensorMap& tRYr = tRY != nullptr ? *tRY : tA;
  const CUtensorMap& tZr = tZ != nullptr ? *tZ : tA;
  int rc;
  if (d.ms == 2) rc = launch_qgemm2_q<TRANS, 2>(qtype, tA, tW, tLA, tLB, tRYr, tZr, p, tiles, st, slot);
  else if (d.ms == 1) rc = launch_qgemm2_q<TRANS, 1>(qtype, tA, tW, tLA, tLB, tRYr, tZr, p, tiles, st, slot);
  else rc = launch_qgemm_q<TRANS, EPI_STORE, 1>(qtype, tA, tW, tLA, tLB, p, std::min(tiles, num_sms()), st, slot);
  if (rc || d.ksplit == 1) return rc;
  if (sum_pending != nullptr) {  // the caller launches the part sum (launch_split_reduce) itself
    *sum_pending = true;
    return QL_OK;
  }
  return launch_split_reduce(split_buf, d.ksplit, (long)M * Nd, (long)M * Nd, out, out_dtype, st);
}

// Small-M forward (M <= 16, Q4_0 / Q8_0, r <= 16): the H partial kernel, then the weight-streaming
// kernel over G = (CTAs per SM) x SMs persistent CTAs, each a balanced range of steps.
struct GvPlan {
  int rows, mt, xr, nrb, ksteps, T, G, maxslots;
  size_t smem;
  size_t hp_bytes, part_bytes;  // workspace: H [16][16], piece partials
};
static GvPlan gemv_plan(int qtype, int64_t N, int64_t K, int64_t M) {
  GvPlan g;
  g.mt = M <= 8 ? 1 : 2;
  g.xr = 8 * g.mt;
  g.rows = qtype == QL_Q4_0 ? GvCfg<QL_Q4_0, 1>::ROWS : GvCfg<QL_Q8_0, 1>::ROWS;
  g.smem = qtype == QL_Q4_0 ? (g.mt == 1 ? GvCfg<QL_Q4_0, 1>::SMEM_BYTES : GvCfg<QL_Q4_0, 2>::SMEM_BYTES)
                            : (g.mt == 1 ? GvCfg<QL_Q8_0, 1>::SMEM_BYTES : GvCfg<QL_Q8_0, 2>::SMEM_BYTES);
  g.nrb = (int)((N + g.rows - 1) / g.rows);
  g.ksteps = (int)(K / 256);
  g.T = g.nrb * g.ksteps;
  const int per_sm = std::max(1, (int)(233472 / (g.smem + 1024)));
  // one SM is left to the H kernel that runs beside the stream: a persistent CTA that could not be
  // placed until it finished would hold up the whole launch
  g.G = std::max(1, std::min(g.T, per_sm * std::max(1, num_sms() - 1)));
  g.maxslots = 1;
  for (int rb = 0; rb < g.nrb; ++rb) {
    const long t0 = (long)rb * g.ksteps;
    g.maxslots = std::max(g.maxslots, gv_cta_of(t0 + g.ksteps - 1, g.T, g.G) - gv_cta_of(t0, g.T, g.G) + 1);
  }
  g.hp_bytes = al256((size_t)256 * 4);
  g.part_bytes = (size_t)g.nrb * g.maxslots * g.xr * g.rows * 4;
  return g;
}

template <int QT, int MT>
static int launch_gemv_q(const CUtensorMap& tW, const CUtensorMap& tX, const GvParams& p, int G, cudaStream_t st,
                         int slot) {
  using C = GvCfg<QT, MT>;
  auto k = qgemv_fwd_kernel<QT, MT>;
  if (set_smem(k, C::SMEM_BYTES) != cudaSuccess)
    return QL_ERR_CUDA;
  PdlLaunch L(dim3(G), dim3(kGvThreads), C::SMEM_BYTES, st);
  ev_record(slot, 0, st);
  const cudaError_t e = cudaLaunchKernelEx(&L.cfg, k, tW, tX, p);
  ev_record(slot, 1, st);
  return launch_result(e);
}

static bool gemv_fwd_applies(int qtype, int64_t M, int r) {
  return M <= 16 && r <= kGvMaxRank && (qtype == QL_Q4_0 || qtype == QL_Q8_0);
}

// ws: the plan's workspace (H [16][16], then piece partials). Three launches: H (one CTA), the
// weight stream (runs beside it), the row-block sums with the adapter term.
static int launch_gemv_fwd(int qtype, const void* wq, int64_t N, int64_t K, const void* X, int64_t M, const void* A,
                           const void* B, int r, float scale, void* Y, int y_dtype, float* H, uint8_t* ws,
                           cudaStream_t st, int slot) {
  const GvPlan g = gemv_plan(qtype, N, K, M);
  CUtensorMap tW, tX;
  if (!tmap_packed(&tW, wq, packed_row_bytes(qtype, K), N, group_bytes(qtype), (uint32_t)g.rows) ||
      !tmap_bf16_rows(&tX, X, K, M, (uint32_t)g.xr))
    return QL_ERR_CUDA;
  float* hf = reinterpret_cast<float*>(ws);
  float* gpart = reinterpret_cast<float*>(ws + g.hp_bytes);
  {
    PdlLaunch L(dim3(1), dim3(kGvHWarps * 32), 0, st);
    const int rc = launch_result(cudaLaunchKernelEx(&L.cfg, gemv_h_kernel, (const __nv_bfloat16*)X,
                                                    (const __nv_bfloat16*)A, (int)M, (int)K, r, hf, H));
    if (rc) return rc;
  }
  GvParams p;
  p.N = (int)N;
  p.K = (int)K;
  p.M = (int)M;
  p.r = r;
  p.nib_mask = 0x000F000Fu;
  p.bf16_magic = 0x43004300u;
  p.ksteps = g.ksteps;
  p.T = g.T;
  p.maxslots = g.maxslots;
  p.gpart = gpart;
  int rc;
  if (qtype == QL_Q4_0)
    rc = g.mt == 1 ? launch_gemv_q<QL_Q4_0, 1>(tW, tX, p, g.G, st, slot)
                   : launch_gemv_q<QL_Q4_0, 2>(tW, tX, p, g.G, st, slot);
  else
    rc = g.mt == 1 ? launch_gemv_q<QL_Q8_0, 1>(tW, tX, p, g.G, st, slot)
                   : launch_gemv_q<QL_Q8_0, 2>(tW, tX, p, g.G, st, slot);
  if (rc) return rc;
  PdlLaunch L(dim3((unsigned)(g.nrb * g.rows / 32)), dim3(128), 0, st);
  return launch_result(cudaLaunchKernelEx(&L.cfg, gemv_finish_kernel, (const float*)gpart, g.maxslots, g.xr, g.rows,
                                          g.ksteps, g.T, g.G, (const float*)hf, (const __nv_bfloat16*)B, (int)N,
                                          (int)M, r, scale, Y, y_dtype));
}

// Small-M input gradient (M <= 16, Q4_0): the dX weight stream, then the k-group sums with G A.
struct GvdPlan {
  int mt, xr, nb, groups, T, G, maxslots;
  size_t smem, part_bytes;
};
// (at 9..16 tokens the doubled B operand work makes it no faster than the tensor-core GEMM)
static bool gemv_dx_applies(int qtype, int64_t M) { return M <= 8 && qtype == QL_Q4_0; }
static GvdPlan gemv_dx_plan(int64_t N, int64_t K, int64_t M) {
  (void)M;  // M <= 8: one token tile
  GvdPlan g;
  g.mt = 1;
  g.xr = 8;
  g.smem = GvdCfg<1>::SMEM_BYTES;
  g.nb = (int)((N + 127) / 128);
  g.groups = (int)(K / 256);
  g.T = g.nb * g.groups;
  const int per_sm = std::max(1, (int)(233472 / (g.smem + 1024)));
  g.G = std::max(1, std::min(g.T, per_sm * num_sms()));
  g.maxslots = 1;
  for (int kg = 0; kg < g.groups; ++kg) {
    const long t0 = (long)kg * g.nb;
    g.maxslots = std::max(g.maxslots, gv_cta_of(t0 + g.nb - 1, g.T, g.G) - gv_cta_of(t0, g.T, g.G) + 1);
  }
  g.part_bytes = (size_t)g.groups * g.maxslots * g.xr * 256 * 4;
  return g;
}

template <int MT>
static int launch_gemv_dx_q(const CUtensorMap& tW, const CUtensorMap& tY, const GvdParams& p, int G, cudaStream_t st,
                            int slot) {
  using C = GvdCfg<MT>;
  auto k = qgemv_dx_kernel<MT>;
  if (set_smem(k, C::SMEM_BYTES) != cudaSuccess) return QL_ERR_CUDA;
  PdlLaunch L(dim3(G), dim3(kGvThreads), C::SMEM_BYTES, st);
  ev_record(slot, 0, st);
  const cudaError_t e = cudaLaunchKernelEx(&L.cfg, k, tW, tY, p);
  ev_record(slot, 1, st);
  return launch_result(e);
}

// dX (the caller's dtype) from W, dY and the row kernel's LA = split(G); part: the plan's partials.
static int launch_gemv_dx(const void* wq, int64_t N, int64_t K, const void* dY, int64_t M, const __nv_bfloat16* LA,
                          int RP, const void* A, int r, void* dX, int dx_dtype, float* part, cudaStream_t st,
                          int slot) {
  const GvdPlan g = gemv_dx_plan(N, K, M);
  CUtensorMap tW, tY;
  if (!tmap_packed(&tW, wq, packed_row_bytes(QL_Q4_0, K), N, group_bytes(QL_Q4_0), 128u) ||
      !tmap_bf16_rows(&tY, dY, N, M, (uint32_t)g.xr))
    return QL_ERR_CUDA;
  GvdParams p;
  p.N = (int)N;
  p.K = (int)K;
  p.M = (int)M;
  p.nib_mask = 0x000F000Fu;
  p.bf16_magic = 0x43004300u;
  p.nb = g.nb;
  p.T = g.T;
  p.maxslots = g.maxslots;
  p.gpart = part;
  const int rc = launch_gemv_dx_q<1>(tW, tY, p, g.G, st, slot);
  if (rc) return rc;
  PdlLaunch L(dim3(g.groups), dim3(256), 0, st);
  return launch_result(cudaLaunchKernelEx(&L.cfg, qgemv_dx_finish_kernel, (const float*)part, g.maxslots, g.xr, g.nb,
                                          g.T, g.G, LA, RP, (const __nv_bfloat16*)A, r, (int)M, (int)K, dX, dx_dtype));
}

// Workspace layout of the dense layer (byte offsets, 256-aligned).
struct LinearWs {
  size_t la, lb, hs, split, cr, fz, hp, dxp, total;
};
static LinearWs linear_ws(int64_t M, int64_t N, int64_t K, int r) {
  LinearWs w;
  const int KL = 2 * lora_rp(r);
  const int64_t NK = N > K ? N : K;
  size_t o = 0;
  w.la = o; o = al256(o + (size_t)M * KL * 2);
  w.lb = o; o = al256(o + (size_t)NK * KL * 2);
  w.hs = o; o = al256(o + (size_t)M * KL * 2);
  const size_t sf = split_bytes(plan_dense(M, N, K, false, true), M, N);
  const size_t sb = split_bytes(plan_dense(M, K, N, true, true), M, K);
  w.split = o; o = al256(o + std::max(sf, sb));
  w.cr = o; o = al256(o + colred_ws_bytes(plan_colred(M, N, K, r), r));
  w.fz = o; o = al256(o + fuse_ctr_bytes(M));
  if (M <= 16) {
    const GvPlan g = gemv_plan(QL_Q4_0, N, K, M), g8 = gemv_plan(QL_Q8_0, N, K, M);
    const size_t gv = std::max(g.hp_bytes + g.part_bytes, g8.hp_bytes + g8.part_bytes);
    w.hp = o; o = al256(o + gv);
    w.dxp = o; o = al256(o + gemv_dx_plan(N, K, M).part_bytes);
  } else {
    w.hp = o;
    w.dxp = o;
  }
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

// ------------------------------------------------------------------------------------------------
// MoE: workspace / saved layouts and launch helpers
// ------------------------------------------------------------------------------------------------
struct MoeSaved {
  size_t g, u, h, hlo, hgu, hd, total;
};
static MoeSaved moe_saved(int64_t T, int k, int64_t H, int64_t I, int r) {
  (void)H;
  const size_t P = (size_t)T * k;
  MoeSaved m;
  size_t o = 0;
  m.g = o; o = al256(o + P * I * 4);
  m.u = o; o = al256(o + P * I * 4);
  m.h = o; o = al256(o + P * I * 2);
  m.hlo = o; o = al256(o + P * I * 2);
  m.hgu = o; o = al256(o + P * r * 4);
  m.hd = o; o = al256(o + P * r * 4);
  m.total = o;
  return m;
}

struct MoeWs {
  size_t xp, yp, row_w, la, lb, g1, g2, dgu, dgulo, dwp, dxp, part, total;
};
static int moe_max_slices(int64_t P, int E) { return (int)((P + 127) / 128 + E); }
static MoeWs moe_ws(int64_t T, int k, int E, int64_t H, int64_t I, int r) {
  const size_t P = (size_t)T * k;
  const size_t KL = 2 * lora_rp(r);
  const size_t HI = (size_t)std::max<int64_t>(H, 2 * I);
  MoeWs w;
  size_t o = 0;
  w.xp = o; o = al256(o + P * H * 2);
  w.yp = o; o = al256(o + P * H * 4);
  w.row_w = o; o = al256(o + P * 4);
  w.la = o; o = al256(o + P * KL * 2);
  w.lb = o; o = al256(o + (size_t)E * HI * KL * 2);
  w.g1 = o; o = al256(o + P * r * 4);
  w.g2 = o; o = al256(o + P * r * 4);
  w.dgu = o; o = al256(o + P * 2 * I * 2);
  w.dgulo = o; o = al256(o + P * 2 * I * 2);
  w.dwp = o; o = al256(o + P * (I / 128) * 4);
  w.dxp = o; o = al256(o + P * H * 4);
  w.part = o; o = al256(o + (size_t)moe_max_slices(P, E) * HI * r * 4);
  w.total = o;
  return w;
}

static int check_moe(int qtype, const void* w_gu, const void* w_d, int E, int64_t H, int64_t I, const void* X, int64_t T,
                     int k, int r) {
  if (!w_gu || !w_d || !X) return QL_ERR_INVALID_ARG;
  if (group_bytes(qtype) == 0) return QL_ERR_UNSUPPORTED;
  if (E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || k > E) return QL_ERR_UNSUPPORTED;
  if (r < 1 || r > 64) return QL_ERR_UNSUPPORTED;
  if (T < 1 || H < 1 || I < 1) return QL_ERR_INVALID_ARG;
  if (H % 256 != 0 || I % 256 != 0) return QL_ERR_SHAPE;
  if (T * k > (1 << 28) || H > (1 << 16) || I > (1 << 16)) return QL_ERR_SHAPE;
  if (!aligned16(w_gu) || !aligned16(w_d) || !aligned16(X)) return QL_ERR_ALIGNMENT;
  return QL_OK;
}

static int launch_rows_seg(const __nv_bfloat16* Y, long ldy, int Kin, const __nv_bfloat16* Z, long zj, long zk, long zes,
                           const int* seg_off, const int* mblk, int E, int r, float oscale, float lscale, float* out,
                           __nv_bfloat16* la, int max_slices, cudaStream_t st) {
  const int RP = lora_rp(r);
  const int NT = r <= 16 ? 2 : (r <= 32 ? 4 : 8);
  const size_t zsm = rows_seg_z_smem(NT, Kin);
  if (Kin % 256 == 0 && zsm <= 220 * 1024) {
    // the expert's whole adapter slice resident in shared memory (two CTAs per SM up to 110 KB)
    cudaError_t e;
    if (NT == 2) {
      e = set_smem(lora_rows_seg_z_kernel<2>, (int)zsm);
      if (e == cudaSuccess)
        launch_pdl(lora_rows_seg_z_kernel<2>, max_slices, 256, zsm, st, Y, ldy, Kin, Z, zj, zk, zes, seg_off, mblk, E, r, oscale,
                                                                lscale, out, la, RP);
    } else if (NT == 4) {
      e = set_smem(lora_rows_seg_z_kernel<4>, (int)zsm);
      if (e == cudaSuccess)
        launch_pdl(lora_rows_seg_z_kernel<4>, max_slices, 256, zsm, st, Y, ldy, Kin, Z, zj, zk, zes, seg_off, mblk, E, r, oscale,
                                                                lscale, out, la, RP);
    } else {
      e = set_smem(lora_rows_seg_z_kernel<8>, (int)zsm);
      if (e == cudaSuccess)
        launch_pdl(lora_rows_seg_z_kernel<8>, max_slices, 256, zsm, st, Y, ldy, Kin, Z, zj, zk, zes, seg_off, mblk, E, r, oscale,
                                                                lscale, out, la, RP);
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return QL_ERR_CUDA;
    return launch_status();
  }
  if (r <= 16)
    launch_pdl(lora_rows_seg_kernel<2>, max_slices, 256, 0, st, Y, ldy, Kin, Z, zj, zk, zes, seg_off, mblk, E, r, oscale, lscale,
                                                        out, la, RP);
  else if (r <= 32)
    launch_pdl(lora_rows_seg_kernel<4>, max_slices, 256, 0, st, Y, ldy, Kin, Z, zj, zk, zes, seg_off, mblk, E, r, oscale, lscale,
                                                        out, la, RP);
  else
    launch_pdl(lora_rows_seg_kernel<8>, max_slices, 256, 0, st, Y, ldy, Kin, Z, zj, zk, zes, seg_off, mblk, E, r, oscale, lscale,
                                                        out, la, RP);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

static int launch_bop_vec(const __nv_bfloat16* Z, long zn, long zjs, long zes, int rows, int nexp, int r,
                          __nv_bfloat16* LB, cudaStream_t st, const int* seg_off = nullptr) {
  const int RP = lora_rp(r);
  // one thread per row of an expert
  const dim3 grid((unsigned)((rows + 255) / 256), nexp);
  launch_pdl(lora_bop_vec_kernel, grid, 256, 0, st, Z, zn, zjs, zes, rows, seg_off, r, RP, LB);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

static int launch_gather(const __nv_bfloat16* src, int cols, const int32_t* perm, int P, int k, __nv_bfloat16* dst,
                         const float* topk_w, float* row_w, cudaStream_t st) {
  const long total = (long)P * (cols / 8);
  const int grid = (int)std::min<long>((total + 255) / 256, (long)num_sms() * 16);
  launch_pdl(moe_gather_rows_kernel, grid, 256, 0, st, src, cols, perm, P, k, dst, topk_w, row_w);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

static int launch_combine(const float* rows, int cols, const int32_t* inv_perm, int T, int k, void* out,
                          int out_dtype, cudaStream_t st) {
  const long total = (long)T * (cols / 4);
  const int grid = (int)std::min<long>((total + 255) / 256, (long)num_sms() * 16);
  launch_pdl(moe_combine_kernel, grid, 256, 0, st, rows, cols, inv_perm, T, k, out, out_dtype);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
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

int qlora_set_rows_fusion(int enable) { return g_rows_fusion.exchange(enable & 3); }

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
  if (group_bytes(qtype) == 0 && qtype != QL_Q6_K && qtype != QL_Q2_K) return QL_ERR_UNSUPPORTED;
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
    case QL_Q5_K: gguf_dequant_kernel<QL_Q5_K><<<grid, 256, 0, st>>>((const uint8_t*)wq, rows, cols, out, out_dtype); break;
    case QL_Q6_K: gguf_dequant_kernel<QL_Q6_K><<<grid, 256, 0, st>>>((const uint8_t*)wq, rows, cols, out, out_dtype); break;
    case QL_Q2_K: gguf_dequant_kernel<QL_Q2_K><<<grid, 256, 0, st>>>((const uint8_t*)wq, rows, cols, out, out_dtype); break;
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
  if (gemv_fwd_applies(qtype, M, r))
    return launch_gemv_fwd(qtype, wq, N, K, X, M, A, B, r, scale, Y, y_dtype, H, wsb + w.hp, st, 0);
  __nv_bfloat16* LA = (__nv_bfloat16*)(wsb + w.la);
  __nv_bfloat16* LB = (__nv_bfloat16*)(wsb + w.lb);
  const int KL = 2 * lora_rp(r);

  // X and A [r x K] in kc-chunk boxes (A's rows past r read as zero)
  CUtensorMap tRY, tZ;
  int kc = 1, stages = 0;
  int rx = dense_fuse_rx(qtype, M, N, K, false, r, st);
  if (rx > 0) {
    fuse_ring(qtype, false, plan_dense(M, N, K, false, true).ms, lora_nt(r), kc, stages);
    if (!tmap_bf16_chunks(&tRY, X, K, M, 128, kc) || !tmap_bf16_chunks(&tZ, A, K, r, 8 * lora_nt(r), kc))
      rx = 0;  // a map is refused: the row kernel instead
  }
  if (rx > 0) {
    // one launch: the GEMM's idle clusters compute H, split(s H) and LB beside the tiles
    RowsFuse f;
    memset(&f, 0, sizeof(f));
    f.r = r;
    f.RP = lora_rp(r);
    f.nt = lora_nt(r);
    f.ztr = 0;
    f.kc = kc;
    f.stages = stages;
    f.oscale = 1.0f;
    f.lscale = scale;
    f.out = H;
    f.la = LA;
    f.lbz = (const __nv_bfloat16*)B;
    f.lbzn = r;
    f.lbzj = 1;
    f.lb_rows = (int)N;
    f.lb = LB;
    f.ctr = (unsigned long long*)(wsb + w.fz);
    f.seq = next_fuse_seq();
    return launch_dense_gemm<false>(qtype, X, M, K, wq, N, K, LA, LB, KL, N, Y, y_dtype, (float*)(wsb + w.split),
                                    true, st, 0, rx, &f, &tRY, &tZ);
  }

  // H = X A^T (saved), the split operand of s*H, and LB = [B | B]
  rc = launch_rows_dense((const __nv_bfloat16*)X, K, (int)M, (int)K, (const __nv_bfloat16*)A, K, 1, r, 1.0f, scale, H,
                         LA, BopArgs{(const __nv_bfloat16*)B, r, 1, (int)N}, LB, st);
  if (rc) return rc;

  return launch_dense_gemm<false>(qtype, X, M, K, wq, N, K, LA, LB, KL, N, Y, y_dtype, (float*)(wsb + w.split), true,
                                  st, 0);
}

static size_t moe_route_ws(int64_t T, int E) { return al256((size_t)((T + kRouteRow - 1) / kRouteRow) * E * 4); }

size_t qlora_moe_route_workspace_bytes(int64_t T, int E, int k) {
  if (T < 1 || E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || k > E) return 0;
  return moe_route_ws(T, E);
}

int qlora_moe_route(const void* logits, int64_t T, int E, int k, int32_t* topk_idx, float* topk_w, int32_t* counts,
                    int32_t* offsets, int32_t* perm, int32_t* inv_perm, int32_t* mblk, void* ws, size_t ws_bytes,
                    void* stream) {
  if (!logits || !topk_idx || !topk_w || !counts || !offsets || !perm || !inv_perm || !mblk) return QL_ERR_INVALID_ARG;
  if (E < 1 || E > kMaxExperts || k < 1 || k > kMaxTopK || k > E) return QL_ERR_UNSUPPORTED;
  if (T < 1) return QL_ERR_INVALID_ARG;
  if (T > (1 << 24)) return QL_ERR_SHAPE;
  if (!ws || ws_bytes < moe_route_ws(T, E)) return QL_ERR_WORKSPACE;
  if (!aligned16(ws)) return QL_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  const int nrow = (int)((T + kRouteRow - 1) / kRouteRow);
  int32_t* hist = (int32_t*)ws;
  launch_pdl(moe_route_select_kernel, nrow, 32 * kRouteRow, 0, st, (const __nv_bfloat16*)logits, (int)T, E, k, topk_idx,
                                                           topk_w, hist);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (launch_status() != QL_OK) return QL_ERR_CUDA;
  launch_pdl(moe_route_scan_kernel, 1, kMaxExperts, 0, st, hist, E, nrow, counts, offsets, mblk);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (launch_status() != QL_OK) return QL_ERR_CUDA;
  launch_pdl(moe_route_place_kernel, (nrow + 7) / 8, 256, 0, st, topk_idx, hist, offsets, (int)T, E, k, perm, inv_perm);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

size_t qlora_moe_saved_bytes(int64_t T, int k, int64_t H, int64_t I, int r) {
  if (T < 1 || k < 1 || H < 1 || I < 1 || r < 1 || r > 64) return 0;
  return moe_saved(T, k, H, I, r).total;
}

size_t qlora_moe_workspace_bytes(int64_t T, int k, int E, int64_t H, int64_t I, int r) {
  if (T < 1 || k < 1 || E < 1 || H < 1 || I < 1 || r < 1 || r > 64) return 0;
  return moe_ws(T, k, E, H, I, r).total;
}

int qlora_moe_fwd(int qtype, const void* w_gu, const void* w_d, int E, int64_t H, int64_t I, const void* X, int64_t T,
                  int k, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets, const int32_t* perm,
                  const int32_t* inv_perm, const int32_t* mblk, const void* A_gu, const void* B_gu, const void* A_d,
                  const void* B_d, int r, float scale, void* Y, int y_dtype, void* saved, size_t saved_bytes, void* ws,
                  size_t ws_bytes, void* stream) {
  int rc = check_moe(qtype, w_gu, w_d, E, H, I, X, T, k, r);
  if (rc) return rc;
  if (!topk_idx || !topk_w || !offsets || !perm || !inv_perm || !mblk || !A_gu || !B_gu || !A_d || !B_d || !Y || !saved)
    return QL_ERR_INVALID_ARG;
  if (y_dtype != QL_F32 && y_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (!aligned16(A_gu) || !aligned16(B_gu) || !aligned16(A_d) || !aligned16(B_d) || !aligned16(Y) || !aligned16(saved))
    return QL_ERR_ALIGNMENT;
  const MoeSaved sv = moe_saved(T, k, H, I, r);
  const MoeWs w = moe_ws(T, k, E, H, I, r);
  if (saved_bytes < sv.total) return QL_ERR_WORKSPACE;
  if (!ws || ws_bytes < w.total) return QL_ERR_WORKSPACE;
  if (!aligned16(ws)) return QL_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  const int P = (int)(T * k);
  const int KL = 2 * lora_rp(r);
  const int ms = moe_max_slices(P, E);
  uint8_t* wb = (uint8_t*)ws;
  uint8_t* sb = (uint8_t*)saved;
  __nv_bfloat16* Xp = (__nv_bfloat16*)(wb + w.xp);
  float* pair_out = (float*)(wb + w.yp);
  float* row_w = (float*)(wb + w.row_w);
  __nv_bfloat16* LA = (__nv_bfloat16*)(wb + w.la);
  __nv_bfloat16* LB = (__nv_bfloat16*)(wb + w.lb);
  float* g = (float*)(sb + sv.g);
  float* u = (float*)(sb + sv.u);
  __nv_bfloat16* h = (__nv_bfloat16*)(sb + sv.h);
  float* Hgu = (float*)(sb + sv.hgu);
  float* Hd = (float*)(sb + sv.hd);
  const int* off = offsets;

  rc = launch_gather((const __nv_bfloat16*)X, (int)H, perm, P, k, Xp, topk_w, row_w, st);
  if (rc) return rc;
  // gate/up: Hgu = Xp A_gu^T (saved), LA = split(s Hgu), LB = [B_gu | B_gu]
  rc = launch_rows_seg(Xp, H, (int)H, (const __nv_bfloat16*)A_gu, H, 1, (long)r * H, off, mblk, E, r, 1.0f, scale, Hgu,
                       LA, ms, st);
  if (rc) return rc;
  rc = launch_bop_vec((const __nv_bfloat16*)B_gu, r, 1, (long)2 * I * r, (int)(2 * I), E, r, LB, st, off);
  if (rc) return rc;
  const int nsm = num_sms();
  {
    CUtensorMap tA, tW, tLA, tLB;
    if (!tmap_bf16_rows(&tA, Xp, H, P, 128) ||
        !tmap_packed(&tW, w_gu, packed_row_bytes(qtype, H), (uint64_t)E * 2 * I, group_bytes(qtype)) ||
        !tmap_bf16_rows(&tLA, LA, KL, P, 128) || !tmap_bf16_rows(&tLB, LB, KL, (uint64_t)E * 2 * I, 64))
      return QL_ERR_CUDA;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    const int bn = grouped_bn(qtype, I, 128);  // a tile holds bn/2 gate and bn/2 up columns
    p.M = P; p.Nd = (int)(2 * I); p.Kd = (int)H; p.n_lora_kb = KL / 64; p.num_n_tiles = (int)(I / (bn / 2));
    p.w_rows_per_expert = (int)(2 * I); p.lb_rows_per_expert = (int)(2 * I); p.I = (int)I;
    p.E = E; p.seg_off = off; p.mblk_off = mblk; p.ksplit = 1;
    p.out_gf = g; p.out_uf = u; p.out_h = h; p.out_lo = (__nv_bfloat16*)(sb + sv.hlo);
    rc = launch_qgemm_q<false, EPI_SWIGLU, 1>(qtype, tA, tW, tLA, tLB, p, nsm, st, 2, bn);
    if (rc) return rc;
  }
  // down: Hd = h A_d^T (saved), LA = split(s Hd), LB = [B_d | B_d]
  rc = launch_rows_seg(h, I, (int)I, (const __nv_bfloat16*)A_d, I, 1, (long)r * I, off, mblk, E, r, 1.0f, scale, Hd, LA,
                       ms, st);
  if (rc) return rc;
  rc = launch_bop_vec((const __nv_bfloat16*)B_d, r, 1, (long)H * r, (int)H, E, r, LB, st, off);
  if (rc) return rc;
  {
    CUtensorMap tA, tW, tLA, tLB;
    if (!tmap_bf16_rows(&tA, h, I, P, 128) ||
        !tmap_packed(&tW, w_d, packed_row_bytes(qtype, I), (uint64_t)E * H, group_bytes(qtype)) ||
        !tmap_bf16_rows(&tLA, LA, KL, P, 128) || !tmap_bf16_rows(&tLB, LB, KL, (uint64_t)E * H, 64))
      return QL_ERR_CUDA;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    const int bn = grouped_bn(qtype, H, 256);
    p.M = P; p.Nd = (int)H; p.Kd = (int)I; p.n_lora_kb = KL / 64; p.num_n_tiles = (int)(H / bn);
    p.w_rows_per_expert = (int)H; p.lb_rows_per_expert = (int)H; p.I = (int)I;
    p.E = E; p.seg_off = off; p.mblk_off = mblk; p.ksplit = 1;
    p.out = pair_out; p.out_dtype = QL_F32; p.ldo = H; p.row_w = row_w;
    rc = launch_qgemm_q<false, EPI_PAIR_OUT, 1>(qtype, tA, tW, tLA, tLB, p, nsm, st, 3, bn);
    if (rc) return rc;
  }
  return launch_combine(pair_out, (int)H, inv_perm, (int)T, k, Y, y_dtype, st);
}

int qlora_moe_bwd(int qtype, const void* w_gu, const void* w_d, int E, int64_t H, int64_t I, const void* X, const void* dY,
                  int64_t T, int k, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                  const int32_t* perm, const int32_t* inv_perm, const int32_t* mblk, const void* A_gu, const void* B_gu,
                  const void* A_d, const void* B_d, int r, float scale, const void* saved, size_t saved_bytes, void* dX,
                  int dx_dtype, float* dA_gu, float* dB_gu, float* dA_d, float* dB_d, float* d_logits, void* ws,
                  size_t ws_bytes, void* stream) {
  int rc = check_moe(qtype, w_gu, w_d, E, H, I, X, T, k, r);
  if (rc) return rc;
  if (!dY || !topk_idx || !topk_w || !offsets || !perm || !inv_perm || !mblk || !A_gu || !B_gu || !A_d || !B_d ||
      !saved || !dX || !dA_gu || !dB_gu || !dA_d || !dB_d)
    return QL_ERR_INVALID_ARG;
  if (dx_dtype != QL_F32 && dx_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(dX) || !aligned16(saved) || !aligned16(dA_gu) || !aligned16(dB_gu) ||
      !aligned16(dA_d) || !aligned16(dB_d) || (d_logits && !aligned16(d_logits)))
    return QL_ERR_ALIGNMENT;
  const MoeSaved sv = moe_saved(T, k, H, I, r);
  const MoeWs w = moe_ws(T, k, E, H, I, r);
  if (saved_bytes < sv.total) return QL_ERR_WORKSPACE;
  if (!ws || ws_bytes < w.total) return QL_ERR_WORKSPACE;
  if (!aligned16(ws)) return QL_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  const int P = (int)(T * k);
  const int KL = 2 * lora_rp(r);
  const int ms = moe_max_slices(P, E);
  uint8_t* wb = (uint8_t*)ws;
  const uint8_t* sb = (const uint8_t*)saved;
  __nv_bfloat16* dYp = (__nv_bfloat16*)(wb + w.yp);
  float* row_w = (float*)(wb + w.row_w);
  __nv_bfloat16* LA = (__nv_bfloat16*)(wb + w.la);
  __nv_bfloat16* LB = (__nv_bfloat16*)(wb + w.lb);
  float* Gd = (float*)(wb + w.g1);
  float* Ggu = (float*)(wb + w.g2);
  __nv_bfloat16* dgu = (__nv_bfloat16*)(wb + w.dgu);
  __nv_bfloat16* dgu_lo = (__nv_bfloat16*)(wb + w.dgulo);
  float* dwp = (float*)(wb + w.dwp);
  float* dxp = (float*)(wb + w.dxp);
  float* part = (float*)(wb + w.part);
  const float* g = (const float*)(sb + sv.g);
  const float* u = (const float*)(sb + sv.u);
  const __nv_bfloat16* h = (const __nv_bfloat16*)(sb + sv.h);
  const __nv_bfloat16* h_lo = (const __nv_bfloat16*)(sb + sv.hlo);
  const float* Hgu = (const float*)(sb + sv.hgu);
  const float* Hd = (const float*)(sb + sv.hd);
  const int* off = offsets;
  const int nsm = num_sms();

  // dY in pair order (and each pair's routing weight); X is read in place by its one consumer
  rc = launch_gather((const __nv_bfloat16*)dY, (int)H, perm, P, k, dYp, topk_w, row_w, st);
  if (rc) return rc;
  int dw_tiles = 0;  // output-column tiles of the down input-gradient GEMM (dw partials per row)
  // down input-gradient: Gd = s dYp B_d, LA = split(Gd), LB[e][i] = [A_d^T | A_d^T]
  rc = launch_rows_seg(dYp, H, (int)H, (const __nv_bfloat16*)B_d, 1, r, (long)H * r, off, mblk, E, r, scale, scale, Gd,
                       LA, ms, st);
  if (rc) return rc;
  rc = launch_bop_vec((const __nv_bfloat16*)A_d, 1, I, (long)r * I, (int)I, E, r, LB, st, off);
  if (rc) return rc;
  {
    CUtensorMap tA, tW, tLA, tLB;
    if (!tmap_bf16_rows(&tA, dYp, H, P, 128) ||
        !tmap_packed(&tW, w_d, packed_row_bytes(qtype, I), (uint64_t)E * H, group_bytes(qtype)) ||
        !tmap_bf16_rows(&tLA, LA, KL, P, 128) || !tmap_bf16_rows(&tLB, LB, KL, (uint64_t)E * I, 64))
      return QL_ERR_CUDA;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    dw_tiles = (int)(I / grouped_bn(qtype, I, 256));
    p.M = P; p.Nd = (int)I; p.Kd = (int)H; p.n_lora_kb = KL / 64; p.num_n_tiles = dw_tiles;
    p.w_rows_per_expert = (int)H; p.lb_rows_per_expert = (int)I; p.I = (int)I;
    p.E = E; p.seg_off = off; p.mblk_off = mblk; p.ksplit = 1;
    p.in_gf = g; p.in_uf = u; p.out_g = dgu; p.out_lo = dgu_lo; p.row_w = row_w; p.dw_part = dwp;
    rc = launch_qgemm_q<true, EPI_SWIGLU_BWD, 1>(qtype, tA, tW, tLA, tLB, p, nsm, st, 4, grouped_bn(qtype, I, 256));
    if (rc) return rc;
  }
  // down adapter gradients: dA_d = sum_p w_p Gd_p^T h_p ; dB_d = s sum_p w_p dYp_p^T Hd_p
  rc = launch_colred(h, I, (int)I, Gd, r, P, row_w, off, mblk, E, ms, part, 1.0f, 1, dA_d, st, h_lo);
  if (rc) return rc;
  rc = launch_colred(dYp, H, (int)H, Hd, r, P, row_w, off, mblk, E, ms, part, scale, 0, dB_d, st);
  if (rc) return rc;
  // gate/up input-gradient: Ggu = s dgu B_gu, LA = split(Ggu), LB[e][hh] = [A_gu^T | A_gu^T]
  rc = launch_rows_seg(dgu, 2 * I, (int)(2 * I), (const __nv_bfloat16*)B_gu, 1, r, (long)2 * I * r, off, mblk, E, r,
                       scale, scale, Ggu, LA, ms, st);
  if (rc) return rc;
  rc = launch_bop_vec((const __nv_bfloat16*)A_gu, 1, H, (long)r * H, (int)H, E, r, LB, st, off);
  if (rc) return rc;
  {
    CUtensorMap tA, tW, tLA, tLB;
    if (!tmap_bf16_rows(&tA, dgu, 2 * I, P, 128) ||
        !tmap_packed(&tW, w_gu, packed_row_bytes(qtype, H), (uint64_t)E * 2 * I, group_bytes(qtype)) ||
        !tmap_bf16_rows(&tLA, LA, KL, P, 128) || !tmap_bf16_rows(&tLB, LB, KL, (uint64_t)E * H, 64))
      return QL_ERR_CUDA;
    GemmParams p;
    memset(&p, 0, sizeof(p));
    const int bn = grouped_bn(qtype, H, 256);
    p.M = P; p.Nd = (int)H; p.Kd = (int)(2 * I); p.n_lora_kb = KL / 64; p.num_n_tiles = (int)(H / bn);
    p.w_rows_per_expert = (int)(2 * I); p.lb_rows_per_expert = (int)H; p.I = (int)I;
    p.E = E; p.seg_off = off; p.mblk_off = mblk; p.ksplit = 1;
    p.out = dxp; p.out_dtype = QL_F32; p.ldo = H;
    rc = launch_qgemm_q<true, EPI_STORE, 1>(qtype, tA, tW, tLA, tLB, p, nsm, st, 5, bn);
    if (rc) return rc;
  }
  rc = launch_combine(dxp, (int)H, inv_perm, (int)T, k, dX, dx_dtype, st);
  if (rc) return rc;
  // gate/up adapter gradients: dA_gu = sum_p Ggu_p^T x_p (x_p = X row perm[p] / k, read in place);
  // dB_gu = s sum_p dgu_p^T Hgu_p
  rc = launch_colred((const __nv_bfloat16*)X, H, (int)H, Ggu, r, P, nullptr, off, mblk, E, ms, part, 1.0f, 1, dA_gu, st,
                     nullptr, perm, k);
  if (rc) return rc;
  rc = launch_colred(dgu, 2 * I, (int)(2 * I), Hgu, r, P, nullptr, off, mblk, E, ms, part, scale, 0, dB_gu, st, dgu_lo);
  if (rc) return rc;
  if (d_logits != nullptr) {
    launch_pdl(moe_dw_dlogits_kernel, (int)((T + 7) / 8), 256, 0, st, dwp, dw_tiles, inv_perm, topk_idx, topk_w,
                                                                  (int)T, E, k, nullptr, d_logits);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return launch_status();
  }
  return QL_OK;
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
  const int KL = 2 * lora_rp(r);

  __nv_bfloat16* HS = (__nv_bfloat16*)(wsb + w.hs);
  uint8_t* crws = wsb + w.cr;
  const int ncr = (int)(colred_ctr_bytes(plan_colred(M, N, K, r)) / 4);
  const ColredOut ob{(int)N, 1.0f, 0, dB};
  const ColredOut oa{(int)K, 1.0f, 1, dA};

  // dY in kc-chunk boxes, and B [N x r] as boxes of 64 kc rows x RN (columns past r read as zero)
  CUtensorMap tRY, tZ;
  int kc = 1, stages = 0;
  int rx = dX != nullptr && !gemv_dx_applies(qtype, M) ? dense_fuse_rx(qtype, M, K, N, true, r, st) : 0;
  if (rx > 0) {
    fuse_ring(qtype, true, plan_dense(M, K, N, true, true).ms, lora_nt(r), kc, stages);
    if (!tmap_bf16_chunks(&tRY, dY, N, M, 128, kc) ||
        !make_tmap(&tZ, B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r, N, (uint64_t)r * 2, 8 * lora_nt(r), 64 * kc,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
      rx = 0;  // a map is refused: the row kernel instead
  }
  if (rx > 0) {
    // one launch for G = s dY B (as LA = split(G)), HS = split(s H), LB = [A^T | A^T] and the dX
    // GEMM; the column reduction then waits for the row clusters' count, not for the GEMM
    RowsFuse f;
    memset(&f, 0, sizeof(f));
    f.r = r;
    f.RP = lora_rp(r);
    f.nt = lora_nt(r);
    f.ztr = 1;
    f.kc = kc;
    f.stages = stages;
    f.oscale = scale;
    f.lscale = scale;
    f.out = nullptr;
    f.la = LA;
    f.lbz = (const __nv_bfloat16*)A;
    f.lbzn = 1;
    f.lbzj = K;
    f.lb_rows = (int)K;
    f.lb = LB;
    f.hin = H;
    f.hscale = scale;
    f.hs = HS;
    f.ctr = (unsigned long long*)(wsb + w.fz);
    f.seq = next_fuse_seq();
    f.zc = (int*)crws;
    f.zn = ncr;
    rc = launch_dense_gemm<true>(qtype, dY, M, N, wq, N, K, LA, LB, KL, K, dX, dx_dtype, (float*)(wsb + w.split),
                                 true, st, 1, rx, &f, &tRY, &tZ);
    if (rc) return rc;
    return launch_colred_dense((const __nv_bfloat16*)dY, (int)N, HS, ob, (const __nv_bfloat16*)X, (int)K, LA, oa,
                               (int)M, r, crws, 1, st, f.ctr + 1, f.seq, 2 * rx);
  }
  // LA = split(G) with G = s dY B, HS = split(s H), and LB[k] = [A^T(k) | A^T(k)]; the column
  // reduction's counters are zeroed on the way
  // (LB only for the tensor-core dX GEMM: the small-M dX path reads A itself)
  const bool need_lb = dX != nullptr && !gemv_dx_applies(qtype, M);
  if (dX != nullptr && gemv_dx_applies(qtype, M) && r <= 16) {
    // a handful of token rows: one CTA (the weight stream after it does not need LB)
    PdlLaunch L(dim3(1), dim3(kGvHWarps * 32), 0, st);
    rc = launch_result(cudaLaunchKernelEx(&L.cfg, gemv_g_kernel, (const __nv_bfloat16*)dY, (const __nv_bfloat16*)B, H,
                                          (int)M, (int)N, r, scale, lora_rp(r), LA, HS, (int*)crws, ncr));
  } else {
    rc = launch_rows_dense((const __nv_bfloat16*)dY, N, (int)M, (int)N, (const __nv_bfloat16*)B, 1, r, r, scale,
                           scale, nullptr, LA,
                           need_lb ? BopArgs{(const __nv_bfloat16*)A, 1, K, (int)K} : BopArgs{nullptr, 0, 0, 0}, LB,
                           st, H, scale, HS, (int*)crws, ncr);
  }
  if (rc) return rc;
  if (dX && gemv_dx_applies(qtype, M)) {
    // weight streaming: W read once, G A added in the finish launch
    rc = launch_gemv_dx(wq, N, K, dY, M, LA, lora_rp(r), A, r, dX, dx_dtype, (float*)(wsb + w.dxp), st, 1);
    if (rc) return rc;
  }
  bool sum_pending = false;
  if (dX && !gemv_dx_applies(qtype, M)) {
    rc = launch_dense_gemm<true>(qtype, dY, M, N, wq, N, K, LA, LB, KL, K, dX, dx_dtype,
                                 (float*)(wsb + w.split), true, st, 1, 0, nullptr, nullptr, nullptr, &sum_pending);
    if (rc) return rc;
  }
  // dB = dY^T split(s H) and dA = split(G)^T X in one launch; after the dX GEMM (which waited for
  // the row kernel) it runs beside the GEMM on the SMs the GEMM leaves idle
  rc = launch_colred_dense((const __nv_bfloat16*)dY, (int)N, HS, ob, (const __nv_bfloat16*)X, (int)K, LA, oa, (int)M,
                           r, crws, dX ? 1 : 0, st);
  if (rc || !sum_pending) return rc;
  // the dX GEMM split K: its fp32 parts are summed after the column reductions (two launches after
  // the GEMM, which has completed by then), so those still run beside the GEMM
  const DensePlan d = plan_dense(M, K, N, true, true);
  return launch_split_reduce((float*)(wsb + w.split), d.ksplit, (long)M * K, (long)M * K, dX, dx_dtype, st);
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
// per device: the context the address was looked up in, and the address
static void* g_static_scratch_ctx[kMaxDevices] = {};
static void* g_static_scratch_dev[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
static CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_static_scratch in the current device's current context. It is looked up
// (cudaGetSymbolAddress) on the first use in a context and again whenever the context differs
// from the one it was looked up in: after a device reset the module is loaded anew and the array
// may sit elsewhere.
static int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return QL_ERR_UNSUPPORTED;
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (get_ctx == nullptr || get_ctx(&ctx) != CUDA_SUCCESS) return QL_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (ctx == nullptr || g_static_scratch_dev[dev] == nullptr || g_static_scratch_ctx[dev] != (void*)ctx) {
    void* ptr = nullptr;
    // also makes the device's primary context current if no context was
    if (cudaGetSymbolAddress((void**)&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr) return QL_ERR_CUDA;
    if (ctx == nullptr && (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr)) return QL_ERR_CUDA;
    g_static_scratch_dev[dev] = ptr;
    g_static_scratch_ctx[dev] = (void*)ctx;
  }
  *out = g_static_scratch_dev[dev];
  return QL_OK;
}

}  // namespace qlora

// ------------------------------------------------------------------------------------------------
// 8-bit AdamW on the adapters
// ------------------------------------------------------------------------------------------------
namespace qlora {

// The dynamic tree code tables: after the optional sign bit, E zero bits (the decade 10^-E), an
// indicator bit and B fraction bits F; |entry| = (0.1 + 0.9 (F + 1/2) / 2^B) / 10^E; no indicator
// codes 0. Entries are formed in fp64 and rounded once to fp32.
static void build_adamw8_tables(Adamw8Tables& T) {
  static const double p10[9] = {1.0, 10.0, 100.0, 1000.0, 1e4, 1e5, 1e6, 1e7, 1e8};
  for (int sg = 0; sg < 2; ++sg) {
    const bool is_signed = sg == 0;
    const int nbits = is_signed ? 7 : 8;
    float* dec = is_signed ? T.dec_s : T.dec_u;
    for (int q = 0; q < 256; ++q) {
      const int bits = q & ((1 << nbits) - 1);
      const bool neg = is_signed && ((q >> 7) & 1);
      double v = 0.0;
      if (bits != 0) {
        int top = 0;
        while ((bits >> (top + 1)) != 0) ++top;          // index of the highest set bit
        const int E = nbits - 1 - top;
        const int B = nbits - E - 1;
        const int F = bits & ((1 << B) - 1);
        v = (0.1 + 0.9 * (F + 0.5) / std::ldexp(1.0, B)) / p10[E];
      }
      dec[q] = (float)(neg ? -v : v);
    }
    // distinct entries ascending (the signed -0 code 0x80 never produced), with their codes
    std::vector<std::pair<float, int>> e;
    for (int q = 0; q < 256; ++q)
      if (!(is_signed && q == 0x80)) e.push_back({dec[q], q});
    std::stable_sort(e.begin(), e.end(), [](const std::pair<float, int>& x, const std::pair<float, int>& y) {
      return x.first < y.first;
    });
    float* srt = is_signed ? T.srt_s : T.srt_u;
    uint8_t* cod = is_signed ? T.cod_s : T.cod_u;
    for (int k = 0; k < 256; ++k) {
      srt[k] = k < (int)e.size() ? e[k].first : 2.0f;
      cod[k] = k < (int)e.size() ? (uint8_t)e[k].second : 0;
    }
    (is_signed ? T.ns : T.nu) = (int)e.size();
  }
}

static const Adamw8Tables& adamw8_tables() {
  static Adamw8Tables T;
  static std::once_flag once;
  std::call_once(once, [] { build_adamw8_tables(T); });
  return T;
}

}  // namespace qlora

// ------------------------------------------------------------------------------------------------
// Quantized lm_head with chunked cross-entropy
// ------------------------------------------------------------------------------------------------
namespace qlora {

struct LmWs {
  size_t logits, dlog, stats, split_f, split_x, total;
};
static LmWs lm_ws(int64_t M, int64_t V, int64_t K, int64_t chunk) {
  const int64_t C = std::min(chunk, M);
  const int64_t tail = M % C;
  size_t sf = 0, sx = 0;
  for (int64_t rows : {C, tail}) {
    if (rows < 1) continue;
    sf = std::max(sf, split_bytes(plan_dense(rows, V, K, false, true), rows, V));
    sx = std::max(sx, split_bytes(plan_dense(rows, K, V, true, true), rows, K));
  }
  LmWs w;
  size_t o = 0;
  w.logits = o; o = al256(o + (size_t)C * V * 4);
  w.dlog = o; o = al256(o + (size_t)C * V * 2);
  w.stats = o; o = al256(o + (size_t)C * ((V + 255) / 256) * 8);  // (max, sum exp) per row and 256 columns
  w.split_f = o; o = al256(o + sf);
  w.split_x = o; o = al256(o + sx);
  w.total = o;
  return w;
}

}  // namespace qlora

extern "C" size_t qlora_lm_head_ce_workspace_bytes(int64_t M, int64_t V, int64_t K, int64_t chunk) {
  if (M < 1 || V < 1 || K < 1 || chunk < 1) return 0;
  return lm_ws(M, V, K, chunk).total;
}

extern "C" int qlora_lm_head_ce(int qtype, const void* wq, int64_t V, int64_t K, const void* X, int64_t M,
                                const int32_t* labels, int64_t chunk, float grad_scale, float* loss, void* dX,
                                int dx_dtype, void* ws, size_t ws_bytes, void* stream) {
  if (!wq || !X || !labels || !loss) return QL_ERR_INVALID_ARG;
  if (group_bytes(qtype) == 0) return QL_ERR_UNSUPPORTED;
  if (M < 1 || V < 64 || K < 256 || chunk < 1) return QL_ERR_INVALID_ARG;
  if (K % 256 != 0 || V % 64 != 0 || M > (1 << 26) || K > (1 << 16) || V > (1 << 22)) return QL_ERR_SHAPE;
  if (dX && dx_dtype != QL_F32 && dx_dtype != QL_BF16) return QL_ERR_INVALID_ARG;
  if (!aligned16(wq) || !aligned16(X) || !aligned16(loss) || (dX && !aligned16(dX))) return QL_ERR_ALIGNMENT;
  const LmWs w = lm_ws(M, V, K, chunk);
  if (!ws || ws_bytes < w.total) return QL_ERR_WORKSPACE;
  if (!aligned16(ws)) return QL_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* wsb = (uint8_t*)ws;
  float* logits = (float*)(wsb + w.logits);
  __nv_bfloat16* dlog = (__nv_bfloat16*)(wsb + w.dlog);
  const int64_t C = std::min(chunk, M);
  const size_t xes = dx_dtype == QL_F32 ? 4 : 2;
  for (int64_t c0 = 0; c0 < M; c0 += C) {
    const int64_t rows = std::min(C, M - c0);
    const __nv_bfloat16* Xc = (const __nv_bfloat16*)X + c0 * K;
    // logits = X_c deq(W)^T, fp32, no adapter; the pair GEMM (more than 128 rows, no K split) also
    // leaves each row's (max, sum exp) per 256 columns, so the CE kernel reads the logits once
    const DensePlan d = plan_dense(rows, V, K, false, true);
    const bool with_stats = d.ms != 0 && d.ksplit == 1 && d.ntiles == (int)((V + 255) / 256);
    float2* stats = with_stats ? (float2*)(wsb + w.stats) : nullptr;
    int rc = launch_dense_gemm<false>(qtype, Xc, rows, K, wq, V, K, nullptr, nullptr, 0, V, logits, QL_F32,
                                      (float*)(wsb + w.split_f), true, st, 0, 0, nullptr, nullptr, nullptr,
                                      nullptr, stats);
    if (rc) return rc;
    // the CE kernel and the input-gradient GEMM each read what the launch right before them wrote:
    // they start only once it has completed
    NoEarlyStart serial;
    lm_ce_kernel<<<(unsigned)std::min<int64_t>(rows, num_sms()), kCeThreads, 0, st>>>(
        logits, (int)V, (int)rows, stats, with_stats ? d.ntiles : 0, labels + c0, grad_scale, loss + c0,
        dX ? dlog : nullptr);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (launch_status() != QL_OK) return QL_ERR_CUDA;
    if (dX) {
      rc = launch_dense_gemm<true>(qtype, dlog, rows, V, wq, V, K, nullptr, nullptr, 0, K,
                                   (uint8_t*)dX + c0 * K * xes, dx_dtype, (float*)(wsb + w.split_x), true, st, 1);
      if (rc) return rc;
    }
  }
  return QL_OK;
}

extern "C" int qlora_rmsnorm_fwd(const void* X, const void* gamma, int64_t M, int64_t K, float eps, void* Xn,
                                 float* rstd, void* stream) {
  if (!X || !gamma || !Xn || !rstd) return QL_ERR_INVALID_ARG;
  if (M < 1 || K < 8 || !(eps >= 0.f)) return QL_ERR_INVALID_ARG;
  if (K % 8 != 0 || M > (1 << 28) || K > (1 << 24)) return QL_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(gamma) || !aligned16(Xn)) return QL_ERR_ALIGNMENT;
  const long threads = M * 32L;
  rmsnorm_fwd_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
      (const __nv_bfloat16*)X, (const __nv_bfloat16*)gamma, (int)M, (int)K, eps, (__nv_bfloat16*)Xn, rstd);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

extern "C" int qlora_rmsnorm_bwd(const void* X, const void* gamma, const float* rstd, const void* dXn, int dxn_dtype,
                                 int64_t M, int64_t K, void* dX, int dx_dtype, void* stream) {
  if (!X || !gamma || !rstd || !dXn || !dX) return QL_ERR_INVALID_ARG;
  if ((dxn_dtype != QL_F32 && dxn_dtype != QL_BF16) || (dx_dtype != QL_F32 && dx_dtype != QL_BF16))
    return QL_ERR_INVALID_ARG;
  if (M < 1 || K < 8) return QL_ERR_INVALID_ARG;
  if (K % 8 != 0 || M > (1 << 28) || K > (1 << 24)) return QL_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(gamma) || !aligned16(dXn) || !aligned16(dX)) return QL_ERR_ALIGNMENT;
  const long threads = M * 32L;
  rmsnorm_bwd_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
      (const __nv_bfloat16*)X, (const __nv_bfloat16*)gamma, rstd, dXn, dxn_dtype, (int)M, (int)K, dX, dx_dtype);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

extern "C" int qlora_adamw8_step(float* p, const float* grad, uint8_t* m_q, float* m_absmax, uint8_t* v_q,
                                 float* v_absmax, int64_t n, float lr, float beta1, float beta2, float eps,
                                 float weight_decay, int64_t step, void* p_bf16, void* stream) {
  if (!p || !grad || !m_q || !m_absmax || !v_q || !v_absmax) return QL_ERR_INVALID_ARG;
  if (n < 1 || step < 1) return QL_ERR_INVALID_ARG;
  if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps > 0.f)) return QL_ERR_INVALID_ARG;
  if (n > ((int64_t)1 << 40)) return QL_ERR_SHAPE;
  Adamw8Args a;
  a.lr = lr;
  a.b1 = beta1;
  a.b2 = beta2;
  a.eps = eps;
  a.wd = weight_decay;
  a.c1 = (float)(1.0 - std::pow((double)beta1, (double)step));
  a.c2 = (float)(1.0 - std::pow((double)beta2, (double)step));
  const long nblk = (long)((n + kAdamBlock - 1) / kAdamBlock);
  adamw8_kernel<<<(unsigned)nblk, kAdamBlock, 0, (cudaStream_t)stream>>>(p, grad, m_q, m_absmax, v_q, v_absmax, (long)n,
                                                                        a, adamw8_tables(),
                                                                        (__nv_bfloat16*)p_bf16);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

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
  const size_t lb_bytes = al256((size_t)N * KL * 2);
  if (la_bytes + lb_bytes > kStaticScratchBytes) return QL_ERR_WORKSPACE;
  void* base = nullptr;
  rc = static_scratch_address(&base);
  if (rc != QL_OK) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  // Both operands are rewritten in full (padding included) before the GEMM reads them, so what
  // an earlier call left in the array does not matter.
  __nv_bfloat16* LA = (__nv_bfloat16*)base;
  __nv_bfloat16* LB = (__nv_bfloat16*)((uint8_t*)base + la_bytes);

  rc = launch_rows_dense((const __nv_bfloat16*)X, K, (int)M, (int)K, (const __nv_bfloat16*)A, K, 1, r, 1.0f, scale, H,
                         LA, BopArgs{(const __nv_bfloat16*)B, r, 1, (int)N}, LB, st);
  if (rc) return rc;
  // no K split here: its partials would need more scratch than the static array holds
  return launch_dense_gemm<false>(qtype, X, M, K, wq, N, K, LA, LB, KL, N, Y, y_dtype, nullptr, false, st, 0);
}
