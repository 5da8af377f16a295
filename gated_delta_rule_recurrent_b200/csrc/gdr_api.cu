// C ABI of libgdr (declared in include/gdr.h): host-side argument checks and
// kernel dispatch for the recurrent gated-delta-rule decode step and the
// standalone LinearAttentionGate op.
//
// Everything here runs on the host before any launch. A failed check returns
// its status with nothing queued; device values (lengths, slot indices) are
// handled by the kernel without traps.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "gdr.h"
#include "gdr_decode.cuh"
#include "gdr_decode_chunk.cuh"
#include "gdr_decode_chunk_tc.cuh"
#include "gdr_decode_rows.cuh"
#include "gdr_decode_tma.cuh"
#include "gdr_gate.cuh"
#include "gdr_prefill_tc.cuh"

namespace {

thread_local std::string g_last_error;
thread_local gdr_launch_info g_last_launch{};

void record_launch(int kernel, int D_k, int tile_cols, bool gated, bool vk, int grid,
                   int threads, int smem, int stages) {
  g_last_launch = gdr_launch_info{kernel, D_k, tile_cols, gated ? 1 : 0,
                                  vk ? GDR_LAYOUT_VK : GDR_LAYOUT_KV, grid, threads, smem, stages};
}

int fail(int status, const std::string& what) {
  g_last_error = what;
  return status;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// Checks shared by both decode entry points. Returns GDR_OK or a failure status.
int check_dims(const gdr_dims* d) {
  if (d == nullptr) return fail(GDR_ERR_NULL, "dims is NULL");
  if (d->B < 0) return fail(GDR_ERR_DIMS, "B must be >= 0");
  if (d->T < 1 || d->T > gdr::kMaxT)
    return fail(GDR_ERR_DIMS, "T must be in [1, 8] (decode only)");
  if (d->H_qk < 1 || d->H_v < 1) return fail(GDR_ERR_DIMS, "H_qk and H_v must be >= 1");
  if (d->H_v % d->H_qk != 0) return fail(GDR_ERR_DIMS, "H_v must be a multiple of H_qk");
  if (d->D_k < 1 || d->D_v < 1) return fail(GDR_ERR_DIMS, "D_k and D_v must be >= 1");
  if (d->pool_size < 1) return fail(GDR_ERR_DIMS, "pool_size must be >= 1");
  if (d->D_k != 64 && d->D_k != 128)
    return fail(GDR_ERR_UNSUPPORTED, "D_k must be 64 or 128");
  if (d->D_v % gdr::kSliceCols != 0)
    return fail(GDR_ERR_UNSUPPORTED, "D_v must be a multiple of 64");
  // Grid size: B * H_v * (D_v / 64) CTAs must fit a 31-bit grid dimension.
  const long long ctas = static_cast<long long>(d->B) * d->H_v * (d->D_v / gdr::kSliceCols);
  if (ctas > 0x7fffffffLL) return fail(GDR_ERR_DIMS, "B * H_v * D_v / 64 exceeds 2^31 - 1");
  if (d->layout != GDR_LAYOUT_KV && d->layout != GDR_LAYOUT_VK)
    return fail(GDR_ERR_DIMS, "layout must be GDR_LAYOUT_KV or GDR_LAYOUT_VK");
  // TMA row coordinates of the pool are 32-bit signed.
  const long long rows_per_slot = d->layout == GDR_LAYOUT_VK ? d->D_v : d->D_k;
  if (static_cast<long long>(d->pool_size) * d->H_v * rows_per_slot > 0x7fffffffLL)
    return fail(GDR_ERR_UNSUPPORTED, "pool_size * H_v * (rows per head) exceeds 2^31 - 1");
  return GDR_OK;
}

// ---------------------------------------------------------------- TMA path

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// The pool seen as a 3-D bf16 array [column blocks of 64][rows][64 columns]
// (row stride = row length * 2 bytes, block stride 128 bytes); one box is a
// whole tile and lands in shared memory as [block][row][64 columns] with the
// 128-byte swizzle: within each 128-byte row segment, 16-byte chunk c is
// stored at position c ^ (row % 8).
//   KV pool [pool, H_v, D_k, D_v]: rows of D_v, box {64, D_k, VS / 64};
//   VK pool [pool, H_v, D_v, D_k]: rows of D_k, box {64, VS, D_k / 64}.
int encode_pool_map(const gdr::DecodeParams& p, int DK, int VS, bool vk, CUtensorMap* map) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return fail(GDR_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int row_len = vk ? DK : p.D_v;          // entries per pool row
  const int rows_per_head = vk ? p.D_v : DK;
  const int box_rows = vk ? VS : DK;
  const cuuint64_t gdim[3] = {64, static_cast<cuuint64_t>(p.pool_size) * p.H_v * rows_per_head,
                              static_cast<cuuint64_t>(row_len / 64)};
  const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(row_len) * 2, 128};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows),
                             static_cast<cuuint32_t>((vk ? DK : VS) / 64)};
  const cuuint32_t estride[3] = {1, 1, 1};
  const CUresult cr = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                             const_cast<uint16_t*>(p.state_pool), gdim, gstride, box, estride,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return fail(GDR_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  return GDR_OK;
}

constexpr int kMaxDevices = 64;
#ifndef GDR_MAX_STAGES
#define GDR_MAX_STAGES 6
#endif
constexpr int kMaxStages = GDR_MAX_STAGES;
// Single-token kernel: at most this many co-resident CTAs per SM, and the
// widest tile that still gives every SM at least GDR_MIN_TILES_PER_SM tiles
// (fewer, larger tiles leave a persistent CTA too few tiles to keep its
// stage ring busy; 16 measured best on the 64-item, 128x128 workload).
#ifndef GDR_MAX_CTAS_PER_SM
#define GDR_MAX_CTAS_PER_SM 6
#endif
#ifndef GDR_MIN_TILES_PER_SM
#define GDR_MIN_TILES_PER_SM 16
#endif

struct DeviceProps {
  int sms = 0;
  int smem_per_sm = 0;
  int smem_optin = 0;
};

int device_props(int dev, DeviceProps* out) {
  static DeviceProps cache[kMaxDevices];
  static std::atomic<bool> ready[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return fail(GDR_ERR_CUDA, "device ordinal out of range");
  if (!ready[dev].load(std::memory_order_acquire)) {
    DeviceProps p;
    if (cudaDeviceGetAttribute(&p.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&p.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                               dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&p.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return fail(GDR_ERR_CUDA, "cudaDeviceGetAttribute failed");
    cache[dev] = p;
    ready[dev].store(true, std::memory_order_release);
  }
  *out = cache[dev];
  return GDR_OK;
}

// Launch shape of one kernel instantiation on one device for one T.
struct LaunchConfig {
  int n_stages = 0;
  int smem = 0;
  int ctas_per_sm = 0;
};

template <int DK, int VS, int R, bool GATED>
int launch_config(int dev, int T, const DeviceProps& props, LaunchConfig* out) {
  using Shape = gdr::TmaShape<DK, VS, R>;
  static LaunchConfig cache[kMaxDevices][gdr::kMaxT + 1];
  static std::atomic<bool> ready[kMaxDevices][gdr::kMaxT + 1];
  if (ready[dev][T].load(std::memory_order_acquire)) {
    *out = cache[dev][T];
    return GDR_OK;
  }
  auto kernel = gdr::decode_tma_kernel<DK, VS, R, GATED>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         props.smem_optin);
  // All of the unified L1/shared storage as shared memory, so that the CTAs
  // the stage budget is split for can be co-resident.
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
  cudaFuncAttributes fa;
  if (err == cudaSuccess) err = cudaFuncGetAttributes(&fa, kernel);
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel attributes: ") + cudaGetErrorString(err));
  // CTAs per SM from the register footprint, then the stage count from the
  // shared-memory budget those CTAs split.
  const int regs_per_warp = ((fa.numRegs * 32 + 255) / 256) * 256;
  int ctas = 65536 / (regs_per_warp * (Shape::kThreads / 32));
  ctas = ctas < 1 ? 1 : (ctas > GDR_MAX_CTAS_PER_SM ? GDR_MAX_CTAS_PER_SM : ctas);
  LaunchConfig c;
  for (; ctas >= 1; --ctas) {
    const int stage_bytes = gdr::stage_layout<DK, VS, R>(T).bytes;
    const int budget = props.smem_per_sm / ctas - 1024;
    int n = (budget - 1024 - gdr::cta_extra_bytes(kMaxStages)) / stage_bytes;
    n = n > kMaxStages ? kMaxStages : n;
    if (n < gdr::kMinStages) n = gdr::kMinStages;
    const int smem = gdr::tma_smem_bytes<DK, VS, R>(T, n);
    if (smem > props.smem_optin) continue;
    // A persistent grid must be co-resident: trust the occupancy calculator.
    int resident = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kernel, Shape::kThreads, smem);
    if (err != cudaSuccess)
      return fail(GDR_ERR_CUDA, std::string("occupancy query: ") + cudaGetErrorString(err));
    if (resident < 1) continue;
    c.n_stages = n;
    c.smem = smem;
    c.ctas_per_sm = resident < ctas ? resident : ctas;
    break;
  }
  if (c.ctas_per_sm == 0) return fail(GDR_ERR_UNSUPPORTED, "tile does not fit in shared memory");
  cache[dev][T] = c;
  ready[dev][T].store(true, std::memory_order_release);
  *out = c;
  return GDR_OK;
}

template <int DK, int VS, int R, bool GATED>
int launch_tma(const gdr::DecodeParams& p, cudaStream_t stream) {
  using Shape = gdr::TmaShape<DK, VS, R>;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(GDR_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(err));
  DeviceProps props;
  int rc = device_props(dev, &props);
  if (rc != GDR_OK) return rc;
  LaunchConfig cfg;
  rc = launch_config<DK, VS, R, GATED>(dev, p.T, props, &cfg);
  if (rc != GDR_OK) return rc;
  const int n_stages = cfg.n_stages;
  const int smem = cfg.smem;
  const int ctas_per_sm = cfg.ctas_per_sm;

  CUtensorMap map;
  rc = encode_pool_map(p, DK, VS, false, &map);
  if (rc != GDR_OK) return rc;

  const int n_tiles = p.B * p.H_v * (p.D_v / VS);
  const int max_ctas = ctas_per_sm * props.sms;
  const int grid = n_tiles < max_ctas ? n_tiles : max_ctas;
  gdr::decode_tma_kernel<DK, VS, R, GATED><<<grid, Shape::kThreads, smem, stream>>>(map, p, n_tiles,
                                                                                 n_stages);
  err = cudaGetLastError();
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  record_launch(GDR_KERNEL_SINGLE_TOKEN, DK, VS, GATED, false, grid, Shape::kThreads, smem,
                n_stages);
  return GDR_OK;
}

// ---------------------------------------------------------------- chunk path (T >= 2)

#ifndef GDR_CHUNK_MAX_STAGES
#define GDR_CHUNK_MAX_STAGES 8
#endif

struct ChunkConfig {
  int n_stages = 0;
  int smem = 0;
  int threads = 0;
};


// One persistent CTA per SM: as many stages as shared memory holds, and one
// consumer group fewer than stages (so no group waits two phases ahead).
template <int DK, int VS, bool GATED, bool VK>
int chunk_config(int dev, int T, const DeviceProps& props, ChunkConfig* out) {
  static ChunkConfig cache[kMaxDevices][gdr::kMaxT + 1];
  static std::atomic<bool> ready[kMaxDevices][gdr::kMaxT + 1];
  if (ready[dev][T].load(std::memory_order_acquire)) {
    *out = cache[dev][T];
    return GDR_OK;
  }
  auto kernel = gdr::decode_chunk_kernel<DK, VS, GATED, VK>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         props.smem_optin);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel attributes: ") + cudaGetErrorString(err));
  constexpr int kMaxStagesChunk = GDR_CHUNK_MAX_STAGES;
  const int stage_bytes = gdr::chunk_stage_bytes<DK, VS>(T);
  int n = (props.smem_optin - 1024 - gdr::kChunkBarriers * 8 * kMaxStagesChunk - 16) / stage_bytes;
  n = n > kMaxStagesChunk ? kMaxStagesChunk : n;
  if (n < 2) return fail(GDR_ERR_UNSUPPORTED, "tile does not fit in shared memory");
  constexpr int cwt = gdr::ChunkShape<DK, VS, VK>::kWarpsPerTile;
  int groups = n - 1;
  const int max_groups = (gdr::kChunkMaxThreads / 32 - 1 - gdr::kChunkFinalizers) / cwt;
  groups = groups > max_groups ? max_groups : groups;
  ChunkConfig c;
  c.n_stages = n;
  c.smem = gdr::chunk_smem_bytes<DK, VS>(T, n);
  c.threads = 32 * (1 + gdr::kChunkFinalizers + groups * cwt);
  int resident = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kernel, c.threads, c.smem);
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("occupancy query: ") + cudaGetErrorString(err));
  if (resident < 1) return fail(GDR_ERR_UNSUPPORTED, "tile does not fit on an SM");
  cache[dev][T] = c;
  ready[dev][T].store(true, std::memory_order_release);
  *out = c;
  return GDR_OK;
}

template <int DK, int VS, bool GATED, bool VK>
int launch_chunk(const gdr::DecodeParams& p, cudaStream_t stream) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(GDR_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(err));
  DeviceProps props;
  int rc = device_props(dev, &props);
  if (rc != GDR_OK) return rc;
  ChunkConfig cfg;
  rc = chunk_config<DK, VS, GATED, VK>(dev, p.T, props, &cfg);
  if (rc != GDR_OK) return rc;
  CUtensorMap map;
  rc = encode_pool_map(p, DK, VS, VK, &map);
  if (rc != GDR_OK) return rc;
  const int n_tiles = p.B * p.H_v * (p.D_v / VS);
  const int grid = n_tiles < props.sms ? n_tiles : props.sms;
  gdr::decode_chunk_kernel<DK, VS, GATED, VK><<<grid, cfg.threads, cfg.smem, stream>>>(
      map, p, n_tiles, cfg.n_stages);
  err = cudaGetLastError();
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  record_launch(GDR_KERNEL_CHUNKED, DK, VS, GATED, VK, grid, cfg.threads, cfg.smem,
                cfg.n_stages);
  return GDR_OK;
}

// ---------------------------------------------------------------- tensor-core path (D_k = 128, 128-column tiles, any T)

// One persistent CTA per SM with kTcGroups consumer groups; each group gets
// as many stages as shared memory holds (at most 4).
template <bool GATED, bool VK, bool SUMS, bool T8>
int chunk_tc_config(int dev, int T, const DeviceProps& props, ChunkConfig* out) {
  static ChunkConfig cache[kMaxDevices][gdr::kMaxT + 1];
  static std::atomic<bool> ready[kMaxDevices][gdr::kMaxT + 1];
  if (ready[dev][T].load(std::memory_order_acquire)) {
    *out = cache[dev][T];
    return GDR_OK;
  }
  auto kernel = gdr::decode_chunk_tc_kernel<GATED, VK, SUMS, T8>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         props.smem_optin);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel attributes: ") + cudaGetErrorString(err));
  constexpr int ng = gdr::kTcGroups;
  int per = 1;
  while (per < 4 && gdr::tc_smem_bytes(T, (per + 1) * ng, ng) <= props.smem_optin) ++per;
  if (gdr::tc_smem_bytes(T, per * ng, ng) > props.smem_optin)
    return fail(GDR_ERR_UNSUPPORTED, "tile does not fit in shared memory");
  ChunkConfig c;
  c.n_stages = per * ng;
  c.smem = gdr::tc_smem_bytes(T, c.n_stages, ng);
  c.threads = gdr::kTcGroups * (gdr::kTcGroupThreads + (SUMS ? 32 : 0)) + 32;
  int resident = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kernel, c.threads, c.smem);
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("occupancy query: ") + cudaGetErrorString(err));
  if (resident < 1) return fail(GDR_ERR_UNSUPPORTED, "tile does not fit on an SM");
  cache[dev][T] = c;
  ready[dev][T].store(true, std::memory_order_release);
  *out = c;
  return GDR_OK;
}

template <bool GATED, bool VK, bool SUMS, bool T8>
int launch_chunk_tc_sums(const gdr::DecodeParams& p, cudaStream_t stream) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(GDR_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(err));
  DeviceProps props;
  int rc = device_props(dev, &props);
  if (rc != GDR_OK) return rc;
  ChunkConfig cfg;
  rc = chunk_tc_config<GATED, VK, SUMS, T8>(dev, p.T, props, &cfg);
  if (rc != GDR_OK) return rc;
  CUtensorMap map;
  rc = encode_pool_map(p, gdr::kTcDK, gdr::kTcVS, VK, &map);
  if (rc != GDR_OK) return rc;
  const int n_tiles = p.B * p.H_v * (p.D_v / gdr::kTcVS);
  const int grid = n_tiles < props.sms ? n_tiles : props.sms;
  gdr::decode_chunk_tc_kernel<GATED, VK, SUMS, T8><<<grid, cfg.threads, cfg.smem, stream>>>(
      map, p, n_tiles, cfg.n_stages);
  err = cudaGetLastError();
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  record_launch(SUMS ? GDR_KERNEL_TENSOR_CORE_ONE : GDR_KERNEL_TENSOR_CORE, gdr::kTcDK,
                gdr::kTcVS, GATED, VK, grid, cfg.threads, cfg.smem, cfg.n_stages);
  return GDR_OK;
}

// Single-token calls take the sums-warp form of the kernel.
template <bool GATED, bool VK>
int launch_chunk_tc(const gdr::DecodeParams& p, cudaStream_t stream) {
  return p.T == 1   ? launch_chunk_tc_sums<GATED, VK, true, false>(p, stream)
         : p.T == 8 ? launch_chunk_tc_sums<GATED, VK, false, true>(p, stream)
                    : launch_chunk_tc_sums<GATED, VK, false, false>(p, stream);
}

// ---------------------------------------------------------------- k-contiguous single token

// One warp per block of RB rows of a head, 8 warps per CTA, as many CTAs as
// stay resident (a grid-stride loop takes the rest). Single-token calls only.
template <int DK, bool GATED, int RB>
int launch_rows(const gdr::DecodeParams& p, cudaStream_t stream) {
  if (p.T != 1 || p.D_v % RB != 0) return GDR_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaGetDevice failed");
  DeviceProps props;
  int rc = device_props(dev, &props);
  if (rc != GDR_OK) return rc;
  static const int resident = [] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gdr::decode_rows_kernel<DK, GATED, RB>,
                                                      gdr::kRowsThreads, 0) != cudaSuccess ||
        n < 1)
      n = 1;
    return n;
  }();
  const long long n_blocks = static_cast<long long>(p.B) * p.H_v * (p.D_v / RB);
  if (n_blocks > 0x7fffffffLL) return fail(GDR_ERR_DIMS, "too many row blocks");
  const long long warps_per_cta = gdr::kRowsThreads / 32;
  const long long need = (n_blocks + warps_per_cta - 1) / warps_per_cta;
  const long long cap = static_cast<long long>(props.sms) * resident;
  const int grid = static_cast<int>(need < cap ? need : cap);
  gdr::decode_rows_kernel<DK, GATED, RB><<<grid, gdr::kRowsThreads, 0, stream>>>(
      p, static_cast<int>(n_blocks));
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  record_launch(GDR_KERNEL_ROWS, DK, RB, GATED, true, grid, gdr::kRowsThreads, 0, 0);
  return GDR_OK;
}

using LaunchFn = int (*)(const gdr::DecodeParams&, cudaStream_t);
struct SliceKernel {
  int vs;
  LaunchFn launch;
};

// Tile widths per path, widest first. Single-token calls use the
// warp-specialised kernel with the rows each consumer thread holds; the
// thread count of a block caps the registers ptxas may give a thread (255 up
// to 256 threads, 168 up to 384, 128 up to 512, 96 up to 640), and a
// single-token call keeps no state in registers (about 75 of them), so a
// full-width 64 x 512 tile can use 16 consumer warps. Single-token calls on
// a k-contiguous pool use the row kernel, whose "width" is the rows of a
// warp's block (64, or 16 for small batches). Multi-token calls use the
// CUDA-core chunked kernel. These tables serve the calls the tensor-core
// kernel does not take (D_k = 64, or D_v not a multiple of 128), and are its
// fallback.
template <bool GATED>
const SliceKernel* slice_kernels(int D_k, bool one, bool vk, int* n) {
  static const SliceKernel k64_one[] = {{512, launch_tma<64, 512, 8, GATED>},
                                        {256, launch_tma<64, 256, 8, GATED>},
                                        {128, launch_tma<64, 128, 8, GATED>},
                                        {64, launch_tma<64, 64, 8, GATED>}};
  // D_k = 128 with D_v a multiple of 128 goes to the tensor-core kernel, so
  // only 64-column tiles remain for it here
  static const SliceKernel k128_one[] = {{64, launch_tma<128, 64, 16, GATED>}};
  static const SliceKernel k64_many[] = {{128, launch_chunk<64, 128, GATED, false>},
                                         {64, launch_chunk<64, 64, GATED, false>}};
  static const SliceKernel k128_many[] = {{64, launch_chunk<128, 64, GATED, false>}};
  // k-contiguous pools: one token per call takes the row kernel (blocks of 64
  // rows, or 16 when a batch gives too few blocks), several the chunked kernel
  static const SliceKernel k64_vk_one[] = {{64, launch_rows<64, GATED, 64>},
                                           {16, launch_rows<64, GATED, 16>}};
  static const SliceKernel k128_vk_one[] = {{64, launch_rows<128, GATED, 64>},
                                            {16, launch_rows<128, GATED, 16>}};
  static const SliceKernel k64_vk[] = {{128, launch_chunk<64, 128, GATED, true>},
                                       {64, launch_chunk<64, 64, GATED, true>}};
  static const SliceKernel k128_vk[] = {{64, launch_chunk<128, 64, GATED, true>}};
  if (vk) {
    *n = one ? 2 : (D_k == 64 ? 2 : 1);
    if (one) return D_k == 64 ? k64_vk_one : k128_vk_one;
    return D_k == 64 ? k64_vk : k128_vk;
  }
  if (D_k == 64) {
    *n = one ? 4 : 2;
    return one ? k64_one : k64_many;
  }
  *n = 1;
  return one ? k128_one : k128_many;
}

// With D_k = 128 and D_v a multiple of 128 every call takes the tensor-core
// kernel (for one token too: on a 64-item, 128 x 128 workload it ran 27 us
// against 31 us for the single-token kernel). Otherwise the column-slice
// width is the widest
// width that divides D_v and still gives every SM GDR_MIN_TILES_PER_SM tiles,
// else the narrowest one; a width whose stage ring does not fit in shared
// memory (long T) falls back to the next narrower one.
int dispatch(const gdr::DecodeParams& p, int D_k, bool gated, bool vk, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaGetDevice failed");
  DeviceProps props;
  int rc = device_props(dev, &props);
  if (rc != GDR_OK) return rc;
  int n = 0;
  const bool one = p.T == 1;
  if (D_k == gdr::kTcDK && p.D_v % gdr::kTcVS == 0) {
    if (vk)
      rc = gated ? launch_chunk_tc<true, true>(p, stream) : launch_chunk_tc<false, true>(p, stream);
    else
      rc = gated ? launch_chunk_tc<true, false>(p, stream) : launch_chunk_tc<false, false>(p, stream);
    if (rc != GDR_ERR_UNSUPPORTED) return rc;
  }
  const SliceKernel* ks = gated ? slice_kernels<true>(D_k, one, vk, &n)
                                : slice_kernels<false>(D_k, one, vk, &n);
  int first = -1;
  for (int i = 0; i < n; ++i) {
    if (p.D_v % ks[i].vs != 0) continue;
    first = i;
    if (static_cast<long long>(p.B) * p.H_v * (p.D_v / ks[i].vs) >=
        static_cast<long long>(GDR_MIN_TILES_PER_SM) * props.sms)
      break;
  }
  if (first < 0) return fail(GDR_ERR_UNSUPPORTED, "no tile width divides D_v");
  for (int i = first; i < n; ++i) {
    if (p.D_v % ks[i].vs != 0) continue;
    rc = ks[i].launch(p, stream);
    if (rc != GDR_ERR_UNSUPPORTED) return rc;
  }
  return rc;
}

// Every kernel form the entry points can launch: the prefill kernel, then,
// per gate variant, the decode dispatcher's: the tensor-core kernel's four
// (layout x token form), then the entries of the tile-width tables.
std::vector<gdr_launch_info> kernel_forms() {
  std::vector<gdr_launch_info> forms;
  for (int gated = 0; gated < 2; ++gated)  // gdr_prefill / gdr_prefill_gated
    forms.push_back(gdr_launch_info{GDR_KERNEL_PREFILL, gdr::kTcDK, gdr::kTcVS, gated,
                                    GDR_LAYOUT_KV, 0, 0, 0, 0});
  for (int gated = 0; gated < 2; ++gated) {
    for (int vk = 0; vk < 2; ++vk)
      for (int kernel : {GDR_KERNEL_TENSOR_CORE_ONE, GDR_KERNEL_TENSOR_CORE})
        forms.push_back(gdr_launch_info{kernel, gdr::kTcDK, gdr::kTcVS, gated, vk, 0, 0, 0, 0});
    for (int D_k : {64, 128})
      for (int vk = 0; vk < 2; ++vk)
        for (int one = 1; one >= 0; --one) {
          int n = 0;
          const SliceKernel* ks = gated ? slice_kernels<true>(D_k, one, vk, &n)
                                        : slice_kernels<false>(D_k, one, vk, &n);
          const int kernel =
              one ? (vk ? GDR_KERNEL_ROWS : GDR_KERNEL_SINGLE_TOKEN) : GDR_KERNEL_CHUNKED;
          for (int i = 0; i < n; ++i)
            forms.push_back(gdr_launch_info{kernel, D_k, ks[i].vs, gated, vk, 0, 0, 0, 0});
        }
  }
  return forms;
}

gdr::DecodeParams base_params(const gdr_dims* d, const gdr_bf16* query, const gdr_bf16* key,
                              const gdr_bf16* value, gdr_bf16* state_pool,
                              const int32_t* asl, const int32_t* idx, const int32_t* nat,
                              const float* gk, float scale, gdr_bf16* out) {
  gdr::DecodeParams p{};
  p.query = query;
  p.key = key;
  p.value = value;
  p.gk = gk;
  p.state_pool = state_pool;
  p.out = out;
  p.seq_lengths = asl;
  p.state_indices = idx;
  p.num_accepted = nat;
  p.scale = scale;
  p.B = d->B;
  p.T = d->T;
  p.H_qk = d->H_qk;
  p.H_v = d->H_v;
  p.D_v = d->D_v;
  p.pool_size = d->pool_size;
  p.group = d->H_v / d->H_qk;
  return p;
}

// ---------------------------------------------------------------- prefill (long T)

int check_prefill_dims(const gdr_dims* d) {
  if (d == nullptr) return fail(GDR_ERR_NULL, "dims is NULL");
  if (d->B < 0) return fail(GDR_ERR_DIMS, "B must be >= 0");
  if (d->T < 1) return fail(GDR_ERR_DIMS, "T must be >= 1");
  if (d->H_qk < 1 || d->H_v < 1) return fail(GDR_ERR_DIMS, "H_qk and H_v must be >= 1");
  if (d->H_v % d->H_qk != 0) return fail(GDR_ERR_DIMS, "H_v must be a multiple of H_qk");
  if (d->D_k < 1 || d->D_v < 1) return fail(GDR_ERR_DIMS, "D_k and D_v must be >= 1");
  if (d->pool_size < 1) return fail(GDR_ERR_DIMS, "pool_size must be >= 1");
  if (d->layout != GDR_LAYOUT_KV && d->layout != GDR_LAYOUT_VK)
    return fail(GDR_ERR_DIMS, "layout must be GDR_LAYOUT_KV or GDR_LAYOUT_VK");
  if (d->D_k != gdr::kTcDK || d->D_v % gdr::kTcVS != 0 || d->layout != GDR_LAYOUT_KV)
    return fail(GDR_ERR_UNSUPPORTED,
                "prefill takes D_k = 128, D_v a multiple of 128 and the [pool, H_v, D_k, D_v] "
                "layout");
  const long long tiles = static_cast<long long>(d->B) * d->H_v * (d->D_v / gdr::kTcVS);
  if (tiles > 0x7fffffffLL) return fail(GDR_ERR_DIMS, "B * H_v * D_v / 128 exceeds 2^31 - 1");
  if (static_cast<long long>(d->pool_size) * d->H_v * d->D_k > 0x7fffffffLL)
    return fail(GDR_ERR_UNSUPPORTED, "pool_size * H_v * D_k exceeds 2^31 - 1");
  // element offsets are 64-bit; keep every tensor's element count below 2^62
  const long long per_item = static_cast<long long>(d->T) *
                             (d->H_v > d->H_qk ? d->H_v : d->H_qk) *
                             (d->D_v > d->D_k ? d->D_v : d->D_k);
  if (per_item > (1LL << 62) / (d->B > 0 ? d->B : 1))
    return fail(GDR_ERR_DIMS, "B * H * T * D exceeds 2^62");
  return GDR_OK;
}

template <bool GATED>
int launch_prefill(const gdr::DecodeParams& p, cudaStream_t stream) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(GDR_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(err));
  DeviceProps props;
  int rc = device_props(dev, &props);
  if (rc != GDR_OK) return rc;
  const int smem = gdr::pf_smem_bytes();
  if (smem > props.smem_optin) return fail(GDR_ERR_UNSUPPORTED, "prefill tile does not fit in shared memory");
  static std::atomic<bool> ready[kMaxDevices];
  auto kernel = gdr::prefill_tc_kernel<GATED>;
  if (!ready[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (err != cudaSuccess)
      return fail(GDR_ERR_CUDA, std::string("kernel attributes: ") + cudaGetErrorString(err));
    ready[dev].store(true, std::memory_order_release);
  }
  CUtensorMap map;
  rc = encode_pool_map(p, gdr::kTcDK, gdr::kTcVS, false, &map);
  if (rc != GDR_OK) return rc;
  // One tile per SM while there are fewer tiles than SMs (each tile is a long
  // sequential chain); past that, a CTA's two groups share an SM.
  const int n_tiles = p.B * p.H_v * (p.D_v / gdr::kTcVS);
  const int grid = n_tiles < props.sms ? n_tiles : props.sms;
  kernel<<<grid, gdr::kPfThreads, smem, stream>>>(map, p, n_tiles);
  err = cudaGetLastError();
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  record_launch(GDR_KERNEL_PREFILL, gdr::kTcDK, gdr::kTcVS, GATED, false, grid, gdr::kPfThreads,
                smem, gdr::kPfStages);
  return GDR_OK;
}

// ---------------------------------------------------------------- standalone gate

// CTAs of 256 threads a kernel keeps resident per SM (its registers decide),
// queried once; the grid-stride grids are that many per SM, one wave.
template <typename K>
int resident_per_sm(K kernel) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, 256, 0) != cudaSuccess || n < 1)
    n = 1;
  return n;
}

template <int TYPE, bool BETA>
int launch_gate(const void* a, const void* b, const float* dt_bias, const float* decay_scale,
                void* decay, void* beta, int64_t n, int H, cudaStream_t stream) {
  using E = gdr::GateElem<TYPE>;
  using bits = typename E::bits;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(GDR_ERR_CUDA, "cudaGetDevice failed");
  DeviceProps props;
  int rc = device_props(dev, &props);
  if (rc != GDR_OK) return rc;
  constexpr int kThreads = 256;
  static const int res_head = resident_per_sm(gdr::gate_vec_kernel<TYPE, BETA, true>);
  static const int res_elem = resident_per_sm(gdr::gate_vec_kernel<TYPE, BETA, false>);
  static const int res_scalar = resident_per_sm(gdr::gate_scalar_kernel<TYPE, BETA>);
  auto blocks_for = [&](int64_t work, int resident) {
    const int64_t max_blocks = static_cast<int64_t>(props.sms) * resident;
    const int64_t blk = (work + kThreads - 1) / kThreads;
    return static_cast<int>(blk < max_blocks ? blk : max_blocks);
  };
  // 16-byte vectors when every tensor allows them; the rest element by element
  const bool vec = aligned16(a) && aligned16(decay) && (!BETA || (aligned16(b) && aligned16(beta)));
  const int64_t n_vec = vec ? n / E::kPerVec : 0;
  // per-head vectors as 16-byte loads when a vector's elements are whole heads
  const bool headvec = H % E::kPerVec == 0 && aligned16(dt_bias) && aligned16(decay_scale);
  const int vec_blocks = blocks_for(n_vec, headvec ? res_head : res_elem);
  if (n_vec > 0) {
    if (headvec)
      gdr::gate_vec_kernel<TYPE, BETA, true><<<vec_blocks, kThreads, 0, stream>>>(
          static_cast<const uint4*>(a), static_cast<const uint4*>(b), dt_bias, decay_scale,
          static_cast<uint4*>(decay), static_cast<uint4*>(beta), n_vec, H);
    else
      gdr::gate_vec_kernel<TYPE, BETA, false><<<vec_blocks, kThreads, 0, stream>>>(
          static_cast<const uint4*>(a), static_cast<const uint4*>(b), dt_bias, decay_scale,
          static_cast<uint4*>(decay), static_cast<uint4*>(beta), n_vec, H);
  }
  const int64_t i_begin = n_vec * E::kPerVec;
  const int scalar_blocks = blocks_for(n - i_begin, res_scalar);
  if (i_begin < n)
    gdr::gate_scalar_kernel<TYPE, BETA><<<scalar_blocks, kThreads, 0, stream>>>(
        static_cast<const bits*>(a), static_cast<const bits*>(b), dt_bias, decay_scale,
        static_cast<bits*>(decay), static_cast<bits*>(beta), i_begin, n, H);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  record_launch(GDR_KERNEL_GATE, 0, 0, true, false, n_vec > 0 ? vec_blocks : scalar_blocks,
                kThreads, 0, 0);
  return GDR_OK;
}

template <int TYPE>
int launch_gate_any(const void* a, const void* b, const float* dt_bias, const float* decay_scale,
                    void* decay, void* beta, int64_t n, int H, cudaStream_t stream) {
  return beta != nullptr
             ? launch_gate<TYPE, true>(a, b, dt_bias, decay_scale, decay, beta, n, H, stream)
             : launch_gate<TYPE, false>(a, b, dt_bias, decay_scale, decay, beta, n, H, stream);
}

int check_common_pointers(const gdr_bf16* query, const gdr_bf16* key, const gdr_bf16* value,
                          gdr_bf16* state_pool, const int32_t* asl, const int32_t* idx,
                          const float* gk, gdr_bf16* out) {
  if (!query || !key || !value || !state_pool || !asl || !idx || !gk || !out)
    return fail(GDR_ERR_NULL, "a required tensor pointer is NULL");
  if (!aligned16(query) || !aligned16(key) || !aligned16(value) || !aligned16(gk) ||
      !aligned16(state_pool) || !aligned16(out))
    return fail(GDR_ERR_ALIGN,
                "query, key, value, gk, state_pool and out must be 16-byte aligned");
  return GDR_OK;
}

}  // namespace

extern "C" {

GDR_API int gdr_decode(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                       const gdr_bf16* value, const gdr_bf16* beta, gdr_bf16* state_pool,
                       const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                       const float* g, const float* gk, const int32_t* num_accepted_tokens,
                       float scale_value, gdr_bf16* out, gdr_stream_t stream) {
  g_last_launch = gdr_launch_info{};
  int rc = check_dims(dims);
  if (rc != GDR_OK) return rc;
  if (dims->B == 0) return GDR_OK;
  rc = check_common_pointers(query, key, value, state_pool, actual_seq_lengths,
                             ssm_state_indices, gk, out);
  if (rc != GDR_OK) return rc;
  if (!beta || !g) return fail(GDR_ERR_NULL, "beta and g must not be NULL");
  gdr::DecodeParams p = base_params(dims, query, key, value, state_pool, actual_seq_lengths,
                                    ssm_state_indices, num_accepted_tokens, gk, scale_value,
                                    out);
  p.beta = beta;
  p.g = g;
  return dispatch(p, dims->D_k, false, dims->layout == GDR_LAYOUT_VK,
                  reinterpret_cast<cudaStream_t>(stream));
}

GDR_API int gdr_gate_fused(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                           const gdr_bf16* value, const gdr_bf16* a, const gdr_bf16* b,
                           const float* dt_bias, const float* decay_scale, gdr_bf16* state_pool,
                           const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                           const float* gk, const int32_t* num_accepted_tokens,
                           float scale_value, gdr_bf16* out, gdr_stream_t stream) {
  g_last_launch = gdr_launch_info{};
  int rc = check_dims(dims);
  if (rc != GDR_OK) return rc;
  if (dims->B == 0) return GDR_OK;
  rc = check_common_pointers(query, key, value, state_pool, actual_seq_lengths,
                             ssm_state_indices, gk, out);
  if (rc != GDR_OK) return rc;
  if (!a || !b || !dt_bias || !decay_scale)
    return fail(GDR_ERR_NULL, "a, b, dt_bias and decay_scale must not be NULL");
  gdr::DecodeParams p = base_params(dims, query, key, value, state_pool, actual_seq_lengths,
                                    ssm_state_indices, num_accepted_tokens, gk, scale_value,
                                    out);
  p.gate_a = a;
  p.gate_b = b;
  p.dt_bias = dt_bias;
  p.decay_scale = decay_scale;
  return dispatch(p, dims->D_k, true, dims->layout == GDR_LAYOUT_VK,
                  reinterpret_cast<cudaStream_t>(stream));
}

GDR_API int gdr_prefill(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                        const gdr_bf16* value, const gdr_bf16* beta, gdr_bf16* state_pool,
                        const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                        const float* g, const float* gk, const int32_t* num_accepted_tokens,
                        float scale_value, gdr_bf16* out, gdr_stream_t stream) {
  g_last_launch = gdr_launch_info{};
  int rc = check_prefill_dims(dims);
  if (rc != GDR_OK) return rc;
  if (dims->B == 0) return GDR_OK;
  rc = check_common_pointers(query, key, value, state_pool, actual_seq_lengths,
                             ssm_state_indices, gk, out);
  if (rc != GDR_OK) return rc;
  if (!beta || !g) return fail(GDR_ERR_NULL, "beta and g must not be NULL");
  gdr::DecodeParams p = base_params(dims, query, key, value, state_pool, actual_seq_lengths,
                                    ssm_state_indices, num_accepted_tokens, gk, scale_value,
                                    out);
  p.beta = beta;
  p.g = g;
  return launch_prefill<false>(p, reinterpret_cast<cudaStream_t>(stream));
}

GDR_API int gdr_prefill_gated(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                              const gdr_bf16* value, const gdr_bf16* a, const gdr_bf16* b,
                              const float* dt_bias, const float* decay_scale,
                              gdr_bf16* state_pool, const int32_t* actual_seq_lengths,
                              const int32_t* ssm_state_indices, const float* gk,
                              const int32_t* num_accepted_tokens, float scale_value,
                              gdr_bf16* out, gdr_stream_t stream) {
  g_last_launch = gdr_launch_info{};
  int rc = check_prefill_dims(dims);
  if (rc != GDR_OK) return rc;
  if (dims->B == 0) return GDR_OK;
  rc = check_common_pointers(query, key, value, state_pool, actual_seq_lengths,
                             ssm_state_indices, gk, out);
  if (rc != GDR_OK) return rc;
  if (!a || !b || !dt_bias || !decay_scale)
    return fail(GDR_ERR_NULL, "a, b, dt_bias and decay_scale must not be NULL");
  gdr::DecodeParams p = base_params(dims, query, key, value, state_pool, actual_seq_lengths,
                                    ssm_state_indices, num_accepted_tokens, gk, scale_value,
                                    out);
  p.gate_a = a;
  p.gate_b = b;
  p.dt_bias = dt_bias;
  p.decay_scale = decay_scale;
  return launch_prefill<true>(p, reinterpret_cast<cudaStream_t>(stream));
}

GDR_API int gdr_linear_attention_gate(const void* a, const void* b, const float* dt_bias,
                                      const float* decay_scale, void* decay, void* beta,
                                      int64_t rows, int32_t H, int dtype, gdr_stream_t stream) {
  g_last_launch = gdr_launch_info{};
  if (!a || !dt_bias || !decay_scale || !decay)
    return fail(GDR_ERR_NULL, "a, dt_bias, decay_scale and decay must not be NULL");
  if (beta != nullptr && b == nullptr)
    return fail(GDR_ERR_NULL, "beta was requested but b is NULL");
  if (rows < 0 || H < 1) return fail(GDR_ERR_DIMS, "rows must be >= 0 and H >= 1");
  if (rows > (static_cast<int64_t>(1) << 62) / H)
    return fail(GDR_ERR_DIMS, "rows * H must be below 2^62");
  if (dtype != GDR_DTYPE_F32 && dtype != GDR_DTYPE_F16 && dtype != GDR_DTYPE_BF16)
    return fail(GDR_ERR_UNSUPPORTED, "dtype must be GDR_DTYPE_F32, GDR_DTYPE_F16 or GDR_DTYPE_BF16");
  if (rows == 0) return GDR_OK;
  const int64_t n = rows * H;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case GDR_DTYPE_F32:
      return launch_gate_any<gdr::kGateF32>(a, b, dt_bias, decay_scale, decay, beta, n, H, st);
    case GDR_DTYPE_F16:
      return launch_gate_any<gdr::kGateF16>(a, b, dt_bias, decay_scale, decay, beta, n, H, st);
    default:
      return launch_gate_any<gdr::kGateBF16>(a, b, dt_bias, decay_scale, decay, beta, n, H, st);
  }
}

GDR_API const char* gdr_status_string(int status) {
  switch (status) {
    case GDR_OK: return "GDR_OK";
    case GDR_ERR_NULL: return "GDR_ERR_NULL";
    case GDR_ERR_DIMS: return "GDR_ERR_DIMS";
    case GDR_ERR_ALIGN: return "GDR_ERR_ALIGN";
    case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
    case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
    default: return "unknown status";
  }
}

GDR_API const char* gdr_last_error(void) { return g_last_error.c_str(); }

GDR_API int gdr_device_error(uint32_t* flags, int reset) {
  if (flags == nullptr) return fail(GDR_ERR_NULL, "flags is NULL");
  unsigned int v = 0;
  cudaError_t err = cudaMemcpyFromSymbol(&v, gdr::g_device_error, sizeof(v));
  if (err == cudaSuccess && reset) {
    const unsigned int zero = 0;
    err = cudaMemcpyToSymbol(gdr::g_device_error, &zero, sizeof(zero));
  }
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("reading the device error word: ") + cudaGetErrorString(err));
  *flags = v;
  return GDR_OK;
}

GDR_API int gdr_last_launch(gdr_launch_info* info) {
  if (info == nullptr) return fail(GDR_ERR_NULL, "info is NULL");
  *info = g_last_launch;
  return GDR_OK;
}

GDR_API int gdr_kernel_form_count(void) { return static_cast<int>(kernel_forms().size()); }

GDR_API int gdr_kernel_form(int i, gdr_launch_info* info) {
  if (info == nullptr) return fail(GDR_ERR_NULL, "info is NULL");
  const std::vector<gdr_launch_info> forms = kernel_forms();
  if (i < 0 || i >= static_cast<int>(forms.size()))
    return fail(GDR_ERR_DIMS, "kernel form index out of range");
  *info = forms[i];
  return GDR_OK;
}

GDR_API int gdr_abi_version(void) { return 6; }

#ifdef GDR_TEST_HOOKS
// Test builds only (libgdr_testhooks.so): shorten the budget of the
// abandonable waits (cycles; <= 0 restores the shipped ~2 s) and hold back the
// tile with index `hold_tile` (< 0: none) in every decode kernel. Synchronous.
// Not part of the library's ABI: the shipped libgdr.so does not contain it.
GDR_API int gdrtest_set_hooks(long long wait_limit_cycles, int hold_tile) {
  const long long limit = wait_limit_cycles > 0 ? wait_limit_cycles : gdr::kWaitLimitCycles;
  cudaError_t err = cudaMemcpyToSymbol(gdr::g_test_wait_limit, &limit, sizeof(limit));
  if (err == cudaSuccess)
    err = cudaMemcpyToSymbol(gdr::g_test_hold_tile, &hold_tile, sizeof(hold_tile));
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("setting the test hooks: ") + cudaGetErrorString(err));
  return GDR_OK;
}
#endif

}  // extern "C"
