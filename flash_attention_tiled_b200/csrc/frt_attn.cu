// frt_attn.cu -- the C ABI of the library (declared in include/frt_attn.h):
// argument validation, work planning, TMA descriptor encoding and kernel
// launches on the caller's stream.  This is the library's single translation
// unit; the kernels live in the .cuh files it includes.
#include <algorithm>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/frt_attn.h"
#include "decode_splitkv.cuh"
#include "frt_device.cuh"
#include "merge_lse.cuh"
#include "prefill_sm100.cuh"

namespace frt {


namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxDevices = 64;

// ------------------------------------------------------- device properties
// Cluster-mode decode kernels (contiguous cache, no workspace), indexed by
// [D == 128][two head tiles].
using DecodeKernel = void (*)(CUtensorMap, CUtensorMap, DecodeParams);
const DecodeKernel kClusterDecode[2][2] = {
    {decode_splitkv_kernel<64, 1, false, true>, decode_splitkv_kernel<64, 2, false, true>},
    {decode_splitkv_kernel<128, 1, false, true>, decode_splitkv_kernel<128, 2, false, true>}};
constexpr size_t kClusterDecodeSmem[2][2] = {
    {DecodeSmem<64, false, 1>::kBytes, DecodeSmem<64, false, 2>::kBytes},
    {DecodeSmem<128, false, 1>::kBytes, DecodeSmem<128, false, 2>::kBytes}};
constexpr int kClusterDecodeThreads[2] = {DecodeCfg<false, 1>::kThreads,
                                          DecodeCfg<false, 2>::kThreads};

struct DeviceInfo {
  int sm_count = 0;
  bool prefill_ok = false;   // register pool of the prefill launch covers its split
  // clusters of c CTAs (index c, 1..16) of each cluster-mode decode kernel
  // that the device holds at once; 0 where that size cannot be scheduled
  int cluster_fit[2][2][17] = {};
  // set (release) once every field above is final; read with acquire
  std::atomic<bool> kernels_configured{false};
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// How many clusters of c CTAs of `kernel` the device holds at once, for
// c = 1..16 (0 where that size cannot be scheduled).
void cluster_fit(DecodeKernel kernel, size_t smem, int threads, int* fit) {
  for (int c = 1; c <= 16; ++c) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();   // a refused size is not an error of the caller's
      n = 0;
    }
    fit[c] = n;
  }
}

frt_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FRT_ERR_CUDA;
  DeviceInfo& di = g_dev[dev];
  if (!di.kernels_configured.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!di.kernels_configured.load(std::memory_order_relaxed)) {
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return FRT_ERR_CUDA;
      di.sm_count = sms;
      if (cudaFuncSetAttribute(decode_splitkv_kernel<128, 1, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               DecodeSmem<128, false, 1>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(decode_splitkv_kernel<128, 2, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               DecodeSmem<128, false, 2>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(decode_splitkv_kernel<64, 1, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               DecodeSmem<64, false, 1>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(decode_splitkv_kernel<64, 2, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               DecodeSmem<64, false, 2>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(decode_splitkv_kernel<128, 1, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               DecodeSmem<128, true, 1>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(decode_splitkv_kernel<128, 2, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               DecodeSmem<128, true, 2>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(prefill_kernel<128, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PrefillSmem<128>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(prefill_kernel<64, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PrefillSmem<64>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(prefill_kernel<128, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PrefillSmem<128>::kBytes) != cudaSuccess ||
          cudaFuncSetAttribute(prefill_kernel<64, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PrefillSmem<64>::kBytes) != cudaSuccess)
        return FRT_ERR_CUDA;
      // The prefill kernel hands registers from its producer warpgroup to
      // its softmax warpgroups (setmaxnreg).  That only works if the launch
      // reserves exactly the pool the split adds up to; otherwise the
      // increase would wait forever, so the kernel is never launched.
      cudaFuncAttributes fa[4];
      if (cudaFuncGetAttributes(&fa[0], prefill_kernel<128, false>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa[1], prefill_kernel<64, false>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa[2], prefill_kernel<128, true>) != cudaSuccess ||
          cudaFuncGetAttributes(&fa[3], prefill_kernel<64, true>) != cudaSuccess)
        return FRT_ERR_CUDA;
      di.prefill_ok = true;
      for (const cudaFuncAttributes& a : fa) di.prefill_ok &= a.numRegs == kPfRegsLaunch;
      for (int d = 0; d < 2; ++d)
        for (int t = 0; t < 2; ++t) {
          if (cudaFuncSetAttribute(kClusterDecode[d][t], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kClusterDecodeSmem[d][t]) != cudaSuccess ||
              cudaFuncSetAttribute(kClusterDecode[d][t],
                                   cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
            return FRT_ERR_CUDA;
          cluster_fit(kClusterDecode[d][t], kClusterDecodeSmem[d][t], kClusterDecodeThreads[t],
                      di.cluster_fit[d][t]);
        }
      di.kernels_configured.store(true, std::memory_order_release);
    }
  }
  *out = &di;
  return FRT_OK;
}

// ------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map (bf16 unless told otherwise) with 128-byte swizzling.  dims/box
// are innermost first; strides_bytes[i] is the stride of dims[i + 1].
bool make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box,
               CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bdim[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estr[i] = 1;
    if (i + 1 < rank) gstr[i] = strides_bytes[i];
  }
  CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base),
                  gdim, gstr, bdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool scale_ok(float scale) { return scale > 0.f && isfinite(scale); }

// ---------------------------------------------------- decode workspace
struct DecodeWorkspace {
  size_t o_off, lse_off, seg_off, total;
};

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Every kernel is launched as a programmatic dependent of the work before it
// in the stream: it is scheduled while that work still runs, and its first
// instruction (griddepcontrol.wait) holds it until that work has finished
// and its writes are visible, so ordering is the same as a plain launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// [segments] piece ranges, [slots, 16] partial LSEs, [slots, 16, D] partial
// outputs; every call writes what it later reads, so nothing carries over.
DecodeWorkspace decode_ws_layout(long long parts, long long segments, int D) {
  DecodeWorkspace w;
  const long long slots = parts + segments;
  w.seg_off = 0;
  w.lse_off = round_up((size_t)segments * sizeof(int2), 256);
  w.o_off = w.lse_off + round_up((size_t)slots * kDecHeadsPerSeg * sizeof(float), 256);
  w.total = w.o_off + round_up((size_t)slots * kDecHeadsPerSeg * D * sizeof(float), 256);
  return w;
}

// Shared launcher of the split-KV decode kernel (paged or contiguous cache).
frt_status launch_decode(const void* q, const void* k_base, const void* v_base,
                         uint64_t cache_rows, const int32_t* block_table, int max_pages,
                         const int32_t* seq_lens, int contig_len, void* o, float* lse, int B,
                         int Hq, int Hkv, int D, float scale, int num_splits, void* workspace,
                         size_t* workspace_bytes, cudaStream_t stream, bool fp8 = false,
                         const float* k_scale = nullptr, const float* v_scale = nullptr) {
  // fp8: the pages hold e4m3 codes with per-KV-head scales (D = 128)
  const bool query = (q == nullptr);
  DeviceInfo* di = nullptr;
  if (!query) {
    frt_status st = device_info(&di);
    if (st != FRT_OK) return st;
  }
  const int g = Hq / Hkv;
  const int hgroups = (g + kDecHeadsPerSeg - 1) / kDecHeadsPerSeg;
  const long long segments = (long long)B * Hkv * hgroups;
  int parts = num_splits;
  if (parts <= 0) {
    if (di == nullptr) {
      frt_status st = device_info(&di);
      if (st != FRT_OK) return st;
    }
    // bf16 cache: enough partitions for kDecInFlightBytes of page copies in
    // flight (192 on a 148-SM B200; measured faster than one or two per SM).
    // FP8 cache: its consumer warps, not HBM, set the pace, so every SM gets
    // as many partitions as it holds CTAs (three with one head tile, else two).
    const long long per_sm = !fp8 ? kDecCtasPerSm
                             : (g <= 8 ? DecodeCfg<true, 1>::kCtasPerSm : DecodeCfg<true, 2>::kCtasPerSm);
    const long long ring = (D == 128) ? DecodeSmem<128>::kRingBytes : DecodeSmem<64>::kRingBytes;
    const long long want = fp8 ? per_sm * di->sm_count : (kDecInFlightBytes + ring - 1) / ring;
    parts = (int)std::min<long long>(std::max<long long>(want, di->sm_count), per_sm * di->sm_count);
  }
  const DecodeWorkspace wl = decode_ws_layout(parts, segments, D);
  if (query) {
    if (workspace_bytes == nullptr) return FRT_ERR_INVALID_ARG;
    *workspace_bytes = wl.total;
    return FRT_OK;
  }
  if (B == 0) return FRT_OK;
  if (workspace == nullptr || workspace_bytes == nullptr || *workspace_bytes < wl.total ||
      !aligned16(workspace))
    return FRT_ERR_WORKSPACE;

  // One TMA box per page.  bf16: (64 columns, 16 rows, D/64 column halves);
  // the half index is the outermost box dimension, so the page lands in
  // shared memory as D/64 consecutive 16x64 swizzled blocks.  FP8: one box of
  // 16 rows x 128 bytes.
  CUtensorMap tk, tv;
  if (fp8) {
    const uint64_t dims[2] = {(uint64_t)D, cache_rows};
    const uint64_t strides[1] = {(uint64_t)D};
    const uint32_t box[2] = {(uint32_t)D, (uint32_t)kDecPage};
    if (!make_tmap(&tk, k_base, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8) ||
        !make_tmap(&tv, v_base, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8))
      return FRT_ERR_CUDA;
  } else {
    const uint64_t dims[3] = {64, cache_rows, (uint64_t)(D / 64)};
    const uint64_t strides[2] = {(uint64_t)D * 2, 128};
    const uint32_t box[3] = {64, (uint32_t)kDecPage, (uint32_t)(D / 64)};
    if (!make_tmap(&tk, k_base, 3, dims, strides, box) ||
        !make_tmap(&tv, v_base, 3, dims, strides, box))
      return FRT_ERR_CUDA;
  }

  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.max_pages = max_pages;
  p.num_pages = block_table != nullptr ? (int)(cache_rows / ((uint64_t)Hkv * kDecPage)) : 0;
  p.bad_row = (int)cache_rows;
  p.contig_len = contig_len;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = g;
  p.hgroups = hgroups;
  p.parts = parts;
  p.scale_log2 = scale * kLog2e;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ws_o = reinterpret_cast<float*>(ws + wl.o_off);
  p.ws_lse = reinterpret_cast<float*>(ws + wl.lse_off);
  p.ws_seg = reinterpret_cast<int2*>(ws + wl.seg_off);

  // one 8-head tile per segment when a KV head serves at most 8 query heads
  const bool one_tile = g <= 8;
  // kernel, its shared memory and block size for this cache type and head tiling
  void (*kernel)(CUtensorMap, CUtensorMap, DecodeParams) = nullptr;
  size_t smem = 0;
  int threads = 0;
  auto pick = [&](auto k, size_t bytes, int nthreads) {
    kernel = k;
    smem = bytes;
    threads = nthreads;
  };
  if (fp8) {
    if (one_tile)
      pick(decode_splitkv_kernel<128, 1, true>, DecodeSmem<128, true, 1>::kBytes, DecodeCfg<true, 1>::kThreads);
    else
      pick(decode_splitkv_kernel<128, 2, true>, DecodeSmem<128, true, 2>::kBytes, DecodeCfg<true, 2>::kThreads);
  } else if (D == 128) {
    if (one_tile)
      pick(decode_splitkv_kernel<128, 1, false>, DecodeSmem<128, false, 1>::kBytes, DecodeCfg<false, 1>::kThreads);
    else
      pick(decode_splitkv_kernel<128, 2, false>, DecodeSmem<128, false, 2>::kBytes, DecodeCfg<false, 2>::kThreads);
  } else {
    if (one_tile)
      pick(decode_splitkv_kernel<64, 1, false>, DecodeSmem<64, false, 1>::kBytes, DecodeCfg<false, 1>::kThreads);
    else
      pick(decode_splitkv_kernel<64, 2, false>, DecodeSmem<64, false, 2>::kBytes, DecodeCfg<false, 2>::kThreads);
  }
  if (launch_pdl(kernel, dim3(parts), dim3(threads), smem, stream, tk, tv, p) != cudaSuccess)
    return FRT_ERR_CUDA;

  // The merge of split segments: its CTAs are scheduled while the kernel
  // above still runs and start when it has finished.  One CTA per row (two
  // fit on an SM), at most two per SM.
  const long long rows = (long long)B * Hq;
  const unsigned merge_grid = (unsigned)std::min<long long>(rows, 2ll * di->sm_count);
  const cudaError_t err =
      launch_pdl((D == 128) ? decode_merge_kernel<128> : decode_merge_kernel<64>, dim3(merge_grid),
                 dim3(kMergeThreads), 0, stream, p);
  return err == cudaSuccess ? FRT_OK : FRT_ERR_CUDA;
}

// Single-token decode over a contiguous cache with no workspace: one cluster
// of C CTAs per segment (sequence, KV head, group of <= 16 query heads), the
// partial states merged through distributed shared memory.  C is the largest
// cluster size whose grid (segments x C CTAs) the device holds in one wave,
// with at most two CTAs per SM and one CTA per page.
frt_status launch_decode_cluster(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int Hq, int Hkv, int Skv, int D, float scale,
                                 cudaStream_t stream) {
  DeviceInfo* di = nullptr;
  frt_status st = device_info(&di);
  if (st != FRT_OK) return st;
  const int g = Hq / Hkv;
  const int hgroups = (g + kDecHeadsPerSeg - 1) / kDecHeadsPerSeg;
  const long long segments = (long long)B * Hkv * hgroups;
  const int d128 = (D == 128) ? 1 : 0, two_tiles = (g > 8) ? 1 : 0;
  const long long pages = (Skv + kDecPage - 1) / kDecPage;
  const long long slots = (long long)kDecCtasPerSm * di->sm_count;
  long long C = std::min<long long>(16, std::min(pages, slots / segments));
  while (C > 1 && di->cluster_fit[d128][two_tiles][C] < segments) --C;
  C = std::max<long long>(1, C);
  if (segments * C > 0x7fffffffLL) return FRT_ERR_UNSUPPORTED;

  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)B * Hkv * Skv;
  const uint64_t dims[3] = {64, rows, (uint64_t)(D / 64)};
  const uint64_t strides[2] = {(uint64_t)D * 2, 128};
  const uint32_t box[3] = {64, (uint32_t)kDecPage, (uint32_t)(D / 64)};
  if (!make_tmap(&tk, k, 3, dims, strides, box) || !make_tmap(&tv, v, 3, dims, strides, box))
    return FRT_ERR_CUDA;
  DecodeParams p = {};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.contig_len = Skv;
  p.bad_row = (int)rows;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = g;
  p.hgroups = hgroups;
  p.parts = (int)(segments * C);
  p.scale_log2 = scale * kLog2e;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(segments * C));
  cfg.blockDim = dim3(kClusterDecodeThreads[two_tiles]);
  cfg.dynamicSmemBytes = kClusterDecodeSmem[d128][two_tiles];
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kClusterDecode[d128][two_tiles], tk, tv, p) == cudaSuccess
             ? FRT_OK
             : FRT_ERR_CUDA;
}

// Tiled tensor-core forward.  Contiguous K/V [B, Hkv, Skv, D] (paged == null),
// or chunked prefill over a paged cache (paged != null: Sq is the padded
// chunk length, lengths per sequence are on the device).
struct PagedKV {
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* q_lens;
  int max_pages, num_pages;
};

// Element strides of a [B, H, S, D] tensor's batch, head and token
// dimensions (d is contiguous).
struct TokStrides {
  long long b, h, t;
};

frt_status launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int Sq, int Skv, int D, int causal,
                          float scale, cudaStream_t stream, const PagedKV* paged = nullptr,
                          const TokStrides* strides = nullptr /* q, k, v, o; null: contiguous */) {
  DeviceInfo* di = nullptr;
  frt_status st = device_info(&di);
  if (st != FRT_OK) return st;
  if (!di->prefill_ok) return FRT_ERR_UNSUPPORTED;
  // An even number of query heads per KV head: a CTA's two tiles are two
  // heads of one group at the same 128 rows; otherwise two row halves of one
  // head (256-row blocks).
  const bool head_pairs = ((Hq / Hkv) % 2) == 0;
  const int blk_rows = head_pairs ? kPfBM : kPfRows;
  const int n_blocks = (Sq + blk_rows - 1) / blk_rows;
  // work items: (sequence, query-head pair or head, query block)
  const long long n_items = (long long)B * (head_pairs ? Hq / 2 : Hq) * n_blocks;
  if (n_items > (1ll << 30)) return FRT_ERR_UNSUPPORTED;
  if (n_items == 0) return FRT_OK;
  // Q, O (and contiguous K, V): 4D maps (d, token, head, batch) with the
  // tensors' own strides, one 128-row box per column half
  CUtensorMap tq, tk, tv, to;
  const TokStrides q_c{(long long)Hq * Sq * D, (long long)Sq * D, D};
  const TokStrides k_c{(long long)Hkv * Skv * D, (long long)Skv * D, D};
  const TokStrides& qs = strides ? strides[0] : q_c;
  const TokStrides& ks = strides ? strides[1] : k_c;
  const TokStrides& vs = strides ? strides[2] : k_c;
  const TokStrides& os = strides ? strides[3] : q_c;
  const uint32_t box[4] = {64, (uint32_t)kPfBM, 1, 1};
  auto map4 = [&](CUtensorMap* m, const void* base, int S, int H, int Bn, const TokStrides& st) {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)S, (uint64_t)H, (uint64_t)Bn};
    const uint64_t str[3] = {(uint64_t)st.t * 2, (uint64_t)st.h * 2, (uint64_t)st.b * 2};
    return make_tmap(m, base, 4, dims, str, box);
  };
  if (!map4(&tq, q, Sq, Hq, B, qs) || !map4(&to, o, Sq, Hq, B, os)) return FRT_ERR_CUDA;
  if (paged == nullptr) {
    if (Skv > 0) {
      if (!map4(&tk, k, Skv, Hkv, B, ks) || !map4(&tv, v, Skv, Hkv, B, vs)) return FRT_ERR_CUDA;
    } else {
      // With Skv == 0 every tile has no key tile to visit (o = 0, lse =
      // -inf); the K/V maps then only need to be valid descriptors, never read.
      const TokStrides one{D, D, D};
      if (!map4(&tk, q, 1, 1, 1, one) || !map4(&tv, q, 1, 1, 1, one)) return FRT_ERR_CUDA;
    }
  } else {
    // page pool as rows of D: one 16-row box per page and column half
    const uint64_t kdims[2] = {(uint64_t)D, (uint64_t)paged->num_pages * Hkv * 16};
    const uint64_t kstr[1] = {(uint64_t)D * 2};
    const uint32_t pbox[2] = {64, 16};
    if (!make_tmap(&tk, k, 2, kdims, kstr, pbox) || !make_tmap(&tv, v, 2, kdims, kstr, pbox))
      return FRT_ERR_CUDA;
  }
  PrefillParams p;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = Hq / Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.causal = causal;
  p.n_blocks = n_blocks;
  p.head_pairs = head_pairs ? 1 : 0;
  p.n_items = (int)n_items;
  p.scale_log2 = scale * kLog2e;
  p.block_table = paged ? paged->block_table : nullptr;
  p.seq_lens = paged ? paged->seq_lens : nullptr;
  p.q_lens = paged ? paged->q_lens : nullptr;
  p.max_pages = paged ? paged->max_pages : 0;
  p.num_pages = paged ? paged->num_pages : 0;
  p.bad_row = paged ? paged->num_pages * Hkv * 16 : 0;
  // persistent: one CTA per SM (the kernel holds a whole SM's shared memory),
  // each walking its share of the items
  const dim3 grid((unsigned)std::min<long long>(n_items, di->sm_count));
  auto* kernel = (paged == nullptr)
                     ? (D == 128 ? prefill_kernel<128, false> : prefill_kernel<64, false>)
                     : (D == 128 ? prefill_kernel<128, true> : prefill_kernel<64, true>);
  const size_t smem = (D == 128) ? PrefillSmem<128>::kBytes : PrefillSmem<64>::kBytes;
  return launch_pdl(kernel, grid, dim3(kPfThreads), smem, stream, tq, tk, tv, to, p) == cudaSuccess
             ? FRT_OK
             : FRT_ERR_CUDA;
}

// ------------------------------------------- decode without caller scratch
// Scratch of frt_attn_decode_paged_noalloc: one fixed buffer per device,
// reserved when the library is loaded and held until the process exits.  In
// host code this name only stands for the device variable; the kernel gets
// its device address from cudaGetSymbolAddress, taken once per device.
constexpr size_t kNoAllocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char frt_noalloc_scratch[kNoAllocScratchBytes];

std::atomic<void*> g_noalloc_ptr[kMaxDevices];   // set once (release), read with acquire
std::mutex g_noalloc_mutex;

// Device address of this device's scratch (looked up on the first call made
// with that device current).
frt_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FRT_ERR_CUDA;
  void* ptr = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (ptr == nullptr) {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    ptr = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (ptr == nullptr) {
      if (cudaGetSymbolAddress(&ptr, frt_noalloc_scratch) != cudaSuccess || ptr == nullptr)
        return FRT_ERR_CUDA;
      g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
    }
  }
  *out = ptr;
  return FRT_OK;
}

// One thread waits on an mbarrier that nothing arrives at, with the bounded
// wait every kernel of the library uses: it must give up after its limit,
// raise the time-out bit of the device error word and return.  *returned
// becomes 2 when the wait gave up, 1 if it (wrongly) completed.
__global__ void wait_timeout_selftest_kernel(int* returned) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    *returned = mbar_wait(&bar, 0u, &abort_flag) ? 1 : 2;
  }
}

__global__ void fp8_decode_selftest_kernel(const uint8_t* codes, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i < n) {
    const uint32_t x = codes[i] | (i + 1 < n ? (uint32_t)codes[i + 1] << 8 : 0u);
    float lo, hi;
    unpack_f16x2(e4m3x2_to_f16x2(x), lo, hi);
    y[i] = lo;
    if (i + 1 < n) y[i + 1] = hi;
  }
}

}  // namespace
}  // namespace frt

using namespace frt;

extern "C" {

frt_status frt_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, int max_pages_per_seq,
                                 const int32_t* seq_lens, int page_size, int num_pages,
                                 void* o, float* lse, int B, int Hq, int Hkv, int D,
                                 float scale, int num_splits, void* workspace,
                                 size_t* workspace_bytes, cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || num_pages < 0 || max_pages_per_seq < 0 ||
      num_splits < 0 || !scale_ok(scale))
    return FRT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FRT_ERR_UNSUPPORTED;
  if (page_size != kDecPage) return FRT_ERR_UNSUPPORTED;
  if (B > kDecMaxBatch) return FRT_ERR_UNSUPPORTED;
  if ((uint64_t)num_pages * Hkv * page_size >= (1ull << 31)) return FRT_ERR_UNSUPPORTED;
  // the kernel's page prefix over the batch and a sequence's token count are 32-bit
  if ((uint64_t)B * max_pages_per_seq >= (1ull << 31) ||
      (uint64_t)max_pages_per_seq * page_size >= (1ull << 31))
    return FRT_ERR_UNSUPPORTED;
  if (q != nullptr && B > 0) {
    if (k_pages == nullptr || v_pages == nullptr || o == nullptr ||
        seq_lens == nullptr || (block_table == nullptr && max_pages_per_seq > 0))
      return FRT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) ||
        (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
      return FRT_ERR_INVALID_ARG;
    if (num_pages == 0) return FRT_ERR_INVALID_ARG;
  }
  return launch_decode(q, k_pages, v_pages, (uint64_t)num_pages * Hkv * page_size, block_table,
                       max_pages_per_seq, seq_lens, 0, o, lse, B, Hq, Hkv, D, scale,
                       num_splits, workspace, workspace_bytes, stream);
}

frt_status frt_attn_decode_paged_fp8(const void* q, const void* k_pages, const void* v_pages,
                                     const float* k_scale, const float* v_scale,
                                     const int32_t* block_table, int max_pages_per_seq,
                                     const int32_t* seq_lens, int page_size, int num_pages,
                                     void* o, float* lse, int B, int Hq, int Hkv, int D,
                                     float scale, int num_splits, void* workspace,
                                     size_t* workspace_bytes, cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || num_pages < 0 || max_pages_per_seq < 0 ||
      num_splits < 0 || !scale_ok(scale))
    return FRT_ERR_INVALID_ARG;
  if (D != 128) return FRT_ERR_UNSUPPORTED;
  if (page_size != kDecPage) return FRT_ERR_UNSUPPORTED;
  if (B > kDecMaxBatch) return FRT_ERR_UNSUPPORTED;
  if ((uint64_t)num_pages * Hkv * page_size >= (1ull << 31)) return FRT_ERR_UNSUPPORTED;
  if ((uint64_t)B * max_pages_per_seq >= (1ull << 31) ||
      (uint64_t)max_pages_per_seq * page_size >= (1ull << 31))
    return FRT_ERR_UNSUPPORTED;
  if (q != nullptr && B > 0) {
    if (k_pages == nullptr || v_pages == nullptr || o == nullptr || k_scale == nullptr ||
        v_scale == nullptr || seq_lens == nullptr ||
        (block_table == nullptr && max_pages_per_seq > 0))
      return FRT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o) ||
        (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
      return FRT_ERR_INVALID_ARG;
    if (num_pages == 0) return FRT_ERR_INVALID_ARG;
  }
  return launch_decode(q, k_pages, v_pages, (uint64_t)num_pages * Hkv * page_size, block_table,
                       max_pages_per_seq, seq_lens, 0, o, lse, B, Hq, Hkv, D, scale, num_splits,
                       workspace, workspace_bytes, stream, true, k_scale, v_scale);
}

frt_status frt_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Sq, int Skv, int D, int causal, float scale,
                        cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Sq < 0 || Skv < 0 ||
      (causal != 0 && causal != 1) || !scale_ok(scale))
    return FRT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FRT_ERR_UNSUPPORTED;
  if ((uint64_t)B * Hkv * Skv >= (1ull << 31) || (uint64_t)B * Hq * Sq >= (1ull << 31))
    return FRT_ERR_UNSUPPORTED;
  if (B == 0 || Sq == 0) return FRT_OK;
  if (q == nullptr || o == nullptr || (Skv > 0 && (k == nullptr || v == nullptr)))
    return FRT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (Skv > 0 && (!aligned16(k) || !aligned16(v))) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FRT_ERR_INVALID_ARG;
  if (Sq == 1 && Skv > 0)
    return launch_decode_cluster(q, k, v, o, lse, B, Hq, Hkv, Skv, D, scale, stream);
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, causal, scale, stream);
}

frt_status frt_attn_fwd_ws(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int Sq, int Skv, int D, int causal,
                           float scale, void* workspace, size_t* workspace_bytes,
                           cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Sq < 0 || Skv < 0 ||
      (causal != 0 && causal != 1) || !scale_ok(scale))
    return FRT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FRT_ERR_UNSUPPORTED;
  if ((uint64_t)B * Hkv * Skv >= (1ull << 31) || (uint64_t)B * Hq * Sq >= (1ull << 31))
    return FRT_ERR_UNSUPPORTED;
  const bool decode = (Sq == 1 && Skv > 0);
  if (q == nullptr) {   // size query
    if (workspace_bytes == nullptr) return FRT_ERR_INVALID_ARG;
    if (!decode) {
      *workspace_bytes = 0;
      return FRT_OK;
    }
    return launch_decode(nullptr, k, v, (uint64_t)B * Hkv * Skv, nullptr, 0, nullptr, Skv, o,
                         lse, B, Hq, Hkv, D, scale, 0, nullptr, workspace_bytes, stream);
  }
  if (B == 0 || Sq == 0) return FRT_OK;
  if (o == nullptr || (Skv > 0 && (k == nullptr || v == nullptr)))
    return FRT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (Skv > 0 && (!aligned16(k) || !aligned16(v))) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FRT_ERR_INVALID_ARG;
  if (decode) {
    if (B > kDecMaxBatch) return FRT_ERR_UNSUPPORTED;
    return launch_decode(q, k, v, (uint64_t)B * Hkv * Skv, nullptr, 0, nullptr, Skv, o, lse, B,
                         Hq, Hkv, D, scale, 0, workspace, workspace_bytes, stream);
  }
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, causal, scale, stream);
}

frt_status frt_attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int Hq, int Hkv, int Sq, int Skv, int D, int causal,
                                float scale, const int64_t* q_strides, const int64_t* k_strides,
                                const int64_t* v_strides, const int64_t* o_strides,
                                cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Sq < 0 || Skv < 0 ||
      (causal != 0 && causal != 1) || !scale_ok(scale))
    return FRT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FRT_ERR_UNSUPPORTED;
  if ((uint64_t)B * Hq * Sq >= (1ull << 31) || (uint64_t)B * Hkv * Skv >= (1ull << 31))
    return FRT_ERR_UNSUPPORTED;
  if (q_strides == nullptr || k_strides == nullptr || v_strides == nullptr || o_strides == nullptr)
    return FRT_ERR_INVALID_ARG;
  TokStrides st[4];
  const int64_t* src[4] = {q_strides, k_strides, v_strides, o_strides};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 3; ++j) {
      // every step of a TMA walk is a multiple of 16 bytes (8 bf16)
      const int64_t x = src[i][j];
      if (x <= 0 || x % 8 != 0 || x >= (1ll << 38)) return FRT_ERR_INVALID_ARG;
    }
    st[i] = TokStrides{src[i][0], src[i][1], src[i][2]};
  }
  if (B == 0 || Sq == 0) return FRT_OK;
  if (q == nullptr || o == nullptr || (Skv > 0 && (k == nullptr || v == nullptr)))
    return FRT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || (Skv > 0 && (!aligned16(k) || !aligned16(v))) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FRT_ERR_INVALID_ARG;
  return launch_prefill(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, causal, scale, stream, nullptr,
                        st);
}

frt_status frt_attn_prefill_paged(const void* q, const void* k_pages, const void* v_pages,
                                  const int32_t* block_table, int max_pages_per_seq,
                                  const int32_t* seq_lens, const int32_t* q_lens, int page_size,
                                  int num_pages, void* o, float* lse, int B, int Hq, int Hkv,
                                  int max_q, int D, int causal, float scale,
                                  cudaStream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_q < 0 || num_pages < 0 ||
      max_pages_per_seq < 0 || (causal != 0 && causal != 1) || !scale_ok(scale))
    return FRT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FRT_ERR_UNSUPPORTED;
  if (page_size != 16) return FRT_ERR_UNSUPPORTED;
  if ((uint64_t)num_pages * Hkv * page_size >= (1ull << 31) ||
      (uint64_t)B * Hq * max_q >= (1ull << 31) ||
      (uint64_t)max_pages_per_seq * page_size >= (1ull << 31))   // 32-bit length bound
    return FRT_ERR_UNSUPPORTED;
  if (B == 0 || max_q == 0) return FRT_OK;
  if (q == nullptr || o == nullptr || k_pages == nullptr || v_pages == nullptr ||
      block_table == nullptr || seq_lens == nullptr || q_lens == nullptr ||
      max_pages_per_seq == 0 || num_pages == 0)
    return FRT_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(k_pages) || !aligned16(v_pages) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(q_lens) & 3u))
    return FRT_ERR_INVALID_ARG;
  PagedKV pk{block_table, seq_lens, q_lens, max_pages_per_seq, num_pages};
  return launch_prefill(q, k_pages, v_pages, o, lse, B, Hq, Hkv, max_q, 0, D, causal, scale,
                        stream, &pk);
}

frt_status frt_attn_merge_lse(const float* o_parts, const float* lse_parts, int S, int B,
                              int Hq, int D, void* o, float* lse, cudaStream_t stream) {
  if (S <= 0 || B < 0 || Hq <= 0) return FRT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FRT_ERR_UNSUPPORTED;
  const long long rows = (long long)B * Hq;
  if (rows == 0) return FRT_OK;
  if (o_parts == nullptr || lse_parts == nullptr || o == nullptr) return FRT_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FRT_ERR_INVALID_ARG;
  const long long blocks = (rows + kMergeWarps - 1) / kMergeWarps;
  if (blocks > 0x7fffffffLL) return FRT_ERR_UNSUPPORTED;
  return launch_pdl(D == 128 ? merge_lse_kernel<128> : merge_lse_kernel<64>, dim3((unsigned)blocks),
                    dim3(kMergeWarps * 32), 0, stream, o_parts, lse_parts, S, rows,
                    static_cast<__nv_bfloat16*>(o), lse) == cudaSuccess
             ? FRT_OK
             : FRT_ERR_CUDA;
}

frt_status frt_attn_decode_paged_noalloc(const void* q, const void* k_pages,
                                         const void* v_pages, const int32_t* block_table,
                                         int max_pages_per_seq, const int32_t* seq_lens,
                                         int page_size, int num_pages, void* o, float* lse,
                                         int B, int Hq, int Hkv, int D, float scale,
                                         int num_splits, cudaStream_t stream) {
  // size this call needs, checked against the fixed scratch before anything runs
  size_t need = 0;
  frt_status st = frt_attn_decode_paged(nullptr, k_pages, v_pages, block_table,
                                        max_pages_per_seq, seq_lens, page_size, num_pages, o,
                                        lse, B, Hq, Hkv, D, scale, num_splits, nullptr, &need,
                                        stream);
  if (st != FRT_OK) return st;
  if (need > kNoAllocScratchBytes) return FRT_ERR_WORKSPACE;
  if (B == 0) return FRT_OK;
  if (q == nullptr) return FRT_ERR_INVALID_ARG;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != FRT_OK) return st;
  // The kernels write every word of the scratch they read later in the
  // call, so whatever a previous call left there is harmless.
  size_t have = kNoAllocScratchBytes;
  return frt_attn_decode_paged(q, k_pages, v_pages, block_table, max_pages_per_seq, seq_lens,
                               page_size, num_pages, o, lse, B, Hq, Hkv, D, scale, num_splits,
                               scratch, &have, stream);
}

frt_status frt_read_device_error(unsigned* flags) {
  if (flags == nullptr) return FRT_ERR_INVALID_ARG;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, frt_device_error, sizeof v) != cudaSuccess) return FRT_ERR_CUDA;
  if (cudaMemcpyToSymbol(frt_device_error, &zero, sizeof zero) != cudaSuccess)
    return FRT_ERR_CUDA;
  *flags = v;
  return FRT_OK;
}

frt_status frt_debug_fp8_decode(const uint8_t* codes, float* y, int n, cudaStream_t stream) {
  if (n < 0 || (n > 0 && (codes == nullptr || y == nullptr))) return FRT_ERR_INVALID_ARG;
  if (n == 0) return FRT_OK;
  const int pairs = (n + 1) / 2;
  fp8_decode_selftest_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(codes, y, n);
  return cudaGetLastError() == cudaSuccess ? FRT_OK : FRT_ERR_CUDA;
}

frt_status frt_debug_wait_timeout(int* returned, cudaStream_t stream) {
  if (returned == nullptr || !aligned16(returned)) return FRT_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(returned);
  return cudaGetLastError() == cudaSuccess ? FRT_OK : FRT_ERR_CUDA;
}

const char* frt_version(void) { return "0.1.0"; }

}  // extern "C"
