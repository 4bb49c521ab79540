// Host side of the C ABI declared in include/pa_b200.h: argument checks,
// launch configuration and dispatch to the sm_100a kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <mutex>

#include <cudaTypedefs.h>

#include "pa_b200.h"
#include "pa_cascade.cuh"
#include "pa_copy.cuh"
#include "pa_kernels.cuh"
#include "pa_prefill.cuh"
#include "pa_mma.cuh"
#include "pa_stream.cuh"

namespace {

thread_local std::string t_last_cuda_error;
std::atomic<uint64_t> g_launches{0};

constexpr int kMaxDevices = 64;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s per bulk-copy wait

struct DeviceInfo {
  int sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mu;

int record(cudaError_t e) {
  t_last_cuda_error = cudaGetErrorString(e);
  return PA_ERR_CUDA;
}

// SM count of the current device (cached per device).
int current_sms(int *sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record(e);
  if (dev < 0 || dev >= kMaxDevices) {
    t_last_cuda_error = "device ordinal beyond the library's table";
    return PA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_devices[dev].sms == 0) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return record(e);
    g_devices[dev].sms = sms;
  }
  *sms_out = g_devices[dev].sms;
  return PA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The address at which the current device reaches `p`: device memory of this
// device as is, pinned (page-locked, mapped) host memory through its device
// alias.  Anything else would fault inside a kernel, so it is refused here.
int device_view(const void *p, const void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record(e);
  cudaPointerAttributes at{};
  e = cudaPointerGetAttributes(&at, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_ADDRESS;
  }
  switch (at.type) {
    case cudaMemoryTypeDevice:
      if (at.device != dev) return PA_ERR_ADDRESS;
      *out = p;
      return PA_OK;
    case cudaMemoryTypeManaged:
      *out = p;
      return PA_OK;
    case cudaMemoryTypeHost:
      if (!at.devicePointer) return PA_ERR_ADDRESS;
      *out = at.devicePointer;
      return PA_OK;
    default:
      return PA_ERR_ADDRESS;
  }
}

// Query heads handled together by one head chunk (the K/V tiles are read once
// for all of them).  Groups of 1 or 2 run on the CUDA-core kernel; larger
// groups run on the tensor-core kernel, whose chunks take up to 8 query heads
// (the largest divisor of the group size not above 8).  Measured on B200 with
// the CUDA-core kernel extended to 3 and 4 heads per chunk: 287 us against
// 165 us for the 32 query / 8 kv head batch (256 sequences) and 112 us against
// 45 us for the shared-prefix step (the extra accumulators spill at head_dim
// 128, and the fp32 FMA work per K/V byte doubles).
bool uses_mma(int group) { return group >= 3; }
int heads_per_unit(int group) {
  if (!uses_mma(group)) return group;
  for (int c = 8; c > 1; --c)
    if (group % c == 0) return c;
  return 1;
}

// Launch shape of the split kernels (warps per block, ring slots per warp);
// overridable at build time for tuning sweeps.
#ifndef PA_WARPS
#define PA_WARPS 4
#endif
#ifndef PA_STAGES
#define PA_STAGES 2
#endif
// Balanced split (see ChunkPlan): per-mille share of each warp's tiles in its
// static first chunk, and queued chunks per warp for the rest of the stream.
// Measured on B200 (Llama-2, long-context, GQA and shared-prefix batches):
// uniform chunks are best -- about 8 per warp for the CUDA-core kernel (fine
// tail balancing), 1 per warp for the tensor-core kernel, whose cut pieces
// carry several heads to merge; a large static first chunk loses more to
// per-warp speed differences than it saves in merging.
#ifndef PA_STATIC_PERMILLE
#define PA_STATIC_PERMILLE 0
#endif
#ifndef PA_TAIL_CHUNKS
#define PA_TAIL_CHUNKS 8
#endif
#ifndef PA_MMA_STATIC_PERMILLE
#define PA_MMA_STATIC_PERMILLE 0
#endif
#ifndef PA_MMA_TAIL_CHUNKS
#define PA_MMA_TAIL_CHUNKS 1
#endif
constexpr int kWarps = PA_WARPS, kStages = PA_STAGES;
int static_permille(int group) { return uses_mma(group) ? PA_MMA_STATIC_PERMILLE : PA_STATIC_PERMILLE; }
int tail_chunks(int group) { return uses_mma(group) ? PA_MMA_TAIL_CHUNKS : PA_TAIL_CHUNKS; }

// Launches `kernel` with programmatic stream serialisation allowed: it may start
// while the previous kernel in the stream finishes, and waits for it on the
// device (griddepcontrol.wait) before touching any input.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
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

// Per-call tag of the chunk counter (never 0: the merge kernel leaves the counter at 0).
std::atomic<uint32_t> g_epoch{0x9e3779b9u};
uint32_t next_epoch() {
  uint32_t e;
  do {
    e = g_epoch.fetch_add(0x61c88647u, std::memory_order_relaxed);
  } while (e == 0);
  return e;
}
constexpr int kMaxSeqs = 32768;         // tile prefix kept in shared memory

template <class E, int D>
const void *split_kernel(int group) {
  if (uses_mma(group)) return reinterpret_cast<const void *>(pa::decode_split_mma_kernel<E, D, kWarps, kStages>);
  if (heads_per_unit(group) == 2) return reinterpret_cast<const void *>(pa::decode_split_kernel<E, D, 2, kWarps, kStages>);
  return reinterpret_cast<const void *>(pa::decode_split_kernel<E, D, 1, kWarps, kStages>);
}
const void *split_kernel_for(int dtype, int head_dim, int group) {
  if (dtype == PA_BFLOAT16) return head_dim == 128 ? split_kernel<pa::BF16, 128>(group) : split_kernel<pa::BF16, 64>(group);
  return head_dim == 128 ? split_kernel<pa::F16, 128>(group) : split_kernel<pa::F16, 64>(group);
}
uint32_t split_smem(int head_dim, int group, int num_seqs) {
  if (uses_mma(group))
    return head_dim == 128 ? pa::MmaSmem<pa::F16, 128, kWarps, kStages>::bytes(num_seqs)
                           : pa::MmaSmem<pa::F16, 64, kWarps, kStages>::bytes(num_seqs);
  return head_dim == 128 ? pa::SplitSmem<kWarps, kStages, 2 * pa::TILE * 128 * 2>::bytes(num_seqs)
                         : pa::SplitSmem<kWarps, kStages, 2 * pa::TILE * 64 * 2>::bytes(num_seqs);
}

// The per-segment kernel (small batches, CUDA-core path): one block of kWarps warps per segment.
template <class E, int D>
const void *segment_kernel(int G) {
  if (G == 2) return reinterpret_cast<const void *>(pa::decode_segment_kernel<E, D, 2, kWarps, kStages>);
  return reinterpret_cast<const void *>(pa::decode_segment_kernel<E, D, 1, kWarps, kStages>);
}
const void *segment_kernel_for(int dtype, int head_dim, int G) {
  if (dtype == PA_BFLOAT16) return head_dim == 128 ? segment_kernel<pa::BF16, 128>(G) : segment_kernel<pa::BF16, 64>(G);
  return head_dim == 128 ? segment_kernel<pa::F16, 128>(G) : segment_kernel<pa::F16, 64>(G);
}
uint32_t segment_smem(int head_dim) {
  return head_dim == 128 ? pa::SplitSmem<kWarps, kStages, 2 * pa::TILE * 128 * 2>::bytes(0)
                         : pa::SplitSmem<kWarps, kStages, 2 * pa::TILE * 64 * 2>::bytes(0);
}
// A segment of at most this many 16-token tiles (kWarps warps x 8) may take the per-segment kernel.
constexpr int kSegmentMaxTiles = kWarps * 8;

// Resident blocks per SM of `kernel` with `smem` bytes of dynamic shared memory (cached).
struct OccEntry {
  int dev;
  const void *kernel;
  uint32_t smem;
  int per_sm;
};
OccEntry g_occ[64];
int g_occ_next = 0;

int blocks_per_sm(const void *kernel, uint32_t smem, int *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record(e);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (const auto &o : g_occ)
      if (o.kernel == kernel && o.smem == smem && o.dev == dev) {
        *out = o.per_sm;
        return PA_OK;
      }
  }
  // the kernel may later be launched with any smem up to the device's opt-in limit
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return record(e);
  if (smem > (uint32_t)optin) return PA_ERR_SHAPE;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  if (e != cudaSuccess) return record(e);
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kWarps * 32, smem);
  if (e != cudaSuccess) return record(e);
  per_sm = std::max(per_sm, 1);
  std::lock_guard<std::mutex> lk(g_mu);
  g_occ[g_occ_next] = OccEntry{dev, kernel, smem, per_sm};
  g_occ_next = (g_occ_next + 1) % 64;
  *out = per_sm;
  return PA_OK;
}

int check_decode_shape(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                       int32_t block_size, int32_t max_context_len) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0) return PA_ERR_SHAPE;
  if (num_seqs > kMaxSeqs) return PA_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_HEADS;
  return PA_OK;
}

// Grid, shared memory and workspace layout of one decode call.  The workspace
// size does not depend on the storage type: it is sized for the larger of the
// two instantiations' grids, and the launch never uses more warps than that.
struct LaunchPlan {
  bool segment_mode;  // the per-segment kernel, no workspace, no merge kernel
  uint32_t smem;
  int grid;          // blocks of the split kernel (for `dtype`; 0 if not asked)
  long long max_chunks;
  int chunk_tiles;   // 0: balanced
  size_t queue_bytes, tiles_bytes, ml_bytes, acc_bytes, total_bytes;
};

int plan_decode(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len,
                int partition_tokens, int dtype, LaunchPlan *lp) {
  if (partition_tokens < 0 || partition_tokens % pa::TILE != 0) return PA_ERR_PARTITION;
  int sms = 0;
  int rc = current_sms(&sms);
  if (rc != PA_OK) return rc;
  const int group = num_q_heads / num_kv_heads;
  const int G = heads_per_unit(group);
  // Small batches on the CUDA-core path: every segment (sequence, head chunk) fits one wave of per-segment
  // blocks and has at most kSegmentMaxTiles tiles.  The choice depends on the sizes only, not on the
  // storage type, so the workspace size query agrees with the call.
  lp->segment_mode = false;
  if (!uses_mma(group) && partition_tokens == 0 && num_seqs > 0 &&
      ((long long)max_context_len + pa::TILE - 1) / pa::TILE <= kSegmentMaxTiles) {
    const uint32_t sm = segment_smem(head_dim);
    int o16 = 0, o_bf = 0;
    if ((rc = blocks_per_sm(segment_kernel_for(PA_FLOAT16, head_dim, G), sm, &o16)) != PA_OK) return rc;
    if ((rc = blocks_per_sm(segment_kernel_for(PA_BFLOAT16, head_dim, G), sm, &o_bf)) != PA_OK) return rc;
    if ((long long)num_seqs * num_kv_heads * (group / G) <= (long long)sms * std::min(o16, o_bf)) {
      lp->segment_mode = true;
      lp->smem = sm;
      lp->grid = num_seqs * num_kv_heads * (group / G);
      lp->chunk_tiles = 0;
      lp->max_chunks = 0;
      lp->queue_bytes = lp->tiles_bytes = lp->ml_bytes = lp->acc_bytes = lp->total_bytes = 0;
      return PA_OK;
    }
  }
  lp->smem = split_smem(head_dim, group, num_seqs);
  if (lp->smem > 227u * 1024u) return PA_ERR_SHAPE;
  int occ_f16 = 0, occ_bf16 = 0;
  if ((rc = blocks_per_sm(split_kernel_for(PA_FLOAT16, head_dim, group), lp->smem, &occ_f16)) != PA_OK) return rc;
  if ((rc = blocks_per_sm(split_kernel_for(PA_BFLOAT16, head_dim, group), lp->smem, &occ_bf16)) != PA_OK) return rc;
  const long long ws_warps = (long long)sms * std::max(occ_f16, occ_bf16) * kWarps;
  lp->grid = dtype == 0 ? 0 : sms * (dtype == PA_BFLOAT16 ? occ_bf16 : occ_f16);
  lp->chunk_tiles = partition_tokens / pa::TILE;
  if (lp->chunk_tiles == 0) {
    lp->max_chunks = ws_warps * (1 + tail_chunks(group)) + 1;
  } else {
    const long long per_seq = ((long long)max_context_len + pa::TILE - 1) / pa::TILE;
    const long long total = (long long)num_seqs * num_kv_heads * (group / G) * per_seq;
    lp->max_chunks = std::max(1LL, (total + lp->chunk_tiles - 1) / lp->chunk_tiles);
  }
  lp->queue_bytes = 256;
  lp->tiles_bytes = (((size_t)num_seqs + 1) * sizeof(int) + 255) / 256 * 256;
  lp->ml_bytes = (size_t)lp->max_chunks * 2 * G * sizeof(float2);
  lp->acc_bytes = (size_t)lp->max_chunks * 2 * G * head_dim * sizeof(float);
  lp->total_bytes = lp->queue_bytes + lp->tiles_bytes + lp->ml_bytes + lp->acc_bytes;
  return PA_OK;
}

// ---- TMA tensor maps of the caches, with the 128-byte swizzle.  2-D (prefill): the cache viewed as
// [num_blocks * num_kv_heads * block_size rows][head_dim], boxes of 16 rows x 64 elements (128 bytes).
// 3-D (decode): the same rows with each row's 64-element halves as a third dimension 128 bytes apart, so
// that one box brings a whole 16-row tile stored as [halves][16 rows][128 bytes]: one copy per K or V
// tile instead of one per half (measured: 43.0 against 44.7 us per call on the shared-prefix step).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder(int *rc) {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!fn) {
    t_last_cuda_error = err != cudaSuccess ? cudaGetErrorString(err) : "cuTensorMapEncodeTiled not available";
    *rc = PA_ERR_CUDA;
  }
  return fn;
}

struct MapKey {
  int dev;
  const void *base;
  long long rows;
  int head_dim, dtype;
  bool three_d;
  bool operator==(const MapKey &o) const {
    return dev == o.dev && base == o.base && rows == o.rows && head_dim == o.head_dim && dtype == o.dtype &&
           three_d == o.three_d;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool used;
};
MapEntry g_maps[32];
int g_map_next = 0;

int cache_tensor_map(const void *base, long long rows, int head_dim, int dtype, bool three_d, CUtensorMap *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record(e);
  const MapKey key{dev, base, rows, head_dim, dtype, three_d};
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto &m : g_maps)
    if (m.used && m.key == key) {
      *out = m.map;
      return PA_OK;
    }
  int rc = PA_OK;
  auto encode = tensor_map_encoder(&rc);
  if (!encode) return rc;
  CUtensorMap map;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3];
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  cuuint32_t rank;
  if (three_d) {
    // [halves][rows][64 elements]: x = element in a half, y = row (head_dim * 2 bytes apart), z = half
    // (128 bytes apart); one box covers a 16-row tile of both halves
    dims[0] = 64, dims[1] = (cuuint64_t)rows, dims[2] = (cuuint64_t)head_dim / 64;
    strides[0] = (cuuint64_t)head_dim * 2, strides[1] = 128;
    box[0] = 64, box[1] = (cuuint32_t)pa::TILE, box[2] = (cuuint32_t)head_dim / 64;
    rank = 3;
  } else {
    dims[0] = (cuuint64_t)head_dim, dims[1] = (cuuint64_t)rows;
    strides[0] = (cuuint64_t)head_dim * 2;
    box[0] = 64, box[1] = (cuuint32_t)pa::TILE;
    rank = 2;
  }
  const CUresult r =
      encode(&map, dtype == PA_BFLOAT16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, rank,
             const_cast<void *>(base), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")";
    return PA_ERR_CUDA;
  }
  g_maps[g_map_next] = MapEntry{key, map, true};
  g_map_next = (g_map_next + 1) % 32;
  *out = map;
  return PA_OK;
}

template <class E, int D>
int launch_decode_d(const pa::DecodeArgs &args, const LaunchPlan &lp, int dtype, cudaStream_t stream) {
  const int threads = kWarps * 32;
  if (lp.segment_mode) {
    cudaError_t e = args.heads_per_unit == 2
                        ? launch_pdl(pa::decode_segment_kernel<E, D, 2, kWarps, kStages>, dim3(lp.grid),
                                     dim3(threads), lp.smem, stream, args)
                        : launch_pdl(pa::decode_segment_kernel<E, D, 1, kWarps, kStages>, dim3(lp.grid),
                                     dim3(threads), lp.smem, stream, args);
    if (e != cudaSuccess) return record(e);
    e = cudaGetLastError();
    if (e != cudaSuccess) return record(e);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PA_OK;
  }
  if (uses_mma(args.group)) {
    const long long rows = args.num_blocks * args.num_kv_heads * args.block_size;
    if (rows > 0x7fffffffLL) return PA_ERR_SHAPE;  // TMA coordinates are signed 32-bit
    CUtensorMap mk, mv;
    int rc = cache_tensor_map(args.k_cache, rows, D, dtype, true, &mk);
    if (rc != PA_OK) return rc;
    rc = cache_tensor_map(args.v_cache, rows, D, dtype, true, &mv);
    if (rc != PA_OK) return rc;
    cudaError_t e = launch_pdl(pa::decode_split_mma_kernel<E, D, kWarps, kStages>, dim3(lp.grid), dim3(threads),
                               lp.smem, stream, mk, mv, args);
    if (e != cudaSuccess) return record(e);
  } else if (args.heads_per_unit == 2) {
    cudaError_t e = launch_pdl(pa::decode_split_kernel<E, D, 2, kWarps, kStages>, dim3(lp.grid), dim3(threads),
                               lp.smem, stream, args);
    if (e != cudaSuccess) return record(e);
  } else {
    cudaError_t e = launch_pdl(pa::decode_split_kernel<E, D, 1, kWarps, kStages>, dim3(lp.grid), dim3(threads),
                               lp.smem, stream, args);
    if (e != cudaSuccess) return record(e);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  // merge: on the tensor-core path (segments of 3 to 8 heads) one warp per two query heads of a segment (one
  // per head for an odd group); on the CUDA-core path one warp per segment (1 or 2 heads); eight warps per
  // block.  Two heads per warp halve the grid, so more of it is resident on the SMs that finish the split
  // early instead of being scheduled after the split drains: 41.0 against 42.2 us on the shared-prefix step,
  // 165.8 against 166.2 on the 32 query / 8 kv head batch; four heads per warp (158 registers) lost on the
  // latter.  Measured and dropped: merging in the tensor-core split kernel itself (the warp that stores a
  // segment's last cut piece merges it, counted through per-segment arrival words): 179 against 167 us on
  // the 32 query / 8 kv head batch and 62 against 43 us on the shared-prefix step -- the merges then run one
  // after another at the end of each warp's stream instead of in parallel across the merge grid.
  const int hw = uses_mma(args.group) ? (args.heads_per_unit % 2 == 0 ? 2 : 1) : args.heads_per_unit;
  const long long warps = (long long)args.num_seqs * args.num_kv_heads * args.n_chunks * (args.heads_per_unit / hw);
  const dim3 mgrid((unsigned)((warps + 7) / 8)), mblock(256);
  if (!uses_mma(args.group))
    e = hw == 2 ? launch_pdl(pa::decode_merge_kernel<E, D, 2, 8>, mgrid, mblock, 0, stream, args)
                : launch_pdl(pa::decode_merge_kernel<E, D, 1, 16>, mgrid, mblock, 0, stream, args);
  else if (hw == 2)
    e = launch_pdl(pa::decode_merge_kernel<E, D, 2, 4>, mgrid, mblock, 0, stream, args);
  else
    e = launch_pdl(pa::decode_merge_kernel<E, D, 1, 4>, mgrid, mblock, 0, stream, args);
  if (e != cudaSuccess) return record(e);
  e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

// Workspace of a cascade plan: per kv head, rows_per_head softmax states (m, l) and partial rows acc[D].
size_t cascade_ml_bytes(const pa_cascade_info &in) {
  return ((size_t)in.num_kv_heads * (size_t)in.rows_per_head * sizeof(float2) + 255) / 256 * 256;
}
size_t cascade_ws_bytes(const pa_cascade_info &in, int head_dim) {
  return std::max<size_t>(256, cascade_ml_bytes(in) + (size_t)in.num_kv_heads * (size_t)in.rows_per_head *
                                                          (size_t)head_dim * sizeof(float));
}

static_assert(pa::CASCADE_CONSUMERS == kWarps, "blocks_per_sm sizes the cascade blocks with kWarps warps");

template <class E, int D>
int launch_cascade_d(const pa::CascadeArgs &a, const void *k_cache, const void *v_cache, int dtype,
                     cudaStream_t stream) {
  if (a.num_jobs > 0) {
    const long long rows = a.num_blocks * a.num_kv_heads * a.block_size;
    if (rows > 0x7fffffffLL) return PA_ERR_SHAPE;  // TMA coordinates are signed 32-bit
    CUtensorMap mk, mv;
    int rc = cache_tensor_map(k_cache, rows, D, dtype, true, &mk);
    if (rc != PA_OK) return rc;
    rc = cache_tensor_map(v_cache, rows, D, dtype, true, &mv);
    if (rc != PA_OK) return rc;
    // one block per prefix job, one per CASCADE_CONSUMERS suffix jobs
    const long long blocks = a.num_prefix_jobs + ((long long)(a.num_jobs - a.num_prefix_jobs) + pa::CASCADE_CONSUMERS - 1) /
                                                     pa::CASCADE_CONSUMERS;
    int per_sm = 0;
    rc = blocks_per_sm(reinterpret_cast<const void *>(pa::cascade_partial_kernel<E, D>), pa::CascadeSmem<D>::bytes(),
                       &per_sm);  // also allows the kernel its shared memory above the default 48 KB
    if (rc != PA_OK) return rc;
    cudaError_t e = launch_pdl(pa::cascade_partial_kernel<E, D>, dim3((unsigned)blocks, (unsigned)a.num_kv_heads),
                               dim3(pa::CASCADE_CONSUMERS * 32), pa::CascadeSmem<D>::bytes(), stream, mk, mv, a);
    if (e != cudaSuccess) return record(e);
    e = cudaGetLastError();
    if (e != cudaSuccess) return record(e);
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  const long long warps = (long long)a.num_seqs * a.num_q_heads;
  cudaError_t e = launch_pdl(pa::cascade_combine_kernel<E, D>, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0,
                             stream, a);
  if (e != cudaSuccess) return record(e);
  e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

// Fixed scratch behind pa_decode_static_workspace, for callers that cannot
// allocate.  In host code this name is only a stand-in for the device
// variable: the kernels are given the address cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];
void *g_static_workspace_addr[kMaxDevices] = {};

// Device address of g_static_workspace on the current device, looked up on
// the first call for that device (with that device current) and cached.
int static_workspace_address(void **addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record(e);
  if (dev < 0 || dev >= kMaxDevices) {
    t_last_cuda_error = "device ordinal beyond the library's table";
    return PA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_workspace_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return record(e);
    g_static_workspace_addr[dev] = p;
  }
  *addr = g_static_workspace_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" {

int pa_write_kv(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int64_t num_blocks,
                int64_t k_token_stride, int64_t v_token_stride, int32_t dtype, void *stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_ERR_SHAPE;
  if (dtype != PA_FLOAT16 && dtype != PA_BFLOAT16) return PA_ERR_DTYPE;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_NULL;
  if (k_token_stride < (int64_t)num_kv_heads * head_dim || v_token_stride < (int64_t)num_kv_heads * head_dim)
    return PA_ERR_SHAPE;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) || (k_token_stride % 8) ||
      (v_token_stride % 8))
    return PA_ERR_ALIGN;
  int sms = 0;
  int rc = current_sms(&sms);
  if (rc != PA_OK) return rc;
  pa::WriteArgs a;
  a.k = static_cast<const uint16_t *>(k);
  a.v = static_cast<const uint16_t *>(v);
  a.k_cache = static_cast<uint16_t *>(k_cache);
  a.v_cache = static_cast<uint16_t *>(v_cache);
  a.slot_mapping = slot_mapping;
  a.num_tokens = num_tokens;
  a.num_blocks = num_blocks;
  a.k_token_stride = k_token_stride;
  a.v_token_stride = v_token_stride;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  const long long chunks = 2LL * num_tokens * num_kv_heads * (head_dim / 8);
  const int grid = (int)std::max(1LL, std::min<long long>((chunks + 255) / 256, (long long)sms * 8));
  cudaError_t e = launch_pdl(pa::write_kv_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), a);
  if (e != cudaSuccess) return record(e);
  e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_context_len, int32_t partition_tokens) {
  if (check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len) != PA_OK)
    return 0;
  LaunchPlan lp;
  if (plan_decode(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_tokens, 0, &lp) != PA_OK)
    return 0;
  return lp.total_bytes;
}

int pa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
              const int32_t *context_lens, float scale, void *out, int32_t num_seqs, int32_t num_q_heads,
              int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int64_t num_blocks,
              int32_t block_table_stride, int32_t max_context_len, int64_t q_seq_stride, int64_t out_seq_stride,
              int32_t partition_tokens, int32_t dtype, void *workspace, size_t workspace_bytes, void *stream) {
  int rc = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len);
  if (rc != PA_OK) return rc;
  if (dtype != PA_FLOAT16 && dtype != PA_BFLOAT16) return PA_ERR_DTYPE;
  if (num_blocks <= 0 || block_table_stride <= 0) return PA_ERR_SHAPE;
  const int64_t row = (int64_t)num_q_heads * head_dim;
  if (q_seq_stride < row || out_seq_stride < row) return PA_ERR_SHAPE;
  if (partition_tokens < 0 || partition_tokens % pa::TILE != 0) return PA_ERR_PARTITION;
  if (num_seqs == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || (q_seq_stride % 8) ||
      (out_seq_stride % 8))
    return PA_ERR_ALIGN;
  if (!std::isfinite(scale)) return PA_ERR_SHAPE;
  LaunchPlan lp;
  rc = plan_decode(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_tokens, dtype, &lp);
  if (rc != PA_OK) return rc;
  if (lp.total_bytes > 0 && (!workspace || workspace_bytes < lp.total_bytes || !aligned16(workspace)))
    return PA_ERR_WORKSPACE;

  const int group = num_q_heads / num_kv_heads;
  const int G = heads_per_unit(group);
  char *ws = static_cast<char *>(workspace);
  pa::DecodeArgs a;
  a.q = static_cast<const uint16_t *>(q);
  a.k_cache = static_cast<const uint16_t *>(k_cache);
  a.v_cache = static_cast<const uint16_t *>(v_cache);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.out = static_cast<uint16_t *>(out);
  if (lp.segment_mode) {  // no workspace
    a.ws_queue = nullptr;
    a.ws_tiles = nullptr;
    a.ws_ml = nullptr;
    a.ws_acc = nullptr;
  } else {
    a.ws_queue = reinterpret_cast<unsigned long long *>(ws);
    a.ws_tiles = reinterpret_cast<int *>(ws + lp.queue_bytes);
    a.ws_ml = reinterpret_cast<float2 *>(ws + lp.queue_bytes + lp.tiles_bytes);
    a.ws_acc = reinterpret_cast<float *>(ws + lp.queue_bytes + lp.tiles_bytes + lp.ml_bytes);
  }
  a.num_blocks = num_blocks;
  a.q_seq_stride = q_seq_stride;
  a.out_seq_stride = out_seq_stride;
  a.max_chunks = lp.max_chunks;
  a.wait_limit_ns = kWaitLimitNs;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);  // log2(e)
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.table_stride = block_table_stride;
  a.max_context_len = max_context_len;
  a.group = group;
  a.heads_per_unit = G;
  a.n_chunks = group / G;
  a.chunk_tiles = lp.chunk_tiles;
  a.split_warps = lp.grid * kWarps;
  a.static_permille = static_permille(group);
  a.tail_chunks_per_warp = tail_chunks(group);
  a.epoch = next_epoch();

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == PA_BFLOAT16;
  if (head_dim == 128)
    return bf16 ? launch_decode_d<pa::BF16, 128>(a, lp, dtype, st) : launch_decode_d<pa::F16, 128>(a, lp, dtype, st);
  return bf16 ? launch_decode_d<pa::BF16, 64>(a, lp, dtype, st) : launch_decode_d<pa::F16, 64>(a, lp, dtype, st);
}

size_t pa_cascade_workspace_size(const pa_cascade_info *info, int32_t head_dim) {
  if (!info || (head_dim != 64 && head_dim != 128) || info->num_kv_heads <= 0 || info->rows_per_head < 0) return 0;
  return cascade_ws_bytes(*info, head_dim);
}

int pa_decode_cascade(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                      const int32_t *context_lens, float scale, void *out, int32_t head_dim, int64_t num_blocks,
                      int32_t block_table_stride, int64_t q_seq_stride, int64_t out_seq_stride, int32_t dtype,
                      const int32_t *plan, const pa_cascade_info *info, void *workspace, size_t workspace_bytes,
                      void *stream) {
  if (!info) return PA_ERR_NULL;
  const pa_cascade_info in = *info;
  int rc = check_decode_shape(in.num_seqs, in.num_q_heads, in.num_kv_heads, head_dim, in.block_size,
                              in.max_context_len);
  if (rc != PA_OK) return rc;
  if (in.num_q_heads / in.num_kv_heads > 8) return PA_ERR_UNSUPPORTED;
  if (dtype != PA_FLOAT16 && dtype != PA_BFLOAT16) return PA_ERR_DTYPE;
  if (num_blocks <= 0 || block_table_stride <= 0) return PA_ERR_SHAPE;
  const int64_t row = (int64_t)in.num_q_heads * head_dim;
  if (q_seq_stride < row || out_seq_stride < row) return PA_ERR_SHAPE;
  if (in.num_jobs < 0 || in.num_prefix_jobs < 0 || in.num_prefix_jobs > in.num_jobs || in.num_members < 0 || in.num_pieces < 0 || in.rows_per_head < 0 ||
      in.plan_ints != (int64_t)in.num_jobs * pa::CJ_INTS + in.num_members + in.num_seqs + 1 + in.num_pieces)
    return PA_ERR_SHAPE;
  if (in.num_seqs == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out || !plan) return PA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || (q_seq_stride % 8) ||
      (out_seq_stride % 8))
    return PA_ERR_ALIGN;
  if (!std::isfinite(scale)) return PA_ERR_SHAPE;
  if (!workspace || workspace_bytes < cascade_ws_bytes(in, head_dim) || !aligned16(workspace)) return PA_ERR_WORKSPACE;

  pa::CascadeArgs a;
  a.q = static_cast<const uint16_t *>(q);
  a.out = static_cast<uint16_t *>(out);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.jobs = plan;
  a.members = plan + (int64_t)in.num_jobs * pa::CJ_INTS;
  a.piece_offsets = a.members + in.num_members;
  a.piece_rows = a.piece_offsets + in.num_seqs + 1;
  a.ws_ml = reinterpret_cast<float2 *>(workspace);
  a.ws_acc = reinterpret_cast<float *>(static_cast<char *>(workspace) + cascade_ml_bytes(in));
  a.q_seq_stride = q_seq_stride;
  a.out_seq_stride = out_seq_stride;
  a.num_blocks = num_blocks;
  a.wait_limit_ns = kWaitLimitNs;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);  // log2(e)
  a.num_seqs = in.num_seqs;
  a.num_q_heads = in.num_q_heads;
  a.num_kv_heads = in.num_kv_heads;
  a.block_size = in.block_size;
  a.table_stride = block_table_stride;
  a.max_context_len = in.max_context_len;
  a.group = in.num_q_heads / in.num_kv_heads;
  a.num_jobs = in.num_jobs;
  a.num_prefix_jobs = in.num_prefix_jobs;
  a.num_members = in.num_members;
  a.num_pieces = in.num_pieces;
  a.rows_per_head = in.rows_per_head;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PA_BFLOAT16)
    return head_dim == 128 ? launch_cascade_d<pa::BF16, 128>(a, k_cache, v_cache, dtype, st)
                           : launch_cascade_d<pa::BF16, 64>(a, k_cache, v_cache, dtype, st);
  return head_dim == 128 ? launch_cascade_d<pa::F16, 128>(a, k_cache, v_cache, dtype, st)
                         : launch_cascade_d<pa::F16, 64>(a, k_cache, v_cache, dtype, st);
}

int pa_get_device_status(uint32_t *status_out, int32_t clear, void *stream) {
  if (!status_out) return PA_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return record(e);
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, pa::g_status, sizeof v);
  if (e != cudaSuccess) return record(e);
  if (clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(pa::g_status, &zero, sizeof zero);
    if (e != cudaSuccess) return record(e);
  }
  *status_out = v;
  return PA_OK;
}

const char *pa_status_string(int32_t status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_NULL: return "a required pointer is NULL";
    case PA_ERR_DTYPE: return "dtype must be PA_FLOAT16 or PA_BFLOAT16";
    case PA_ERR_SHAPE: return "a size or stride is negative or inconsistent";
    case PA_ERR_ALIGN: return "a pointer is not 16-byte aligned or a stride is not a multiple of 8 elements";
    case PA_ERR_UNSUPPORTED: return "head_dim must be 64 or 128 and block_size 16 or 32";
    case PA_ERR_HEADS: return "num_q_heads must be a multiple of num_kv_heads";
    case PA_ERR_WORKSPACE: return "workspace missing, smaller than pa_decode_workspace_size() or misaligned";
    case PA_ERR_PARTITION: return "partition_tokens must be 0 or a positive multiple of 16";
    case PA_ERR_CUDA: return "a CUDA runtime call failed (see pa_last_cuda_error)";
    case PA_ERR_ADDRESS: return "a pointer is neither this device's memory nor mapped pinned host memory";
    case PA_ERR_STATIC_WORKSPACE:
      return "the problem needs more split-context scratch than the library's fixed 32 MiB array; "
             "use pa_decode with a caller workspace or a larger partition_tokens";
    default: return "unknown status";
  }
}

const char *pa_last_cuda_error(void) { return t_last_cuda_error.c_str(); }

uint64_t pa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int pa_debug_wait_timeout(int64_t limit_ns, void *stream) {
  const unsigned long long lim = (unsigned long long)std::min<int64_t>(std::max<int64_t>(limit_ns, 1000), 1000000000);
  pa::wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(lim);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

int pa_decode_static_workspace(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_tables, const int32_t *context_lens, float scale, void *out,
                               int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                               int32_t block_size, int64_t num_blocks, int32_t block_table_stride,
                               int32_t max_context_len, int64_t q_seq_stride, int64_t out_seq_stride,
                               int32_t partition_tokens, int32_t dtype, void *stream) {
  int rc = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len);
  if (rc != PA_OK) return rc;
  if (num_seqs > 0) {  // an empty batch needs no scratch and launches nothing
    const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                 max_context_len, partition_tokens);
    if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_STATIC_WORKSPACE;
  }
  void *scratch = nullptr;
  rc = static_workspace_address(&scratch);
  if (rc != PA_OK) return rc;
  return pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out, num_seqs, num_q_heads, num_kv_heads,
                   head_dim, block_size, num_blocks, block_table_stride, max_context_len, q_seq_stride,
                   out_seq_stride, partition_tokens, dtype, scratch, PA_STATIC_WORKSPACE_BYTES, stream);
}

int pa_swap_blocks(const void *src_k, const void *src_v, void *dst_k, void *dst_v, const int64_t *block_mapping,
                   int64_t num_pairs, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                   int64_t src_num_blocks, int64_t dst_num_blocks, void *stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || src_num_blocks <= 0 || dst_num_blocks <= 0) return PA_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!src_k || !src_v || !dst_k || !dst_v || !block_mapping) return PA_ERR_NULL;
  if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v) ||
      (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
    return PA_ERR_ALIGN;
  const void *view[5];
  const void *ptrs[5] = {src_k, src_v, dst_k, dst_v, block_mapping};
  for (int i = 0; i < 5; ++i) {
    const int rc = device_view(ptrs[i], &view[i]);
    if (rc != PA_OK) return rc;
  }
  int sms = 0;
  int rc = current_sms(&sms);
  if (rc != PA_OK) return rc;
  pa::CopyArgs a;
  a.src_k = static_cast<const uint4 *>(view[0]);
  a.src_v = static_cast<const uint4 *>(view[1]);
  a.dst_k = static_cast<uint4 *>(const_cast<void *>(view[2]));
  a.dst_v = static_cast<uint4 *>(const_cast<void *>(view[3]));
  a.mapping = static_cast<const int64_t *>(view[4]);
  a.num_pairs = num_pairs;
  a.chunks_per_block = (long long)num_kv_heads * block_size * head_dim * 2 / 16;
  a.src_blocks = src_num_blocks;
  a.dst_blocks = dst_num_blocks;
  const long long warp_tiles = num_pairs * 2 * ((a.chunks_per_block + pa::COPY_TILE - 1) / pa::COPY_TILE);
  const int grid = (int)std::max(1LL, std::min<long long>((warp_tiles + 7) / 8, (long long)sms * 8));
  cudaError_t e = launch_pdl(pa::copy_blocks_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream), a);
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int64_t num_pairs,
                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int64_t num_blocks, void *stream) {
  return pa_swap_blocks(k_cache, v_cache, k_cache, v_cache, block_mapping, num_pairs, num_kv_heads, head_dim,
                        block_size, num_blocks, num_blocks, stream);
}

// Work counters of pa_prefill calls: a call takes the next of 64 slots and zeroes it on its own stream
// before the launch, so calls in flight on different streams (up to 64) never share a counter.
static __device__ unsigned int g_prefill_queue[64];
void *g_prefill_queue_addr[kMaxDevices] = {};
std::atomic<uint32_t> g_prefill_slot{0};

int prefill_queue_slot(unsigned int **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record(e);
  if (dev < 0 || dev >= kMaxDevices) {
    t_last_cuda_error = "device ordinal beyond the library's table";
    return PA_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_prefill_queue_addr[dev]) {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_prefill_queue);
      if (e != cudaSuccess) return record(e);
      g_prefill_queue_addr[dev] = p;
    }
  }
  *out = static_cast<unsigned int *>(g_prefill_queue_addr[dev]) + g_prefill_slot.fetch_add(1) % 64;
  return PA_OK;
}

int pa_prefill(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
               const int32_t *query_start, const int32_t *context_lens, float scale, void *out, int32_t num_seqs,
               int64_t num_query_tokens, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
               int32_t block_size, int64_t num_blocks, int32_t block_table_stride, int32_t max_query_len,
               int64_t q_token_stride, int64_t out_token_stride, int32_t dtype, void *stream) {
  if (num_seqs < 0 || num_query_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_query_len < 0 ||
      num_blocks < 0 || block_table_stride < 0)
    return PA_ERR_SHAPE;
  if (num_seqs > 65535 || num_q_heads > 65535 || num_query_tokens > 0x7fffffffLL) return PA_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_HEADS;
  if (dtype != PA_FLOAT16 && dtype != PA_BFLOAT16) return PA_ERR_DTYPE;
  if (!std::isfinite(scale)) return PA_ERR_SHAPE;
  if (num_seqs == 0 || num_query_tokens == 0 || max_query_len == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !query_start || !context_lens || !out) return PA_ERR_NULL;
  if (q_token_stride < (long long)num_q_heads * head_dim || out_token_stride < (long long)num_q_heads * head_dim)
    return PA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || (q_token_stride % 8) ||
      (out_token_stride % 8))
    return PA_ERR_ALIGN;
  const long long rows = num_blocks * num_kv_heads * block_size;
  if (rows > 0x7fffffffLL || rows == 0) return PA_ERR_SHAPE;  // TMA coordinates are signed 32-bit
  int rc = PA_OK;
  auto encode = tensor_map_encoder(&rc);
  if (!encode) return rc;
  CUtensorMap mq, mk, mv;
  {
    // q viewed as [tokens][heads][head_dim]; one box = 128 tokens x 64 dims of one head
    const cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads, (cuuint64_t)num_query_tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)q_token_stride * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)pa::PF_BM};
    const cuuint32_t elem_strides[3] = {1, 1, 1};
    const CUresult r =
        encode(&mq, dtype == PA_BFLOAT16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
               const_cast<void *>(q), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
      t_last_cuda_error = "cuTensorMapEncodeTiled failed for q (code " + std::to_string((int)r) + ")";
      return PA_ERR_CUDA;
    }
  }
  rc = cache_tensor_map(k_cache, rows, head_dim, dtype, false, &mk);
  if (rc != PA_OK) return rc;
  rc = cache_tensor_map(v_cache, rows, head_dim, dtype, false, &mv);
  if (rc != PA_OK) return rc;

  pa::PrefillArgs a;
  a.block_tables = block_tables;
  a.query_start = query_start;
  a.context_lens = context_lens;
  a.out = static_cast<uint16_t *>(out);
  a.num_blocks = num_blocks;
  a.out_token_stride = out_token_stride;
  a.num_query_tokens = num_query_tokens;
  a.wait_limit_ns = kWaitLimitNs;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);  // log2(e)
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.table_stride = block_table_stride;
  a.q_tiles = (max_query_len + pa::PF_ROWS - 1) / pa::PF_ROWS;
  a.num_items = (long long)a.q_tiles * num_q_heads * num_seqs;
  int sms = 0;
  rc = current_sms(&sms);
  if (rc != PA_OK) return rc;
  // persistent: one CTA per SM (the shared-memory footprint admits no second one)
  const dim3 grid((unsigned)std::min<long long>(a.num_items, sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (a.num_items > 0xffffffffLL) return PA_ERR_SHAPE;
  rc = prefill_queue_slot(&a.queue);
  if (rc != PA_OK) return rc;
  cudaError_t me = cudaMemsetAsync(a.queue, 0, sizeof(unsigned int), st);
  if (me != cudaSuccess) return record(me);
  auto launch = [&](auto kernel, uint32_t smem) -> int {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return record(e);
    e = launch_pdl(kernel, grid, dim3(pa::PF_THREADS), smem, st, mq, mk, mv, a);
    if (e != cudaSuccess) return record(e);
    e = cudaGetLastError();
    if (e != cudaSuccess) return record(e);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return PA_OK;
  };
  if (dtype == PA_BFLOAT16) {
    if (head_dim == 128) return launch(pa::prefill_tc_kernel<pa::BF16, 128>, pa::PrefillSmem<128>::ALLOC);
    return launch(pa::prefill_tc_kernel<pa::BF16, 64>, pa::PrefillSmem<64>::ALLOC);
  }
  if (head_dim == 128) return launch(pa::prefill_tc_kernel<pa::F16, 128>, pa::PrefillSmem<128>::ALLOC);
  return launch(pa::prefill_tc_kernel<pa::F16, 64>, pa::PrefillSmem<64>::ALLOC);
}

int pa_read_bandwidth_probe(const void *src, int64_t bytes, uint32_t *sink, void *stream) {
  if (bytes < 0) return PA_ERR_SHAPE;
  if (bytes == 0) return PA_OK;
  if (!src || !sink) return PA_ERR_NULL;
  if (!aligned16(src) || (bytes % 16) || (reinterpret_cast<uintptr_t>(sink) & 3u)) return PA_ERR_ALIGN;
  int sms = 0;
  int rc = current_sms(&sms);
  if (rc != PA_OK) return rc;
  // four blocks of 512 threads fill an SM's 2048 thread slots
  const long long n16 = bytes / 16;
  const long long want = (n16 + pa::STREAM_THREADS - 1) / pa::STREAM_THREADS;
  const int grid = (int)std::max(1LL, std::min<long long>(want, (long long)sms * 4));
  pa::stream_read_kernel<<<grid, pa::STREAM_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(src), n16, reinterpret_cast<unsigned int *>(sink));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

uint32_t pa_build_flags(void) { return pa::kDebugChecks ? PA_BUILD_DEBUG : 0u; }

int32_t pa_version(void) { return 100; }

}  // extern "C"
