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

#include "pa_b200.h"
#include "pa_kernels.cuh"

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

// Query heads handled together by one work unit: the largest of 4, 2, 1
// dividing the group size (a unit reads its K/V tiles once for all of them).
int heads_per_unit(int group) { return (group % 4 == 0) ? 4 : (group % 2 == 0) ? 2 : 1; }

// Per-head-dim launch shape of the partition kernel.
template <int D>
struct Shape;
template <>
struct Shape<128> {
  static constexpr int WARPS = 4, STAGES = 3;
};
template <>
struct Shape<64> {
  static constexpr int WARPS = 4, STAGES = 4;
};

template <int D>
constexpr int partition_smem() {
  return ((Shape<D>::WARPS * Shape<D>::STAGES * 8 + 127) / 128) * 128 +
         Shape<D>::WARPS * Shape<D>::STAGES * 2 * pa::TILE * D * 2;
}

int warps_per_sm_estimate(int head_dim) {
  // resident warps per SM that the shared-memory budget of the partition kernel allows
  const int smem = head_dim == 128 ? partition_smem<128>() : partition_smem<64>();
  const int warps = head_dim == 128 ? Shape<128>::WARPS : Shape<64>::WARPS;
  const int ctas = std::max(1, (227 * 1024) / (smem + 1024));
  return ctas * warps;
}

int resolve_partition(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                      int max_context_len, int requested, int sms) {
  if (requested != 0) {
    if (requested < 0 || requested % block_size != 0 || requested % pa::TILE != 0 || requested > 32 * block_size)
      return PA_ERR_PARTITION;
    return requested;
  }
  const int group = num_q_heads / num_kv_heads;
  const long long base_units = (long long)num_seqs * num_kv_heads * (group / heads_per_unit(group));
  const long long want = 2LL * sms * warps_per_sm_estimate(head_dim);
  const int cap = 32 * block_size;
  const int ctx = std::max(max_context_len, 1);
  int part = cap;
  // shrink until the (rough) number of units fills the GPU twice over; a
  // context that fits one partition is never split
  while (part > 2 * pa::TILE && part > block_size) {
    const long long mean_parts = std::max(1LL, ((long long)ctx / 2 + part - 1) / part);
    if (base_units * mean_parts >= want) break;
    part /= 2;
  }
  const int fit = ((ctx + block_size - 1) / block_size) * block_size;
  if (fit <= cap && fit <= part) part = std::max(fit, pa::TILE);
  if (part % block_size) part = ((part + block_size - 1) / block_size) * block_size;
  return part;
}

size_t workspace_bytes_for(int num_seqs, int num_q_heads, int head_dim, int max_context_len, int part) {
  const long long n_part_max = std::max(1LL, ((long long)max_context_len + part - 1) / part);
  if (n_part_max <= 1) return 0;
  const size_t rows = (size_t)num_seqs * num_q_heads * n_part_max;
  return rows * head_dim * sizeof(float) + rows * sizeof(float2);
}

int check_decode_shape(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                       int32_t block_size, int32_t max_context_len) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0) return PA_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_HEADS;
  return PA_OK;
}

template <class E, int D, int G>
int launch_partition(const pa::DecodeArgs &args, int sms, cudaStream_t stream) {
  constexpr int WARPS = Shape<D>::WARPS, STAGES = Shape<D>::STAGES;
  constexpr int SMEM = partition_smem<D>();
  auto kernel = pa::decode_partition_kernel<E, D, G, WARPS, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return record(e);
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, WARPS * 32, SMEM);
  if (e != cudaSuccess) return record(e);
  per_sm = std::max(per_sm, 1);
  const long long need = (args.n_slots + WARPS - 1) / WARPS;
  const int grid = (int)std::max(1LL, std::min<long long>((long long)sms * per_sm, need));
  kernel<<<grid, WARPS * 32, SMEM, stream>>>(args);
  e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

template <class E, int D>
int launch_decode_d(const pa::DecodeArgs &args, int G, int sms, cudaStream_t stream) {
  int rc;
  switch (G) {
    case 4: rc = launch_partition<E, D, 4>(args, sms, stream); break;
    case 2: rc = launch_partition<E, D, 2>(args, sms, stream); break;
    default: rc = launch_partition<E, D, 1>(args, sms, stream); break;
  }
  if (rc != PA_OK || args.n_part_max <= 1) return rc;
  const long long warps = (long long)args.num_seqs * args.num_q_heads;
  const int grid = (int)std::max(1LL, std::min<long long>((warps + 7) / 8, (long long)sms * 8));
  pa::decode_reduce_kernel<E, D><<<grid, 256, 0, stream>>>(args);
  cudaError_t e = cudaGetLastError();
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
  pa::write_kv_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record(e);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return PA_OK;
}

int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   int32_t block_size, int32_t max_context_len) {
  int rc = check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len);
  if (rc != PA_OK) return rc;
  int sms = 0;
  rc = current_sms(&sms);
  if (rc != PA_OK) return rc;
  return resolve_partition(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, 0, sms);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_context_len, int32_t partition_tokens) {
  if (check_decode_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len) != PA_OK)
    return 0;
  int part = partition_tokens;
  if (part == 0) {
    int sms = 0;
    if (current_sms(&sms) != PA_OK) return 0;
    part = resolve_partition(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, 0, sms);
  } else if (resolve_partition(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, part,
                               1) < 0) {
    return 0;
  }
  return workspace_bytes_for(num_seqs, num_q_heads, head_dim, max_context_len, part);
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
  if (num_seqs == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || (q_seq_stride % 8) ||
      (out_seq_stride % 8))
    return PA_ERR_ALIGN;
  if (!std::isfinite(scale)) return PA_ERR_SHAPE;
  int sms = 0;
  rc = current_sms(&sms);
  if (rc != PA_OK) return rc;
  const int part = resolve_partition(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                     partition_tokens, sms);
  if (part < 0) return part;
  const int n_part_max = (int)std::max(1LL, ((long long)max_context_len + part - 1) / part);
  const size_t need = workspace_bytes_for(num_seqs, num_q_heads, head_dim, max_context_len, part);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PA_ERR_WORKSPACE;

  const int group = num_q_heads / num_kv_heads;
  const int G = heads_per_unit(group);
  pa::DecodeArgs a;
  a.q = static_cast<const uint16_t *>(q);
  a.k_cache = static_cast<const uint16_t *>(k_cache);
  a.v_cache = static_cast<const uint16_t *>(v_cache);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.out = static_cast<uint16_t *>(out);
  a.ws_acc = need ? static_cast<float *>(workspace) : nullptr;
  a.ws_ml = need ? reinterpret_cast<float2 *>(static_cast<char *>(workspace) +
                                              (size_t)num_seqs * num_q_heads * n_part_max * head_dim * sizeof(float))
                 : nullptr;
  a.num_blocks = num_blocks;
  a.q_seq_stride = q_seq_stride;
  a.out_seq_stride = out_seq_stride;
  a.wait_limit_ns = kWaitLimitNs;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);  // log2(e)
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.table_stride = block_table_stride;
  a.max_context_len = max_context_len;
  a.part_tokens = part;
  a.n_part_max = n_part_max;
  a.group = group;
  a.n_chunks = group / G;
  a.n_slots = (long long)n_part_max * num_seqs * num_kv_heads * a.n_chunks;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == PA_BFLOAT16;
  if (head_dim == 128)
    return bf16 ? launch_decode_d<pa::BF16, 128>(a, G, sms, st) : launch_decode_d<pa::F16, 128>(a, G, sms, st);
  return bf16 ? launch_decode_d<pa::BF16, 64>(a, G, sms, st) : launch_decode_d<pa::F16, 64>(a, G, sms, st);
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
    case PA_ERR_PARTITION: return "partition_tokens must be a multiple of block_size and of 16, at most 32 blocks";
    case PA_ERR_CUDA: return "a CUDA runtime call failed (see pa_last_cuda_error)";
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

int32_t pa_version(void) { return 100; }

}  // extern "C"
