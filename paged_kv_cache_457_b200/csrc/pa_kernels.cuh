// sm_100a kernels of the paged decode path.
//
//   write_kv_kernel        slot-mapped scatter of this step's new K/V rows
//                          ("4. vLLM核心机制" section 4.3, layout of 4.2).
//   decode_split_kernel    attention of one query token per sequence over the
//                          block-paged cache, reached through the per-sequence
//                          block table ("4. vLLM核心机制" 4.2; "vLLM：大型语言模型
//                          推理优化的革命性突破" 2.1), on the CUDA cores, over a
//                          balanced stream of 16-token tiles (the tensor-core
//                          variant for query groups of 3 to 8 heads is in
//                          pa_mma.cuh).
//   decode_segment_kernel  the same attention for small batches: one block per
//                          (sequence, head chunk), no workspace, no merge.
//   decode_merge_kernel    merges the partial softmax states of the segments
//                          that the split kernel cut across chunks.
//
// Cache layout: [num_blocks][num_kv_heads][block_size][head_dim], so the
// 16 consecutive tokens of one (block, kv head) form one contiguous tile of
// 16 * head_dim * 2 bytes (2 or 4 KiB), moved by a single bulk copy.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "pa_b200.h"
#include "pa_ptx.cuh"

namespace pa {

constexpr unsigned FULL = 0xffffffffu;
constexpr int TILE = 16;  // tokens per bulk-copied tile

// Device status word (one per device; see pa_get_device_status).
__device__ unsigned int g_status = 0;

// Index checks of the debug build (PA_DEBUG): dcheck(ok) flags PA_DEV_ERR_INTERNAL when ok is false and
// returns ok, so the caller skips the access.  In the release build it is the constant true and the
// checks compile away.
#ifdef PA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool dcheck(bool ok) {
  if constexpr (kDebugChecks) {
    if (!ok) atomicOr(&g_status, PA_DEV_ERR_INTERNAL);
    return ok;
  } else {
    return true;
  }
}

// ---------------------------------------------------------------- element types
__device__ __forceinline__ float dot8_f16(const uint32_t (&q)[4], const uint4 k, float c);
__device__ __forceinline__ float dot8_bf16(const uint32_t (&q)[4], const uint4 k, float c);

struct F16 {
  static __device__ __forceinline__ float dot8(const uint32_t (&q)[4], const uint4 k, float c) {
    return dot8_f16(q, k, c);
  }
  static __device__ __forceinline__ void widen8(const uint4 w, float (&f)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2 *>(&u[i]);
      const float2 t = __half22float2(h);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  static __device__ __forceinline__ uint32_t narrow2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
  }
};

struct BF16 {
  static __device__ __forceinline__ float dot8(const uint32_t (&q)[4], const uint4 k, float c) {
    return dot8_bf16(q, k, c);
  }
  static __device__ __forceinline__ void widen8(const uint4 w, float (&f)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(u[i] << 16);
      f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ uint32_t narrow2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
  }
};

template <class E>
__device__ __forceinline__ uint4 narrow8(const float (&f)[8]) {
  return make_uint4(E::narrow2(f[0], f[1]), E::narrow2(f[2], f[3]), E::narrow2(f[4], f[5]), E::narrow2(f[6], f[7]));
}

// ---------------------------------------------------------------- K1: KV write
struct WriteArgs {
  const uint16_t *k;
  const uint16_t *v;
  uint16_t *k_cache;
  uint16_t *v_cache;
  const int64_t *slot_mapping;
  long long num_tokens, num_blocks, k_token_stride, v_token_stride;
  int num_kv_heads, head_dim, block_size;
};

// One thread per 16-byte chunk of a (token, kv head) row, K rows then V rows.
__global__ void __launch_bounds__(256) write_kv_kernel(const WriteArgs a) {
  grid_dependency_wait();  // the new rows may come from the previous kernel in the stream
  grid_launch_dependents();
  const int cpr = a.head_dim / 8;
  const long long per = a.num_tokens * a.num_kv_heads * cpr;
  const long long cap = a.num_blocks * a.block_size;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * per;
       i += (long long)gridDim.x * blockDim.x) {
    const bool is_v = i >= per;
    const long long r = is_v ? i - per : i;
    const long long t = r / (a.num_kv_heads * cpr);
    const int rem = (int)(r - t * a.num_kv_heads * cpr);
    const int h = rem / cpr;
    const int c = rem - h * cpr;
    const long long slot = __ldg(a.slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= cap) {
      if (rem == 0 && !is_v) atomicOr(&g_status, PA_DEV_ERR_SLOT);
      continue;
    }
    const long long blk = slot / a.block_size;
    const int row = (int)(slot - blk * a.block_size);
    if (!dcheck(t < a.num_tokens && h < a.num_kv_heads && blk < a.num_blocks && row < a.block_size)) continue;
    const uint16_t *src = (is_v ? a.v + t * a.v_token_stride : a.k + t * a.k_token_stride) + h * a.head_dim + c * 8;
    uint16_t *dst = (is_v ? a.v_cache : a.k_cache) + ((blk * a.num_kv_heads + h) * a.block_size + row) * a.head_dim +
                    c * 8;
    *reinterpret_cast<uint4 *>(dst) = __ldg(reinterpret_cast<const uint4 *>(src));
  }
}

// ---------------------------------------------------------------- K2/K3: decode
//
// Work decomposition ("split over a tile stream"): every sequence s with a
// valid, non-empty context owns nt(s) = ceil(L_s / 16) tiles per head chunk
// (a head chunk = one kv head and up to 8 of its query heads).  All tiles are
// laid in one stream, ordered by sequence, then head chunk, then tile, and the
// stream is cut into chunks of consecutive tiles (ChunkPlan): warp w of the
// split kernel takes chunk w, and later chunks come from a queue (ChunkQueue),
// so a warp that runs ahead takes more.  The boundaries depend only on the
// lengths and the launch shape, never on timing, so the output is the same on
// every run.  The part of a chunk that falls in one (sequence, head chunk)
// is a piece: a piece that covers its whole segment writes the final output,
// the others write a partial softmax state that the merge kernel combines.
struct DecodeArgs {
  const uint16_t *q;
  const uint16_t *k_cache;
  const uint16_t *v_cache;
  const int32_t *block_tables;
  const int32_t *context_lens;
  uint16_t *out;
  unsigned long long *ws_queue;  // chunk queue word: (call epoch << 32) | next ticket; reset to 0 by the merge kernel
  int *ws_tiles;   // [num_seqs + 1] tile prefix, written by block 0 of the split kernel for the merge kernel
  float2 *ws_ml;   // [max_chunks][2][heads_per_unit] (running max in base-2 units, running sum) of partial pieces
  float *ws_acc;   // [max_chunks][2][heads_per_unit][head_dim] un-normalised partial outputs
  long long num_blocks, q_seq_stride, out_seq_stride, max_chunks;
  unsigned long long wait_limit_ns;
  float scale_log2;  // scale * log2(e)
  int num_seqs, num_q_heads, num_kv_heads, block_size, table_stride, max_context_len;
  int group;           // query heads per kv head
  int n_chunks;        // head chunks per kv head
  int heads_per_unit;  // query heads per head chunk (group / n_chunks)
  int chunk_tiles;     // tiles per chunk; 0: total tiles / split_warps
  int split_warps;     // warps in the split kernel's grid
  int static_permille;       // balanced split: share of each warp's tiles in its static first chunk (per mille)
  int tail_chunks_per_warp;  // balanced split: queued chunks per warp for the rest of the stream
  unsigned epoch;      // non-zero, different for every call
};

__device__ __forceinline__ bool context_ok(const DecodeArgs &a, int L) {
  return L >= 0 && (long long)L <= (long long)a.table_stride * a.block_size && L <= a.max_context_len;
}

__device__ __forceinline__ int seq_tiles(const DecodeArgs &a, int L) {
  return (context_ok(a, L) && L > 0) ? (L + TILE - 1) / TILE : 0;
}

// pt[s] = tiles (per head chunk) of the sequences before s, s = 0..num_seqs.
// Called by every thread of the block; ends with a block barrier.
// `scratch` holds one int per warp.
__device__ __forceinline__ void build_tile_prefix(const DecodeArgs &a, int *pt, int *scratch) {
  const int S = a.num_seqs;
  const int nth = blockDim.x, tid = threadIdx.x;
  const int per = (S + nth - 1) / nth;
  const int i0 = min(S, tid * per), i1 = min(S, i0 + per);
  int sum = 0;
  for (int i = i0; i < i1; ++i) {
    const int nt = seq_tiles(a, __ldg(a.context_lens + i));
    pt[i + 1] = nt;
    sum += nt;
  }
  const int lane = tid & 31, warp = tid >> 5;
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(FULL, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int run = incl - sum;
  for (int w = 0; w < warp; ++w) run += scratch[w];
  for (int i = i0; i < i1; ++i) {
    run += pt[i + 1];
    pt[i + 1] = run;
  }
  if (tid == 0) pt[0] = 0;
  __syncthreads();
}

constexpr int MIN_CHUNK_TILES = 4;  // never cut the stream finer than this (>= ring depth)

// How the tile stream is cut.  The first `n1` chunks (one per warp of the
// split kernel) hold `c1` tiles each; the rest of the stream is cut into
// chunks of `c2` tiles, handed out through the queue.  With the balanced
// split, c1 covers static_permille / 1000 of each warp's share and the tail
// gives every warp about tail_chunks_per_warp more chunks; with a fixed
// chunk length c1 = c2.  Boundaries depend only on the stream length and
// the arguments, so every kernel of the call computes the same ones.
struct ChunkPlan {
  long long total, c1, c2, n1, count;
  __device__ __forceinline__ long long start(long long c) const {
    return c < n1 ? c * c1 : n1 * c1 + (c - n1) * c2;
  }
  __device__ __forceinline__ int length(long long c) const {
    return (int)min(c < n1 ? c1 : c2, total - start(c));
  }
  __device__ __forceinline__ long long chunk_of(long long t) const {
    return t < n1 * c1 ? t / c1 : n1 + (t - n1 * c1) / c2;
  }
};

__device__ __forceinline__ ChunkPlan plan_chunks(const DecodeArgs &a, int tiles_per_head_chunk_set) {
  ChunkPlan p;
  p.total = (long long)tiles_per_head_chunk_set * a.num_kv_heads * a.n_chunks;
  const long long W = a.split_warps;
  if (a.chunk_tiles > 0) {
    p.c1 = p.c2 = max((long long)a.chunk_tiles, (long long)MIN_CHUNK_TILES);
  } else {
    p.c1 = p.total * a.static_permille / 1000 / W;
    p.c2 = max((long long)MIN_CHUNK_TILES, (p.total - W * p.c1 + W * a.tail_chunks_per_warp - 1) /
                                                max(1LL, W * a.tail_chunks_per_warp));
    if (p.c1 < MIN_CHUNK_TILES) p.c1 = p.c2;  // a small stream: uniform chunks
  }
  // never more chunks than the workspace holds
  p.n1 = min(W, (p.total + p.c1 - 1) / p.c1);
  long long rest = max(0LL, p.total - p.n1 * p.c1);
  if (a.max_chunks > p.n1 && rest > 0)
    p.c2 = max(p.c2, (rest + (a.max_chunks - p.n1) - 1) / (a.max_chunks - p.n1));
  p.count = p.n1 + (rest + p.c2 - 1) / p.c2;
  return p;
}

// Chunk hand-out: chunk w goes to warp w; later chunks come from a counter in
// the workspace.  Block 0 installs (epoch << 32) in the counter word at the
// start of the call (the epoch is non-zero and new for every call, and the
// merge kernel leaves the word at 0), so a ticket drawn before the install is
// recognised by its stale upper half and drawn again.  A warp requests its
// next ticket TICKET_AHEAD tiles before its current chunk runs out: late
// enough that a slow warp does not reserve work a faster one could take (a
// request half a chunk ahead pinned most of the queue to warps that were
// still busy), early enough that the atomic's round trip is hidden behind
// the tiles already in flight.
constexpr int TICKET_AHEAD = 3;

struct ChunkQueue {
  unsigned long long *word;
  unsigned epoch;
  long long first_dynamic, count;
  unsigned long long pending;  // lane 0: result of the last atomicAdd

  __device__ __forceinline__ void request(int lane) {
    if (lane == 0) pending = atomicAdd(word, 1ull);
  }
  // The chunk of the last request (>= count: none left).
  __device__ __forceinline__ long long take(int lane, unsigned long long limit_ns) {
    unsigned long long ticket = 0;
    if (lane == 0) {
      unsigned long long old = pending;
      const uint64_t t0 = global_ns();
      while ((unsigned)(old >> 32) != epoch) {  // drawn before this call's counter was installed
        if (global_ns() - t0 > limit_ns) {
          atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
          old = ~0ull;
          break;
        }
        __nanosleep(256);
        old = atomicAdd(word, 1ull);
      }
      ticket = old == ~0ull ? ~0ull : (old & 0xffffffffull);
    }
    ticket = __shfl_sync(FULL, ticket, 0);
    if (ticket == ~0ull) return count;
    const long long c = first_dynamic + (long long)ticket;
    return c < count ? c : count;
  }
};

// A position in the tile stream: tile j of head chunk hc of sequence s (nt tiles).
struct TilePos {
  int s, hc, j, nt;
};

__device__ __forceinline__ TilePos locate_tile(const int *pt, int S, int HC, long long t) {
  int lo = 0, hi = S - 1;  // largest s with pt[s] * HC <= t; that sequence has tiles
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)pt[mid] * HC <= t)
      lo = mid;
    else
      hi = mid - 1;
  }
  TilePos p;
  p.s = lo;
  p.nt = pt[lo + 1] - pt[lo];
  if (!dcheck(p.nt > 0 && t >= 0 && t < (long long)pt[S] * HC)) {  // a stream position past the tiles
    p.hc = p.j = 0;
    p.nt = 1;
    return p;
  }
  const long long r = t - (long long)pt[lo] * HC;
  p.hc = (int)(r / p.nt);
  p.j = (int)(r - (long long)p.hc * p.nt);
  return p;
}

__device__ __forceinline__ void advance_tile(TilePos &p, const int *pt, int S, int HC) {
  if (++p.j < p.nt) return;
  p.j = 0;
  if (++p.hc < HC) return;
  p.hc = 0;
  do {
    ++p.s;
  } while (p.s < S && pt[p.s + 1] == pt[p.s]);
  p.nt = p.s < S ? pt[p.s + 1] - pt[p.s] : 0;
}

// First query head of head chunk hc (kv head hc / n_chunks).
__device__ __forceinline__ int chunk_first_head(const DecodeArgs &a, int hc) {
  const int h = hc / a.n_chunks;
  return h * a.group + (hc - h * a.n_chunks) * a.heads_per_unit;
}

// The copy side of a warp's tile stream: walks the chunk ahead of the
// consumer, looks the physical block of each tile up in a 32-entry window of
// the sequence's table (one entry per lane), and starts the copies of the
// tile into a ring slot.  A tile whose table entry lies outside the pool is
// not copied: its slot's barrier is completed with a plain arrive and the
// slot is flagged in `bad_slots`.
struct TileProducer {
  TilePos pos;
  int win_s, win_base, ent;  // the table window in use: entries [win_base, win_base + 32) of row win_s
  uint32_t bad_slots;        // ring slots whose tile was not copied (set or cleared at every issue)

  __device__ __forceinline__ void init() {
    win_s = -1;
    win_base = 0;
    ent = -1;
    bad_slots = 0;
  }

  // Moves the producer to a new position.  The window stays valid (it depends on the table row only), and
  // so do the flags of the slots still in flight from the previous chunk.
  __device__ __forceinline__ void start(const TilePos &p) { pos = p; }

  // Returns the physical block of the producer's current tile (or -1), loading a new window when needed.
  // The row's block count comes from the sequence's tile count nt = ceil(L / 16)
  // (ceil(nt * 16 / block_size) = ceil(L / block_size)), so no length load stands between the producer and
  // the table; entries at or past it are not read.
  __device__ __forceinline__ int lookup(const DecodeArgs &a, int lane) {
    const int blk = (pos.j * TILE) / a.block_size;
    if (pos.s != win_s || blk < win_base || blk >= win_base + 32) {
      win_s = pos.s;
      win_base = blk & ~31;
      const int nblk = (pos.nt * TILE + a.block_size - 1) / a.block_size;
      const bool in_row = dcheck(pos.s < a.num_seqs && nblk <= a.table_stride);
      ent = (in_row && win_base + lane < nblk)
                ? __ldg(a.block_tables + (long long)pos.s * a.table_stride + win_base + lane)
                : -1;
    }
    const int phys = __shfl_sync(FULL, ent, blk - win_base);
    if (phys < 0 || (long long)phys >= a.num_blocks) return -1;
    // the tile's 16 rows lie inside the (block, kv head) slab
    if (!dcheck(pos.hc / a.n_chunks < a.num_kv_heads && (pos.j * TILE) % a.block_size + TILE <= a.block_size))
      return -1;
    return phys;
  }

  // Global row (in [num_blocks * num_kv_heads * block_size)) of the tile's first token.
  __device__ __forceinline__ long long first_row(const DecodeArgs &a, int phys) const {
    return ((long long)phys * a.num_kv_heads + pos.hc / a.n_chunks) * a.block_size + (pos.j * TILE) % a.block_size;
  }
};

// Sums, over the lanes of one row group (lane bits 0..log2(2R)-1), R partial
// dot products held by every lane, with R/2 + R/4 + ... + 1 + 1 shuffles
// (a reduce-scatter butterfly).  Lane l ends with the full dot of its local
// row (l & (2R-2)) >> 1; lanes l and l^1 hold the same value.
template <int R>
__device__ __forceinline__ float row_group_reduce(float (&v)[R], int lane) {
#pragma unroll
  for (int n = R; n >= 2; n >>= 1) {
    const int half = n >> 1;
    const bool upper = (lane & n) != 0;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float send = upper ? v[k] : v[k + half];
      const float keep = upper ? v[k + half] : v[k];
      v[k] = keep + __shfl_xor_sync(FULL, send, n);
    }
  }
  return v[0] + __shfl_xor_sync(FULL, v[0], 1);
}

// Element-type specific arithmetic used by the partition kernel.
//   dot8: sum of 8 products q_i * k_i of packed 2-byte values (4 words each),
//         computed by the mixed-precision fma (2-byte inputs widened exactly,
//         fp32 accumulation) so no separate conversion is issued.
//   widen8: 8 packed values -> fp32.
__device__ __forceinline__ float dot8_f16(const uint32_t (&q)[4], const uint4 k, float c) {
  float d;
  asm("{\n\t.reg .b16 q0, q1, k0, k1;\n\t.reg .f32 t;\n\t"
      "mov.b32 {q0, q1}, %1;\n\tmov.b32 {k0, k1}, %5;\n\tfma.rn.f32.f16 t, q0, k0, %9;\n\tfma.rn.f32.f16 t, q1, k1, t;\n\t"
      "mov.b32 {q0, q1}, %2;\n\tmov.b32 {k0, k1}, %6;\n\tfma.rn.f32.f16 t, q0, k0, t;\n\tfma.rn.f32.f16 t, q1, k1, t;\n\t"
      "mov.b32 {q0, q1}, %3;\n\tmov.b32 {k0, k1}, %7;\n\tfma.rn.f32.f16 t, q0, k0, t;\n\tfma.rn.f32.f16 t, q1, k1, t;\n\t"
      "mov.b32 {q0, q1}, %4;\n\tmov.b32 {k0, k1}, %8;\n\tfma.rn.f32.f16 t, q0, k0, t;\n\tfma.rn.f32.f16 %0, q1, k1, t;\n\t}"
      : "=f"(d)
      : "r"(q[0]), "r"(q[1]), "r"(q[2]), "r"(q[3]), "r"(k.x), "r"(k.y), "r"(k.z), "r"(k.w), "f"(c));
  return d;
}
__device__ __forceinline__ float dot8_bf16(const uint32_t (&q)[4], const uint4 k, float c) {
  float d;
  asm("{\n\t.reg .b16 q0, q1, k0, k1;\n\t.reg .f32 t;\n\t"
      "mov.b32 {q0, q1}, %1;\n\tmov.b32 {k0, k1}, %5;\n\tfma.rn.f32.bf16 t, q0, k0, %9;\n\tfma.rn.f32.bf16 t, q1, k1, t;\n\t"
      "mov.b32 {q0, q1}, %2;\n\tmov.b32 {k0, k1}, %6;\n\tfma.rn.f32.bf16 t, q0, k0, t;\n\tfma.rn.f32.bf16 t, q1, k1, t;\n\t"
      "mov.b32 {q0, q1}, %3;\n\tmov.b32 {k0, k1}, %7;\n\tfma.rn.f32.bf16 t, q0, k0, t;\n\tfma.rn.f32.bf16 t, q1, k1, t;\n\t"
      "mov.b32 {q0, q1}, %4;\n\tmov.b32 {k0, k1}, %8;\n\tfma.rn.f32.bf16 t, q0, k0, t;\n\tfma.rn.f32.bf16 %0, q1, k1, t;\n\t}"
      : "=f"(d)
      : "r"(q[0]), "r"(q[1]), "r"(q[2]), "r"(q[3]), "r"(k.x), "r"(k.y), "r"(k.z), "r"(k.w), "f"(c));
  return d;
}

// Shared-memory layout of the split kernels: [ring slots][per-warp barriers][tile prefix][scan scratch].
template <int WARPS, int STAGES, uint32_t STAGE_BYTES>
struct SplitSmem {
  static constexpr uint32_t RING = WARPS * STAGES * STAGE_BYTES;
  static constexpr uint32_t BARS = ((WARPS * STAGES * 8 + 127) / 128) * 128;
  static __host__ __device__ constexpr uint32_t bytes(int num_seqs) {
    return RING + BARS + (uint32_t)(num_seqs + 1 + WARPS) * 4u;
  }
};

// Waits (bounded) for ring slot `it`; on a timeout flags the status, lets the
// copies still in flight land (bounded) and returns false.
template <int STAGES>
__device__ __forceinline__ bool wait_slot(uint64_t *bars, uint32_t it, int in_flight, unsigned long long limit_ns,
                                          int lane) {
  const bool arrived = mbar_wait_bounded(&bars[it % STAGES], (it / STAGES) & 1u, limit_ns);
  if (!__any_sync(FULL, !arrived)) return true;
  if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
  for (int k = 0; k < in_flight; ++k) {
    const uint32_t i2 = it + k;
    mbar_wait_bounded(&bars[i2 % STAGES], (i2 / STAGES) & 1u, limit_ns);
  }
  return false;
}

constexpr float RESCALE_SLACK = 8.f;

// The arithmetic of the CUDA-core kernels for one piece (a run of tiles of one segment: G query heads of
// one kv head), shared by the split and the per-segment kernels: the query rows, the online-softmax state
// and accumulators, and the step for one 16-token tile.
//
// Per tile, lane l holds 16 bytes (8 head dims, cl * 8 ..) of rows r * NGRP + grp (r < R) of K and of V.
// QK^T uses the mixed-precision fma (2-byte inputs, fp32 accumulation); the 16 dot products are finished
// by a reduce-scatter butterfly.  The online softmax keeps, per query head, a running maximum m that is
// raised only when a logit exceeds it by more than RESCALE_SLACK (base-2 units), so most tiles need no max
// reduction; m cancels between numerator and denominator, and weights stay below 2^RESCALE_SLACK.
template <class E, int D, int G>
struct CoreMath {
  static constexpr int LPR = D / 8;      // lanes covering one K/V row
  static constexpr int NGRP = 32 / LPR;  // rows one warp-wide 16-byte load covers
  static constexpr int R = TILE / NGRP;  // rows per lane per tile
  int grp, cl, my_tok;
  uint32_t qw[G][4];
  float m[G], lsum[G];
  float2 acc[G][4];

  __device__ __forceinline__ void setup(int lane) {
    grp = lane / LPR;
    cl = lane % LPR;
    my_tok = ((lane & (LPR - 2)) >> 1) * NGRP + grp;  // token whose logit this lane ends with
  }

  // A new piece: the G query rows starting at qrow (D elements apart), zeros when !ok; a fresh state.
  __device__ __forceinline__ void begin(const uint16_t *qrow, bool ok) {
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const uint4 w = ok ? __ldg(reinterpret_cast<const uint4 *>(qrow + gg * D + cl * 8)) : make_uint4(0, 0, 0, 0);
      qw[gg][0] = w.x;
      qw[gg][1] = w.y;
      qw[gg][2] = w.z;
      qw[gg][3] = w.w;
      m[gg] = -INFINITY;
      lsum[gg] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) acc[gg][kk] = make_float2(0.f, 0.f);
    }
  }

  // This lane's rows of the K tile at kt and the V tile at vt (zeros for a tile that was not copied).
  __device__ __forceinline__ void read_tile(const unsigned char *kt, const unsigned char *vt, bool bad, uint4 (&kr)[R],
                                            uint4 (&vr)[R]) const {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      kr[r] = bad ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4 *>(kt + ((r * NGRP + grp) * D + cl * 8) * 2);
      vr[r] = bad ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4 *>(vt + ((r * NGRP + grp) * D + cl * 8) * 2);
    }
  }

  // One tile of nvalid live rows (the rest masked): QK^T, scale, mask, online softmax, P.V.
  __device__ __forceinline__ void tile(const uint4 (&kr)[R], const uint4 (&vr)[R], int nvalid, float scale_log2,
                                       int lane) {
    const bool tok_live = my_tok < nvalid;
    // QK^T for this lane's R rows, the butterfly, scale, mask
    float z[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float part[R];
#pragma unroll
      for (int r = 0; r < R; ++r) part[r] = E::dot8(qw[gg], kr[r], 0.f);
      const float t = row_group_reduce<R>(part, lane) * scale_log2;
      z[gg] = tok_live ? t : -INFINITY;
    }
    // softmax state: raise m only when some logit passes it by more than the slack
    float pr[G][R];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      if (__any_sync(FULL, z[gg] > m[gg] + RESCALE_SLACK)) {
        float mt = z[gg];
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 2));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 4));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 8));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 16));
        const float alpha = exp2f(m[gg] - mt);  // 0 on the piece's first tile (m = -inf)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) acc[gg][kk] = make_float2(acc[gg][kk].x * alpha, acc[gg][kk].y * alpha);
        lsum[gg] *= alpha;
        m[gg] = mt;
      }
      const float pz = exp2f(z[gg] - m[gg]);
      lsum[gg] += (lane & 1) ? 0.f : pz;
#pragma unroll
      for (int r = 0; r < R; ++r) pr[gg][r] = __shfl_sync(FULL, pz, grp * LPR + 2 * r);
    }
    // P.V over this lane's 8 dims and R rows (packed fp32 fma)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float vf[8];
      E::widen8(vr[r], vf);
      if (nvalid < TILE) {  // rows past the sequence may hold anything (NaN): never let them in
        const bool row_live = (r * NGRP + grp) < nvalid;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) vf[kk] = row_live ? vf[kk] : 0.f;
      }
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        const float2 pp = make_float2(pr[gg][r], pr[gg][r]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) acc[gg][kk] = __ffma2_rn(pp, make_float2(vf[2 * kk], vf[2 * kk + 1]), acc[gg][kk]);
      }
    }
  }

  // End of the piece: merges the row groups (lanes < LPR then hold dims cl * 8 .. cl * 8 + 7 of every head,
  // un-normalised) and totals the sums in every lane.
  __device__ __forceinline__ void finish() {
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          acc[gg][kk].x += __shfl_xor_sync(FULL, acc[gg][kk].x, off);
          acc[gg][kk].y += __shfl_xor_sync(FULL, acc[gg][kk].y, off);
        }
      }
      float l = lsum[gg];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(FULL, l, off);
      lsum[gg] = l;
    }
  }

  // Lanes < LPR: the normalised rows (zeros when bad) of the G heads, heads D elements apart from out_row.
  __device__ __forceinline__ void store_output(uint16_t *out_row, bool bad) const {
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float o[8];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        o[2 * kk] = bad ? 0.f : acc[gg][kk].x / lsum[gg];
        o[2 * kk + 1] = bad ? 0.f : acc[gg][kk].y / lsum[gg];
      }
      *reinterpret_cast<uint4 *>(out_row + gg * D + cl * 8) = narrow8<E>(o);
    }
  }
};

// CUDA-core split kernel, for head chunks of G = 1 or 2 query heads.
//
// Each warp streams the tiles of its chunks through a private STAGES-deep ring
// of shared-memory slots filled by bulk copies (K tile + V tile of one
// (block, kv head), 2 x 16 * D * 2 bytes).  Per tile, each lane copies its
// rows of K and V from the slot into registers and the slot is refilled at
// once, before the math (CoreMath).
template <class E, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, 12 / WARPS) decode_split_kernel(const DecodeArgs a) {
  constexpr int LPR = CoreMath<E, D, G>::LPR;
  constexpr uint32_t TILE_BYTES = TILE * D * 2;
  constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;
  using Smem = SplitSmem<WARPS, STAGES, STAGE_BYTES>;

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  unsigned char *ring = smem + warp * STAGES * STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Smem::RING) + warp * STAGES;
  int *pt = reinterpret_cast<int *>(smem + Smem::RING + Smem::BARS);
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
  }
  grid_dependency_wait();    // every input may come from the previous kernel in the stream
  grid_launch_dependents();  // the merge kernel may launch now and wait for this grid
  if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(a.ws_queue, (unsigned long long)a.epoch << 32);
  const int S = a.num_seqs;
  build_tile_prefix(a, pt, pt + S + 1);
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= S; i += blockDim.x) a.ws_tiles[i] = pt[i];
  const ChunkPlan plan = plan_chunks(a, pt[S]);
  const int HC = a.num_kv_heads * a.n_chunks;

  uint32_t iter = 0;  // tiles consumed by this warp: ring slot iter % STAGES, phase (iter / STAGES) & 1
  TileProducer prod;

  long long cons_c = (long long)blockIdx.x * WARPS + warp;  // chunk the consumer is in (the first one is static)
  if (cons_c < plan.count) {
    ChunkQueue queue{a.ws_queue, a.epoch, (long long)a.split_warps, plan.count, 0ull};
    bool requested = false;  // a ticket for the producer's next chunk is on its way
    long long prod_c = cons_c;
    int prod_left = plan.length(prod_c);
    bool prod_done = false;
    TilePos cp = locate_tile(pt, S, HC, plan.start(cons_c));
    prod.init();
    prod.start(cp);
    uint32_t issued = iter;  // tiles issued by this warp: the next goes to ring slot issued % STAGES

    // issue the producer's next tile, moving it into its next chunk when the current one is done
    auto issue_next = [&]() {
      if (prod_left == 0) {
        if (prod_done) return;
        if (!requested) queue.request(lane);
        requested = false;
        const long long nc = queue.take(lane, a.wait_limit_ns);
        if (nc >= plan.count) {
          prod_done = true;
          return;
        }
        prod_c = nc;
        prod_left = plan.length(nc);
        prod.start(locate_tile(pt, S, HC, plan.start(nc)));
      }
      const uint32_t it = issued++;
      const int phys = prod.lookup(a, lane);
      const int st = (int)(it % STAGES);
      prod.bad_slots = phys >= 0 ? (prod.bad_slots & ~(1u << st)) : (prod.bad_slots | (1u << st));
      if (lane == 0) {
        fence_proxy_async_smem();
        if (phys >= 0) {
          const long long row0 = prod.first_row(a, phys);
          unsigned char *dst = ring + st * STAGE_BYTES;
          mbar_arrive_expect_tx(&bars[st], STAGE_BYTES);
          bulk_copy_g2s(dst, a.k_cache + row0 * D, TILE_BYTES, &bars[st]);
          bulk_copy_g2s(dst + TILE_BYTES, a.v_cache + row0 * D, TILE_BYTES, &bars[st]);
        } else {
          mbar_arrive(&bars[st]);
        }
      }
      advance_tile(prod.pos, pt, S, HC);
      --prod_left;
      if (!requested && prod_left <= TICKET_AHEAD) {
        queue.request(lane);
        requested = true;
      }
    };
    for (int k = 0; k < STAGES; ++k) issue_next();

    CoreMath<E, D, G> cm;
    cm.setup(lane);
    int L = 0, hq0 = 0, slot = 0;
    bool full = false, piece_bad = false;

    int cons_left = plan.length(cons_c);
    int k = 0;  // tile index within the consumer's chunk
    while (true) {
      if (cons_left == 0) {  // the consumer's chunk is done: follow the producer into its next chunk
        if (prod_c == cons_c) break;
        cons_c = prod_c;
        cons_left = plan.length(cons_c);
        cp = locate_tile(pt, S, HC, plan.start(cons_c));
        k = 0;
      }
      if (k == 0 || cp.j == 0) {  // a new piece: segment (cp.s, cp.hc) from tile cp.j on
        const int len = min(cp.nt - cp.j, cons_left);
        full = (cp.j == 0 && len == cp.nt);
        slot = (k == 0) ? 0 : 1;
        hq0 = chunk_first_head(a, cp.hc);
        const bool q_ok = dcheck(cp.s < S && hq0 + G <= a.num_q_heads);
        L = q_ok ? __ldg(a.context_lens + cp.s) : 0;
        piece_bad = false;
        cm.begin(a.q + (long long)cp.s * a.q_seq_stride + (long long)hq0 * D, q_ok);
      }
      const int st = (int)(iter % STAGES);
      if (!wait_slot<STAGES>(bars, iter, (int)(issued - iter), a.wait_limit_ns, lane)) return;
      const bool tile_bad = (prod.bad_slots >> st) & 1u;
      // copy this lane's rows out of the slot, then hand the slot straight back to the copy engine
      uint4 kr[CoreMath<E, D, G>::R], vr[CoreMath<E, D, G>::R];
      cm.read_tile(ring + st * STAGE_BYTES, ring + st * STAGE_BYTES + TILE_BYTES, tile_bad, kr, vr);
      __syncwarp();
      issue_next();
      ++iter;
      piece_bad |= tile_bad;
      if (!piece_bad) cm.tile(kr, vr, min(TILE, L - cp.j * TILE), a.scale_log2, lane);

      if (cp.j + 1 == cp.nt || cons_left == 1) {
        // ---- end of the piece: merge the row groups, total the sums, store the output or the partial
        cm.finish();
        if (piece_bad && lane == 0) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
        if (full) {
          if (lane < LPR && dcheck(cp.s < S && hq0 + G <= a.num_q_heads))
            cm.store_output(a.out + (long long)cp.s * a.out_seq_stride + (long long)hq0 * D, piece_bad);
        } else {
          const long long prow = (cons_c * 2 + slot) * G;
          const bool row_ok = dcheck(cons_c < a.max_chunks);
#pragma unroll
          for (int gg = 0; gg < G; ++gg) {
            if (!row_ok) break;
            if (lane < LPR && !piece_bad) {
              float4 *dst = reinterpret_cast<float4 *>(a.ws_acc + (prow + gg) * D + cm.cl * 8);
              dst[0] = make_float4(cm.acc[gg][0].x, cm.acc[gg][0].y, cm.acc[gg][1].x, cm.acc[gg][1].y);
              dst[1] = make_float4(cm.acc[gg][2].x, cm.acc[gg][2].y, cm.acc[gg][3].x, cm.acc[gg][3].y);
            }
            if (lane == 0)
              a.ws_ml[prow + gg] = piece_bad ? make_float2(-INFINITY, -1.f) : make_float2(cm.m[gg], cm.lsum[gg]);
          }
        }
      }
      advance_tile(cp, pt, S, HC);
      --cons_left;
      ++k;
    }
  }
}

// Per-segment kernel for small batches on the CUDA-core path: block b handles segment b (sequence
// s = b / HC, head chunk hc = b % HC) whole.  Its WARPS warps take the segment's tiles in turn (tile j to
// warp j mod WARPS), each through its own ring of bulk copies as in the split kernel; at the end the warps'
// softmax states are merged in shared memory, in warp order (deterministic), and warp 0 writes the rows.
// It needs no workspace and no merge kernel, and a block touches only its own sequence's length and table
// row: chosen when all segments fit one wave of blocks and are short, where the split kernel's tile
// prefix, chunk queue and separate merge launch would cost more than the work.
template <class E, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32) decode_segment_kernel(const DecodeArgs a) {
  using CM = CoreMath<E, D, G>;
  constexpr int LPR = CM::LPR;
  constexpr uint32_t TILE_BYTES = TILE * D * 2;
  constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;
  using Smem = SplitSmem<WARPS, STAGES, STAGE_BYTES>;

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  unsigned char *ring = smem + warp * STAGES * STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Smem::RING) + warp * STAGES;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
  }
  grid_dependency_wait();  // every input may come from the previous kernel in the stream
  grid_launch_dependents();
  const int HC = a.num_kv_heads * a.n_chunks;
  const int s = (int)(blockIdx.x / HC), hc = (int)(blockIdx.x - (unsigned)s * HC);
  const int hq0 = chunk_first_head(a, hc);
  const int h = hc / a.n_chunks;
  const int L = __ldg(a.context_lens + s);
  uint16_t *out_row = a.out + (long long)s * a.out_seq_stride + (long long)hq0 * D;
  if (!context_ok(a, L) || L == 0) {  // zero rows; the status bit once per sequence
    if (warp == 0) {
      if (lane == 0 && L != 0 && hc == 0)
        atomicOr(&g_status, (L < 0 || (long long)L > (long long)a.table_stride * a.block_size) ? PA_DEV_ERR_CONTEXT
                                                                                              : PA_DEV_ERR_CONTEXT_HINT);
      for (int c = lane; c < G * D / 8; c += 32) reinterpret_cast<uint4 *>(out_row)[c] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const int nt = (L + TILE - 1) / TILE;
  const int nblk = (L + a.block_size - 1) / a.block_size;
  const int my_tiles = warp < nt ? (nt - warp + WARPS - 1) / WARPS : 0;

  // physical block of tile j, through a 32-entry window of the table row (entries >= nblk not read)
  int win_base = -1, ent = -1;
  auto phys_of = [&](int j) -> int {
    const int blk = (j * TILE) / a.block_size;
    const int base = blk & ~31;
    if (base != win_base) {
      win_base = base;
      ent = (base + lane < nblk && dcheck(nblk <= a.table_stride))
                ? __ldg(a.block_tables + (long long)s * a.table_stride + base + lane)
                : -1;
    }
    const int phys = __shfl_sync(FULL, ent, blk - base);
    return (phys >= 0 && (long long)phys < a.num_blocks) ? phys : -1;
  };
  uint32_t bad_slots = 0;
  auto issue = [&](int t) {  // this warp's t-th tile into slot t % STAGES
    const int j = warp + t * WARPS;
    const int phys = phys_of(j);
    const int st = t % STAGES;
    bad_slots = phys >= 0 ? (bad_slots & ~(1u << st)) : (bad_slots | (1u << st));
    if (lane == 0) {
      fence_proxy_async_smem();
      if (phys >= 0) {
        const long long row0 = ((long long)phys * a.num_kv_heads + h) * a.block_size + (j * TILE) % a.block_size;
        unsigned char *dst = ring + st * STAGE_BYTES;
        mbar_arrive_expect_tx(&bars[st], STAGE_BYTES);
        bulk_copy_g2s(dst, a.k_cache + row0 * D, TILE_BYTES, &bars[st]);
        bulk_copy_g2s(dst + TILE_BYTES, a.v_cache + row0 * D, TILE_BYTES, &bars[st]);
      } else {
        mbar_arrive(&bars[st]);
      }
    }
  };

  CM cm;
  cm.setup(lane);
  cm.begin(a.q + (long long)s * a.q_seq_stride + (long long)hq0 * D, true);
  int issued = 0;
  for (; issued < STAGES && issued < my_tiles; ++issued) issue(issued);
  bool bad = false;
  for (int t = 0; t < my_tiles; ++t) {
    const int st = t % STAGES;
    if (!wait_slot<STAGES>(bars, (uint32_t)t, issued - t, a.wait_limit_ns, lane)) {
      bad = true;  // timed out (flagged; the copies in flight were waited for): this segment's rows become zeros
      break;
    }
    uint4 kr[CM::R], vr[CM::R];
    const bool tile_bad = (bad_slots >> st) & 1u;
    cm.read_tile(ring + st * STAGE_BYTES, ring + st * STAGE_BYTES + TILE_BYTES, tile_bad, kr, vr);
    __syncwarp();
    if (issued < my_tiles) issue(issued++);
    bad |= tile_bad;
    const int j = warp + t * WARPS;
    if (!bad) cm.tile(kr, vr, min(TILE, L - j * TILE), a.scale_log2, lane);
  }
  cm.finish();

  // merge the warps' states through shared memory (the rings are free: every copy issued was waited for)
  __syncthreads();
  float *x_acc = reinterpret_cast<float *>(smem);                  // [WARPS][G][D]
  float2 *x_ml = reinterpret_cast<float2 *>(x_acc + WARPS * G * D);  // [WARPS][G]
  int *x_bad = reinterpret_cast<int *>(x_ml + WARPS * G);          // [WARPS]
#pragma unroll
  for (int gg = 0; gg < G; ++gg) {
    if (lane < LPR) {
      float4 *dst = reinterpret_cast<float4 *>(x_acc + (warp * G + gg) * D + cm.cl * 8);
      dst[0] = make_float4(cm.acc[gg][0].x, cm.acc[gg][0].y, cm.acc[gg][1].x, cm.acc[gg][1].y);
      dst[1] = make_float4(cm.acc[gg][2].x, cm.acc[gg][2].y, cm.acc[gg][3].x, cm.acc[gg][3].y);
    }
    if (lane == 0) x_ml[warp * G + gg] = make_float2(cm.m[gg], cm.lsum[gg]);
  }
  if (lane == 0) x_bad[warp] = bad ? 1 : 0;
  __syncthreads();
  if (warp != 0) return;
  bool any_bad = false;
#pragma unroll
  for (int w = 0; w < WARPS; ++w) any_bad |= x_bad[w] != 0;
  if (any_bad && lane == 0) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
  if (lane < LPR) {
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < WARPS; ++w) M = fmaxf(M, x_ml[w * G + gg].x);
      float l = 0.f, o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < WARPS; ++w) {
        const float2 ml = x_ml[w * G + gg];
        const float wt = ml.y > 0.f ? exp2f(ml.x - M) : 0.f;  // a warp with no tiles has m = -inf, l = 0
        l = fmaf(ml.y, wt, l);
        const float *src = x_acc + (w * G + gg) * D + cm.cl * 8;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) o[kk] = fmaf(wt, src[kk], o[kk]);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) o[kk] = any_bad ? 0.f : o[kk] / l;
      *reinterpret_cast<uint4 *>(out_row + gg * D + cm.cl * 8) = narrow8<E>(o);
    }
  }
}

// One warp per HW query heads of a segment (sequence s, head chunk: G query heads of one kv head): writes
// the zero rows of empty or invalid sequences (setting the status bits of the invalid ones) and merges the
// partial pieces of segments that the split kernel cut across chunks:
//   out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p,  M = max_p m_p,
// summed in increasing chunk order (deterministic).  Built for latency, since it runs after the split grid
// has drained: the pieces' (m, l) and the partial rows of the first MB pieces are requested together, so a
// segment cut into at most MB pieces costs two dependent trips to memory after the wait (tile prefix, then
// pieces).  Eight warps per block: with more, smaller blocks the grid took measurably longer to get
// through the SMs behind the split kernel (4096 blocks of two warps: +20 us on a 256-sequence batch).
template <class E, int D, int HW, int MB>
__global__ void __launch_bounds__(256, 1) decode_merge_kernel(const DecodeArgs a) {
  static_assert(32 % MB == 0, "a batch of pieces never straddles a 32-piece window");
  constexpr int DPL = D / 32;  // dims per lane (4 or 2)
  const int lane = threadIdx.x & 31;
  grid_dependency_wait();  // the split kernel's pieces and tile prefix
  grid_launch_dependents();
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.ws_queue = 0ull;  // leave the chunk counter clear
  const int S = a.num_seqs;
  const int HC = a.num_kv_heads * a.n_chunks;
  const int G = a.heads_per_unit;
  const int subs = G / HW;  // warps per segment
  const long long w = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (w >= (long long)S * HC * subs) return;
  const long long seg = w / subs;
  const int gg0 = (int)(w - seg * subs) * HW;  // first head of this warp within the chunk
  const int s = (int)(seg / HC);
  const int hc = (int)(seg - (long long)s * HC);
  const int L = __ldg(a.context_lens + s);
  const int pt0 = __ldg(a.ws_tiles + s), pt1 = __ldg(a.ws_tiles + s + 1), pts = __ldg(a.ws_tiles + S);
  uint16_t *dst =
      a.out + (long long)s * a.out_seq_stride + (long long)(chunk_first_head(a, hc) + gg0) * D + lane * DPL;
  float o[HW][DPL];
#pragma unroll
  for (int gg = 0; gg < HW; ++gg)
#pragma unroll
    for (int k = 0; k < DPL; ++k) o[gg][k] = 0.f;
  if (!context_ok(a, L) || L == 0) {
    if (lane == 0 && L != 0 && hc == 0 && gg0 == 0)
      atomicOr(&g_status, (L < 0 || (long long)L > (long long)a.table_stride * a.block_size) ? PA_DEV_ERR_CONTEXT
                                                                                            : PA_DEV_ERR_CONTEXT_HINT);
  } else {
    const ChunkPlan plan = plan_chunks(a, pts);
    const int nt = pt1 - pt0;
    const long long seg0 = (long long)pt0 * HC + (long long)hc * nt;
    if (!dcheck(nt > 0 && pt0 >= 0 && pt1 <= pts)) return;  // a sequence with a context owns tiles
    const long long c_first = plan.chunk_of(seg0), c_last = plan.chunk_of(seg0 + nt - 1);
    if (c_first == c_last) return;  // one chunk held the whole segment: the split kernel wrote the rows
    if (!dcheck(c_first >= 0 && c_last < plan.count && c_last < a.max_chunks)) return;
    const int n = (int)(c_last - c_first + 1);
    auto piece_row = [&](int p) -> long long {  // partial row of this warp's first head in piece p
      const long long c = c_first + p;
      const int slot = (p == 0 && seg0 > plan.start(c)) ? 1 : 0;
      return (c * 2 + slot) * G + gg0;
    };
    // (m, l) of the first 32 pieces (lane p holds piece p) and the partial rows of the first batch, together
    float2 ml0[HW];
#pragma unroll
    for (int gg = 0; gg < HW; ++gg) ml0[gg] = make_float2(-INFINITY, 0.f);
    if (lane < n) {
      const long long r = piece_row(lane);
#pragma unroll
      for (int gg = 0; gg < HW; ++gg) ml0[gg] = __ldg(a.ws_ml + r + gg);
    }
    float t[MB][HW][DPL];
    auto load_batch = [&](int base) {
#pragma unroll
      for (int i = 0; i < MB; ++i) {
        const bool ok = base + i < n;
        const long long r = ok ? piece_row(base + i) : 0;
#pragma unroll
        for (int gg = 0; gg < HW; ++gg) {
          const float *src = a.ws_acc + (r + gg) * D + lane * DPL;
          if constexpr (DPL == 4) {
            const float4 v = ok ? __ldg(reinterpret_cast<const float4 *>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
            t[i][gg][0] = v.x;
            t[i][gg][1] = v.y;
            t[i][gg][2] = v.z;
            t[i][gg][3] = v.w;
          } else {
            const float2 v = ok ? __ldg(reinterpret_cast<const float2 *>(src)) : make_float2(0.f, 0.f);
            t[i][gg][0] = v.x;
            t[i][gg][1] = v.y;
          }
        }
      }
    };
    load_batch(0);
    // maximum and validity over all pieces, per head
    float M[HW];
    bool err = false;
#pragma unroll
    for (int gg = 0; gg < HW; ++gg) {
      M[gg] = ml0[gg].x;
      err |= lane < n && ml0[gg].y < 0.f;
    }
    for (int p = lane + 32; p < n; p += 32) {
      const long long r = piece_row(p);
#pragma unroll
      for (int gg = 0; gg < HW; ++gg) {
        const float2 ml = __ldg(a.ws_ml + r + gg);
        M[gg] = fmaxf(M[gg], ml.x);
        err |= ml.y < 0.f;
      }
    }
#pragma unroll
    for (int gg = 0; gg < HW; ++gg)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) M[gg] = fmaxf(M[gg], __shfl_xor_sync(FULL, M[gg], off));
    if (!__any_sync(FULL, err)) {
      // lane p of the current 32-piece window holds piece p's weight per head; the sum of weighted l runs per lane
      float wt[HW], l[HW];
#pragma unroll
      for (int gg = 0; gg < HW; ++gg) {
        wt[gg] = lane < n ? exp2f(ml0[gg].x - M[gg]) : 0.f;
        l[gg] = ml0[gg].y * wt[gg];
      }
      for (int base = 0; base < n; base += MB) {
        if (base > 0) {
          if ((base & 31) == 0) {  // next window of 32 pieces: their (m, l)
            const int p = base + lane;
            const long long r = p < n ? piece_row(p) : 0;
#pragma unroll
            for (int gg = 0; gg < HW; ++gg) {
              const float2 ml = p < n ? __ldg(a.ws_ml + r + gg) : make_float2(-INFINITY, 0.f);
              wt[gg] = p < n ? exp2f(ml.x - M[gg]) : 0.f;
              l[gg] = fmaf(ml.y, wt[gg], l[gg]);
            }
          }
          load_batch(base);
        }
#pragma unroll
        for (int i = 0; i < MB; ++i) {
          const int src_lane = (base + i) & 31;
#pragma unroll
          for (int gg = 0; gg < HW; ++gg) {
            const float wq = __shfl_sync(FULL, wt[gg], src_lane);  // 0 past the last piece
#pragma unroll
            for (int k = 0; k < DPL; ++k) o[gg][k] = fmaf(wq, t[i][gg][k], o[gg][k]);
          }
        }
      }
#pragma unroll
      for (int gg = 0; gg < HW; ++gg) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) l[gg] += __shfl_xor_sync(FULL, l[gg], off);
#pragma unroll
        for (int k = 0; k < DPL; ++k) o[gg][k] = o[gg][k] / l[gg];
      }
    }
  }
#pragma unroll
  for (int gg = 0; gg < HW; ++gg) {
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint2 *>(dst + gg * D) =
          make_uint2(E::narrow2(o[gg][0], o[gg][1]), E::narrow2(o[gg][2], o[gg][3]));
    } else {
      *reinterpret_cast<uint32_t *>(dst + gg * D) = E::narrow2(o[gg][0], o[gg][1]);
    }
  }
}

// One warp waits on a barrier nothing will complete; after limit_ns it gives
// up, flags PA_DEV_ERR_TIMEOUT and returns (self-test of the bounded wait).
__global__ void wait_timeout_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const bool done = mbar_wait_bounded(&bar, 0, limit_ns);
  if (__any_sync(FULL, !done) && threadIdx.x == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
}

}  // namespace pa
