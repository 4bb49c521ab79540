// sm_100a kernels of the paged decode path.
//
//   write_kv_kernel          slot-mapped scatter of this step's new K/V rows
//                            ("4. vLLM核心机制" section 4.3, layout of 4.2).
//   decode_partition_kernel  attention of one query token per sequence over
//                            the block-paged cache, reached through the
//                            per-sequence block table ("4. vLLM核心机制" 4.2;
//                            "vLLM：大型语言模型推理优化的革命性突破" 2.1).
//   decode_reduce_kernel     merges the partial softmax states of sequences
//                            split along the context into several units.
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
    const uint16_t *src = (is_v ? a.v + t * a.v_token_stride : a.k + t * a.k_token_stride) + h * a.head_dim + c * 8;
    uint16_t *dst = (is_v ? a.v_cache : a.k_cache) + ((blk * a.num_kv_heads + h) * a.block_size + row) * a.head_dim +
                    c * 8;
    *reinterpret_cast<uint4 *>(dst) = __ldg(reinterpret_cast<const uint4 *>(src));
  }
}

// ---------------------------------------------------------------- K2/K3: decode
struct DecodeArgs {
  const uint16_t *q;
  const uint16_t *k_cache;
  const uint16_t *v_cache;
  const int32_t *block_tables;
  const int32_t *context_lens;
  uint16_t *out;
  float *ws_acc;  // [S][Hq][n_part_max][D] un-normalised partial outputs
  float2 *ws_ml;  // [S][Hq][n_part_max] (running max in log2 units, running sum)
  long long num_blocks, q_seq_stride, out_seq_stride, n_slots;
  unsigned long long wait_limit_ns;
  float scale_log2;  // scale * log2(e): logits are kept in base-2 units
  int num_seqs, num_q_heads, num_kv_heads, block_size, table_stride;
  int max_context_len, part_tokens, n_part_max, group, n_chunks;
  int heads_per_unit;  // query heads sharing one kv head handled by one unit (group / n_chunks)
};

__device__ __forceinline__ bool context_ok(const DecodeArgs &a, int L) {
  return L >= 0 && (long long)L <= (long long)a.table_stride * a.block_size && L <= a.max_context_len;
}

// One work unit: partition p of sequence s, kv head h, query heads
// hq0 .. hq0 + heads_per_unit - 1.
struct Unit {
  int s, h, p, hq0, L, tok_begin, tok_end, blk_begin, nblk;
  bool work;  // context valid and non-empty: tiles to stream
};

// A warp's static, strided list of unit slots.  Slot order is partition
// index outermost, then sequence, kv head, query-head chunk; slot p of a
// sequence is empty when p * part_tokens >= L (slot p = 0 always exists: it
// zeroes the rows of empty or invalid sequences).
struct UnitList {
  long long base, nwarps, per_part, per_seq;
  int lane;

  __device__ __forceinline__ UnitList(const DecodeArgs &a, int warps_per_block) {
    lane = threadIdx.x & 31;
    nwarps = (long long)gridDim.x * warps_per_block;
    per_seq = (long long)a.num_kv_heads * a.n_chunks;
    per_part = (long long)a.num_seqs * per_seq;
    base = (long long)blockIdx.x * warps_per_block + (threadIdx.x >> 5);
  }

  // Next non-empty slot (32 candidates per step, one per lane); -1 when none is left.
  __device__ __forceinline__ long long next(const DecodeArgs &a, int &L_out) {
    while (base < a.n_slots) {
      const long long c = base + (long long)lane * nwarps;
      bool live = false;
      int Lc = 0;
      if (c < a.n_slots) {
        const int p = (int)(c / per_part);
        const int s = (int)((c - (long long)p * per_part) / per_seq);
        Lc = __ldg(a.context_lens + s);
        live = (p == 0) || (context_ok(a, Lc) && (long long)p * a.part_tokens < Lc);
      }
      const unsigned m = __ballot_sync(FULL, live);
      if (m) {
        const int idx = __ffs(m) - 1;
        L_out = __shfl_sync(FULL, Lc, idx);
        const long long slot = base + (long long)idx * nwarps;
        base = slot + nwarps;
        return slot;
      }
      base += 32LL * nwarps;
    }
    return -1;
  }

  __device__ __forceinline__ Unit describe(const DecodeArgs &a, long long slot, int L) const {
    Unit u;
    u.p = (int)(slot / per_part);
    long long rem = slot - (long long)u.p * per_part;
    u.s = (int)(rem / per_seq);
    rem -= (long long)u.s * per_seq;
    u.h = (int)(rem / a.n_chunks);
    u.hq0 = u.h * a.group + (int)(rem - (long long)u.h * a.n_chunks) * a.heads_per_unit;
    u.L = L;
    u.work = context_ok(a, L) && L > 0;
    u.tok_begin = u.p * a.part_tokens;
    u.tok_end = u.work ? min(L, u.tok_begin + a.part_tokens) : u.tok_begin;
    u.blk_begin = u.tok_begin / a.block_size;
    u.nblk = (u.tok_end - u.tok_begin + a.block_size - 1) / a.block_size;  // <= 32
    return u;
  }
};

// The unit's table entry for this lane (block blk_begin + lane), or 0.
__device__ __forceinline__ int unit_table_entry(const DecodeArgs &a, const Unit &u, int lane) {
  return (u.work && lane < u.nblk) ? __ldg(a.block_tables + (long long)u.s * a.table_stride + u.blk_begin + lane) : 0;
}

// Status bits and zero rows for a unit that streams nothing (empty or invalid
// context, or a table entry outside the pool).
__device__ __forceinline__ void unit_without_tiles(const DecodeArgs &a, const Unit &u, bool bad_entry, int lane,
                                                   int D) {
  const int n_parts = u.work ? (u.L + a.part_tokens - 1) / a.part_tokens : 1;
  if (lane == 0) {
    if (!u.work && u.L != 0)
      atomicOr(&g_status, (u.L < 0 || (long long)u.L > (long long)a.table_stride * a.block_size)
                              ? PA_DEV_ERR_CONTEXT
                              : PA_DEV_ERR_CONTEXT_HINT);
    if (u.work && bad_entry) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
  }
  if (n_parts == 1) {
    for (int i = lane; i < a.heads_per_unit * D / 8; i += 32) {
      const int gg = i / (D / 8), c = i - gg * (D / 8);
      *reinterpret_cast<uint4 *>(a.out + (long long)u.s * a.out_seq_stride + (long long)(u.hq0 + gg) * D + c * 8) =
          make_uint4(0, 0, 0, 0);
    }
  } else if (lane < a.heads_per_unit) {
    // a partial marked invalid: the merge kernel zeroes the row
    a.ws_ml[((long long)u.s * a.num_q_heads + u.hq0 + lane) * a.n_part_max + u.p] = make_float2(-INFINITY, -1.f);
  }
}

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

// Each warp is an independent worker: it walks its own static, strided list
// of work units (UnitList) and streams each unit's 16-token K/V tiles through
// a private STAGES-deep ring of shared-memory buffers filled by bulk copies.
// There is no block-level barrier.  Used for groups of G <= 2 query heads per
// kv head (CUDA cores).
//
// Per tile, lane l copies 16 bytes (8 head dims) of rows r*NGRP + l/LPR
// (r < R) of K and of V from the ring into registers, and the ring slot is
// refilled at once, before any arithmetic, so the copies in flight never wait
// on the math.  The next unit's table entries and query rows are loaded while
// the current unit runs.  QK^T uses the mixed-precision fma (2-byte inputs,
// fp32 accumulation); the 16 dot products are finished by a reduce-scatter
// butterfly.  The online softmax keeps, per query head, a running maximum m
// that is raised only when a logit exceeds it by more than RESCALE_SLACK
// (base-2 units), so most tiles need no max reduction; m cancels between the
// numerator and the denominator, and the weights stay below 2^RESCALE_SLACK.
constexpr float RESCALE_SLACK = 8.f;

template <class E, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32) decode_partition_kernel(const DecodeArgs a) {
  constexpr int LPR = D / 8;       // lanes covering one K/V row
  constexpr int NGRP = 32 / LPR;   // rows one warp-wide 16-byte load covers
  constexpr int R = TILE / NGRP;   // rows per lane per tile
  constexpr uint32_t TILE_BYTES = TILE * D * 2;
  constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;
  constexpr int BAR_BYTES = ((WARPS * STAGES * 8 + 127) / 128) * 128;

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem) + warp * STAGES;
  unsigned char *ring = smem + BAR_BYTES + warp * STAGES * STAGE_BYTES;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const int grp = lane / LPR;
  const int cl = lane % LPR;
  const int my_tok = ((lane & (LPR - 2)) >> 1) * NGRP + grp;  // token whose logit this lane ends with
  uint32_t iter = 0;  // tiles consumed by this warp so far: ring slot iter % STAGES, phase (iter / STAGES) & 1

  UnitList list(a, WARPS);
  auto fetch_q = [&](const Unit &u, uint4 (&qraw)[G]) {
#pragma unroll
    for (int gg = 0; gg < G; ++gg)
      qraw[gg] = u.work ? __ldg(reinterpret_cast<const uint4 *>(a.q + (long long)u.s * a.q_seq_stride +
                                                                (long long)(u.hq0 + gg) * D + cl * 8))
                        : make_uint4(0, 0, 0, 0);
  };

  int L0 = 0;
  const long long first = list.next(a, L0);
  if (first < 0) return;
  Unit cur = list.describe(a, first, L0);
  int ent = unit_table_entry(a, cur, lane);
  uint4 qraw[G];
  fetch_q(cur, qraw);

  while (true) {
    const int n_parts = cur.work ? (cur.L + a.part_tokens - 1) / a.part_tokens : 1;
    const int ntiles = (cur.tok_end - cur.tok_begin + TILE - 1) / TILE;
    const bool bad = __any_sync(FULL, cur.work && lane < cur.nblk && (ent < 0 || (long long)ent >= a.num_blocks));

    // ---- issue one tile: K and V rows [tok0, tok0 + 16) of (block, h) into ring slot it % STAGES
    auto issue = [&](int j, uint32_t it) {
      const int tok0 = cur.tok_begin + j * TILE;
      const int phys = __shfl_sync(FULL, ent, tok0 / a.block_size - cur.blk_begin);
      if (lane == 0) {
        const int st = (int)(it % STAGES);
        const long long row0 = ((long long)phys * a.num_kv_heads + cur.h) * a.block_size + (tok0 % a.block_size);
        unsigned char *dst = ring + st * STAGE_BYTES;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[st], STAGE_BYTES);
        bulk_copy_g2s(dst, a.k_cache + row0 * D, TILE_BYTES, &bars[st]);
        bulk_copy_g2s(dst + TILE_BYTES, a.v_cache + row0 * D, TILE_BYTES, &bars[st]);
      }
    };
    const int npro = (cur.work && !bad) ? min(ntiles, STAGES) : 0;
    for (int j = 0; j < npro; ++j) issue(j, iter + j);

    // ---- look up and prefetch the next unit while those copies are in flight
    int Ln = 0;
    const long long nslot = list.next(a, Ln);
    Unit nxt = cur;
    int ent_n = 0;
    uint4 qraw_n[G];
    if (nslot >= 0) {
      nxt = list.describe(a, nslot, Ln);
      ent_n = unit_table_entry(a, nxt, lane);
      fetch_q(nxt, qraw_n);
    }

    if (!cur.work || bad) {
      unit_without_tiles(a, cur, bad, lane, D);
    } else {
      uint16_t *out_row = a.out + (long long)cur.s * a.out_seq_stride + (long long)cur.hq0 * D + cl * 8;
      uint32_t qw[G][4];
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        qw[gg][0] = qraw[gg].x;
        qw[gg][1] = qraw[gg].y;
        qw[gg][2] = qraw[gg].z;
        qw[gg][3] = qraw[gg].w;
      }
      float m[G], lsum[G];
      float2 acc[G][4];
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        m[gg] = -INFINITY;
        lsum[gg] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[gg][k] = make_float2(0.f, 0.f);
      }

      for (int j = 0; j < ntiles; ++j) {
        const int st = (int)(iter % STAGES);
        const uint32_t parity = (iter / STAGES) & 1u;
        const bool arrived = mbar_wait_bounded(&bars[st], parity, a.wait_limit_ns);
        if (__any_sync(FULL, !arrived)) {
          // A copy never landed: report, let every copy still in flight finish (bounded), stop.
          if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
          const int last = min(ntiles, j + STAGES);
          for (int jj = j; jj < last; ++jj) {
            const uint32_t it = iter + (jj - j);
            mbar_wait_bounded(&bars[it % STAGES], (it / STAGES) & 1u, a.wait_limit_ns);
          }
          return;
        }
        // copy this lane's rows out of the ring, then hand the slot straight back to the copy engine
        const unsigned char *kt = ring + st * STAGE_BYTES;
        const unsigned char *vt = kt + TILE_BYTES;
        uint4 kr[R], vr[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          kr[r] = *reinterpret_cast<const uint4 *>(kt + ((r * NGRP + grp) * D + cl * 8) * 2);
          vr[r] = *reinterpret_cast<const uint4 *>(vt + ((r * NGRP + grp) * D + cl * 8) * 2);
        }
        __syncwarp();
        if (j + STAGES < ntiles) issue(j + STAGES, iter + STAGES);
        ++iter;
        const int nvalid = min(TILE, cur.tok_end - (cur.tok_begin + j * TILE));
        const bool tok_live = my_tok < nvalid;

        // QK^T for this lane's R rows, the butterfly, scale, mask
        float z[G];
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          float part[R];
#pragma unroll
          for (int r = 0; r < R; ++r) part[r] = E::dot8(qw[gg], kr[r], 0.f);
          const float t = row_group_reduce<R>(part, lane) * a.scale_log2;
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
            const float alpha = exp2f(m[gg] - mt);  // 0 on the first tile (m = -inf)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[gg][k] = make_float2(acc[gg][k].x * alpha, acc[gg][k].y * alpha);
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
            for (int k = 0; k < 8; ++k) vf[k] = row_live ? vf[k] : 0.f;
          }
#pragma unroll
          for (int gg = 0; gg < G; ++gg) {
            const float2 pp = make_float2(pr[gg][r], pr[gg][r]);
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[gg][k] = __ffma2_rn(pp, make_float2(vf[2 * k], vf[2 * k + 1]), acc[gg][k]);
          }
        }
      }

      // ---- merge the row groups, total the running sums, store
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            acc[gg][k].x += __shfl_xor_sync(FULL, acc[gg][k].x, off);
            acc[gg][k].y += __shfl_xor_sync(FULL, acc[gg][k].y, off);
          }
        }
        float l = lsum[gg];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) l += __shfl_xor_sync(FULL, l, off);
        lsum[gg] = l;
      }
      if (n_parts == 1) {
        if (lane < LPR) {
#pragma unroll
          for (int gg = 0; gg < G; ++gg) {
            float o[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              o[2 * k] = acc[gg][k].x / lsum[gg];
              o[2 * k + 1] = acc[gg][k].y / lsum[gg];
            }
            *reinterpret_cast<uint4 *>(out_row + gg * D) = narrow8<E>(o);
          }
        }
      } else {
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          const long long prow = ((long long)cur.s * a.num_q_heads + cur.hq0 + gg) * a.n_part_max + cur.p;
          if (lane < LPR) {
            float4 *dst = reinterpret_cast<float4 *>(a.ws_acc + prow * D + cl * 8);
            dst[0] = make_float4(acc[gg][0].x, acc[gg][0].y, acc[gg][1].x, acc[gg][1].y);
            dst[1] = make_float4(acc[gg][2].x, acc[gg][2].y, acc[gg][3].x, acc[gg][3].y);
          }
          if (lane == 0) a.ws_ml[prow] = make_float2(m[gg], lsum[gg]);
        }
      }
    }

    if (nslot < 0) break;
    cur = nxt;
    ent = ent_n;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) qraw[gg] = qraw_n[gg];
  }
}

// One warp per (sequence, query head) whose context spans more than one
// partition: out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p with
// M = max_p m_p, in increasing p order (deterministic).
template <class E, int D>
__global__ void __launch_bounds__(256) decode_reduce_kernel(const DecodeArgs a) {
  constexpr int DPL = D / 32;  // dims per lane (4 or 2)
  const int lane = threadIdx.x & 31;
  const long long total = (long long)a.num_seqs * a.num_q_heads;
  const long long nw = (long long)gridDim.x * (blockDim.x / 32);
  for (long long w = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); w < total; w += nw) {
    const int s = (int)(w / a.num_q_heads);
    const int L = __ldg(a.context_lens + s);
    if (L <= 0 || !context_ok(a, L)) continue;
    const int n = (L + a.part_tokens - 1) / a.part_tokens;
    if (n <= 1) continue;
    const long long row0 = w * a.n_part_max;
    float M = -INFINITY;
    bool err = false;
    for (int p = lane; p < n; p += 32) {
      const float2 ml = a.ws_ml[row0 + p];
      M = fmaxf(M, ml.x);
      err |= ml.y < 0.f;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
    err = __any_sync(FULL, err);
    float o[DPL];
#pragma unroll
    for (int k = 0; k < DPL; ++k) o[k] = 0.f;
    if (!err) {
      float l = 0.f;
#pragma unroll 4
      for (int p = 0; p < n; ++p) {
        const float2 ml = a.ws_ml[row0 + p];
        const float wgt = exp2f(ml.x - M);
        l = fmaf(ml.y, wgt, l);
        const float *src = a.ws_acc + (row0 + p) * D + lane * DPL;
        float v[DPL];
        if constexpr (DPL == 4) {
          const float4 t = *reinterpret_cast<const float4 *>(src);
          v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2 *>(src);
          v[0] = t.x; v[1] = t.y;
        }
#pragma unroll
        for (int k = 0; k < DPL; ++k) o[k] = fmaf(wgt, v[k], o[k]);
      }
#pragma unroll
      for (int k = 0; k < DPL; ++k) o[k] = o[k] / l;
    }
    uint16_t *dst = a.out + (long long)s * a.out_seq_stride + (long long)(w - (long long)s * a.num_q_heads) * D +
                    lane * DPL;
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint2 *>(dst) = make_uint2(E::narrow2(o[0], o[1]), E::narrow2(o[2], o[3]));
    } else {
      *reinterpret_cast<uint32_t *>(dst) = E::narrow2(o[0], o[1]);
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
