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
struct F16 {
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
};

__device__ __forceinline__ bool context_ok(const DecodeArgs &a, int L) {
  return L >= 0 && (long long)L <= (long long)a.table_stride * a.block_size && L <= a.max_context_len;
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

// Each warp is an independent worker: it walks its own list of work units
// (sequence s, kv head h, query-head chunk ch, partition p) and streams the
// unit's 16-token K/V tiles through a private STAGES-deep ring of shared
// memory buffers filled by bulk copies.  There is no block-level barrier.
//
// Within a tile, lane l reads 16 bytes (8 head dims) of rows
// r*NGRP + l/LPR (r < R) of K and of V; q lives in registers as fp32 pre-
// multiplied by scale*log2(e).  The online softmax keeps a running max m,
// running sum and un-normalised output per query head.
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

  const long long nwarps = (long long)gridDim.x * WARPS;
  const long long per_part = (long long)a.num_seqs * a.num_kv_heads * a.n_chunks;
  const long long per_seq = (long long)a.num_kv_heads * a.n_chunks;
  long long base = (long long)blockIdx.x * WARPS + warp;
  uint32_t iter = 0;  // tiles consumed by this warp so far: ring slot iter % STAGES, phase (iter / STAGES) & 1

  while (true) {
    // ---- next non-empty unit of this warp's static list, 32 candidates per step
    long long slot = -1;
    while (base < a.n_slots) {
      const long long c = base + (long long)lane * nwarps;
      bool live = false;
      if (c < a.n_slots) {
        const int p = (int)(c / per_part);
        const int s = (int)((c - (long long)p * per_part) / per_seq);
        const int L = __ldg(a.context_lens + s);
        live = (p == 0) || (context_ok(a, L) && (long long)p * a.part_tokens < L);
      }
      const unsigned m = __ballot_sync(FULL, live);
      if (m) {
        slot = base + (long long)(__ffs(m) - 1) * nwarps;
        base = slot + nwarps;
        break;
      }
      base += 32LL * nwarps;
    }
    if (slot < 0) break;

    const int p = (int)(slot / per_part);
    long long rem = slot - (long long)p * per_part;
    const int s = (int)(rem / per_seq);
    rem -= (long long)s * per_seq;
    const int h = (int)(rem / a.n_chunks);
    const int ch = (int)(rem - (long long)h * a.n_chunks);
    const int hq0 = h * a.group + ch * G;
    const int L = __ldg(a.context_lens + s);
    uint16_t *out_row = a.out + (long long)s * a.out_seq_stride + (long long)hq0 * D + cl * 8;

    if (!context_ok(a, L) || L == 0) {  // only the p == 0 unit reaches here
      if (lane == 0 && L != 0)
        atomicOr(&g_status, (L < 0 || (long long)L > (long long)a.table_stride * a.block_size)
                                ? PA_DEV_ERR_CONTEXT
                                : PA_DEV_ERR_CONTEXT_HINT);
      if (lane < LPR) {
#pragma unroll
        for (int gg = 0; gg < G; ++gg) *reinterpret_cast<uint4 *>(out_row + gg * D) = make_uint4(0, 0, 0, 0);
      }
      continue;
    }

    const int n_parts = (L + a.part_tokens - 1) / a.part_tokens;
    const int tok_begin = p * a.part_tokens;
    const int tok_end = min(L, tok_begin + a.part_tokens);
    const int ntiles = (tok_end - tok_begin + TILE - 1) / TILE;
    const int blk_begin = tok_begin / a.block_size;
    const int nblk = (tok_end - tok_begin + a.block_size - 1) / a.block_size;  // <= 32

    // ---- this unit's table entries, one per lane; validated before any copy
    int ent = 0;
    bool bad = false;
    if (lane < nblk) {
      ent = __ldg(a.block_tables + (long long)s * a.table_stride + blk_begin + lane);
      bad = ent < 0 || (long long)ent >= a.num_blocks;
    }
    if (__any_sync(FULL, bad)) {
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
      if (n_parts == 1) {
        if (lane < LPR) {
#pragma unroll
          for (int gg = 0; gg < G; ++gg) *reinterpret_cast<uint4 *>(out_row + gg * D) = make_uint4(0, 0, 0, 0);
        }
      } else if (lane == 0) {
#pragma unroll
        for (int gg = 0; gg < G; ++gg)
          a.ws_ml[((long long)s * a.num_q_heads + hq0 + gg) * a.n_part_max + p] = make_float2(-INFINITY, -1.f);
      }
      continue;
    }

    // ---- issue one tile: K and V rows [tok0, tok0 + 16) of (block, h) into ring slot it % STAGES
    auto issue = [&](int j, uint32_t it) {
      const int tok0 = tok_begin + j * TILE;
      const int phys = __shfl_sync(FULL, ent, tok0 / a.block_size - blk_begin);
      if (lane == 0) {
        const int st = (int)(it % STAGES);
        const long long row0 = ((long long)phys * a.num_kv_heads + h) * a.block_size + (tok0 % a.block_size);
        unsigned char *dst = ring + st * STAGE_BYTES;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[st], STAGE_BYTES);
        bulk_copy_g2s(dst, a.k_cache + row0 * D, TILE_BYTES, &bars[st]);
        bulk_copy_g2s(dst + TILE_BYTES, a.v_cache + row0 * D, TILE_BYTES, &bars[st]);
      }
    };
    const int npro = ntiles < STAGES ? ntiles : STAGES;
    for (int j = 0; j < npro; ++j) issue(j, iter + j);

    // ---- query rows (fp32, pre-scaled into base-2 logits)
    float qf[G][8];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      const uint4 w = __ldg(reinterpret_cast<const uint4 *>(a.q + (long long)s * a.q_seq_stride +
                                                            (long long)(hq0 + gg) * D + cl * 8));
      E::widen8(w, qf[gg]);
#pragma unroll
      for (int k = 0; k < 8; ++k) qf[gg][k] *= a.scale_log2;
    }

    float m[G], lsum[G], acc[G][8];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
      m[gg] = -INFINITY;
      lsum[gg] = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[gg][k] = 0.f;
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
      const unsigned char *kt = ring + st * STAGE_BYTES;
      const unsigned char *vt = kt + TILE_BYTES;
      const int nvalid = min(TILE, tok_end - (tok_begin + j * TILE));

      // QK^T: partial dots of this lane's 8 dims for its R rows, then the butterfly
      float part[G][R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint4 kw = *reinterpret_cast<const uint4 *>(kt + ((r * NGRP + grp) * D + cl * 8) * 2);
        float kf[8];
        E::widen8(kw, kf);
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          float dot = qf[gg][0] * kf[0];
#pragma unroll
          for (int k = 1; k < 8; ++k) dot = fmaf(qf[gg][k], kf[k], dot);
          part[gg][r] = dot;
        }
      }
      const bool tok_live = my_tok < nvalid;
      float pr[G][R];
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        float z = row_group_reduce<R>(part[gg], lane);
        z = tok_live ? z : -INFINITY;
        float mt = z;
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 2));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 4));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 8));
        mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 16));
        if (mt > m[gg]) {  // warp-uniform: every lane holds the same mt and m
          const float alpha = exp2f(m[gg] - mt);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[gg][k] *= alpha;
          lsum[gg] *= alpha;
          m[gg] = mt;
        }
        const float pz = exp2f(z - m[gg]);
        lsum[gg] += (lane & 1) ? 0.f : pz;
#pragma unroll
        for (int r = 0; r < R; ++r) pr[gg][r] = __shfl_sync(FULL, pz, grp * LPR + 2 * r);
      }

      // P.V: accumulate this lane's 8 dims over its R rows
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint4 vw = *reinterpret_cast<const uint4 *>(vt + ((r * NGRP + grp) * D + cl * 8) * 2);
        float vf[8];
        E::widen8(vw, vf);
        if (nvalid < TILE) {  // rows past the sequence may hold anything (NaN): never let them in
          const bool row_live = (r * NGRP + grp) < nvalid;
#pragma unroll
          for (int k = 0; k < 8; ++k) vf[k] = row_live ? vf[k] : 0.f;
        }
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[gg][k] = fmaf(pr[gg][r], vf[k], acc[gg][k]);
        }
      }
      __syncwarp();
      if (j + STAGES < ntiles) issue(j + STAGES, iter + STAGES);
      ++iter;
    }

    // ---- merge the row groups, total the running sums
#pragma unroll
    for (int gg = 0; gg < G; ++gg) {
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[gg][k] += __shfl_xor_sync(FULL, acc[gg][k], off);
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
          for (int k = 0; k < 8; ++k) o[k] = acc[gg][k] / lsum[gg];
          *reinterpret_cast<uint4 *>(out_row + gg * D) = narrow8<E>(o);
        }
      }
    } else {
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        const long long prow = ((long long)s * a.num_q_heads + hq0 + gg) * a.n_part_max + p;
        if (lane < LPR) {
          float4 *dst = reinterpret_cast<float4 *>(a.ws_acc + prow * D + cl * 8);
          dst[0] = make_float4(acc[gg][0], acc[gg][1], acc[gg][2], acc[gg][3]);
          dst[1] = make_float4(acc[gg][4], acc[gg][5], acc[gg][6], acc[gg][7]);
        }
        if (lane == 0) a.ws_ml[prow] = make_float2(m[gg], lsum[gg]);
      }
    }
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
