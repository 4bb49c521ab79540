// Causal prefill / chunked-prefill attention through the page table on the
// sm_100a tensor cores ("4. vLLM核心机制" section 4.3: the prompt's tokens
// enter the cache before decoding, possibly a chunk per iteration).
//
// One CTA computes 128 consecutive new tokens of one sequence for one query
// head.  Per key tile of 128 tokens (8 pages of 16 or 4 of 32):
//   S = Q K^T      tcgen05.mma M=128 N=128 K=d, Q and K tiles in swizzled smem,
//                  S in tensor memory (two buffers, so the next tile's S is
//                  computed while this one's softmax runs);
//   softmax        4 warps, one row each: S read from tensor memory, causal
//                  mask, online max with a lazy rescale of O, P rounded to the
//                  storage type and written to smem in the MMA's swizzled layout;
//   O += P V       tcgen05.mma M=128 N=d K=128, V read MN-major straight from
//                  its TMA tile, O accumulated in tensor memory.
// Warp roles: 0-3 softmax and epilogue, 4 TMA producer (Q once, then K/V
// pages through the table into a STAGES-deep ring), 5 MMA issue (one lane).
// Every wait is bounded: on a timeout the CTA flags PA_DEV_ERR_TIMEOUT, drains
// its copies and MMAs in flight, frees its tensor memory and returns.
#pragma once

#include <cuda.h>

#include <cstdint>
#include <type_traits>

#include "pa_kernels.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

struct PrefillArgs {
  const int32_t *block_tables;
  const int32_t *query_start;   // [num_seqs + 1]
  const int32_t *context_lens;  // [num_seqs], new tokens included
  uint16_t *out;                // [num_query_tokens][num_q_heads][head_dim]
  long long num_blocks, out_token_stride, num_query_tokens;
  unsigned long long wait_limit_ns;
  float scale_log2;
  int num_seqs, num_q_heads, num_kv_heads, block_size, table_stride, q_tiles;
};

constexpr int PF_BM = 128;  // query rows per CTA
constexpr int PF_BN = 128;  // keys per tile
constexpr int PF_THREADS = 192;
constexpr uint32_t PF_TMEM_COLS = 512;  // S double buffer (2 x 128) + O (<= 128), rounded to a power of two

template <int D, int STAGES>
struct PrefillSmem {
  static constexpr uint32_t REGION = 128 * 128;  // 128 rows of 128 bytes (64 elements)
  static constexpr uint32_t HALVES = D / 64;
  static constexpr uint32_t Q = 0;
  static constexpr uint32_t K = Q + HALVES * REGION;
  static constexpr uint32_t V = K + STAGES * HALVES * REGION;
  static constexpr uint32_t P = V + STAGES * HALVES * REGION;
  static constexpr uint32_t BARS = P + 2 * REGION;
  static constexpr uint32_t BYTES = BARS + 256;
  // + alignment slack; at least 120 KB so that one CTA holds an SM (and its tensor memory) alone
  static constexpr uint32_t ALLOC = (BYTES + 1024 > 120 * 1024) ? BYTES + 1024 : 120 * 1024;
};

// All lanes wait on the same barrier phase; the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned long long limit_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, limit_ns);
  return __all_sync(FULL, ok);
}

template <class E, int D, int STAGES>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const PrefillArgs a) {
  using L = PrefillSmem<D, STAGES>;
  constexpr int HALVES = D / 64;
  constexpr uint32_t REGION = L::REGION;
  constexpr bool kBf16 = std::is_same<E, BF16>::value;

  grid_dependency_wait();  // inputs may come from the previous kernel in the stream
  const int s = blockIdx.z, hq = blockIdx.y;
  const int qt = a.q_tiles - 1 - (int)blockIdx.x;  // late (heavier) query tiles first
  const int q0 = a.query_start[s];
  const int n = a.query_start[s + 1] - q0;
  const int ctx = a.context_lens[s];
  if (q0 < 0 || n < 0 || (long long)q0 + n > a.num_query_tokens) {  // rows outside q / out: write nothing
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) atomicOr(&g_status, PA_DEV_ERR_CONTEXT);
    return;
  }
  if (n == 0 || qt * PF_BM >= n) return;
  const int t0 = qt * PF_BM;
  const int rows = min(PF_BM, n - t0);
  if (ctx < n || (long long)ctx > (long long)a.table_stride * a.block_size) {
    if (threadIdx.x == 0) atomicOr(&g_status, PA_DEV_ERR_CONTEXT);
    for (int i = threadIdx.x; i < rows * (D / 8); i += blockDim.x) {
      const int r = i / (D / 8), c = i % (D / 8);
      *reinterpret_cast<uint4 *>(a.out + (long long)(q0 + t0 + r) * a.out_token_stride + (long long)hq * D + c * 8) =
          make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const int pos0 = ctx - n + t0;           // logical position of row 0
  const int kmax = min(ctx, pos0 + rows);  // keys [0, kmax) are visible to some row
  const int nt = (kmax + PF_BN - 1) / PF_BN;
  const int h = hq / (a.num_q_heads / a.num_kv_heads);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t *sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_addr(sm);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
  uint64_t *q_full = bars;
  uint64_t *k_full = bars + 1;
  uint64_t *v_full = k_full + STAGES;
  uint64_t *kv_empty = v_full + STAGES;
  uint64_t *s_full = kv_empty + STAGES;
  uint64_t *p_full = s_full + 2;
  uint64_t *o_done = p_full + 1;
  uint64_t *drained = o_done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drained + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *bad_pages = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drained, 1);
    *abort_flag = 0;
    *bad_pages = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tc::alloc(tmem_slot, PF_TMEM_COLS);
    tc::relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const unsigned long long limit = a.wait_limit_ns;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    const int bs = a.block_size;
    const int ppt = PF_BN / bs;  // pages per key tile
    int last_issued[STAGES];
#pragma unroll
    for (int i = 0; i < STAGES; ++i) last_issued[i] = -1;
    if (lane == 0) {
      prefetch_tensor_map(&tmap_q);
      prefetch_tensor_map(&tmap_k);
      prefetch_tensor_map(&tmap_v);
      mbar_arrive_expect_tx(q_full, PF_BM * D * 2);
#pragma unroll
      for (int hh = 0; hh < HALVES; ++hh) tc::tma_load_3d(sm + L::Q + hh * REGION, &tmap_q, hh * 64, hq, q0 + t0, q_full);
    }
    for (int j = 0; j < nt; ++j) {
      const int st = j % STAGES;
      if (j >= STAGES && !warp_wait(&kv_empty[st], ((j / STAGES) - 1) & 1, limit)) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      if (__any_sync(FULL, *abort_flag != 0)) break;
      const int page = j * ppt + lane;
      int blk = -1;
      bool bad = false;
      if (lane < ppt && page * bs < kmax) {
        blk = a.block_tables[(long long)s * a.table_stride + page];
        if (blk < 0 || (long long)blk >= a.num_blocks) {
          bad = true;
          blk = -1;
        }
      }
      if (__any_sync(FULL, bad) && lane == 0) {
        *bad_pages = 1;
        atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
      }
      const unsigned loaded = __ballot_sync(FULL, blk >= 0);
      int ids[PF_BN / 16];
#pragma unroll
      for (int p = 0; p < PF_BN / 16; ++p) ids[p] = __shfl_sync(FULL, blk, p);
      if (lane == 0) {
        const uint32_t bytes = (uint32_t)__popc(loaded) * bs * 128u * HALVES;
        const int boxes = bs / TILE;
        uint8_t *kdst = sm + L::K + st * HALVES * REGION;
        uint8_t *vdst = sm + L::V + st * HALVES * REGION;
        mbar_arrive_expect_tx(&k_full[st], bytes);
        for (int p = 0; p < ppt; ++p) {
          if (!((loaded >> p) & 1u)) continue;
          const long long row = ((long long)ids[p] * a.num_kv_heads + h) * bs;
          for (int hh = 0; hh < HALVES; ++hh)
            for (int b = 0; b < boxes; ++b)
              tma_load_2d(kdst + hh * REGION + (p * bs + b * TILE) * 128, &tmap_k, hh * 64, (int)(row + b * TILE),
                          &k_full[st]);
        }
        mbar_arrive_expect_tx(&v_full[st], bytes);
        for (int p = 0; p < ppt; ++p) {
          if (!((loaded >> p) & 1u)) continue;
          const long long row = ((long long)ids[p] * a.num_kv_heads + h) * bs;
          for (int hh = 0; hh < HALVES; ++hh)
            for (int b = 0; b < boxes; ++b)
              tma_load_2d(vdst + hh * REGION + (p * bs + b * TILE) * 128, &tmap_v, hh * 64, (int)(row + b * TILE),
                          &v_full[st]);
        }
      }
      last_issued[st] = j;
    }
    // Every copy this warp started has landed before the CTA's smem is given back.
    bool ok = warp_wait(q_full, 0, limit);
#pragma unroll
    for (int i = 0; i < STAGES; ++i)
      if (last_issued[i] >= 0) {
        ok = warp_wait(&k_full[i], (last_issued[i] / STAGES) & 1, limit) && ok;
        ok = warp_wait(&v_full[i], (last_issued[i] / STAGES) & 1, limit) && ok;
      }
    if (!ok && lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_f16(kBf16, false, PF_BM, PF_BN);
      constexpr uint32_t idesc_pv = tc::idesc_f16(kBf16, true, PF_BM, D);
      const uint32_t qs = sbase + L::Q, ps = sbase + L::P;
      bool ok = mbar_wait_bounded(q_full, 0, limit);
      for (int j = 0; ok && j <= nt; ++j) {
        if (*abort_flag) break;
        if (j < nt) {
          const int st = j % STAGES;
          if (!(ok = mbar_wait_bounded(&k_full[st], (j / STAGES) & 1, limit))) break;
          tc::fence_after_sync();
          const uint32_t ks = sbase + L::K + st * HALVES * REGION;
          const uint32_t d = tmem + (uint32_t)(j & 1) * PF_BN;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k / 4) * REGION + (k % 4) * 32;
            tc::mma_ss(d, tc::desc_sw128(qs + off, 16, 1024), tc::desc_sw128(ks + off, 16, 1024), idesc_qk, k > 0);
          }
          tc::commit(&s_full[j & 1]);
        }
        if (j >= 1) {
          const int jj = j - 1, st = jj % STAGES;
          if (!(ok = mbar_wait_bounded(p_full, jj & 1, limit))) break;
          if (!(ok = mbar_wait_bounded(&v_full[st], (jj / STAGES) & 1, limit))) break;
          tc::fence_after_sync();
          const uint32_t vs = sbase + L::V + st * HALVES * REGION;
#pragma unroll
          for (int k = 0; k < PF_BN / 16; ++k) {
            const uint32_t a_off = (k / 4) * REGION + (k % 4) * 32;
            tc::mma_ss(tmem + 2 * PF_BN, tc::desc_sw128(ps + a_off, 16, 1024),
                       tc::desc_sw128(vs + k * 16 * 128, REGION, 1024), idesc_pv, jj > 0 || k > 0);
          }
          tc::commit(o_done);
          tc::commit(&kv_empty[st]);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
      }
      // Every MMA issued has finished before tensor memory and smem are released.
      tc::commit(drained);
      if (!mbar_wait_bounded(drained, 0, limit)) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3, one row per thread)
    const int r = warp * 32 + lane;
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;
    // last key this row sees; rows past the tile's tokens stop at kmax - 1 too, so that no row reads
    // a page the producer did not load
    const int vis = min(pos0 + r, kmax - 1);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      if (__any_sync(FULL, *abort_flag != 0)) {
        ok = false;
        break;
      }
      if (!(ok = warp_wait(&s_full[j & 1], (j >> 1) & 1, limit))) break;
      tc::fence_after_sync();
      float sv[PF_BN];
#pragma unroll
      for (int c = 0; c < PF_BN / 32; ++c) {
        float t[32];
        tc::ld32(tmem + lanes + (uint32_t)(j & 1) * PF_BN + c * 32, t);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = t[i];
      }
      tc::wait_ld();
      const int key0 = j * PF_BN;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < PF_BN; ++c) {
        const float x = (key0 + c <= vis) ? sv[c] * a.scale_log2 : -INFINITY;
        sv[c] = x;
        mx = fmaxf(mx, x);
      }
      const float m_new = fmaxf(m, mx);
      const bool need = m_new > m + RESCALE_SLACK;
      float factor = 1.f;
      if (need) {
        factor = exp2f(m - m_new);
        m = m_new;
      }
      uint32_t pk[PF_BN / 2];
      float rowsum = 0.f;
#pragma unroll
      for (int c = 0; c < PF_BN / 2; ++c) {
        pk[c] = E::narrow2(exp2f(sv[2 * c] - m), exp2f(sv[2 * c + 1] - m));
        float w[8];
        if (c % 4 == 3) {  // sum the rounded weights (the ones the MMA uses), 8 at a time
          E::widen8(make_uint4(pk[c - 3], pk[c - 2], pk[c - 1], pk[c]), w);
#pragma unroll
          for (int i = 0; i < 8; ++i) rowsum += w[i];
        }
      }
      const int st = j % STAGES;
      if (j == nt - 1 && key0 + PF_BN > kmax) {
        // V rows from kmax on are either past the context (whatever the pool
        // holds there, possibly NaN) or in pages this CTA never loaded (stale
        // smem); P is 0 for them but 0 * NaN is not, so they are zeroed.
        if (!(ok = warp_wait(&v_full[st], (j / STAGES) & 1, limit))) break;
        if (key0 + r >= kmax) {
#pragma unroll
          for (int hh = 0; hh < HALVES; ++hh) {
            uint4 *row = reinterpret_cast<uint4 *>(sm + L::V + (st * HALVES + hh) * REGION + r * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      if (j > 0) {
        if (!(ok = warp_wait(o_done, (j - 1) & 1, limit))) break;
        tc::fence_after_sync();
        if (__any_sync(FULL, need)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tc::ld32(tmem + lanes + 2 * PF_BN + c * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= factor;
            tc::st32(tmem + lanes + 2 * PF_BN + c * 32, o);
          }
          tc::wait_st();
        }
      }
      l = l * factor + rowsum;
      // P row r, 128-byte swizzle: 16-byte chunk c of a 128-byte row goes to chunk c ^ (r & 7).
#pragma unroll
      for (int c = 0; c < PF_BN / 8; ++c) {
        uint4 *dst = reinterpret_cast<uint4 *>(sm + L::P + (c / 8) * REGION + r * 128 + (((c % 8) ^ (r & 7)) * 16));
        *dst = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      mbar_arrive(p_full);
    }
    if (ok) ok = warp_wait(o_done, (nt - 1) & 1, limit);
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
    }
    tc::fence_before_sync();
    // the epilogue runs after the barrier below
    __syncthreads();
    tc::fence_after_sync();
    if (!*abort_flag) {  // uniform: read after the barrier
      uint16_t *dst = a.out + (long long)(q0 + t0 + r) * a.out_token_stride + (long long)hq * D;
      const bool zero = *bad_pages != 0;
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tc::ld32(tmem + lanes + 2 * PF_BN + c * 32, o);  // every lane: the load is warp-collective
        tc::wait_ld();
        if (r < rows) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = zero ? 0.f : o[i * 8 + e] * inv;
            *reinterpret_cast<uint4 *>(dst + c * 32 + i * 8) = narrow8<E>(f);
          }
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();
    return;
  }
  // producer and MMA warps
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc::fence_after_sync();
    tc::dealloc(tmem, PF_TMEM_COLS);
  }
}

}  // namespace pa
