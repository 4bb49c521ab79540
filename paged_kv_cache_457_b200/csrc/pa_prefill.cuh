// Causal prefill / chunked-prefill attention through the page table on the
// sm_100a tensor cores ("4. vLLM核心机制" section 4.3: the prompt's tokens
// enter the cache before decoding, possibly a chunk per iteration).
//
// Work item: 128 consecutive new tokens of one sequence for one query head.
// Persistent CTAs (one per SM) walk the items round-robin; the items of one
// (sequence, head) are adjacent, so the CTAs working on them at the same time
// share that head's K/V through L2, and the latest (heaviest) query tiles of
// a sequence come first.  Per key tile of 128 tokens (8 pages of 16 or 4 of 32):
//   S = Q K^T      tcgen05.mma M=128 N=128 K=d, Q and K tiles in swizzled smem,
//                  S in tensor memory (two buffers, so the next tile's S is
//                  computed while this one's softmax runs);
//   softmax        4 warps, one row each: S read from tensor memory, causal
//                  mask, online max with a lazy rescale of O, P rounded to the
//                  storage type and written to smem in the MMA's swizzled layout;
//   O += P V       tcgen05.mma M=128 N=d K=128, V read MN-major straight from
//                  its TMA tile, O accumulated in tensor memory.
// Warp roles: 0-3 softmax and epilogue, 4 TMA producer of Q (two buffers) and
// K pages, 5 MMA issue (one lane), 6 TMA producer of V pages.  A K slot frees
// when its QK^T has run, a V slot when its PV has, so K runs ahead of V.  The
// MMA lane keeps one software pipeline across items: QK^T of tile g, then PV
// of tile g-1.  Every wait is bounded: on a timeout the CTA flags
// PA_DEV_ERR_TIMEOUT, drains its copies and MMAs in flight, frees its tensor
// memory and returns.
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
  long long num_blocks, out_token_stride, num_query_tokens, num_items;
  unsigned long long wait_limit_ns;
  float scale_log2;
  int num_seqs, num_q_heads, num_kv_heads, block_size, table_stride, q_tiles;
};

constexpr int PF_BM = 128;  // query rows per item
constexpr int PF_BN = 128;  // keys per tile
constexpr int PF_THREADS = 224;
constexpr int PF_KST = 2;  // K ring
constexpr int PF_VST = 2;  // V ring
constexpr uint32_t PF_TMEM_COLS = 512;  // S double buffer (2 x 128) + O (<= 128), rounded to a power of two

template <int D>
struct PrefillSmem {
  static constexpr uint32_t REGION = 128 * 128;  // 128 rows of 128 bytes (64 elements)
  static constexpr uint32_t HALVES = D / 64;
  static constexpr uint32_t Q = 0;  // two buffers
  static constexpr uint32_t K = Q + 2 * HALVES * REGION;
  static constexpr uint32_t V = K + PF_KST * HALVES * REGION;
  static constexpr uint32_t P = V + PF_VST * HALVES * REGION;
  static constexpr uint32_t BARS = P + 2 * REGION;
  static constexpr uint32_t BYTES = BARS + 256;
  // + alignment slack; at least 120 KB so that one CTA holds an SM (and its tensor memory) alone
  static constexpr uint32_t ALLOC = (BYTES + 1024 > 120 * 1024) ? BYTES + 1024 : 120 * 1024;
};

// 2^x with the SFU's approximate exponential (documented PTX; relative error about 2^-22, 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// All lanes wait on the same barrier phase; the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned long long limit_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, limit_ns);
  return __all_sync(FULL, ok);
}

// One work item as every role sees it (all values uniform across the CTA).
struct PrefillItem {
  int s, hq, h, q0, t0, rows, ctx, pos0, kmax, nt;
  bool work, bad_ctx;
};

__device__ __forceinline__ PrefillItem prefill_item(const PrefillArgs &a, long long item) {
  PrefillItem it;
  const int per_seq = a.q_tiles * a.num_q_heads;
  it.s = (int)(item / per_seq);
  const int rem = (int)(item - (long long)it.s * per_seq);
  it.hq = rem / a.q_tiles;
  const int qt = a.q_tiles - 1 - rem % a.q_tiles;  // latest (heaviest) query tiles first
  it.h = it.hq / (a.num_q_heads / a.num_kv_heads);
  it.q0 = a.query_start[it.s];
  const int n = a.query_start[it.s + 1] - it.q0;
  it.ctx = a.context_lens[it.s];
  it.t0 = qt * PF_BM;
  it.work = false;
  it.bad_ctx = false;
  it.rows = it.pos0 = it.kmax = it.nt = 0;
  if (it.q0 < 0 || n < 0 || (long long)it.q0 + n > a.num_query_tokens) {  // rows outside q / out
    if (qt == a.q_tiles - 1 && it.hq == 0 && threadIdx.x == 0) atomicOr(&g_status, PA_DEV_ERR_CONTEXT);
    return it;
  }
  if (it.t0 >= n) return it;
  it.rows = min(PF_BM, n - it.t0);
  if (it.ctx < n || (long long)it.ctx > (long long)a.table_stride * a.block_size) {
    it.bad_ctx = true;
    return it;
  }
  it.work = true;
  it.pos0 = it.ctx - n + it.t0;              // logical position of row 0
  it.kmax = min(it.ctx, it.pos0 + it.rows);  // keys [0, kmax) are visible to some row
  it.nt = (it.kmax + PF_BN - 1) / PF_BN;
  return it;
}

// Page id of key tile j of an item for this lane (lanes >= pages per tile: -1);
// entries outside the pool count as missing and set *bad.
__device__ __forceinline__ int tile_page(const PrefillArgs &a, const PrefillItem &it, int j, int lane, bool *bad) {
  const int bs = a.block_size;
  const int page = j * (PF_BN / bs) + lane;
  int blk = -1;
  *bad = false;
  if (lane < PF_BN / bs && page * bs < it.kmax) {
    blk = a.block_tables[(long long)it.s * a.table_stride + page];
    if (blk < 0 || (long long)blk >= a.num_blocks) {
      *bad = true;
      blk = -1;
    }
  }
  return blk;
}

// Issues the TMA boxes of one key tile (K or V) into `dst`, completing on `bar`.
template <int HALVES>
__device__ __forceinline__ void load_tile(const PrefillArgs &a, const PrefillItem &it, int blk, int lane,
                                          uint8_t *dst, const CUtensorMap *map, uint64_t *bar) {
  const int bs = a.block_size;
  const unsigned loaded = __ballot_sync(FULL, blk >= 0);
  int ids[PF_BN / 16];
#pragma unroll
  for (int p = 0; p < PF_BN / 16; ++p) ids[p] = __shfl_sync(FULL, blk, p);
  if (lane == 0) {
    mbar_arrive_expect_tx(bar, (uint32_t)__popc(loaded) * bs * 128u * HALVES);
    for (int p = 0; p < PF_BN / bs; ++p) {
      if (!((loaded >> p) & 1u)) continue;
      const long long row = ((long long)ids[p] * a.num_kv_heads + it.h) * bs;
      for (int hh = 0; hh < HALVES; ++hh)
        for (int b = 0; b < bs / TILE; ++b)
          tma_load_2d(dst + hh * 128 * 128 + (p * bs + b * TILE) * 128, map, hh * 64, (int)(row + b * TILE), bar);
    }
  }
}

template <class E, int D>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v, const PrefillArgs a) {
  using L = PrefillSmem<D>;
  constexpr int HALVES = D / 64;
  constexpr uint32_t REGION = L::REGION;
  constexpr bool kBf16 = std::is_same<E, BF16>::value;

  grid_dependency_wait();  // inputs may come from the previous kernel in the stream

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  uint8_t *sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_addr(sm);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::BARS);
  uint64_t *q_full = bars;              // [2]
  uint64_t *q_empty = q_full + 2;       // [2]
  uint64_t *k_full = q_empty + 2;       // [PF_KST]
  uint64_t *k_empty = k_full + PF_KST;  // [PF_KST]
  uint64_t *v_full = k_empty + PF_KST;  // [PF_VST]
  uint64_t *v_empty = v_full + PF_VST;  // [PF_VST]
  uint64_t *s_full = v_empty + PF_VST;  // [2]
  uint64_t *p_full = s_full + 2;
  uint64_t *o_done = p_full + 1;
  uint64_t *drained = o_done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drained + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *bad_pages = abort_flag + 1;  // [4]: per item, a ring of 4

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
    }
    for (int i = 0; i < PF_KST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < PF_VST; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(drained, 1);
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) bad_pages[i] = 0;
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
  const long long first = blockIdx.x, stride = gridDim.x;

  if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------ TMA producers: Q and K (warp 4), V (warp 6)
    const bool is_k = warp == 4;
    if (lane == 0) {
      prefetch_tensor_map(is_k ? &tmap_k : &tmap_v);
      if (is_k) prefetch_tensor_map(&tmap_q);
    }
    const int nst = is_k ? PF_KST : PF_VST;
    uint64_t *full = is_k ? k_full : v_full;
    uint64_t *empty = is_k ? k_empty : v_empty;
    uint8_t *ring = sm + (is_k ? L::K : L::V);
    long long g = 0;  // tiles issued so far
    int n_items = 0;
    bool ok = true;
    for (long long item = first; ok && item < a.num_items; item += stride) {
      const PrefillItem it = prefill_item(a, item);
      if (!it.work) continue;
      if (is_k) {
        const int qb = n_items & 1;
        if (n_items >= 2 && !(ok = warp_wait(&q_empty[qb], ((n_items >> 1) - 1) & 1, limit))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&q_full[qb], PF_BM * D * 2);
#pragma unroll
          for (int hh = 0; hh < HALVES; ++hh)
            tc::tma_load_3d(sm + L::Q + (qb * HALVES + hh) * REGION, &tmap_q, hh * 64, it.hq, it.q0 + it.t0,
                            &q_full[qb]);
        }
      }
      bool bad_next;
      int blk_next = tile_page(a, it, 0, lane, &bad_next);
      for (int j = 0; j < it.nt; ++j, ++g) {
        const int blk = blk_next;
        const bool bad = bad_next;
        if (j + 1 < it.nt) blk_next = tile_page(a, it, j + 1, lane, &bad_next);  // in flight during the wait
        const int st = (int)(g % nst);
        if (g >= nst && !(ok = warp_wait(&empty[st], (uint32_t)(((g / nst) - 1) & 1), limit))) break;
        if (__any_sync(FULL, *abort_flag != 0)) {
          ok = false;
          break;
        }
        if (!is_k && __any_sync(FULL, bad) && lane == 0) {
          bad_pages[n_items & 3] = 1;  // published by this tile's v_full arrival
          atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
        }
        load_tile<HALVES>(a, it, blk, lane, ring + st * HALVES * REGION, is_k ? &tmap_k : &tmap_v, &full[st]);
      }
      ++n_items;
    }
    if (!ok && lane == 0) *abort_flag = 1;
    // Every copy this warp started has landed before the CTA's smem is given back: for each slot,
    // the phase of the last tile issued into it.
    bool drained_ok = true;
    for (int i = 0; i < nst; ++i) {
      if (g <= i) continue;
      const long long last = i + ((g - 1 - i) / nst) * nst;
      drained_ok = warp_wait(&full[i], (uint32_t)((last / nst) & 1), limit) && drained_ok;
    }
    if (is_k)
      for (int i = 0; i < 2 && i < n_items; ++i) {
        const int last = i + ((n_items - 1 - i) / 2) * 2;
        drained_ok = warp_wait(&q_full[i], (uint32_t)((last >> 1) & 1), limit) && drained_ok;
      }
    if (!drained_ok && lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issue (one lane)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_f16(kBf16, false, PF_BM, PF_BN);
      constexpr uint32_t idesc_pv = tc::idesc_f16(kBf16, true, PF_BM, D);
      const uint32_t ps = sbase + L::P;
      long long g = 0;         // tiles whose QK^T has been issued
      long long pending = -1;  // tile whose PV is due next
      bool pending_first = false;
      int n_items = 0;
      bool ok = true;
      // PV of tile t (O += P V), once its softmax has written P.
      auto issue_pv = [&](long long t, bool first_of_item) -> bool {
        if (!mbar_wait_bounded(p_full, (uint32_t)(t & 1), limit)) return false;
        const int st = (int)(t % PF_VST);
        if (!mbar_wait_bounded(&v_full[st], (uint32_t)((t / PF_VST) & 1), limit)) return false;
        tc::fence_after_sync();
        const uint32_t vs = sbase + L::V + st * HALVES * REGION;
#pragma unroll
        for (int k = 0; k < PF_BN / 16; ++k) {
          const uint32_t a_off = (k / 4) * REGION + (k % 4) * 32;
          tc::mma_ss(tmem + 2 * PF_BN, tc::desc_sw128(ps + a_off, 16, 1024),
                     tc::desc_sw128(vs + k * 16 * 128, REGION, 1024), idesc_pv, !first_of_item || k > 0);
        }
        tc::commit(o_done);
        tc::commit(&v_empty[st]);
        return true;
      };
      for (long long item = first; ok && item < a.num_items; item += stride) {
        const PrefillItem it = prefill_item(a, item);
        if (!it.work) continue;
        const int qb = n_items & 1;
        if (!(ok = mbar_wait_bounded(&q_full[qb], (uint32_t)((n_items >> 1) & 1), limit))) break;
        const uint32_t qs = sbase + L::Q + qb * HALVES * REGION;
        for (int j = 0; j < it.nt; ++j, ++g) {
          if (*abort_flag) {
            ok = false;
            break;
          }
          const int st = (int)(g % PF_KST);
          if (!(ok = mbar_wait_bounded(&k_full[st], (uint32_t)((g / PF_KST) & 1), limit))) break;
          tc::fence_after_sync();
          const uint32_t ks = sbase + L::K + st * HALVES * REGION;
          const uint32_t d = tmem + (uint32_t)(g & 1) * PF_BN;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k / 4) * REGION + (k % 4) * 32;
            tc::mma_ss(d, tc::desc_sw128(qs + off, 16, 1024), tc::desc_sw128(ks + off, 16, 1024), idesc_qk, k > 0);
          }
          tc::commit(&s_full[g & 1]);
          tc::commit(&k_empty[st]);
          if (j == it.nt - 1) tc::commit(&q_empty[qb]);
          if (pending >= 0 && !(ok = issue_pv(pending, pending_first))) break;
          pending = g;
          pending_first = j == 0;
        }
        ++n_items;
      }
      if (ok && pending >= 0) ok = issue_pv(pending, pending_first);
      if (!ok) {
        *abort_flag = 1;
        atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
      }
      // Every MMA issued has finished before tensor memory and smem are released.
      tc::commit(drained);
      if (!mbar_wait_bounded(drained, 0, limit)) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ softmax and epilogue (warps 0-3, one row each)
    const int r = warp * 32 + lane;
    const uint32_t lanes = (uint32_t)(warp * 32) << 16;
    long long g = 0;
    int n_items = 0;
    bool ok = true;
    for (long long item = first; ok && item < a.num_items; item += stride) {
      const PrefillItem it = prefill_item(a, item);
      if (it.bad_ctx) {
        if (r == 0) atomicOr(&g_status, PA_DEV_ERR_CONTEXT);
        if (r < it.rows) {
          uint4 *dst = reinterpret_cast<uint4 *>(a.out + (long long)(it.q0 + it.t0 + r) * a.out_token_stride +
                                                 (long long)it.hq * D);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
        }
      }
      if (!it.work) continue;
      // last key this row sees; rows past the item's tokens stop at kmax - 1 too, so that no row
      // reads a page the producers did not load
      const int vis = min(it.pos0 + r, it.kmax - 1);
      const int vis_min = min(it.pos0, it.kmax - 1);  // the smallest vis of the item's rows
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < it.nt; ++j, ++g) {
        if (__any_sync(FULL, *abort_flag != 0)) {
          ok = false;
          break;
        }
        if (!(ok = warp_wait(&s_full[g & 1], (uint32_t)((g >> 1) & 1), limit))) break;
        tc::fence_after_sync();
        float sv[PF_BN];
#pragma unroll
        for (int c = 0; c < PF_BN / 32; ++c) {
          float t[32];
          tc::ld32(tmem + lanes + (uint32_t)(g & 1) * PF_BN + c * 32, t);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[c * 32 + i] = t[i];
        }
        tc::wait_ld();
        const int key0 = j * PF_BN;
        if (key0 + PF_BN - 1 > vis_min) {  // a tile on the diagonal or at the end: mask (uniform branch)
#pragma unroll
          for (int c = 0; c < PF_BN; ++c)
            if (key0 + c > vis) sv[c] = -INFINITY;
        }
        // row max of the raw scores in four independent chains (scale_log2 > 0 keeps the order)
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < PF_BN; c += 4)
#pragma unroll
          for (int u = 0; u < 4; ++u) mx4[u] = fmaxf(mx4[u], sv[c + u]);
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.scale_log2;
        const float m_new = fmaxf(m, mx);
        const bool need = m_new > m + RESCALE_SLACK;
        float factor = 1.f;
        if (need) {
          factor = ex2(m - m_new);
          m = m_new;
        }
        // p = 2^(s * scale_log2 - m): one FFMA and one SFU op per score; fp32 sums in four chains
        uint32_t pk[PF_BN / 2];
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < PF_BN / 2; ++c) {
          const float p0 = ex2(fmaf(sv[2 * c], a.scale_log2, -m));
          const float p1 = ex2(fmaf(sv[2 * c + 1], a.scale_log2, -m));
          sum4[(2 * c) & 3] += p0;
          sum4[(2 * c + 1) & 3] += p1;
          pk[c] = E::narrow2(p0, p1);
        }
        const float rowsum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
        if (j == it.nt - 1) {
          // The V producer publishes the item's missing pages with this tile's arrival.  V rows from
          // kmax on are past the context (whatever the pool holds there, possibly NaN) or in pages
          // never loaded (stale smem); P is 0 for them but 0 * NaN is not, so they are zeroed.
          const int st = (int)(g % PF_VST);
          if (!(ok = warp_wait(&v_full[st], (uint32_t)((g / PF_VST) & 1), limit))) break;
          if (key0 + PF_BN > it.kmax && key0 + r >= it.kmax) {
#pragma unroll
            for (int hh = 0; hh < HALVES; ++hh) {
              uint4 *row = reinterpret_cast<uint4 *>(sm + L::V + (st * HALVES + hh) * REGION + r * 128);
#pragma unroll
              for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
            }
          }
        }
        if (g > 0) {  // the previous PV has read P (and, within an item, O is settled)
          if (!(ok = warp_wait(o_done, (uint32_t)((g - 1) & 1), limit))) break;
          tc::fence_after_sync();
          if (j > 0 && __any_sync(FULL, need)) {
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
      if (!ok) break;
      // epilogue: O after the item's last PV, normalised
      if (!(ok = warp_wait(o_done, (uint32_t)((g - 1) & 1), limit))) break;
      tc::fence_after_sync();
      const bool zero = bad_pages[n_items & 3] != 0;
      __syncwarp();
      if (r == 0) bad_pages[n_items & 3] = 0;  // free the slot for item n_items + 4
      uint16_t *dst = a.out + (long long)(it.q0 + it.t0 + r) * a.out_token_stride + (long long)it.hq * D;
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tc::ld32(tmem + lanes + 2 * PF_BN + c * 32, o);  // every lane: the load is warp-collective
        tc::wait_ld();
        if (r < it.rows) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = zero ? 0.f : o[i * 8 + e] * inv;
            *reinterpret_cast<uint4 *>(dst + c * 32 + i * 8) = narrow8<E>(f);
          }
        }
      }
      tc::fence_before_sync();
      ++n_items;
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc::fence_after_sync();
    tc::dealloc(tmem, PF_TMEM_COLS);
  }
}

}  // namespace pa
