// Causal prefill / chunked-prefill attention through the page table on the
// sm_100a tensor cores ("4. vLLM核心机制" section 4.3: the prompt's tokens
// enter the cache before decoding, possibly a chunk per iteration).
//
// Work item: 256 consecutive new tokens of one sequence for one query head,
// as two 128-row sub-tiles A and B that share every K/V tile (half the K/V
// bytes per flop of one 128-row tile).  Persistent CTAs (one per SM) take
// items from a per-call counter, latest (heaviest) query tiles of every
// sequence first; the producer warp fetches each item and hands it to the
// other roles through a 4-deep ring in shared memory.  Per key tile of 128 tokens
// (8 pages of 16 or 4 of 32), for each sub-tile x:
//   S_x = Q_x K^T    tcgen05.mma M=128 N=128 K=d, Q and K from swizzled smem,
//                    S_x in tensor memory;
//   softmax_x        one warpgroup per sub-tile, one row per thread: S_x read
//                    from tensor memory into registers (four loads, one
//                    wait), causal mask, online max with a lazy rescale of O_x, P_x
//                    rounded to the storage type and stored back into the
//                    first half of S_x's columns;
//   O_x += P_x V     tcgen05.mma M=128 N=d K=128 with P_x read from tensor
//                    memory and V MN-major from its TMA tile.
// The MMA lane issues QK_A(j), PV_B(j-1), QK_B(j), PV_A(j): each warpgroup's
// softmax runs while the tensor core works on the other sub-tile.  Tensor
// memory (512 columns): S_A, S_B (128 each), O_A, O_B (d each).
// Warp roles: 0-3 softmax of A, 4-7 softmax of B, 8 TMA producer of Q and K
// pages, 9 TMA producer of V pages, 10 MMA issue (one lane).  A K slot frees
// once both QK^T of its tile ran, a V slot once both PV did.  Every wait is
// bounded: on a timeout the CTA flags PA_DEV_ERR_TIMEOUT, drains its copies
// and MMAs in flight, frees its tensor memory and returns.
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
  unsigned int *queue;          // work counter of this call, zero at launch
  long long num_blocks, out_token_stride, num_query_tokens, num_items;
  unsigned long long wait_limit_ns;
  float scale_log2;
  int num_seqs, num_q_heads, num_kv_heads, block_size, table_stride, q_tiles;
};

constexpr int PF_BM = 128;             // query rows per sub-tile
constexpr int PF_ROWS = 2 * PF_BM;     // query rows per item (sub-tiles A and B)
constexpr int PF_BN = 128;             // keys per tile
constexpr int PF_THREADS = 11 * 32;
constexpr int PF_KST = 3;              // K ring
constexpr int PF_VST = 2;              // V ring
constexpr uint32_t PF_TMEM_COLS = 512;
constexpr int PF_ITEM_READERS = 10;  // V producer, MMA lane, 8 softmax warps

template <int D>
struct PrefillSmem {
  static constexpr uint32_t REGION = 128 * 128;  // 128 rows of 128 bytes (64 elements)
  static constexpr uint32_t HALVES = D / 64;
  static constexpr uint32_t Q = 0;  // sub-tiles A and B
  static constexpr uint32_t K = Q + 2 * HALVES * REGION;
  static constexpr uint32_t V = K + PF_KST * HALVES * REGION;
  static constexpr uint32_t BARS = V + PF_VST * HALVES * REGION;
  // 27 mbarriers, the item ring, the tensor-memory address and flags: 272 bytes used
  static constexpr uint32_t BYTES = BARS + 512;
  // + alignment slack; at least 120 KB so that one CTA holds an SM (and its tensor memory) alone
  static constexpr uint32_t ALLOC = (BYTES + 1024 > 120 * 1024) ? BYTES + 1024 : 120 * 1024;
  // tensor memory columns
  static constexpr uint32_t T_S = 0;      // S_x at T_S + x * 128; P_x in its first 64 columns
  static constexpr uint32_t T_O = 256;    // O_x at T_O + x * D
};

// 2^x with the SFU's approximate exponential (documented PTX; relative error about 2^-22, 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe, for the share of the softmax's exponentials taken off the SFU (x <= RESCALE_SLACK;
// x below -126, -inf included, gives 0).  2^x = 2^n * 2^f with n = round(x) -- adding 1.5 * 2^23 leaves n in
// the low mantissa bits -- and f = x - n in [-1/2, 1/2]; 2^f by a cubic fitted to 2^f on [-1/2, 1/2] (least
// squares at Chebyshev nodes, reweighted toward equal relative error: at most 7.5e-5, below the 2-byte rounding
// of P that follows); n is then added to the exponent field.
// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// c + lo + hi of two packed 2-byte values, widened exactly by the mixed-precision fma (times 1.0):
// the row sum adds the rounded P values that the PV product uses, so the weights sum to one.
template <class E>
__device__ __forceinline__ float add_packed(uint32_t pk, float c) {
  float d;
  if constexpr (std::is_same<E, BF16>::value) {
    asm("{\n\t.reg .b16 p0, p1, one;\n\tmov.b16 one, 0x3F80;\n\tmov.b32 {p0, p1}, %1;\n\t"
        "fma.rn.f32.bf16 %0, p0, one, %2;\n\tfma.rn.f32.bf16 %0, p1, one, %0;\n\t}"
        : "=f"(d)
        : "r"(pk), "f"(c));
  } else {
    asm("{\n\t.reg .b16 p0, p1, one;\n\tmov.b16 one, 0x3C00;\n\tmov.b32 {p0, p1}, %1;\n\t"
        "fma.rn.f32.f16 %0, p0, one, %2;\n\tfma.rn.f32.f16 %0, p1, one, %0;\n\t}"
        : "=f"(d)
        : "r"(pk), "f"(c));
  }
  return d;
}

// All lanes wait on the same barrier phase; the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned long long limit_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, limit_ns);
  return __all_sync(FULL, ok);
}

// One work item as every role sees it (all values uniform across the CTA).
struct PrefillItem {
  int s, hq, h, q0, t0, rows, ctx, pos0, kmax, nt, nt_a;
  bool work, bad_ctx, bad_rows, has_b, past_grid;
};

__device__ __forceinline__ PrefillItem prefill_item(const PrefillArgs &a, long long item) {
  PrefillItem it;
  // Item order: query tile (latest, i.e. heaviest, first), then sequence, then head -- the longest work
  // first, so the tail of the persistent grid is made of light items.  Measured against two orders that
  // keep a pair's K/V pages in L2 between its query tiles (llama2_7b_prefill / gqa_chunked_prefill,
  // TFLOP/s): this order 556 / 845 with DRAM reads 2.6x the algorithmic bytes; (sequence, head, tile)
  // 450 / 766 at 1.0x; bands of one pair per CTA, heaviest tiles of a band first, 527 / 834 at 1.6x.
  // The kernel is bound by its per-tile softmax chain, not by HBM, so the re-reads cost nothing and the
  // better balance wins.
  const long long per_tile = (long long)a.num_seqs * a.num_q_heads;
  const int qt = a.q_tiles - 1 - (int)(item / per_tile);
  const int rem = (int)(item % per_tile);
  it.s = rem / a.num_q_heads;
  it.hq = rem % a.num_q_heads;
  it.h = it.hq / (a.num_q_heads / a.num_kv_heads);
  it.q0 = a.query_start[it.s];
  const int n = a.query_start[it.s + 1] - it.q0;
  it.ctx = a.context_lens[it.s];
  it.t0 = qt * PF_ROWS;
  it.work = it.bad_ctx = it.bad_rows = it.has_b = it.past_grid = false;
  it.rows = it.pos0 = it.kmax = it.nt = it.nt_a = 0;
  if (it.q0 < 0 || n < 0 || (long long)it.q0 + n > a.num_query_tokens) {  // rows outside q / out
    it.bad_rows = true;
    return it;
  }
  it.past_grid = (long long)n > (long long)a.q_tiles * PF_ROWS;  // more new tokens than max_query_len covers
  if (it.t0 >= n) return it;
  it.rows = min(PF_ROWS, n - it.t0);
  if (it.ctx < n || (long long)it.ctx > (long long)a.table_stride * a.block_size) {
    it.bad_ctx = true;
    return it;
  }
  it.work = true;
  it.has_b = it.rows > PF_BM;
  it.pos0 = it.ctx - n + it.t0;              // logical position of row 0 of sub-tile A
  it.kmax = min(it.ctx, it.pos0 + it.rows);  // keys [0, kmax) are visible to some row
  it.nt = (it.kmax + PF_BN - 1) / PF_BN;
  // sub-tile A sees keys up to pos0 + 127 only; its tiles are a prefix of the item's
  it.nt_a = (min(it.kmax, it.pos0 + PF_BM) + PF_BN - 1) / PF_BN;
  return it;
}

// Page id of key tile j of an item for this lane (lanes >= pages per tile: -1);
// entries outside the pool count as missing and set *bad.
__device__ __forceinline__ int tile_page(const PrefillArgs &a, const PrefillItem &it, int j, int lane, bool *bad) {
  const int bs = a.block_size;
  const int page = j * (PF_BN / bs) + lane;
  int blk = -1;
  *bad = false;
  if (lane < PF_BN / bs && page * bs < it.kmax && dcheck(page < a.table_stride && it.s < a.num_seqs)) {
    blk = a.block_tables[(long long)it.s * a.table_stride + page];
    if (blk < 0 || (long long)blk >= a.num_blocks) {
      *bad = true;
      blk = -1;
    }
  }
  return blk;
}

// Issues the TMA boxes of one key tile (K or V) into `dst`, completing on `bar`: lane 0 posts the
// expected bytes, then lane p issues the boxes of the tile's page p (its `blk`), so the pages' copies
// go out together rather than one after another from a single thread.
template <int HALVES>
__device__ __forceinline__ void load_tile(const PrefillArgs &a, const PrefillItem &it, int blk, int lane,
                                          uint8_t *dst, const CUtensorMap *map, uint64_t *bar) {
  const int bs = a.block_size;
  const unsigned loaded = __ballot_sync(FULL, blk >= 0);
  if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)__popc(loaded) * bs * 128u * HALVES);
  __syncwarp();
  if (blk >= 0) {
    const long long row = ((long long)blk * a.num_kv_heads + it.h) * bs;
    for (int hh = 0; hh < HALVES; ++hh)
      for (int b = 0; b < bs / TILE; ++b)
        tma_load_2d(dst + hh * 128 * 128 + (lane * bs + b * TILE) * 128, map, hh * 64, (int)(row + b * TILE), bar);
  }
}

static_assert(PrefillSmem<128>::ALLOC <= 232448, "prefill smem over the per-block opt-in limit");

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
  uint64_t *q_full = bars;
  uint64_t *q_empty = q_full + 1;
  uint64_t *k_full = q_empty + 1;       // [PF_KST]
  uint64_t *k_empty = k_full + PF_KST;  // [PF_KST]
  uint64_t *v_full = k_empty + PF_KST;  // [PF_VST]
  uint64_t *v_empty = v_full + PF_VST;  // [PF_VST]
  uint64_t *s_full = v_empty + PF_VST;  // [2]: S_A, S_B written (and every earlier MMA done)
  uint64_t *p_full = s_full + 2;        // [2]: P_A, P_B written
  uint64_t *o_done = p_full + 2;        // [2]: an item's last PV of A, of B done
  uint64_t *drained = o_done + 2;
  uint64_t *item_full = drained + 1;   // [4]: the ring of items handed out by the producer warp
  uint64_t *item_empty = item_full + 4;
  volatile long long *items = reinterpret_cast<volatile long long *>(item_empty + 4);  // [4]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(const_cast<long long *>(items + 4));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *bad_pages = abort_flag + 1;  // [4]: per item, a ring of 4

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < PF_KST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < PF_VST; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drained, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], PF_ITEM_READERS);
    }
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) bad_pages[i] = 0;
    fence_mbar_init();
  }
  if (warp == 10) {
    tc::alloc(tmem_slot, PF_TMEM_COLS);
    tc::relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const unsigned long long limit = a.wait_limit_ns;
  // The k-th item the producer warp handed out (-1: none left), for one warp or one lane.
  auto take_item = [&](int k, bool whole_warp, long long *idx) -> bool {
    const int slot = k & 3;
    const bool ok = whole_warp ? warp_wait(&item_full[slot], (uint32_t)((k >> 2) & 1), limit)
                               : mbar_wait_bounded(&item_full[slot], (uint32_t)((k >> 2) & 1), limit);
    *idx = items[slot];
    if (whole_warp) __syncwarp();
    if (!whole_warp || lane == 0) mbar_arrive(&item_empty[slot]);
    return ok;
  };

  if (warp == 8 || warp == 9) {
    // ------------------------------------------------------------ TMA producers: Q and K (warp 8), V (warp 9)
    const bool is_k = warp == 8;
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
    for (int k = 0; ok; ++k) {
      long long item;
      PrefillItem it;
      if (is_k) {
        // fetch the next item with work; items whose rows or context are invalid are settled here
        const int slot = k & 3;
        if (k >= 4 && !(ok = warp_wait(&item_empty[slot], (uint32_t)(((k >> 2) - 1) & 1), limit))) break;
        for (;;) {
          unsigned int t = 0;
          if (lane == 0) t = atomicAdd(a.queue, 1u);
          item = (long long)__shfl_sync(FULL, t, 0);
          if (item >= a.num_items) {
            item = -1;
            break;
          }
          it = prefill_item(a, item);
          if (!dcheck(it.s < a.num_seqs && it.hq < a.num_q_heads)) {
            it.work = false;
            it.bad_ctx = false;
            continue;
          }
          if (it.past_grid && it.t0 == 0 && it.hq == 0 && lane == 0) atomicOr(&g_status, PA_DEV_ERR_CONTEXT_HINT);
          if (it.work) break;
          if (!it.bad_ctx && lane == 0) {
            // no rows of this sequence at this query tile (or no valid rows at all): the same holds for
            // the sequence's remaining heads, which are the next items; move the counter past them
            atomicMax(a.queue, (unsigned int)(item + a.num_q_heads - it.hq));
            if (it.bad_rows) atomicOr(&g_status, PA_DEV_ERR_CONTEXT);
          }
          if (it.bad_ctx) {  // zero the item's rows
            if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_CONTEXT);
            for (int r = lane; r < it.rows; r += 32) {
              if (!dcheck((long long)it.q0 + it.t0 + r < a.num_query_tokens)) break;
              uint4 *dst = reinterpret_cast<uint4 *>(a.out + (long long)(it.q0 + it.t0 + r) * a.out_token_stride +
                                                     (long long)it.hq * D);
#pragma unroll
              for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
            }
          }
        }
        if (lane == 0) {
          items[slot] = item;
          mbar_arrive(&item_full[slot]);  // release: the item index is visible to the readers
        }
        if (item < 0) break;
      } else {
        if (!(ok = take_item(k, true, &item))) break;
        if (item < 0) break;
        it = prefill_item(a, item);
      }
      if (is_k) {
        if (n_items >= 1 && !(ok = warp_wait(q_empty, (uint32_t)((n_items - 1) & 1), limit))) break;
        if (lane == 0) mbar_arrive_expect_tx(q_full, 2 * PF_BM * D * 2);
        __syncwarp();
        if (lane < 2 * HALVES) {  // lane = sub-tile * HALVES + half
          const int x = lane / HALVES, hh = lane % HALVES;
          tc::tma_load_3d(sm + L::Q + lane * REGION, &tmap_q, hh * 64, it.hq, it.q0 + it.t0 + x * PF_BM, q_full);
        }
      }
      bool any_bad = false;
      bool bad_next;
      int blk_next = tile_page(a, it, 0, lane, &bad_next);
      for (int j = 0; j < it.nt; ++j, ++g) {
        const int blk = blk_next;
        any_bad = any_bad || bad_next;
        if (j + 1 < it.nt) blk_next = tile_page(a, it, j + 1, lane, &bad_next);  // in flight during the wait
        const int st = (int)(g % nst);
        if (g >= nst && !(ok = warp_wait(&empty[st], (uint32_t)(((g / nst) - 1) & 1), limit))) break;
        if (__any_sync(FULL, *abort_flag != 0)) {
          ok = false;
          break;
        }
        if (!is_k && j == it.nt - 1) {  // published by this tile's v_full arrival
          const bool bad_item = __any_sync(FULL, any_bad);
          if (lane == 0) {
            bad_pages[n_items & 3] = bad_item ? 1 : 0;
            if (bad_item) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
          }
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
    if (is_k && n_items > 0) drained_ok = warp_wait(q_full, (uint32_t)((n_items - 1) & 1), limit) && drained_ok;
    if (!drained_ok && lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
  } else if (warp == 10) {
    // ------------------------------------------------------------ MMA issue (one lane)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_f16(kBf16, false, PF_BM, PF_BN);
      constexpr uint32_t idesc_pv = tc::idesc_f16(kBf16, true, PF_BM, D);
      const uint32_t qs = sbase + L::Q;
      long long g = 0;           // K/V tiles
      long long gx[2] = {0, 0};  // tiles of sub-tile A, B
      int n_items = 0;
      bool ok = true;
      // S_x = Q_x K(t)^T
      auto issue_qk = [&](int x, long long t) {
        const uint32_t ks = sbase + L::K + (uint32_t)(t % PF_KST) * HALVES * REGION;
        const uint32_t qx = qs + x * HALVES * REGION;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k / 4) * REGION + (k % 4) * 32;
          tc::mma_ss(tmem + L::T_S + x * 128, tc::desc_sw128(qx + off, 16, 1024), tc::desc_sw128(ks + off, 16, 1024),
                     idesc_qk, k > 0);
        }
        tc::commit(&s_full[x]);
      };
      // O_x += P_x V(t), once softmax_x has written P_x for its tile gx
      auto issue_pv = [&](int x, long long t, long long tx, bool first_of_item) -> bool {
        if (!mbar_wait_bounded(&p_full[x], (uint32_t)(tx & 1), limit)) return false;
        const int st = (int)(t % PF_VST);
        if (!mbar_wait_bounded(&v_full[st], (uint32_t)((t / PF_VST) & 1), limit)) return false;
        tc::fence_after_sync();
        const uint32_t vs = sbase + L::V + st * HALVES * REGION;
#pragma unroll
        for (int k = 0; k < PF_BN / 16; ++k)
          tc::mma_ts(tmem + L::T_O + x * D, tmem + L::T_S + x * 128 + k * 8,
                     tc::desc_sw128(vs + k * 16 * 128, REGION, 1024), idesc_pv, !first_of_item || k > 0);
        return true;
      };
      for (int k = 0; ok; ++k) {
        long long item;
        if (!(ok = take_item(k, false, &item))) break;
        if (item < 0) break;
        const PrefillItem it = prefill_item(a, item);
        if (!(ok = mbar_wait_bounded(q_full, (uint32_t)(n_items & 1), limit))) break;
        long long pend_t = -1, pend_tb = 0;  // PV_B due next: K/V tile and B's tile
        bool pend_first = false;
        for (int j = 0; j < it.nt; ++j, ++g) {
          if (*abort_flag) {
            ok = false;
            break;
          }
          const bool a_on = j < it.nt_a, b_on = it.has_b;
          if (!(ok = mbar_wait_bounded(&k_full[g % PF_KST], (uint32_t)((g / PF_KST) & 1), limit))) break;
          tc::fence_after_sync();
          if (a_on) issue_qk(0, g);
          if (pend_t >= 0) {
            if (!(ok = issue_pv(1, pend_t, pend_tb, pend_first))) break;
            tc::commit(&v_empty[pend_t % PF_VST]);
            pend_t = -1;
          }
          if (b_on) issue_qk(1, g);
          tc::commit(&k_empty[g % PF_KST]);
          if (j == it.nt - 1) tc::commit(q_empty);
          if (a_on) {
            if (!(ok = issue_pv(0, g, gx[0], j == 0))) break;
            if (j == it.nt_a - 1) tc::commit(&o_done[0]);
            if (!b_on) tc::commit(&v_empty[g % PF_VST]);
            ++gx[0];
          }
          if (b_on) {
            pend_t = g;
            pend_tb = gx[1]++;
            pend_first = j == 0;
          }
        }
        if (ok && pend_t >= 0) {  // the item's last PV_B
          if ((ok = issue_pv(1, pend_t, pend_tb, pend_first))) {
            tc::commit(&v_empty[pend_t % PF_VST]);
            tc::commit(&o_done[1]);
          }
        }
        ++n_items;
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
    // ------------------------------------------------------------ softmax and epilogue of sub-tile x (warps 0-3: A, 4-7: B)
    const int x = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lanes + L::T_S + x * 128, t_o = tmem + lanes + L::T_O + x * D;
    long long g = 0;   // K/V tiles
    long long gx = 0;  // this sub-tile's tiles
    int n_items = 0, nx_items = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      long long item;
      if (!(ok = take_item(k, true, &item))) break;
      if (item < 0) break;
      const PrefillItem it = prefill_item(a, item);
      const int ntx = x == 0 ? it.nt_a : (it.has_b ? it.nt : 0);
      const bool zeroes_v = x == 0 ? it.nt_a == it.nt : it.nt_a < it.nt;  // first PV reader of the last tile
      // last key this row sees; rows past the item's tokens stop at kmax - 1 too, so that no row
      // reads a page the producers did not load
      const int pos0 = it.pos0 + x * PF_BM;
      const int vis = min(pos0 + r, it.kmax - 1);
      const int vis_min = min(pos0, it.kmax - 1);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < ntx; ++j, ++gx) {
        if (__any_sync(FULL, *abort_flag != 0)) {
          ok = false;
          break;
        }
        // S_x(j) is in tensor memory, and every earlier MMA (PV_x of the previous tile) is done
        if (!(ok = warp_wait(&s_full[x], (uint32_t)(gx & 1), limit))) break;
        tc::fence_after_sync();
        const int key0 = j * PF_BN;
        const bool masked = key0 + PF_BN - 1 > vis_min;  // a tile on the diagonal or at the end (uniform)
        // the row of S_x: four loads, one wait
        float sv[PF_BN];
#pragma unroll
        for (int c = 0; c < PF_BN / 32; ++c) tc::ld32(t_s + c * 32, *reinterpret_cast<float(*)[32]>(&sv[c * 32]));
        tc::wait_ld();
        if (masked) {
#pragma unroll
          for (int c = 0; c < PF_BN; ++c)
            if (key0 + c > vis) sv[c] = -INFINITY;
        }
        // row max of the raw scores in four chains, two scores per three-input max (scale_log2 > 0 keeps the order)
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < PF_BN; c += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u) mx4[u] = fmax3(mx4[u], sv[c + u], sv[c + 4 + u]);
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.scale_log2;
        const float m_new = fmaxf(m, mx);
        const bool need = m_new > m + RESCALE_SLACK;
        float factor = 1.f;
        if (need) {
          factor = ex2(m - m_new);
          m = m_new;
        }
        // p = 2^(s * scale_log2 - m) (0 where masked), rounded to the storage type, into P_x: the
        // first 64 columns of S_x, whose scores are all in registers by now.
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < PF_BN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            // masked scores are -inf: 2^-inf = 0
            // scale and shift two scores in one packed fma
            const float2 x = __ffma2_rn(make_float2(sv[c * 32 + 2 * i], sv[c * 32 + 2 * i + 1]),
                                        make_float2(a.scale_log2, a.scale_log2), make_float2(-m, -m));
            const float p0 = ex2(x.x);
            const float p1 = ex2(x.y);
            pk[i] = E::narrow2(p0, p1);
            sum4[i & 3] = add_packed<E>(pk[i], sum4[i & 3]);
          }
          tc::st16(t_s + c * 16, pk);
        }
        const float rowsum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
        if (j > 0 && __any_sync(FULL, need)) {  // O_x is settled: the previous PV_x is done
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tc::ld32(t_o + c * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= factor;
            tc::st32(t_o + c * 32, o);
          }
        }
        tc::wait_st();
        l = l * factor + rowsum;
        if (j == it.nt - 1) {
          // The V producer publishes the item's missing pages with this tile's arrival.  V rows from
          // kmax on are past the context (whatever the pool holds there, possibly NaN) or in pages
          // never loaded (stale smem); P is 0 for them but 0 * NaN is not, so the sub-tile whose PV
          // reads the last tile first zeroes them.
          const int st = (int)(g % PF_VST);
          if (!(ok = warp_wait(&v_full[st], (uint32_t)((g / PF_VST) & 1), limit))) break;
          if (zeroes_v && key0 + PF_BN > it.kmax && key0 + r >= it.kmax) {
#pragma unroll
            for (int hh = 0; hh < HALVES; ++hh) {
              uint4 *row = reinterpret_cast<uint4 *>(sm + L::V + (st * HALVES + hh) * REGION + r * 128);
#pragma unroll
              for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
        }
        tc::fence_before_sync();
        mbar_arrive(&p_full[x]);
        ++g;
      }
      if (!ok) break;
      g += it.nt - ntx;  // tiles this sub-tile does not read
      if (ntx == 0) {
        ++n_items;
        continue;
      }
      if (ntx < it.nt) {  // sub-tile A skips the last tiles: it still needs the item's missing-page flag
        const long long gl = g - 1;
        if (!(ok = warp_wait(&v_full[gl % PF_VST], (uint32_t)((gl / PF_VST) & 1), limit))) break;
      }
      // epilogue: O_x after the item's last PV_x, normalised
      if (!(ok = warp_wait(&o_done[x], (uint32_t)(nx_items & 1), limit))) break;
      tc::fence_after_sync();
      const bool zero = bad_pages[n_items & 3] != 0;
      const int row = x * PF_BM + r;
      uint16_t *dst = a.out + (long long)(it.q0 + it.t0 + row) * a.out_token_stride + (long long)it.hq * D;
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tc::ld32(t_o + c * 32, o);  // every lane: the load is warp-collective
        tc::wait_ld();
        if (row < it.rows && dcheck((long long)it.q0 + it.t0 + row < a.num_query_tokens)) {
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
      ++nx_items;
    }
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 10) {
    __syncwarp();
    tc::fence_after_sync();
    tc::dealloc(tmem, PF_TMEM_COLS);
  }
}

}  // namespace pa
