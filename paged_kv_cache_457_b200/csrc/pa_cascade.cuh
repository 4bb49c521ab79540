// Cascade decode: the attention pa_decode computes, for a batch whose sequences share leading blocks, with
// every shared K/V tile fetched once per group of sequences instead of once per sequence ("4. vLLM核心机制"
// section 4.2: the pages of a shared prefix -- one prompt sampled several times, a common system prompt --
// are named by several block tables).  Only the order of the work differs from pa_decode:
//
//   cascade_partial_kernel   one block per plan job and kv head.  A prefix job streams a chunk of a group's
//                            shared tiles through one TMA ring that all of the block's consumer warps read;
//                            consumer warp w multiplies each tile against the query heads of its own members
//                            (the mma's 8 columns: 8 / G members of G heads each), so one 16-token tile
//                            serves up to 32 (member, head) columns.  A suffix job streams a chunk of one
//                            sequence's own tiles (one consumer warp).  Every job leaves, per (member, head),
//                            the unnormalised softmax state (m, l, acc[D]) of its tiles; a job with no tiles
//                            leaves (-inf, 0), a failed one (-inf, -1).
//   cascade_combine_kernel   one warp per (sequence, query head): merges the sequence's pieces in plan order,
//                              out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p,   M = max_p m_p,
//                            and rounds to the storage type (nearest even).
//
// The per-tile arithmetic is the tensor-core split kernel's (pa_mma.cuh): S^T = K Q^T and O^T += V^T P^T on
// mma.sync m16n8k16 with fp32 accumulation, P split into a 2-byte head and residual, lazy rescaling.
#pragma once

#include <cuda.h>

#include "pa_mma.cuh"
#include "pa_plan_layout.h"

namespace pa {

static_assert(CASCADE_TILE == TILE, "one plan tile is one ring tile");
constexpr int CASCADE_SLOTS = 8;  // ring slots per block: all shared by a prefix job, two per warp for suffix jobs
constexpr int CASCADE_WARP_SLOTS = CASCADE_SLOTS / CASCADE_CONSUMERS;

struct CascadeArgs {
  const uint16_t *q;
  uint16_t *out;
  const int *block_tables;
  const int *context_lens;
  const int *jobs;           // [num_jobs][CJ_INTS]: the num_prefix_jobs prefix jobs first, then the suffix jobs
  const int *members;        // [num_members]
  const int *piece_offsets;  // [num_seqs + 1]: pieces of sequence s are [piece_offsets[s], piece_offsets[s+1])
  const int *piece_rows;     // [num_pieces]: partial row of the piece's head 0, in merge order
  float2 *ws_ml;             // [num_kv_heads][rows_per_head]
  float *ws_acc;             // [num_kv_heads][rows_per_head][D]
  long long q_seq_stride, out_seq_stride, num_blocks;
  unsigned long long wait_limit_ns;
  float scale_log2;
  int num_seqs, num_q_heads, num_kv_heads, block_size, table_stride, max_context_len, group;
  int num_jobs, num_prefix_jobs, num_members, num_pieces, rows_per_head;
};

template <int D>
struct CascadeSmem {
  static constexpr uint32_t STAGE_BYTES = 2 * TILE * D * 2;
  static constexpr uint32_t RING = CASCADE_SLOTS * STAGE_BYTES;
  // 1024: alignment slack (the swizzle pattern repeats every 1024 bytes); full and empty barriers, slot flags,
  // member mask
  static __host__ __device__ constexpr uint32_t bytes() { return 1024 + RING + CASCADE_SLOTS * 20 + 16; }
};

// Tokens of a context that the library accepts: within the table row and the call's bound.
__device__ __forceinline__ bool cascade_context_ok(const CascadeArgs &a, int L) {
  return L >= 0 && (long long)L <= (long long)a.table_stride * a.block_size && L <= a.max_context_len;
}

// The table entries of one row, 32 at a time (lane i holds entry base + i); entries at or past nblk are not read.
struct RowWindow {
  int base = -1, ent = -1;
  __device__ __forceinline__ int lookup(const int *row, int blk, int nblk, int lane) {
    if (base < 0 || blk >= base + 32) {
      base = blk & ~31;
      ent = base + lane < nblk ? __ldg(row + base + lane) : -1;
    }
    return __shfl_sync(FULL, ent, blk - base);
  }
};

// Lane 0: K and V of tile t of (block phys, kv head h), one 3-D TMA box each, into `dst`, completing on `bar`;
// an entry outside the pool flags the slot instead and completes the barrier without data.
template <int D>
__device__ __forceinline__ void cascade_issue(const CascadeArgs &a, const CUtensorMap *mk, const CUtensorMap *mv,
                                              int phys, int t, int h, unsigned char *dst, uint64_t *bar, int *bad) {
  constexpr uint32_t TILE_BYTES = TILE * D * 2;
  const bool ok = phys >= 0 && (long long)phys < a.num_blocks;
  *bad = ok ? 0 : 1;
  if (ok) {
    const int row = (int)(((long long)phys * a.num_kv_heads + h) * a.block_size + (t * TILE) % a.block_size);
    fence_proxy_async_smem();  // the slot's previous contents were read through the generic proxy
    mbar_arrive_expect_tx(bar, 2 * TILE_BYTES);
    tc::tma_load_3d(dst, mk, 0, row, 0, bar);
    tc::tma_load_3d(dst + TILE_BYTES, mv, 0, row, 0, bar);
  } else {
    mbar_arrive(bar);
  }
}

// One warp's 8 query columns (column c: member c / G of the warp's members, head c % G) and their online
// softmax state over the tiles it has consumed.  The arithmetic of the tensor-core split kernel.
template <class E, int D>
struct ColumnTile {
  static constexpr int KSTEPS = D / 16;
  uint32_t qb[KSTEPS][2];
  float o[KSTEPS][4];
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
  int gid, tig, ka_tok, ka_c, va_tok, va_c;

  __device__ __forceinline__ void init(const CascadeArgs &a, int lane, int seq_of_gid, int head_of_gid) {
    gid = lane >> 2;
    tig = lane & 3;
    const int mi = lane >> 3, mr = lane & 7;
    ka_tok = 8 * (mi & 1) + mr, ka_c = mi >> 1;  // K as A (non-transposed)
    va_tok = 8 * (mi >> 1) + mr, va_c = mi & 1;  // V^T as A (transposed)
    const bool q_ok = seq_of_gid >= 0;
    const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
        a.q + (long long)(q_ok ? seq_of_gid : 0) * a.q_seq_stride + (long long)(q_ok ? head_of_gid : 0) * D);
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      qb[ks][0] = q_ok ? __ldg(qrow + 8 * ks + tig) : 0u;
      qb[ks][1] = q_ok ? __ldg(qrow + 8 * ks + 4 + tig) : 0u;
      o[ks][0] = o[ks][1] = o[ks][2] = o[ks][3] = 0.f;
    }
  }

  // S^T = K Q^T from the slot at shared address kt, and the V^T fragments; the slot may be reused after this
  __device__ __forceinline__ void scores(uint32_t kt, float (&sc)[4], uint32_t (&vf)[KSTEPS][4]) const {
    constexpr uint32_t TILE_BYTES = TILE * D * 2;
    sc[0] = sc[1] = sc[2] = sc[3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      uint32_t kf[4];
      ldsm_x4(kf, kt + swizzled(ka_tok, 2 * ks + ka_c));
      MmaOps<E>::mma(sc, kf, qb[ks][0], qb[ks][1]);
    }
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) ldsm_x4_trans(vf[ks], kt + TILE_BYTES + swizzled(va_tok, 2 * ks + va_c));
  }

  // online softmax of the tile's scores (rows >= nvalid masked) and O^T += V^T P^T
  __device__ __forceinline__ void accumulate(const CascadeArgs &a, const float (&sc)[4], uint32_t (&vf)[KSTEPS][4],
                                             int nvalid) {
    const bool lo_live = gid < nvalid, hi_live = gid + 8 < nvalid;
    const float z0 = lo_live ? sc[0] * a.scale_log2 : -INFINITY;
    const float z1 = lo_live ? sc[1] * a.scale_log2 : -INFINITY;
    const float z2 = hi_live ? sc[2] * a.scale_log2 : -INFINITY;
    const float z3 = hi_live ? sc[3] * a.scale_log2 : -INFINITY;
    const bool need = z0 > ma + RESCALE_SLACK || z2 > ma + RESCALE_SLACK || z1 > mb + RESCALE_SLACK ||
                      z3 > mb + RESCALE_SLACK;
    if (__any_sync(FULL, need)) {
      float ca = fmaxf(z0, z2), cb = fmaxf(z1, z3);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        ca = fmaxf(ca, __shfl_xor_sync(FULL, ca, off));
        cb = fmaxf(cb, __shfl_xor_sync(FULL, cb, off));
      }
      const float na = fmaxf(ma, ca), nb = fmaxf(mb, cb);
      const float alpha_a = exp2f(ma - na), alpha_b = exp2f(mb - nb);  // 0 on the first tile
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        o[mt][0] *= alpha_a;
        o[mt][1] *= alpha_b;
        o[mt][2] *= alpha_a;
        o[mt][3] *= alpha_b;
      }
      la *= alpha_a;
      lb *= alpha_b;
      ma = na;
      mb = nb;
    }
    const float p0 = exp2f(z0 - ma), p1 = exp2f(z1 - mb), p2 = exp2f(z2 - ma), p3 = exp2f(z3 - mb);
    la += p0 + p2;
    lb += p1 + p3;
    uint32_t h01, l01, h23, l23;
    MmaOps<E>::split(p0, p1, h01, l01);
    MmaOps<E>::split(p2, p3, h23, l23);
    const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
    const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);
    if (nvalid < TILE) {  // V rows past the context may hold NaN: zero them (0 * NaN would leak in)
      const uint32_t m_lo = (2 * tig < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 1 < nvalid ? 0xffff0000u : 0u);
      const uint32_t m_hi = (2 * tig + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 9 < nvalid ? 0xffff0000u : 0u);
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        vf[ks][0] &= m_lo;
        vf[ks][1] &= m_lo;
        vf[ks][2] &= m_hi;
        vf[ks][3] &= m_hi;
      }
    }
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt) {
      MmaOps<E>::mma(o[mt], vf[mt], bh0, bh1);
      MmaOps<E>::mma(o[mt], vf[mt], bl0, bl1);
    }
  }

  // Writes the state of the live columns c < ncols to rows row + c (per kv head): (m, l) and acc[D], or
  // (-inf, -1) for a column in `bad_cols` (bit c); a state with no tiles is (-inf, 0) and writes no acc.
  __device__ __forceinline__ void store(const CascadeArgs &a, long long row, int ncols, uint32_t bad_cols,
                                        bool any_tiles) {
    float lta = la, ltb = lb;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      lta += __shfl_xor_sync(FULL, lta, off);
      ltb += __shfl_xor_sync(FULL, ltb, off);
    }
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      const int c = 2 * tig + c2;
      if (c >= ncols) continue;
      const bool cbad = (bad_cols >> c) & 1u;
      if (gid == 0) a.ws_ml[row + c] = cbad ? make_float2(-INFINITY, -1.f) : make_float2(c2 ? mb : ma, c2 ? ltb : lta);
      if (!cbad && any_tiles) {
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
          const int d0 = 16 * mt + gid;
          a.ws_acc[(row + c) * D + d0] = c2 ? o[mt][1] : o[mt][0];
          a.ws_acc[(row + c) * D + d0 + 8] = c2 ? o[mt][3] : o[mt][2];
        }
      }
    }
  }
};

// One job of the plan, read and checked (the plan lives in the caller's memory).
struct CascadeJob {
  int ts, t0, t1, mbase, nm, row0, kind;
  __device__ __forceinline__ bool load(const CascadeArgs &a, int j, int mpo) {
    const int *job = a.jobs + (long long)j * CJ_INTS;
    ts = __ldg(job + CJ_SEQ), t0 = __ldg(job + CJ_T0), t1 = __ldg(job + CJ_T1);
    mbase = __ldg(job + CJ_MEMBERS), nm = __ldg(job + CJ_NM), row0 = __ldg(job + CJ_ROW), kind = __ldg(job + CJ_KIND);
    const bool prefix = j < a.num_prefix_jobs;
    return ts >= 0 && ts < a.num_seqs && t0 >= 0 && t1 >= t0 && nm >= 1 && mbase >= 0 &&
           mbase <= a.num_members - nm && row0 >= 0 && row0 <= a.rows_per_head - nm * a.group &&
           (prefix ? (kind == CJ_PREFIX && nm <= CASCADE_CONSUMERS * mpo)
                   : (kind == CJ_SUFFIX && nm == 1 && __ldg(a.members + mbase) == ts));
  }
};

// Blocks [0, num_prefix_jobs): one prefix job each.  The block's warps share one ring of CASCADE_SLOTS tiles
// that warp 0 refills: before consuming tile i it makes sure tile i has been issued (waiting for the slot's
// previous tile to be released by every consuming warp) and issues further tiles whose slots are already
// free.  Blocks after them: CASCADE_CONSUMERS suffix jobs each, one per warp, every warp streaming its own
// tiles through its own CASCADE_WARP_SLOTS slots and issuing them itself.
template <class E, int D>
__global__ void __launch_bounds__(CASCADE_CONSUMERS * 32)
    cascade_partial_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                           const CascadeArgs a) {
  constexpr int KSTEPS = D / 16;
  constexpr uint32_t STAGE_BYTES = CascadeSmem<D>::STAGE_BYTES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *ring = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + CascadeSmem<D>::RING);
  uint64_t *empty = full + CASCADE_SLOTS;
  int *tile_bad = reinterpret_cast<int *>(empty + CASCADE_SLOTS);  // per slot: its tile was not copied
  int *member_bad = tile_bad + CASCADE_SLOTS;                       // bit i: member i failed the prefix checks
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int h = blockIdx.y;
  const int G = a.group;
  const int mpo = 8 / G;  // members per warp (the host accepts G <= 8)

  grid_dependency_wait();    // the step's new K/V rows and every other input may come from the previous kernel
  grid_launch_dependents();  // the combine kernel may launch now; it waits for this grid

  if ((int)blockIdx.x >= a.num_prefix_jobs) {
    // ---------------- suffix jobs: warp `warp` streams job num_prefix_jobs + 4 * (block - num_prefix) + warp
    const long long j = a.num_prefix_jobs + (long long)((int)blockIdx.x - a.num_prefix_jobs) * CASCADE_CONSUMERS + warp;
    if (j >= a.num_jobs) return;
    CascadeJob jb;
    if (!jb.load(a, (int)j, mpo)) {
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_PLAN);
      return;
    }
    const int L = __ldg(a.context_lens + jb.ts);
    const int nt = cascade_context_ok(a, L) ? max(0, min(jb.t1, (L + TILE - 1) / TILE) - jb.t0) : 0;
    uint64_t *wfull = full + warp * CASCADE_WARP_SLOTS;
    int *wbad = tile_bad + warp * CASCADE_WARP_SLOTS;
    unsigned char *wring = ring + warp * CASCADE_WARP_SLOTS * STAGE_BYTES;
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < CASCADE_WARP_SLOTS; ++k) mbar_init(&wfull[k], 1);
      fence_mbar_init();
      prefetch_tensor_map(&tmap_k);
      prefetch_tensor_map(&tmap_v);
    }
    __syncwarp();
    const int *row = a.block_tables + (long long)jb.ts * a.table_stride;
    const int nblk = ((jb.t0 + nt) * TILE + a.block_size - 1) / a.block_size;  // entries read: < nblk
    RowWindow win;
    auto issue = [&](int i) {  // tile i of the job into slot i % CASCADE_WARP_SLOTS (whole warp)
      const int t = jb.t0 + i;
      const int phys = win.lookup(row, t * TILE / a.block_size, nblk, lane);
      const int st = i % CASCADE_WARP_SLOTS;
      if (lane == 0) cascade_issue<D>(a, &tmap_k, &tmap_v, phys, t, h, wring + st * STAGE_BYTES, &wfull[st], &wbad[st]);
    };
    for (int i = 0; i < CASCADE_WARP_SLOTS && i < nt; ++i) issue(i);
    ColumnTile<E, D> ct;
    ct.init(a, lane, (lane >> 2) < G ? jb.ts : -1, h * G + ((lane >> 2) < G ? (lane >> 2) : 0));
    bool bad = false;
    int i = 0;
    for (; i < nt; ++i) {
      const int st = i % CASCADE_WARP_SLOTS;
      const bool arrived = mbar_wait_bounded(&wfull[st], (uint32_t)(i / CASCADE_WARP_SLOTS) & 1u, a.wait_limit_ns);
      if (__any_sync(FULL, !arrived)) {
        if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
        bad = true;
        break;
      }
      if (wbad[st] != 0) {  // warp-uniform
        if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
        bad = true;
      }
      float sc[4];
      uint32_t vf[KSTEPS][4];
      if (!bad) ct.scores(smem_addr(wring + st * STAGE_BYTES), sc, vf);
      __syncwarp();
      if (i + CASCADE_WARP_SLOTS < nt) issue(i + CASCADE_WARP_SLOTS);
      if (!bad) ct.accumulate(a, sc, vf, min(TILE, L - (jb.t0 + i) * TILE));
    }
    // copies still in flight after a timeout land (bounded) before the warp leaves
    for (int k = i + 1; k < nt && k < i + CASCADE_WARP_SLOTS; ++k)
      mbar_wait_bounded(&wfull[k % CASCADE_WARP_SLOTS], (uint32_t)(k / CASCADE_WARP_SLOTS) & 1u, a.wait_limit_ns);
    ct.store(a, (long long)h * a.rows_per_head + jb.row0, G, bad ? 0xffu : 0u, nt > 0);
    return;
  }

  // ---------------- a prefix job: the block's warps share the ring
  CascadeJob jb;
  if (!jb.load(a, (int)blockIdx.x, mpo)) {
    if (threadIdx.x == 0) atomicOr(&g_status, PA_DEV_ERR_PLAN);
    return;
  }
  const int L_lead = __ldg(a.context_lens + jb.ts);
  const bool lead_ok = cascade_context_ok(a, L_lead);
  const bool prefix_short = lead_ok && (long long)jb.t1 * TILE > L_lead;  // the leader does not hold the range
  const int nt = (lead_ok && !prefix_short) ? jb.t1 - jb.t0 : 0;
  const int n_oct = (jb.nm + mpo - 1) / mpo;  // warps with columns
  if (threadIdx.x == 0) {
#pragma unroll
    for (int st = 0; st < CASCADE_SLOTS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], n_oct);
      tile_bad[st] = 0;
    }
    // a leader that fails, or does not hold the range, fails the job for every member
    *member_bad = (!lead_ok || prefix_short) ? -1 : 0;
    if (prefix_short) atomicOr(&g_status, PA_DEV_ERR_PLAN);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp >= n_oct) return;  // no columns for this warp
  const int *lead_row = a.block_tables + (long long)jb.ts * a.table_stride;
  const int nblk = nt > 0 ? (jb.t1 * TILE + a.block_size - 1) / a.block_size : 0;
  RowWindow win;
  int issued = 0;
  bool issue_failed = false;
  // warp 0: issue tiles up to `upto` (inclusive) that are not issued yet; tile `need` and those before it are
  // waited for, later ones only if their slot is already free.  Returns false if a wait ran out.
  auto refill = [&](int need, int upto) {
    while (issued < nt && issued <= upto) {
      const int jt = issued, st = jt % CASCADE_SLOTS;
      if (jt >= CASCADE_SLOTS) {
        const uint32_t par = (uint32_t)(jt / CASCADE_SLOTS - 1) & 1u;
        bool free_slot;
        if (jt <= need) {
          free_slot = __all_sync(FULL, mbar_wait_bounded(&empty[st], par, a.wait_limit_ns));
          if (!free_slot) return false;
        } else {
          free_slot = __all_sync(FULL, mbar_try_wait(&empty[st], par));
          if (!free_slot) return true;
        }
      }
      const int t = jb.t0 + jt;
      const int phys = win.lookup(lead_row, t * TILE / a.block_size, nblk, lane);
      if (lane == 0) cascade_issue<D>(a, &tmap_k, &tmap_v, phys, t, h, ring + st * STAGE_BYTES, &full[st], &tile_bad[st]);
      __syncwarp();
      ++issued;
    }
    return true;
  };
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensor_map(&tmap_k);
      prefetch_tensor_map(&tmap_v);
    }
    refill(-1, CASCADE_SLOTS - 1);
  }
  const int mo = warp * mpo;  // the warp's first member
  ColumnTile<E, D> ct;
  {
    const int gid = lane >> 2;
    const bool live = gid < mpo * G && mo + gid / G < jb.nm;
    int m = live ? __ldg(a.members + jb.mbase + mo + gid / G) : -1;
    if (m >= a.num_seqs) m = -1;  // flagged by the member checks below
    ct.init(a, lane, m, h * G + (live ? gid % G : 0));
  }
  bool bad = false;
  for (int i = 0; i < nt; ++i) {
    const int st = i % CASCADE_SLOTS;
    if (warp == 0 && !issue_failed && !refill(i, i + CASCADE_SLOTS - 1)) {
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
      issue_failed = true;
    }
    const bool arrived = !issue_failed &&
                         __all_sync(FULL, mbar_wait_bounded(&full[st], (uint32_t)(i / CASCADE_SLOTS) & 1u, a.wait_limit_ns));
    if (!arrived) {
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_TIMEOUT);
      bad = true;
      break;
    }
    if (!bad && tile_bad[st] != 0) {  // warp-uniform
      if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
      bad = true;
    }
    float sc[4];
    uint32_t vf[KSTEPS][4];
    if (!bad) ct.scores(smem_addr(ring + st * STAGE_BYTES), sc, vf);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the slot
    if (!bad) ct.accumulate(a, sc, vf, TILE);
  }
  if (warp == 0) {
    // every member's table must name the leader's blocks over the job's range, and its context must hold it
    if (nt > 0) {
      const int b0 = jb.t0 * TILE / a.block_size;
      for (int k = lane; k < jb.nm; k += 32) {
        const int m = __ldg(a.members + jb.mbase + k);
        bool plan_ok = m >= 0 && m < a.num_seqs;
        const int L = plan_ok ? __ldg(a.context_lens + m) : 0;
        const bool ctx_ok = plan_ok && cascade_context_ok(a, L);
        plan_ok = plan_ok && (!ctx_ok || (long long)jb.t1 * TILE <= L);
        for (int b = b0; plan_ok && ctx_ok && b < nblk; ++b)
          plan_ok = __ldg(a.block_tables + (long long)m * a.table_stride + b) == __ldg(lead_row + b);
        if (!plan_ok || !ctx_ok) atomicOr(member_bad, 1 << k);
        if (!plan_ok) atomicOr(&g_status, PA_DEV_ERR_PLAN);  // a bad context is flagged by the combine kernel
      }
    }
    // every copy issued has landed before the block can finish (bounded)
    for (int k = 0; k < CASCADE_SLOTS && k < issued; ++k) {
      const int i = issued - 1 - k;
      mbar_wait_bounded(&full[i % CASCADE_SLOTS], (uint32_t)(i / CASCADE_SLOTS) & 1u, a.wait_limit_ns);
    }
  }
  asm volatile("bar.sync 1, %0;" ::"r"((uint32_t)n_oct * 32u) : "memory");  // member_bad is final
  const uint32_t mbad = (uint32_t)*member_bad;
  uint32_t bad_cols = bad ? 0xffu : 0u;
  for (int c = 0; c < 8; ++c)
    if ((mbad >> min(31, mo + c / G)) & 1u) bad_cols |= 1u << c;
  const int ncols = min(mpo, jb.nm - mo) * G;
  ct.store(a, (long long)h * a.rows_per_head + jb.row0 + (long long)mo * G, ncols, bad_cols, nt > 0);
}

// One warp per (sequence, query head).  Pieces with l = 0 (no tiles) take no part; a piece with l < 0 (a
// job that failed and set its own status bit) zeroes the row.  A context outside [0, min(table capacity, max_context_len)] gives a zero row
// and its status bit, as in pa_decode.
template <class E, int D>
__global__ void __launch_bounds__(256) cascade_combine_kernel(const CascadeArgs a) {
  constexpr int DPL = D / 32;  // dims per lane
  constexpr int MB = 8;        // partial rows requested together
  grid_dependency_wait();      // the partial kernel's rows
  grid_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (w >= (long long)a.num_seqs * a.num_q_heads) return;
  const int s = (int)(w / a.num_q_heads);
  const int hq = (int)(w - (long long)s * a.num_q_heads);
  const int h = hq / a.group, hh = hq - h * a.group;
  const long long head_rows = (long long)h * a.rows_per_head;
  float o[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) o[k] = 0.f;
  const int L = __ldg(a.context_lens + s);
  if (!cascade_context_ok(a, L)) {
    if (lane == 0 && hq == 0)
      atomicOr(&g_status, (L < 0 || (long long)L > (long long)a.table_stride * a.block_size) ? PA_DEV_ERR_CONTEXT
                                                                                            : PA_DEV_ERR_CONTEXT_HINT);
  } else if (L > 0) {
    const int p0 = __ldg(a.piece_offsets + s), p1 = __ldg(a.piece_offsets + s + 1);
    bool err = !(p0 >= 0 && p0 <= p1 && p1 <= a.num_pieces);  // plan indices out of range
    bool failed = false;                                       // a piece whose job flagged its own error
    const int n = err ? 0 : p1 - p0;
    // pass 1: the maximum over the pieces with tokens, and whether any piece failed
    float M = -INFINITY;
    for (int p = lane; p < n; p += 32) {
      const int r = __ldg(a.piece_rows + p0 + p);
      if (r < 0 || r > a.rows_per_head - a.group) {
        err = true;
        continue;
      }
      const float2 ml = __ldg(a.ws_ml + head_rows + r + hh);
      if (ml.y < 0.f) failed = true;
      if (ml.y > 0.f) M = fmaxf(M, ml.x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
    err = __any_sync(FULL, err);
    failed = __any_sync(FULL, failed);
    if (err && lane == 0) atomicOr(&g_status, PA_DEV_ERR_PLAN);
    if (!err && !failed) {
      // pass 2, in plan order: lane p of a 32-piece window holds piece p's row and weight
      float l = 0.f;
      for (int base = 0; base < n; base += 32) {
        const int p = base + lane;
        int r = 0;
        float wt = 0.f, lp = 0.f;
        if (p < n) {
          r = __ldg(a.piece_rows + p0 + p);
          const float2 ml = __ldg(a.ws_ml + head_rows + r + hh);
          if (ml.y > 0.f) {
            wt = exp2f(ml.x - M);
            lp = ml.y;
          }
        }
        const int nw = min(32, n - base);
        for (int i0 = 0; i0 < nw; i0 += MB) {
          float t[MB][DPL];
#pragma unroll
          for (int i = 0; i < MB; ++i) {
            const int ri = __shfl_sync(FULL, r, (i0 + i) & 31);
            const float wi = __shfl_sync(FULL, wt, (i0 + i) & 31);
            const bool use = i0 + i < nw && wi > 0.f;  // warp-uniform
            const float *src = a.ws_acc + (head_rows + ri + hh) * D + lane * DPL;
            if constexpr (DPL == 4) {
              const float4 v = use ? __ldg(reinterpret_cast<const float4 *>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
              t[i][0] = v.x;
              t[i][1] = v.y;
              t[i][2] = v.z;
              t[i][3] = v.w;
            } else {
              const float2 v = use ? __ldg(reinterpret_cast<const float2 *>(src)) : make_float2(0.f, 0.f);
              t[i][0] = v.x;
              t[i][1] = v.y;
            }
          }
#pragma unroll
          for (int i = 0; i < MB; ++i) {
            const float wi = __shfl_sync(FULL, wt, (i0 + i) & 31);
            const float li = __shfl_sync(FULL, lp, (i0 + i) & 31);
            if (i0 + i < nw && wi > 0.f) {
              l = fmaf(li, wi, l);
#pragma unroll
              for (int k = 0; k < DPL; ++k) o[k] = fmaf(wi, t[i][k], o[k]);
            }
          }
        }
      }
      if (l > 0.f) {
#pragma unroll
        for (int k = 0; k < DPL; ++k) o[k] = o[k] / l;
      } else {  // a context with tokens that no piece covered: the plan does not fit the call
        if (lane == 0) atomicOr(&g_status, PA_DEV_ERR_PLAN);
#pragma unroll
        for (int k = 0; k < DPL; ++k) o[k] = 0.f;
      }
    }
  }
  uint16_t *dst = a.out + (long long)s * a.out_seq_stride + (long long)hq * D + lane * DPL;
  if constexpr (DPL == 4) {
    *reinterpret_cast<uint2 *>(dst) = make_uint2(E::narrow2(o[0], o[1]), E::narrow2(o[2], o[3]));
  } else {
    *reinterpret_cast<uint32_t *>(dst) = E::narrow2(o[0], o[1]);
  }
}

}  // namespace pa
