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
#ifndef CASCADE_MIN_BLOCKS
#define CASCADE_MIN_BLOCKS 3
#endif

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
// an entry outside the pool flags the slot instead and completes the barrier without data.  The caller has
// fenced the generic-proxy reads of the slot's previous contents against the copy (fence_proxy_async_smem, once
// for any number of copies issued after it).
template <int D>
__device__ __forceinline__ void cascade_issue(const CascadeArgs &a, const CUtensorMap *mk, const CUtensorMap *mv,
                                              int phys, int t, int h, unsigned char *dst, uint64_t *bar, int *bad) {
  constexpr uint32_t TILE_BYTES = TILE * D * 2;
  const bool ok = phys >= 0 && (long long)phys < a.num_blocks;
  *bad = ok ? 0 : 1;
  if (ok) {
    const int row = (int)(((long long)phys * a.num_kv_heads + h) * a.block_size + (t * TILE) % a.block_size);
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

// One warp's 16 query rows (row r: member r / G of the warp's row tile, head r % G) against a 16-token tile, with
// the queries as the mma's M dimension (prefix jobs, where many rows share each tile):
//   S[16 rows x 16 tokens]  = Q[16 x d] . K^T[d x 16]        (two 8-token halves, d/16 mma each)
//   O[16 rows x d]         += P[16 x 16 tokens] . V[16 x d]  (d/8 mma, twice: P's 2-byte head and residual)
// P's accumulator layout is the A operand's, so it feeds the second product without a transpose.  Each thread
// holds rows gid and gid + 8 and keeps their online softmax state.
template <class E, int D>
struct RowTile {
  static constexpr int KSTEPS = D / 16, NT = D / 8;
  uint32_t qa[KSTEPS][4];
  float o[NT][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows gid, gid + 8
  int gid, tig, kb_tok, kb_c, vb_tok, vb_c;

  __device__ __forceinline__ void init(const CascadeArgs &a, int lane, int seq_lo, int head_lo, int seq_hi,
                                       int head_hi) {
    gid = lane >> 2;
    tig = lane & 3;
    const int mi = lane >> 3, mr = lane & 7;
    kb_tok = 8 * (mi >> 1) + mr, kb_c = mi & 1;  // K rows as the B operand: [tokens 0-7 | 8-15] x [dims lo | hi]
    vb_tok = 8 * (mi & 1) + mr, vb_c = mi >> 1;  // V rows as the B operand, transposed: two 8-dim column tiles
    const uint32_t *qlo = reinterpret_cast<const uint32_t *>(a.q + (long long)max(seq_lo, 0) * a.q_seq_stride +
                                                             (long long)head_lo * D);
    const uint32_t *qhi = reinterpret_cast<const uint32_t *>(a.q + (long long)max(seq_hi, 0) * a.q_seq_stride +
                                                             (long long)head_hi * D);
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      qa[ks][0] = seq_lo >= 0 ? __ldg(qlo + 8 * ks + tig) : 0u;
      qa[ks][1] = seq_hi >= 0 ? __ldg(qhi + 8 * ks + tig) : 0u;
      qa[ks][2] = seq_lo >= 0 ? __ldg(qlo + 8 * ks + 4 + tig) : 0u;
      qa[ks][3] = seq_hi >= 0 ? __ldg(qhi + 8 * ks + 4 + tig) : 0u;
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  }

  // S = Q K^T from the slot at shared address kt, and the V fragments; the slot may be reused after this
  __device__ __forceinline__ void scores(uint32_t kt, float (&s)[2][4], uint32_t (&vf)[NT / 2][4]) const {
    constexpr uint32_t TILE_BYTES = TILE * D * 2;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) s[h2][0] = s[h2][1] = s[h2][2] = s[h2][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      uint32_t kf[4];
      ldsm_x4(kf, kt + swizzled(kb_tok, 2 * ks + kb_c));
      MmaOps<E>::mma(s[0], qa[ks], kf[0], kf[1]);
      MmaOps<E>::mma(s[1], qa[ks], kf[2], kf[3]);
    }
#pragma unroll
    for (int c2 = 0; c2 < NT / 2; ++c2) ldsm_x4_trans(vf[c2], kt + TILE_BYTES + swizzled(vb_tok, 2 * c2 + vb_c));
  }

  __device__ __forceinline__ void accumulate(const CascadeArgs &a, const float (&s)[2][4], uint32_t (&vf)[NT / 2][4],
                                             int nvalid) {
    // z[h2][0..1]: row gid, tokens 8*h2 + 2tig, +1; z[h2][2..3]: row gid + 8
    float z[2][4];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
      for (int k = 0; k < 4; ++k) z[h2][k] = 8 * h2 + 2 * tig + (k & 1) < nvalid ? s[h2][k] * a.scale_log2 : -INFINITY;
    const float c0 = fmaxf(fmaxf(z[0][0], z[0][1]), fmaxf(z[1][0], z[1][1]));
    const float c1 = fmaxf(fmaxf(z[0][2], z[0][3]), fmaxf(z[1][2], z[1][3]));
    if (__any_sync(FULL, c0 > m0 + RESCALE_SLACK || c1 > m1 + RESCALE_SLACK)) {
      float r0 = fmaxf(c0, __shfl_xor_sync(FULL, c0, 1)), r1 = fmaxf(c1, __shfl_xor_sync(FULL, c1, 1));
      r0 = fmaxf(r0, __shfl_xor_sync(FULL, r0, 2));
      r1 = fmaxf(r1, __shfl_xor_sync(FULL, r1, 2));
      const float n0 = fmaxf(m0, r0), n1 = fmaxf(m1, r1);
      const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);  // 0 on the first tile
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        o[nt][0] *= al0;
        o[nt][1] *= al0;
        o[nt][2] *= al1;
        o[nt][3] *= al1;
      }
      l0 *= al0;
      l1 *= al1;
      m0 = n0;
      m1 = n1;
    }
    float p[2][4];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      p[h2][0] = exp2f(z[h2][0] - m0);
      p[h2][1] = exp2f(z[h2][1] - m0);
      p[h2][2] = exp2f(z[h2][2] - m1);
      p[h2][3] = exp2f(z[h2][3] - m1);
    }
    l0 += (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]);
    l1 += (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]);
    // A operand of P . V: a0 row gid tokens 2tig..; a1 row gid + 8; a2, a3 the same rows, tokens 8 + 2tig..
    uint32_t ah[4], al[4];
    MmaOps<E>::split(p[0][0], p[0][1], ah[0], al[0]);
    MmaOps<E>::split(p[0][2], p[0][3], ah[1], al[1]);
    MmaOps<E>::split(p[1][0], p[1][1], ah[2], al[2]);
    MmaOps<E>::split(p[1][2], p[1][3], ah[3], al[3]);
    if (nvalid < TILE) {  // V rows past the context may hold NaN: zero them (0 * NaN would leak in)
      const uint32_t m_lo = (2 * tig < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 1 < nvalid ? 0xffff0000u : 0u);
      const uint32_t m_hi = (2 * tig + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 9 < nvalid ? 0xffff0000u : 0u);
#pragma unroll
      for (int c2 = 0; c2 < NT / 2; ++c2) {
        vf[c2][0] &= m_lo;
        vf[c2][1] &= m_hi;
        vf[c2][2] &= m_lo;
        vf[c2][3] &= m_hi;
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t b0 = vf[nt >> 1][(nt & 1) * 2], b1 = vf[nt >> 1][(nt & 1) * 2 + 1];
      MmaOps<E>::mma(o[nt], ah, b0, b1);
      MmaOps<E>::mma(o[nt], al, b0, b1);
    }
  }

  // Writes rows gid and gid + 8 (if live) to partial rows row_lo / row_hi (per kv head), as ColumnTile::store.
  __device__ __forceinline__ void store(const CascadeArgs &a, long long row_lo, long long row_hi, bool live_lo,
                                        bool live_hi, bool bad_lo, bool bad_hi, bool any_tiles) {
    float t0 = l0 + __shfl_xor_sync(FULL, l0, 1), t1 = l1 + __shfl_xor_sync(FULL, l1, 1);
    t0 += __shfl_xor_sync(FULL, t0, 2);
    t1 += __shfl_xor_sync(FULL, t1, 2);
    if (tig == 0) {
      if (live_lo) a.ws_ml[row_lo] = bad_lo ? make_float2(-INFINITY, -1.f) : make_float2(m0, t0);
      if (live_hi) a.ws_ml[row_hi] = bad_hi ? make_float2(-INFINITY, -1.f) : make_float2(m1, t1);
    }
    if (!any_tiles) return;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (live_lo && !bad_lo)
        *reinterpret_cast<float2 *>(a.ws_acc + row_lo * D + 8 * nt + 2 * tig) = make_float2(o[nt][0], o[nt][1]);
      if (live_hi && !bad_hi)
        *reinterpret_cast<float2 *>(a.ws_acc + row_hi * D + 8 * nt + 2 * tig) = make_float2(o[nt][2], o[nt][3]);
    }
  }
};

// One job of the plan, read and checked (the plan lives in the caller's memory).  `per` is the members one
// warp holds: 8 / G columns for a suffix job's warp, 16 / G rows for a prefix job's row tile.
struct CascadeJob {
  int ts, t0, t1, mbase, nm, row0, kind, split;
  __device__ __forceinline__ bool load(const CascadeArgs &a, int j, int per) {
    const int *job = a.jobs + (long long)j * CJ_INTS;
    ts = __ldg(job + CJ_SEQ), t0 = __ldg(job + CJ_T0), t1 = __ldg(job + CJ_T1);
    mbase = __ldg(job + CJ_MEMBERS), nm = __ldg(job + CJ_NM), row0 = __ldg(job + CJ_ROW), kind = __ldg(job + CJ_KIND);
    split = __ldg(job + CJ_SPLIT);
    const bool prefix = j < a.num_prefix_jobs;
    const int n_rt = (nm + per - 1) / per;
    const bool shape_ok = prefix ? (kind == CJ_PREFIX && (split == 1 || split == 2 || split == 4) &&
                                    nm <= CASCADE_CONSUMERS * per && n_rt * split <= CASCADE_CONSUMERS)
                                 : (kind == CJ_SUFFIX && split == 1 && nm == 1);
    return shape_ok && ts >= 0 && ts < a.num_seqs && t0 >= 0 && t1 >= t0 && nm >= 1 && mbase >= 0 &&
           mbase <= a.num_members - nm && row0 >= 0 && (long long)row0 + (long long)nm * a.group * split <= a.rows_per_head &&
           (prefix || __ldg(a.members + mbase) == ts);
  }
};

// Blocks [0, num_prefix_jobs): one prefix job each.  The block's warps share one ring of CASCADE_SLOTS tiles
// that warp 0 refills: before consuming tile i it makes sure tile i has been issued (waiting for the slot's
// previous tile to be released by every consuming warp) and issues further tiles whose slots are already
// free.  Blocks after them: CASCADE_CONSUMERS suffix jobs each, one per warp, every warp streaming its own
// tiles through its own CASCADE_WARP_SLOTS slots and issuing them itself.
template <class E, int D>
__global__ void __launch_bounds__(CASCADE_CONSUMERS * 32, CASCADE_MIN_BLOCKS)
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
      if (lane == 0) {
        fence_proxy_async_smem();  // the slot's previous tile was read through the generic proxy
        cascade_issue<D>(a, &tmap_k, &tmap_v, phys, t, h, wring + st * STAGE_BYTES, &wfull[st], &wbad[st]);
      }
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

  // ---------------- a prefix job: the block's warps share the ring.  Warp w takes row tile w % n_rt (16 of the
  // job's member x head rows) and tiles i = w / n_rt (mod split) of the job.
  CascadeJob jb;
  const int mpr = 16 / G;  // members per row tile
  if (!jb.load(a, (int)blockIdx.x, mpr)) {
    if (threadIdx.x == 0) atomicOr(&g_status, PA_DEV_ERR_PLAN);
    return;
  }
  const int n_rt = (jb.nm + mpr - 1) / mpr;
  const int split = jb.split;
  const int L_lead = __ldg(a.context_lens + jb.ts);
  const bool lead_ok = cascade_context_ok(a, L_lead);
  const bool prefix_short = lead_ok && (long long)jb.t1 * TILE > L_lead;  // the leader does not hold the range
  const int nt = (lead_ok && !prefix_short) ? jb.t1 - jb.t0 : 0;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int st = 0; st < CASCADE_SLOTS; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], n_rt);  // tile i is read by the n_rt warps of split i % split
      tile_bad[st] = 0;
    }
    // a leader that fails, or does not hold the range, fails the job for every member
    *member_bad = (!lead_ok || prefix_short) ? -1 : 0;
    if (prefix_short) atomicOr(&g_status, PA_DEV_ERR_PLAN);
    fence_mbar_init();
  }
  __syncthreads();
  const int n_warps = n_rt * split;
  if (warp >= n_warps) return;
  const int rt = warp % n_rt, sp = warp / n_rt;
  const int *lead_row = a.block_tables + (long long)jb.ts * a.table_stride;
  const int nblk = nt > 0 ? (jb.t1 * TILE + a.block_size - 1) / a.block_size : 0;
  int issued = 0;
  bool issue_failed = false;
  // warp 0: issue tiles up to `upto` (inclusive) that are not issued yet; tiles up to `need` are waited for,
  // later ones only if their slot is already free.  Lane k takes the k-th next tile, so a run of free slots is
  // filled by one round of copies.  Returns false if a wait ran out.
  auto refill = [&](int need, int upto) {
    while (issued < nt && issued <= upto) {
      const int jt = issued + lane;
      bool ready = jt < nt && jt <= upto;
      if (ready && jt >= CASCADE_SLOTS)
        ready = mbar_try_wait(&empty[jt % CASCADE_SLOTS], (uint32_t)(jt / CASCADE_SLOTS - 1) & 1u);
      const unsigned run = __ballot_sync(FULL, ready);
      const int c = run == FULL ? 32 : __ffs(~run) - 1;  // lanes 0 .. c-1 issue
      if (c == 0) {
        if (issued > need) return true;
        const int st = issued % CASCADE_SLOTS;  // a tile that is needed now: wait for its slot
        if (!__all_sync(FULL, mbar_wait_bounded(&empty[st], (uint32_t)(issued / CASCADE_SLOTS - 1) & 1u, a.wait_limit_ns)))
          return false;
        continue;
      }
      if (lane < c) {
        const int t = jb.t0 + jt;
        const int phys = __ldg(lead_row + t * TILE / a.block_size);  // an entry below nblk
        fence_proxy_async_smem();  // the freed slot was read through the generic proxy
        cascade_issue<D>(a, &tmap_k, &tmap_v, phys, t, h, ring + (jt % CASCADE_SLOTS) * STAGE_BYTES,
                         &full[jt % CASCADE_SLOTS], &tile_bad[jt % CASCADE_SLOTS]);
      }
      __syncwarp();
      issued += c;
    }
    return true;
  };
  // this lane's rows gid and gid + 8 of the row tile: member rt * mpr + r / G, head r % G
  const int gid = lane >> 2;
  const int r_lo = gid, r_hi = gid + 8;
  const int ml_lo = rt * mpr + r_lo / G, ml_hi = rt * mpr + r_hi / G;
  const bool live_lo = r_lo < mpr * G && ml_lo < jb.nm, live_hi = r_hi < mpr * G && ml_hi < jb.nm;
  RowTile<E, D> rtile;
  {
    int m_lo = live_lo ? __ldg(a.members + jb.mbase + ml_lo) : -1;
    int m_hi = live_hi ? __ldg(a.members + jb.mbase + ml_hi) : -1;
    if (m_lo >= a.num_seqs) m_lo = -1;  // flagged by the member checks below
    if (m_hi >= a.num_seqs) m_hi = -1;
    rtile.init(a, lane, m_lo, h * G + r_lo % G, m_hi, h * G + r_hi % G);
  }
  if (warp == 0) {  // the first tiles, while the Q loads above are in flight
    if (lane == 0) {
      prefetch_tensor_map(&tmap_k);
      prefetch_tensor_map(&tmap_v);
    }
    refill(-1, CASCADE_SLOTS - 1);
  }
  bool bad = false;
  int done = 0;  // tiles this warp consumed
  for (int i = sp; i < nt; i += split) {
    const int st = i % CASCADE_SLOTS;
    if (warp == 0 && !issue_failed && !refill(i + split - 1, i + CASCADE_SLOTS - 1)) {
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
    float sc[2][4];
    uint32_t vf[RowTile<E, D>::NT / 2][4];
    if (!bad) rtile.scores(smem_addr(ring + st * STAGE_BYTES), sc, vf);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the slot
    if (!bad) rtile.accumulate(a, sc, vf, TILE);
    ++done;
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
  asm volatile("bar.sync 1, %0;" ::"r"((uint32_t)n_warps * 32u) : "memory");  // member_bad is final
  const uint32_t mbad = (uint32_t)*member_bad;
  // rows of split sp: row0 + sp * nm * G + member * G + head
  const long long base = (long long)h * a.rows_per_head + jb.row0 + (long long)sp * jb.nm * G + (long long)rt * mpr * G;
  rtile.store(a, base + r_lo, base + r_hi, live_lo, live_hi, bad || ((mbad >> min(31, ml_lo)) & 1u),
              bad || ((mbad >> min(31, ml_hi)) & 1u), done > 0);
}

// Partial rows [i0, i0 + MB) of a 32-piece window whose lane p holds piece p's row r and range flag bad, for
// query head hh of the kv head whose rows start at head_rows: lane l takes dims [l * DPL, (l + 1) * DPL).  Rows
// at or past nw, or out of range, are not read (zeros).
template <int D, int MB>
__device__ __forceinline__ void cascade_load_rows(const CascadeArgs &a, float (&t)[MB][D / 32], long long head_rows,
                                                  int hh, int r, bool bad, int i0, int nw, int lane) {
  constexpr int DPL = D / 32;
#pragma unroll
  for (int i = 0; i < MB; ++i) {
    const int ri = __shfl_sync(FULL, r, (i0 + i) & 31);
    const bool bi = __shfl_sync(FULL, bad ? 1 : 0, (i0 + i) & 31) != 0;
    const bool use = i0 + i < nw && !bi;  // warp-uniform
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
}

// One warp per (sequence, query head).  Pieces with l = 0 (no tiles) take no part; a piece with l < 0 (a
// job that failed and set its own status bit) zeroes the row.  A context outside [0, min(table capacity, max_context_len)] gives a zero row
// and its status bit, as in pa_decode.
//
// Memory trips.  Behind the partial kernel (num_jobs > 0) the length, the piece offsets and the first 32 piece
// rows are read before the grid-dependency wait: they are inputs of the call, which the partial kernel does not
// write, and that kernel triggers this launch only after its own wait, so every earlier write in the stream is
// complete by then.  After the wait, the pieces' (m, l) and the partial rows of the first MB pieces are requested
// in one trip.  Without a partial kernel the wait comes first, as the inputs may come from the previous kernel.
template <class E, int D>
__global__ void __launch_bounds__(256) cascade_combine_kernel(const CascadeArgs a) {
  constexpr int DPL = D / 32;  // dims per lane
  constexpr int MB = 8;        // partial rows requested together
  const bool after_partial = a.num_jobs > 0;
  if (!after_partial) grid_dependency_wait();  // the inputs may come from the previous kernel in the stream
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (w >= (long long)a.num_seqs * a.num_q_heads) return;
  const int s = (int)(w / a.num_q_heads);
  const int hq = (int)(w - (long long)s * a.num_q_heads);
  const int h = hq / a.group, hh = hq - h * a.group;
  const long long head_rows = (long long)h * a.rows_per_head;
  const int L = __ldg(a.context_lens + s);
  const int p0 = __ldg(a.piece_offsets + s), p1 = __ldg(a.piece_offsets + s + 1);
  const bool ctx_ok = cascade_context_ok(a, L);
  bool err = ctx_ok && L > 0 && !(p0 >= 0 && p0 <= p1 && p1 <= a.num_pieces);  // plan indices out of range
  const int n = ctx_ok && L > 0 && !err ? p1 - p0 : 0;
  // the first window's pieces: lane p holds piece p's row and whether it lies inside the workspace
  int r0 = 0;
  bool bad0 = false;
  if (lane < n) {
    r0 = __ldg(a.piece_rows + p0 + lane);
    bad0 = r0 < 0 || r0 > a.rows_per_head - a.group;
  }
  if (after_partial) grid_dependency_wait();  // the partial kernel's rows
  grid_launch_dependents();

  float o[DPL];
#pragma unroll
  for (int k = 0; k < DPL; ++k) o[k] = 0.f;
  if (!ctx_ok) {
    if (lane == 0 && hq == 0)
      atomicOr(&g_status, (L < 0 || (long long)L > (long long)a.table_stride * a.block_size) ? PA_DEV_ERR_CONTEXT
                                                                                            : PA_DEV_ERR_CONTEXT_HINT);
  } else if (L > 0) {
    // one trip: the first window's (m, l) and the first MB partial rows
    float2 ml0 = make_float2(-INFINITY, 0.f);
    if (lane < n && !bad0) ml0 = __ldg(a.ws_ml + head_rows + r0 + hh);
    const int nw0 = min(32, n);
    float t[MB][DPL];
    cascade_load_rows<D, MB>(a, t, head_rows, hh, r0, bad0, 0, nw0, lane);
    // pass 1: the maximum over the pieces with tokens, and whether any piece failed
    bool failed = lane < n && !bad0 && ml0.y < 0.f;  // a piece whose job flagged its own error
    err = err || (lane < n && bad0);
    float M = lane < n && !bad0 && ml0.y > 0.f ? ml0.x : -INFINITY;
    for (int p = 32 + lane; p < n; p += 32) {
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
        int r = r0;
        float2 ml = ml0;
        if (base > 0) {
          r = 0;
          ml = make_float2(-INFINITY, 0.f);
          if (p < n) {
            r = __ldg(a.piece_rows + p0 + p);
            ml = __ldg(a.ws_ml + head_rows + r + hh);
          }
        }
        float wt = 0.f, lp = 0.f;
        if (p < n && ml.y > 0.f) {
          wt = exp2f(ml.x - M);
          lp = ml.y;
        }
        const int nw = min(32, n - base);
        for (int i0 = 0; i0 < nw; i0 += MB) {
          if (base > 0 || i0 > 0) cascade_load_rows<D, MB>(a, t, head_rows, hh, r, false, i0, nw, lane);
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
