// Tensor-core partition kernel for grouped-query decode: 3 to 8 query heads
// of one unit share each K/V tile, so the query-group x tile product is a
// real dense contraction and runs on mma.sync (m16n8k16, fp32 accumulation).
//
// Per 16-token tile, with the unit's query heads as the N = 8 columns:
//   S^T[16 tokens x 8 heads]  = K[16 x d] . Q^T[d x 8]          (d/16 mma)
//   O^T[d x 8 heads]         += V^T[d x 16 tokens] . P^T[16 x 8] (2 * d/16 mma)
// K and V tiles arrive by TMA tensor copies with the 128-byte swizzle (one
// 3-D box per tile: the D / 64 halves of the 16 rows, each stored as 16 rows
// of 128 bytes), so the ldmatrix loads of both operands are free of bank
// conflicts.  P is
// split into a 2-byte head and a 2-byte residual (P ~= Ph + Pl, relative
// error ~2^-16) so the product keeps fp32-level accuracy although the mma
// takes 2-byte operands; movmatrix turns P^T's accumulator layout into the
// B operand layout.  The online softmax runs along the token (M) axis, per
// head column, with the same lazy rescaling as the CUDA-core kernel.
#pragma once

#include <cuda.h>

#include "pa_kernels.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <class E>
struct MmaOps;

template <>
struct MmaOps<F16> {
  static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    mma_16816_f16(d, a, b0, b1);
  }
  // p0, p1 -> packed head (nearest) and packed residual
  static __device__ __forceinline__ void split(float p0, float p1, uint32_t &hi, uint32_t &lo) {
    __half2 h = __floats2half2_rn(p0, p1);
    const float2 f = __half22float2(h);
    __half2 l = __floats2half2_rn(p0 - f.x, p1 - f.y);
    hi = *reinterpret_cast<uint32_t *>(&h);
    lo = *reinterpret_cast<uint32_t *>(&l);
  }
};

template <>
struct MmaOps<BF16> {
  static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    mma_16816_bf16(d, a, b0, b1);
  }
  // head = upper 16 bits (truncation; the residual is then exact in fp32)
  static __device__ __forceinline__ void split(float p0, float p1, uint32_t &hi, uint32_t &lo) {
    const uint32_t u0 = __float_as_uint(p0) & 0xffff0000u;
    const uint32_t u1 = __float_as_uint(p1) & 0xffff0000u;
    hi = (u0 >> 16) | u1;
    __nv_bfloat162 l = __floats2bfloat162_rn(p0 - __uint_as_float(u0), p1 - __uint_as_float(u1));
    lo = *reinterpret_cast<uint32_t *>(&l);
  }
};

// Offset of 16-byte chunk c (8 head dims) of token row r in a tile stored as
// D/64 boxes of [16 rows x 128 bytes] with the TMA 128-byte swizzle.
__device__ __forceinline__ uint32_t swizzled(int r, int c) {
  return (uint32_t)((c >> 3) * 2048 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <class E, int D, int WARPS, int STAGES>
struct MmaSmem {
  static constexpr uint32_t STAGE_BYTES = 2 * TILE * D * 2;
  static constexpr uint32_t RING = WARPS * STAGES * STAGE_BYTES;
  static constexpr uint32_t BARS = ((WARPS * STAGES * 8 + 127) / 128) * 128;
  static __host__ __device__ constexpr uint32_t bytes(int num_seqs) {
    return 1024 + RING + BARS + (uint32_t)(num_seqs + 1 + WARPS) * 4u;  // 1024: alignment slack
  }
};

template <class E, int D, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, 12 / WARPS)
    decode_split_mma_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                            const DecodeArgs a) {
  constexpr int KSTEPS = D / 16;  // 16-dim steps of QK^T, and 16-dim row tiles of O^T
  constexpr uint32_t TILE_BYTES = TILE * D * 2;
  using Smem = MmaSmem<E, D, WARPS, STAGES>;
  constexpr uint32_t STAGE_BYTES = Smem::STAGE_BYTES;

  extern __shared__ unsigned char smem_raw[];
  // ring slots start on a 1024-byte boundary (the swizzle pattern repeats every 1024 bytes)
  unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  unsigned char *ring = smem + warp * STAGES * STAGE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Smem::RING) + warp * STAGES;
  int *pt = reinterpret_cast<int *>(smem + Smem::RING + Smem::BARS);
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < STAGES; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
    prefetch_tensor_map(&tmap_k);
    prefetch_tensor_map(&tmap_v);
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
  const int G = a.heads_per_unit;

  const int gid = lane >> 2;  // mma row group
  const int tig = lane & 3;   // thread in group
  // ldmatrix row addresses: lane supplies row (lane & 7) of matrix (lane >> 3)
  const int mi = lane >> 3, mr = lane & 7;
  const int ka_tok = 8 * (mi & 1) + mr, ka_c = mi >> 1;  // K as A (non-transposed)
  const int va_tok = 8 * (mi >> 1) + mr, va_c = mi & 1;  // V^T as A (transposed)
  const int ha = 2 * tig, hb = 2 * tig + 1;              // this lane's head columns
  uint32_t iter = 0;
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
      // one 3-D box per K and per V tile: [D / 64 halves][16 rows][64 elements] (see cache_tensor_map)
      if (lane == 0) {
        fence_proxy_async_smem();
        if (phys >= 0) {
          const int row0 = (int)prod.first_row(a, phys);  // lookup() checked the tile lies in its slab
          unsigned char *dst = ring + st * STAGE_BYTES;
          mbar_arrive_expect_tx(&bars[st], STAGE_BYTES);
          tc::tma_load_3d(dst, &tmap_k, 0, row0, 0, &bars[st]);
          tc::tma_load_3d(dst + TILE_BYTES, &tmap_v, 0, row0, 0, &bars[st]);
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

    uint32_t qb[KSTEPS][2];
    float o[KSTEPS][4];
    float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
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
        // Q^T as the B operand: b0 = Q[head gid][16ks + 2tig, +1], b1 = the same 8 dims later
        const bool row_live = gid < G && q_ok;
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(a.q + (long long)cp.s * a.q_seq_stride +
                                                                  (long long)(hq0 + (row_live ? gid : 0)) * D);
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          qb[ks][0] = row_live ? __ldg(qrow + 8 * ks + tig) : 0u;
          qb[ks][1] = row_live ? __ldg(qrow + 8 * ks + 4 + tig) : 0u;
          o[ks][0] = o[ks][1] = o[ks][2] = o[ks][3] = 0.f;
        }
        ma = mb = -INFINITY;
        la = lb = 0.f;
      }
      const int st = (int)(iter % STAGES);
      if (!wait_slot<STAGES>(bars, iter, (int)(issued - iter), a.wait_limit_ns, lane)) return;
      const bool tile_bad = (prod.bad_slots >> st) & 1u;  // warp-uniform
      piece_bad |= tile_bad;
      // S^T = K Q^T (K fragments loaded just before use), then the V^T fragments; then the slot is free
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t vf[KSTEPS][4];
      if (!piece_bad) {
        const uint32_t kt = smem_addr(ring + st * STAGE_BYTES);
        const uint32_t vt = kt + TILE_BYTES;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          uint32_t kf[4];
          ldsm_x4(kf, kt + swizzled(ka_tok, 2 * ks + ka_c));
          MmaOps<E>::mma(sc, kf, qb[ks][0], qb[ks][1]);
        }
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) ldsm_x4_trans(vf[ks], vt + swizzled(va_tok, 2 * ks + va_c));
      }
      __syncwarp();
      issue_next();
      ++iter;

      if (!piece_bad) {
        const int nvalid = min(TILE, L - cp.j * TILE);
        // s0 = (token gid, head ha), s1 = (gid, hb), s2 = (gid + 8, ha), s3 = (gid + 8, hb)
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
          const float alpha_a = exp2f(ma - na), alpha_b = exp2f(mb - nb);  // 0 on the piece's first tile
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

        // P^T (tokens x heads) in accumulator layout -> P as the B operand (k = tokens, n = heads)
        uint32_t h01, l01, h23, l23;
        MmaOps<E>::split(p0, p1, h01, l01);
        MmaOps<E>::split(p2, p3, h23, l23);
        const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
        const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);

        if (nvalid < TILE) {  // V rows past the sequence may hold NaN: zero them (0 * NaN would leak in)
          const uint32_t m_lo = (2 * tig < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 1 < nvalid ? 0xffff0000u : 0u);
          const uint32_t m_hi =
              (2 * tig + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 9 < nvalid ? 0xffff0000u : 0u);
#pragma unroll
          for (int ks = 0; ks < KSTEPS; ++ks) {
            vf[ks][0] &= m_lo;
            vf[ks][1] &= m_lo;
            vf[ks][2] &= m_hi;
            vf[ks][3] &= m_hi;
          }
        }
        // O^T += V^T P^T, head part then residual part
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
          MmaOps<E>::mma(o[mt], vf[mt], bh0, bh1);
          MmaOps<E>::mma(o[mt], vf[mt], bl0, bl1);
        }
      }

      if (cp.j + 1 == cp.nt || cons_left == 1) {
        // ---- end of the piece: totals per head column (lanes with the same tig), then store
        float lta = la, ltb = lb;
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          lta += __shfl_xor_sync(FULL, lta, off);
          ltb += __shfl_xor_sync(FULL, ltb, off);
        }
        if (piece_bad && lane == 0) atomicOr(&g_status, PA_DEV_ERR_BLOCK_ID);
        if (full) {
          // normalise, narrow, transpose 8x8 blocks back to [head][dims]: lane then holds head gid, dims 2tig, 2tig+1
          const float ia = piece_bad ? 0.f : 1.f / lta, ib = piece_bad ? 0.f : 1.f / ltb;
          uint16_t *orow = a.out + (long long)cp.s * a.out_seq_stride + (long long)(hq0 + (gid < G ? gid : 0)) * D + 2 * tig;
#pragma unroll
          for (int mt = 0; mt < KSTEPS; ++mt) {
            const uint32_t t0w = movmatrix_trans(E::narrow2(piece_bad ? 0.f : o[mt][0] * ia, piece_bad ? 0.f : o[mt][1] * ib));
            const uint32_t t1w = movmatrix_trans(E::narrow2(piece_bad ? 0.f : o[mt][2] * ia, piece_bad ? 0.f : o[mt][3] * ib));
            if (gid < G && dcheck(cp.s < S && hq0 + G <= a.num_q_heads)) {
              *reinterpret_cast<uint32_t *>(orow + 16 * mt) = t0w;
              *reinterpret_cast<uint32_t *>(orow + 16 * mt + 8) = t1w;
            }
          }
        } else {
          const long long prow = (cons_c * 2 + slot) * G;
          const bool row_ok = dcheck(cons_c < a.max_chunks);
          if (!piece_bad && row_ok) {
#pragma unroll
            for (int mt = 0; mt < KSTEPS; ++mt) {
              const int d0 = 16 * mt + gid;
              if (ha < G) {
                a.ws_acc[(prow + ha) * D + d0] = o[mt][0];
                a.ws_acc[(prow + ha) * D + d0 + 8] = o[mt][2];
              }
              if (hb < G) {
                a.ws_acc[(prow + hb) * D + d0] = o[mt][1];
                a.ws_acc[(prow + hb) * D + d0 + 8] = o[mt][3];
              }
            }
          }
          if (gid == 0 && row_ok) {
            if (ha < G) a.ws_ml[prow + ha] = piece_bad ? make_float2(-INFINITY, -1.f) : make_float2(ma, lta);
            if (hb < G) a.ws_ml[prow + hb] = piece_bad ? make_float2(-INFINITY, -1.f) : make_float2(mb, ltb);
          }
        }
      }
      advance_tile(cp, pt, S, HC);
      --cons_left;
      ++k;
    }
  }
}

}  // namespace pa
