// Fused projection + pool for the scalar-logit form of the compressor ("Ch 04 · CSA" §3
// symbol table: one score z_j per token and stream, Z = H w^{Z} with w^{Z} in R^d, an
// m-dimensional position bias, and one weight S_j for the whole vector C_j).  Included by
// fused_proj.cu: it uses that file's pair wrappers, work schedule and device error word.
//
// The value streams C = H W^{KV} are accumulated on the tensor cores by CTA pairs
// (tcgen05 cta_group::2, M = 256) as in fused_pair_kernel, but the pair is split by
// channel: each CTA holds two 128-lane accumulators of its own channels, C^a and C^b of one
// channel group (CSA), or C of two channel groups (HCA), so no value crosses CTAs.  The
// scores are a matrix-vector product, d multiply-adds per token and stream, far too few
// for an MMA of their own (and TMEM is full): while the tensor cores run the K loop, the
// 16 epilogue warps read each stage's H rows from shared memory (the same tile the MMAs
// read, 128-byte swizzled), multiply them by the matching 64 entries of w^{Z_a} and w^{Z_b}
// in fp32 and, when the tile's K loop ends, hand the peer the scores of their half of the
// tokens through distributed shared memory.  The epilogue then forms each window's
// weights once from the scalar logits (shared by all channels) and pools.
//
// CSA: entry i of a tile pools its a-block from the C^a accumulator and the b-block
// i - 1 from the C^b one; the b-block of a tile's first entry is the last block of the tile
// before, whose C^b values the last epilogue group hands to the first one through shared
// memory (its scores stay in the previous tile's score buffer: there are three).
// Tiles advance by 64 blocks; pieces and the tile budget are those of fused_pair_kernel,
// over channel-group pairs.  HCA: a tile holds two 128-token windows; each window's
// weights are normalised once, so the two epilogue groups of a window add partial sums.
#pragma once

namespace scal {

constexpr int kEpiWarps = pair::kGroups * 4;        // 16
// warp 0 TMA, warp 1 MMA, warp 2 relay (leader: tells the peer's score readers that a
// stage landed; a release-ordered remote arrive in the MMA thread would hold its MMAs
// back, measured 0.33 -> 0.71 ms), warps 3..18 epilogue
constexpr int kThreads = 96 + kEpiWarps * 32;
// scores [tile % 3][stream][token].  Three buffers: pooling tile t reads those of t and
// t - 1, while the other CTA may already write those of t + 1 (its score readers can run
// through a short K loop on prefetched stages); those of t + 2 wait for the MMAs of t + 2,
// which wait for every epilogue group of both CTAs to finish pooling t + 1.
constexpr int kZBufs = 3;
constexpr int kZFloats = kZBufs * 2 * 256;
constexpr int kCarryFloats = 128 * 4;               // CSA: C^b of a tile's last block
constexpr int kWFloats = pair::kGroups * 128;       // weights, per epilogue group
constexpr int kHFloats = 2 * 128 * 2;               // HCA: second-half sums [window][row][acc]
constexpr int kRedFloats = pair::kGroups * 8;       // HCA: per-warp maxima / sums

struct Cfg {
  using P = pair::Cfg;
  static constexpr int XS = (kZFloats + kCarryFloats + kWFloats + kHFloats + kRedFloats) * 4;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(P::STAGES) * P::STAGE + XS + 512;
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

// HCA unit u = (sequence, 256-token tile, channel quad q), quad fastest; the leader takes
// channel groups 4q and 4q + 1, the peer 4q + 2 and 4q + 3 (cg = the CTA's first group).
__device__ __forceinline__ pair::Unit hca_unit(const Args& a, int64_t u, uint32_t rank) {
  pair::Unit h;
  const int nq = a.ncg;  // channel quads
  const int64_t tiles_per_seq = (a.ne + 1) / 2;
  const int q = static_cast<int>(u % nq);
  const int64_t r = u / nq;
  h.b = static_cast<int>(r / tiles_per_seq);
  h.j = r - static_cast<int64_t>(h.b) * tiles_per_seq;
  h.cg = 4 * q + 2 * static_cast<int>(rank);
  h.row0 = static_cast<int64_t>(h.b) * a.n + h.j * 256;
  const int64_t wins = a.ne - 2 * h.j < 2 ? a.ne - 2 * h.j : 2;
  h.rows = 128 * wins;
  h.stride = 256;
  h.ntiles = 1;
  h.e0 = h.e1 = h.first_block = 0;
  return h;
}

template <bool CSA>
__device__ __forceinline__ bool next_unit(const Args& a, pair::Sched* s, uint32_t rank,
                                          pair::Unit* q) {
  if constexpr (CSA) {
    return pair::sched_next<true>(a, s, rank, q);  // pieces over channel-group pairs
  } else {
    if (s->u >= s->units) return false;
    *q = hca_unit(a, s->u, rank);
    s->u += s->step;
    return true;
  }
}

// First channel group of this CTA's two accumulators, and the group of each accumulator.
template <bool CSA>
__device__ __forceinline__ int acc_group(const pair::Unit& q, uint32_t rank, int slot) {
  if constexpr (CSA) {
    return 2 * q.cg + static_cast<int>(rank);  // C^a and C^b of one group
  } else {
    return q.cg + slot;  // two groups of C
  }
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// acc (two fp32 lanes) += x * w over the 8 bf16 of two 16-byte vectors, pairwise (the
// products of bf16 values are exact in fp32).
__device__ __forceinline__ float2 dot8(const uint4& x, const uint4& w, float2 acc) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    acc = f2_fma(make_float2(__uint_as_float(xs[i] << 16), __uint_as_float(xs[i] & 0xffff0000u)),
                 make_float2(__uint_as_float(ws[i] << 16), __uint_as_float(ws[i] & 0xffff0000u)),
                 acc);
  return acc;
}

}  // namespace scal

// W maps: CSA W0 = W^{KV_a}, W1 = W^{KV_b} (each CTA loads its own channels of both); HCA
// W0 = W1 = W^{KV}.  a.wz0 / a.wz1: w^{Z_a} / w^{Z_b} (CSA) or w^{Z} (HCA), bf16 [d];
// a.B0 / a.B1: the position biases [m] fp32.
template <bool CSA, typename OutT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(scal::kThreads, 1)
    fused_scalar_kernel(const __grid_constant__ CUtensorMap tmH,
                        const __grid_constant__ CUtensorMap tmW0,
                        const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ Args a) {
  using C = pair::Cfg;
  constexpr int S = C::STAGES;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* zbuf = reinterpret_cast<float*>(smem + S * C::STAGE);  // [3][2][256]
  float* carry = zbuf + scal::kZFloats;                          // [128][4]
  float* wbuf = carry + scal::kCarryFloats;                      // [kGroups][128]
  float* hbuf = wbuf + scal::kWFloats;                           // [2][128][2]
  float* red = hbuf + scal::kHFloats;                            // [kGroups][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE + scal::Cfg::XS);
  uint64_t* full = bars;              // [S] leader: both CTAs' bytes of a stage
  uint64_t* empty = bars + S;         // [S] each CTA: MMAs and score readers are done
  uint64_t* pfull = bars + 2 * S;     // [S] peer: the leader saw the stage land
  uint64_t* tmem_full = bars + 3 * S;
  uint64_t* tmem_empty = tmem_full + 1;
  uint64_t* final_bar = tmem_full + 2;
  uint64_t* zfull = tmem_full + 3;    // [3] each CTA: both halves of a tile's scores
  uint64_t* carry_full = zfull + scal::kZBufs;   // CSA: group 3 wrote the carry
  uint64_t* carry_empty = carry_full + 1;        // CSA: group 0 read it
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(carry_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(carry_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = blockIdx.x & 1u;
  const uint32_t peer = rank ^ 1u;
  const int64_t cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const uint32_t peer_abort = cluster_addr(smem_u32(const_cast<int*>(abort_flag)), peer);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + scal::kEpiWarps);
      mbar_init(&pfull[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 2 * pair::kGroups);
    mbar_init(final_bar, 1);
    for (int zb = 0; zb < scal::kZBufs; ++zb) mbar_init(&zfull[zb], 2 * scal::kEpiWarps);
    mbar_init(carry_full, 1);
    mbar_init(carry_empty, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  cluster_sync_all();
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int pending_parity[S];
      for (int s = 0; s < S; ++s) pending_parity[s] = -1;
      bool ok = true;
      const uint64_t wpol = l2_evict_last_policy();  // W stays in L2 while H streams past
      pair::Sched sc = pair::sched_begin<CSA>(a, cid, ncl);
      pair::Unit q;
      while (ok && scal::next_unit<CSA>(a, &sc, rank, &q)) {
        const int g0 = scal::acc_group<CSA>(q, rank, 0), g1 = scal::acc_group<CSA>(q, rank, 1);
        for (int t = 0; t < q.ntiles && ok; ++t) {
          const int nt = pair::tile_tokens(q, t);
          const int y = static_cast<int>(q.row0 + static_cast<int64_t>(t) * q.stride +
                                         static_cast<int64_t>(rank) * (nt / 2));
          for (int kstep = 0; kstep < a.nk; ++kstep) {
            if (!pair::wait_pair(&empty[stage], phase ^ 1u, abort_flag, peer_abort)) {
              ok = false;
              break;
            }
            if (rank == 0) {
              mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE);
              pending_parity[stage] = static_cast<int>(phase);
            }
            const uint32_t lbar = cluster_addr(smem_u32(&full[stage]), 0);
            uint8_t* st = smem + stage * C::STAGE;
            const int x = kstep * C::BK;
            tma_load_2d_pair(smem_u32(st + C::A_BYTES), &tmH, lbar, x, y);
            tma_load_2d_pair_hint(smem_u32(st + 0 * C::A_BOX), &tmW0, lbar, g0 * kCh, x, wpol);
            tma_load_2d_pair_hint(smem_u32(st + 1 * C::A_BOX), &tmW0, lbar, g0 * kCh + 64, x, wpol);
            tma_load_2d_pair_hint(smem_u32(st + 2 * C::A_BOX), CSA ? &tmW1 : &tmW0, lbar, g1 * kCh,
                                  x, wpol);
            tma_load_2d_pair_hint(smem_u32(st + 3 * C::A_BOX), CSA ? &tmW1 : &tmW0, lbar,
                                  g1 * kCh + 64, x, wpol);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < S; ++s)
          if (pending_parity[s] >= 0)
            pair::wait_pair(&full[s], static_cast<uint32_t>(pending_parity[s]), abort_flag,
                            peer_abort, false);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0) {
      if (rank == 0) {
        int stage = 0;
        uint32_t phase = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        pair::Sched sc = pair::sched_begin<CSA>(a, cid, ncl);
        pair::Unit q;
        while (ok && scal::next_unit<CSA>(a, &sc, 0, &q)) {
          for (int t = 0; t < q.ntiles && ok; ++t) {
            const uint32_t idesc = pair::idesc_pair(pair::tile_tokens(q, t));
            if (!pair::wait_pair(tmem_empty, acc_phase ^ 1u, abort_flag, peer_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            for (int kstep = 0; kstep < a.nk; ++kstep) {
              if (!pair::wait_pair(&full[stage], phase, abort_flag, peer_abort)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t st = smem_u32(smem + stage * C::STAGE);
#pragma unroll
              for (int s = 0; s < 2; ++s) {
#pragma unroll
                for (int ks = 0; ks < C::BK / 16; ++ks) {
                  const uint64_t ad = smem_desc(st + (2 * s) * C::A_BOX + ks * 16 * 128,
                                                C::A_BOX, 1024, 2);
                  const uint64_t bd = smem_desc(st + C::A_BYTES + ks * 32, 16, 1024, 2);
                  umma_bf16_pair(tmem_base + s * 256, ad, bd, idesc,
                                       (kstep | ks) != 0 ? 1u : 0u);
                }
              }
              umma_commit_pair(cluster_addr(smem_u32(&empty[stage]), 0));
              umma_commit_pair(cluster_addr(smem_u32(&empty[stage]), 1));
              if (++stage == S) {
                stage = 0;
                phase ^= 1u;
              }
            }
            if (!ok) break;
            umma_commit_pair(cluster_addr(smem_u32(tmem_full), 0));
            umma_commit_pair(cluster_addr(smem_u32(tmem_full), 1));
            acc_phase ^= 1u;
          }
        }
        umma_commit_pair(cluster_addr(smem_u32(final_bar), 0));
        umma_commit_pair(cluster_addr(smem_u32(final_bar), 1));
      }
      pair::wait_pair(final_bar, 0, abort_flag, peer_abort, false);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ relay (leader)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      pair::Sched sc = pair::sched_begin<CSA>(a, cid, ncl);
      pair::Unit q;
      while (ok && scal::next_unit<CSA>(a, &sc, 0, &q)) {
        for (int t = 0; t < q.ntiles && ok; ++t) {
          for (int kstep = 0; kstep < a.nk; ++kstep) {
            if (!pair::wait_pair(&full[stage], phase, abort_flag, peer_abort)) {
              ok = false;
              break;
            }
            // the peer's score readers learn here that their half of the stage landed
            mbar_arrive_cluster(cluster_addr(smem_u32(&pfull[stage]), 1));
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 3..18)
    const int ew = warp - 3;              // epilogue warp 0..15
    const int eg = ew >> 2;               // group: tokens [64 eg, 64 eg + 64) of a tile
    const int qw = warp & 3;              // TMEM lane quarter this warp may access
    const int row = qw * 32 + lane;       // TMEM lane = channel within an accumulator
    const bool elected = (ew & 3) == 0 && lane == 0;
    const int gbar = 1 + eg;              // the group's named barrier (128 threads)
    const int gi = (ew & 3) * 32 + lane;  // thread within the group
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(qw * 32) << 16);
    const uint32_t leader_tmem_empty = cluster_addr(smem_u32(tmem_empty), 0);
    // score readers: row lr of this CTA's half of a stage's H tile, k quarter lq
    const int lt = ew * 32 + lane, lr = lt >> 2, lq = lt & 3;
    const __nv_bfloat16* wz0 = static_cast<const __nv_bfloat16*>(a.wz0);
    const __nv_bfloat16* wz1 = static_cast<const __nv_bfloat16*>(a.wz1);
    OutT* out = static_cast<OutT*>(a.out);
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0, tcount = 0, ccount = 0;
    bool ok = true;
    pair::Sched sc = pair::sched_begin<CSA>(a, cid, ncl);
    pair::Unit q;
    while (ok && scal::next_unit<CSA>(a, &sc, rank, &q)) {
      for (int t = 0; t < q.ntiles && ok; ++t, ++tcount) {
        const int nt = pair::tile_tokens(q, t);
        const uint32_t par = tcount % scal::kZBufs;  // this tile's score buffer
        // ---- the tile's scores for this CTA's H rows, stage by stage, beside the MMAs; the
        // w slices of the next stage are loaded while this one is summed
        float2 z0 = make_float2(0.f, 0.f), z1 = make_float2(0.f, 0.f);
        uint4 wn[4] = {};
        {
          const uint4* p0 = reinterpret_cast<const uint4*>(wz0 + 16 * lq);
          const uint4* p1 = reinterpret_cast<const uint4*>(wz1 + 16 * lq);
          wn[0] = __ldg(p0);
          wn[1] = __ldg(p0 + 1);
          if constexpr (CSA) {
            wn[2] = __ldg(p1);
            wn[3] = __ldg(p1 + 1);
          }
        }
        for (int kstep = 0; kstep < a.nk; ++kstep) {
          const bool got = rank == 0
                               ? pair::wait_pair(&full[stage], phase, abort_flag, peer_abort)
                               : pair::wait_pair(&pfull[stage], phase, abort_flag, peer_abort);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          // 128-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ (r % 8)
          const uint8_t* hb = smem + stage * C::STAGE + C::A_BYTES + lr * 128;
          const int sw = lr & 7;
          const uint4 h0 = *reinterpret_cast<const uint4*>(hb + (((2 * lq) ^ sw) << 4));
          const uint4 h1 = *reinterpret_cast<const uint4*>(hb + (((2 * lq + 1) ^ sw) << 4));
          uint4 wc[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) wc[i] = wn[i];
          if (kstep + 1 < a.nk) {
            const int k1 = (kstep + 1) * C::BK + 16 * lq;
            const uint4* p0 = reinterpret_cast<const uint4*>(wz0 + k1);
            wn[0] = __ldg(p0);
            wn[1] = __ldg(p0 + 1);
            if constexpr (CSA) {
              const uint4* p1 = reinterpret_cast<const uint4*>(wz1 + k1);
              wn[2] = __ldg(p1);
              wn[3] = __ldg(p1 + 1);
            }
          }
          // the stage's bytes are in registers: release it (MMA commit + 16 reader warps)
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          z0 = scal::dot8(h0, wc[0], z0);
          z0 = scal::dot8(h1, wc[1], z0);
          if constexpr (CSA) {
            z1 = scal::dot8(h0, wc[2], z1);
            z1 = scal::dot8(h1, wc[3], z1);
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        float s0 = z0.x + z0.y, s1 = z1.x + z1.y;
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
        if (lq == 0 && lr < nt / 2) {  // this CTA's tokens are [rank nt/2, (rank + 1) nt/2)
          const int pos = static_cast<int>(rank) * (nt / 2) + lr;
          float* zl = zbuf + par * 512;
          zl[pos] = s0;
          zl[256 + pos] = s1;
          scal::st_cluster_f32(cluster_addr(smem_u32(zl + pos), peer), s0);
          scal::st_cluster_f32(cluster_addr(smem_u32(zl + 256 + pos), peer), s1);
        }
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&zfull[par]);
          mbar_arrive_cluster(cluster_addr(smem_u32(&zfull[par]), peer));
        }
        const bool got = pair::wait_pair(tmem_full, acc_phase, abort_flag, peer_abort) &&
                         pair::wait_pair(&zfull[par], (tcount / scal::kZBufs) & 1u, abort_flag,
                                         peer_abort);
        if constexpr (CSA) {
          // ---- pool: entry lb of the tile takes a-block lb (C^a) and b-block lb - 1 (C^b)
          if (!bar_and(gbar, 128, got)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float* za = zbuf + par * 512;
          const float* zb = za + 256;
          // the tile before's (when t > 0)
          const float* zbp = zbuf + ((par + scal::kZBufs - 1) % scal::kZBufs) * 512 + 256;
          const int64_t ch = static_cast<int64_t>(scal::acc_group<true>(q, rank, 0)) * kCh + row;
          const bool live = ch < a.c;
          const int nch = nt / 16;
          const int c_lo = 4 * eg, c_hi = 4 * eg + 4 < nch ? 4 * eg + 4 : nch;
          const int64_t kb_tile = q.first_block + static_cast<int64_t>(t) * 64;
          {
            // the window weights of the group's 16 entries: thread gi takes row j = gi % 8
            // (a-rows 0..3, b-rows 4..7) of entry gi / 8; the 8 rows are 8 adjacent lanes
            const int j = gi & 7, lb = 16 * eg + (gi >> 3);
            float l = -INFINITY;
            if (lb < 4 * nch) {
              if (j < 4) {
                l = fmaf(za[4 * lb + j], kLog2e, __ldg(a.B0 + j) * kLog2e);
              } else if (lb > 0) {
                l = fmaf(zb[4 * (lb - 1) + j - 4], kLog2e, __ldg(a.B1 + j - 4) * kLog2e);
              } else if (t > 0) {  // b-block = the previous tile's last block
                l = fmaf(zbp[252 + j - 4], kLog2e, __ldg(a.B1 + j - 4) * kLog2e);
              }  // else: the sequence's entry 0 (no b-rows) or the piece's halo block
            }
            float mx = l;
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            const float w = mx == -INFINITY ? 0.f : ex2_ftz(l - mx);
            float sum = w;
            sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            sum += __shfl_xor_sync(0xffffffffu, sum, 4);
            wbuf[eg * 128 + gi] = sum > 0.f ? __fdividef(w, sum) : 0.f;
          }
          bar_named(gbar, 128);  // the group's weights are in place
          float pb[4] = {0.f, 0.f, 0.f, 0.f};  // C^b of the block before the next entry
          if (eg > 0 && c_lo < nch) {
            float cb[16];
            tmem_ld16(lane_addr + 256 + (c_lo - 1) * 16, cb);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 4; ++k) pb[k] = cb[12 + k];
          } else if (eg == 0 && t > 0) {
            if (!bar_and(gbar, 128, pair::wait_pair(carry_full, ccount & 1u, abort_flag,
                                                    peer_abort))) {
              ok = false;
              break;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) pb[k] = carry[row * 4 + k];
            bar_named(gbar, 128);  // every thread of the group has read the carry
            if (elected) mbar_arrive(carry_empty);
            ++ccount;
          }
#pragma unroll 1
          for (int c = c_lo; c < c_hi; ++c) {
            float ca[16], cb[16];
            tmem_ld16(lane_addr + c * 16, ca);
            tmem_ld16(lane_addr + 256 + c * 16, cb);
            tmem_wait_ld();
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
              const int lb = 4 * c + blk;
              const int64_t kb = kb_tile + lb;
              if (live && kb >= q.e0 && kb < q.e1) {
                const float* w8 = wbuf + eg * 128 + (lb - 16 * eg) * 8;
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) acc = fmaf(w8[k], ca[4 * blk + k], acc);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  acc = fmaf(w8[4 + k], blk == 0 ? pb[k] : cb[4 * (blk - 1) + k], acc);
                store_scalar<OutT>(out + (static_cast<int64_t>(q.b) * a.ne + kb) * a.c + ch, acc);
              }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) pb[k] = cb[12 + k];
          }
          // the last group hands C^b of the tile's last block to group 0's next tile
          if (ok && eg == pair::kGroups - 1 && t + 1 < q.ntiles) {
            if (!bar_and(gbar, 128, pair::wait_pair(carry_empty, (ccount & 1u) ^ 1u, abort_flag,
                                                    peer_abort))) {
              ok = false;
              break;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) carry[row * 4 + k] = pb[k];
            bar_named(gbar, 128);  // every thread of the group has written
            if (elected) mbar_arrive(carry_full);
            ++ccount;
          }
        } else {
          // ---- pool: window w of the tile, rows [64 half, 64 half + 64) of it
          const int wins = static_cast<int>(q.rows / 128);
          const int w = eg >> 1, half = eg & 1;
          const bool active = w < wins;
          const int wbar = 5 + w;  // the window's two groups (256 threads)
          if (!(active ? bar_and(wbar, 256, got) : bar_and(gbar, 128, got))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (active) {
            // the window's weights, once: thread gi takes token gi of the window
            const float* z = zbuf + par * 512;
            const float l = fmaf(z[w * 128 + gi], kLog2e, __ldg(a.B0 + gi) * kLog2e);
            float mx = l;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float* rg = red + eg * 8;
            if (lane == 0) rg[ew & 3] = mx;
            bar_named(gbar, 128);
            mx = fmaxf(fmaxf(rg[0], rg[1]), fmaxf(rg[2], rg[3]));
            const float e = ex2_ftz(l - mx);
            float sum = e;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (lane == 0) rg[4 + (ew & 3)] = sum;
            bar_named(gbar, 128);
            sum = (rg[4] + rg[5]) + (rg[6] + rg[7]);
            wbuf[eg * 128 + gi] = __fdividef(e, sum);
            bar_named(gbar, 128);  // the weights are in place
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              const int cc = 4 * half + c;  // chunk within the window
              float c0[16], c1[16];
              const uint32_t col = static_cast<uint32_t>(w * 128 + cc * 16);
              tmem_ld16(lane_addr + col, c0);
              tmem_ld16(lane_addr + 256 + col, c1);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                const float wk = wbuf[eg * 128 + cc * 16 + k];
                acc0 = fmaf(wk, c0[k], acc0);
                acc1 = fmaf(wk, c1[k], acc1);
              }
            }
            float* hs = hbuf + (w * 128 + row) * 2;
            if (half == 1) {
              hs[0] = acc0;
              hs[1] = acc1;
            }
            bar_named(wbar, 256);
            if (half == 0) {
              acc0 += hs[0];
              acc1 += hs[1];
              const int64_t ch0 = static_cast<int64_t>(q.cg) * kCh + row, ch1 = ch0 + kCh;
              OutT* o = out + (static_cast<int64_t>(q.b) * a.ne + q.j * 2 + w) * a.c;
              if (ch0 < a.c) store_scalar<OutT>(o + ch0, acc0);
              if (ch1 < a.c) store_scalar<OutT>(o + ch1, acc1);
            }
          }
        }
        if (!ok) break;
        tc_fence_before();
        bar_named(gbar, 128);  // the group's TMEM reads of this tile are done
        if (elected) {
          if (rank == 0) {
            mbar_arrive(tmem_empty);
          } else {
            mbar_arrive_cluster(leader_tmem_empty);
          }
        }
        acc_phase ^= 1u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote access of either CTA is still in flight
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(512));
  }
  cluster_sync_all();
}
