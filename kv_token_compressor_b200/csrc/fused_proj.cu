// Fused projection + softmax-pool on the 5th-generation tensor cores (sm_100a).
//
// What it computes ("序列压缩注意力", eq. attn-seqcomp-csa-proj followed by
// eqs. attn-seqcomp-csa-softmax / -csa-pool / -overlap-bound, or eq. attn-seqcomp-hca):
// the streams C = H W^{KV}, Z = H W^{Z} (four for CSA, two for HCA) are accumulated in
// fp32 in tensor memory and pooled straight out of it; they never reach device memory.
//
// Layout ("swap AB").  The GEMM is D[ch, tok] = sum_k W[k, ch] H[tok, k]: the 128
// channels of a tile sit on the MMA M dimension (TMEM lanes) and the tokens on N (TMEM
// columns).  A = W tile is MN-major (W is d x c, channel-contiguous), B = H tile is
// K-major.  After tcgen05.ld.32x32b every epilogue thread owns one channel and holds
// that channel's stream values for consecutive tokens in its own registers, so the
// softmax over a window is thread-local (no shuffles).
//
// Two kernels.  fused_pair_kernel (further down) runs on clusters of two CTAs sharing
// M = 256 MMAs and is the one launched; fused_pool_kernel below, one CTA per SM, is
// taken when no CTA pair can be resident, and for HCA when the channel groups of 128 are
// odd in number (they cannot pair up).
//
// fused_pool_kernel, per CTA (persistent, one per SM, 192 threads):
//   warp 0        TMA producer: H tile [TN tokens x 64] + the W tiles [64 x 128] of
//                 every stream per pipeline stage (128-byte swizzle, mbarrier tx count)
//   warp 1        TMEM allocator and MMA issuer (one thread): NS x 4 tcgen05.mma
//                 (M=128, N=TN, K=16) per stage, tcgen05.commit frees the stage
//   warps 2..5    epilogue: tcgen05.ld the accumulators, bias + softmax + weighted sum
//                 in fp32 registers, store the entries
// TMEM holds NS accumulators of 128 lanes x TN columns (NS * TN = 512 columns).
// CSA (NS = 4, TN = 128): a CTA walks a contiguous range of entries of one sequence and
// channel group; its first tile starts one block early (the b-rows of its first entry)
// and the b-part of each block is carried in registers to the next entry.
// HCA (NS = 2, TN = 256): each tile holds two 128-token windows.
//
// Every mbarrier wait is bounded in time; a wait that gives up sets the library's device
// error word and an abort flag, the CTA drains its own TMA copies and MMAs (again with a
// bound), frees its TMEM and returns.
#include <cuda.h>

#include "kvc_common.cuh"
#include "kvc_host.h"
#include "kvc_launch.h"
#include "tc_ptx.cuh"

#include <mutex>
#include <type_traits>

namespace kvc {

// Set by kernels whose bounded waits give up; read and cleared by kvc_device_status().
__device__ unsigned int g_device_error = 0;

namespace fused {

constexpr int kCh = 128;         // channels per tile (MMA M, TMEM lanes)
constexpr int kThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

// NS streams; BK = K per pipeline stage: 64 (H rows of 128 bytes, 128-byte swizzle) or
// 32 (H rows of 64 bytes, 64-byte swizzle; half the stage size, twice the stages).
template <int NS, int BK_>
struct Cfg {
  static constexpr int BK = BK_;
  static constexpr int TN = 512 / NS;               // tokens per tile (MMA N)
  static constexpr int A_BOX = BK * 64 * 2;         // one [BK k x 64 ch] bf16 W box
  static constexpr int A_BYTES = NS * 2 * A_BOX;    // NS streams x 2 boxes (128 channels)
  static constexpr int B_BYTES = TN * BK * 2;       // H tile [TN tokens x BK k]
  static constexpr uint32_t B_SBO = BK * 2 * 8;     // 8 H rows
  static constexpr uint64_t B_LAYOUT = BK == 64 ? 2 : 4;  // SWIZZLE_128B / SWIZZLE_64B
  static_assert(BK == 64 || BK == 32, "stage K");
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE + 256;
  static_assert(STAGES >= 2, "pipeline needs two stages");
  static_assert(A_BYTES % 1024 == 0 && STAGE % 1024 == 0, "1024-byte swizzle atoms");
};

// ------------------------------------------------------------------ PTX wrappers
// (the generic ones are in tc_ptx.cuh)
using namespace tcx;

// Bounded wait for the phase of `parity` to complete.  Gives up (returns false) when the
// CTA's abort flag is raised or after kWaitLimitNs, in which case it raises the flag and
// records the timeout in the device error word.
__device__ __noinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(&g_device_error, 1u);
      return false;
    }
  }
}

// Instruction descriptor of kind::f16: D fp32, A and B bf16, A MN-major, B K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kCh >> 4) << 24);
}

// ------------------------------------------------------------------ CTA-pair wrappers
// (a cluster of two CTAs on two SMs sharing one M = 256 MMA: tcgen05 cta_group::2)

// The same shared-memory variable in CTA `rank` of the cluster (shared::cluster address).
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// Arrive on an mbarrier of either CTA; release orders this thread's earlier writes
// (including remote shared-memory stores) before the arrival, at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
// try_wait on a local barrier whose arrivals may come from the other CTA (acquire at
// cluster scope, so the other CTA's released writes are visible afterwards).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Generic-proxy shared-memory writes of this thread become visible to async copies.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Arm a barrier of either CTA with an arrival plus `bytes` of expected transfer.
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cluster_bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
                   cluster_bar),
               "r"(bytes)
               : "memory");
}
// Bulk copy of `bytes` from this CTA's shared memory into the other CTA's, counted on a
// barrier there (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t dst_cluster, uint32_t src_cta,
                                                     uint32_t bytes, uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src_cta), "r"(bytes), "r"(cluster_bar)
      : "memory");
}
// All threads of both CTAs.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Tile load into this CTA's shared memory whose completion is counted on the pair
// leader's barrier (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t leader_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y)
      : "memory");
}
// The same with an L2 policy (l2_evict_last_policy for the weights).
__device__ __forceinline__ void tma_load_2d_pair_hint(uint32_t dst, const CUtensorMap* map,
                                                      uint32_t leader_bar, int x, int y, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y), "l"(pol)
      : "memory");
}
// M = 256 MMA over the pair: A rows 0..127 from the leader's shared memory, 128..255 from
// the peer's (same offsets); B columns split in halves the same way; each CTA's TMEM
// receives its own 128 rows.  Issued by one leader thread.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Arrive on a barrier (of either CTA, cluster address) once this thread's pair MMAs finish.
__device__ __forceinline__ void umma_commit_pair(uint32_t cluster_bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   cluster_bar)
               : "memory");
}

// ------------------------------------------------------------------ work schedules

constexpr int kMaxClusters = 96;  // CSA CTA-pair schedule table (B200: 74 pairs)

struct Args {
  const float* B0;  // CSA: B^a [m, c]; HCA: B [m, c]
  const float* B1;  // CSA: B^b [m, c]
  void* out;
  int64_t batch, n, c, ne;
  int ncg;          // channel groups of 128
  int nk;           // K steps of 64
  int pieces_per_unit;  // single-CTA CSA: entry ranges per (sequence, channel group)
  int64_t units;        // single-CTA CSA: pieces; HCA: tiles; CTA-pair CSA: busy clusters
  // CTA-pair CSA: tiles per cluster, token ranges per sequence, and each cluster's first
  // piece (flat piece index)
  int64_t tile_budget;
  int64_t ranges;
  int32_t start_k[kMaxClusters + 1];  // start_k[units] = the number of pieces
  // scalar-logit form: the score vectors w^{Z_a}, w^{Z_b} (CSA) or w^{Z} (HCA), bf16 [d]
  const void* wz0;
  const void* wz1;
};

// Extra kernel argument of the cache-layout instantiations (empty otherwise).
template <bool CACHE>
using FusedCacheArg = typename std::conditional<CACHE, CacheFmt, NoCache>::type;

// Stores the result v of channel ch of entry `entry` of sequence b: as OutT into the plain
// output, or in the cache layout (E4M3 below c - r, RoPE'd bf16 above).  Every lane of the
// warp calls it together (the lanes hold consecutive channels; the RoPE pairs are
// exchanged by a shuffle).
template <bool CACHE, typename OutT>
__device__ __forceinline__ void store_entry(const Args& a, const FusedCacheArg<CACHE>& cf, int b,
                                            int64_t entry, int64_t ch, float v) {
  const int64_t orow = static_cast<int64_t>(b) * a.ne + entry;
  if constexpr (CACHE) {
    store_cache_lane(cf, orow, ch, entry, v, true);
  } else {
    store_scalar<OutT>(static_cast<OutT*>(a.out) + orow * a.c + ch, v);
  }
}

// CSA m = 4: piece p = (sequence b, channel group cg, entries [e0, e1)).  Its token rows
// start one block before e0 (the b-rows of entry e0) unless e0 = 0.
struct CsaPiece {
  int b, cg;
  int64_t e0, e1, first_block, row0;  // row0: first H row (global)
  int ntiles;
};
template <int TN>
__device__ __forceinline__ CsaPiece csa_piece(const Args& a, int64_t p) {
  CsaPiece q;
  const int64_t P = a.pieces_per_unit;
  const int64_t u = p / P, r = p - u * P;
  q.b = static_cast<int>(u / a.ncg);
  q.cg = static_cast<int>(u - static_cast<int64_t>(q.b) * a.ncg);
  q.e0 = (r * a.ne) / P;
  q.e1 = ((r + 1) * a.ne) / P;
  q.first_block = q.e0 > 0 ? q.e0 - 1 : 0;
  const int64_t rows = 4 * q.e1 - 4 * q.first_block;
  q.ntiles = q.e1 > q.e0 ? static_cast<int>((rows + TN - 1) / TN) : 0;
  q.row0 = static_cast<int64_t>(q.b) * a.n + 4 * q.first_block;
  return q;
}

// HCA m' = 128: tile t = (sequence b, token tile j, channel group cg), cg fastest so the
// CTAs sharing an H tile run side by side.
struct HcaTile {
  int b, cg;
  int64_t j, row0;
};
template <int TN>
__device__ __forceinline__ HcaTile hca_tile(const Args& a, int64_t t) {
  HcaTile h;
  const int64_t tiles_per_seq = (a.ne * 128 + TN - 1) / TN;
  h.cg = static_cast<int>(t % a.ncg);
  const int64_t r = t / a.ncg;
  h.b = static_cast<int>(r / tiles_per_seq);
  h.j = r - static_cast<int64_t>(h.b) * tiles_per_seq;
  h.row0 = static_cast<int64_t>(h.b) * a.n + h.j * TN;
  return h;
}

// ------------------------------------------------------------------ the kernel

template <bool CSA, int BK, typename OutT, bool CACHE>
__global__ void __launch_bounds__(kThreads, 1)
    fused_pool_kernel(const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmW0,
                      const __grid_constant__ CUtensorMap tmW1,
                      const __grid_constant__ CUtensorMap tmW2,
                      const __grid_constant__ CUtensorMap tmW3, const __grid_constant__ Args a,
                      const FusedCacheArg<CACHE> cf) {
  constexpr int NS = CSA ? 4 : 2;
  using C = Cfg<NS, BK>;
  constexpr int TN = C::TN;
  constexpr uint32_t IDESC = idesc_bf16(TN);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = bars + C::STAGES;          // [STAGES]
  uint64_t* tmem_full = bars + 2 * C::STAGES;  // [1]
  uint64_t* tmem_empty = tmem_full + 1;        // [1]
  uint64_t* final_bar = tmem_full + 2;         // [1]
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(tmem_full + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_full + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 4 * 32);
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {  // the whole warp allocates all 512 TMEM columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t units = a.units;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int pending_parity[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) pending_parity[s] = -1;
      bool ok = true;
      const uint64_t wpol = l2_evict_last_policy();  // W stays in L2 while H streams past
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int ntiles, cg;
        int64_t row0;
        if constexpr (CSA) {
          const CsaPiece q = csa_piece<TN>(a, u);
          ntiles = q.ntiles;
          cg = q.cg;
          row0 = q.row0;
        } else {
          const HcaTile h = hca_tile<TN>(a, u);
          ntiles = 1;
          cg = h.cg;
          row0 = h.row0;
        }
        for (int t = 0; t < ntiles && ok; ++t) {
          const int y = static_cast<int>(row0 + static_cast<int64_t>(t) * TN);
          for (int kstep = 0; kstep < a.nk; ++kstep) {
            if (!wait_phase(&empty[stage], phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* st = smem + stage * C::STAGE;
            mbar_arrive_expect_tx(&full[stage], C::STAGE);
            pending_parity[stage] = static_cast<int>(phase);
            const int x = kstep * BK;
            tma_load_2d(smem_u32(st + C::A_BYTES), &tmH, &full[stage], x, y);
            const CUtensorMap* maps[4] = {&tmW0, &tmW1, &tmW2, &tmW3};
#pragma unroll
            for (int s = 0; s < NS; ++s) {
              tma_load_2d_hint(smem_u32(st + (2 * s) * C::A_BOX), maps[s], &full[stage], cg * kCh,
                               x, wpol);
              tma_load_2d_hint(smem_u32(st + (2 * s + 1) * C::A_BOX), maps[s], &full[stage],
                               cg * kCh + 64, x, wpol);
            }
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (!ok) {  // drain the copies this thread issued before giving up
        for (int s = 0; s < C::STAGES; ++s)
          if (pending_parity[s] >= 0)
            wait_phase(&full[s], static_cast<uint32_t>(pending_parity[s]), abort_flag, false);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int ntiles;
        if constexpr (CSA) {
          ntiles = csa_piece<TN>(a, u).ntiles;
        } else {
          ntiles = 1;
        }
        for (int t = 0; t < ntiles && ok; ++t) {
          if (!wait_phase(tmem_empty, acc_phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kstep = 0; kstep < a.nk; ++kstep) {
            if (!wait_phase(&full[stage], phase, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = smem_u32(smem + stage * C::STAGE);
#pragma unroll
            for (int s = 0; s < NS; ++s) {
#pragma unroll
              for (int ks = 0; ks < BK / 16; ++ks) {
                // A: W tile of stream s, MN-major, 128-byte swizzle: 64-channel blocks
                // A_BOX apart (LBO), 8-row k groups 1024 B apart (SBO); k-slice ks starts
                // 16 rows in.
                const uint64_t ad =
                    smem_desc(st + (2 * s) * C::A_BOX + ks * 16 * 128, C::A_BOX, 1024, 2);
                // B: H tile, K-major: token rows of 2*BK bytes, 8-row groups B_SBO apart;
                // k-slice ks starts 32 bytes into the swizzled row.
                const uint64_t bd =
                    smem_desc(st + C::A_BYTES + ks * 32, 16, C::B_SBO, C::B_LAYOUT);
                umma_bf16(tmem_base + s * TN, ad, bd, IDESC, (kstep | ks) != 0 ? 1u : 0u);
              }
            }
            umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit(tmem_full);  // accumulators of this tile are complete
          acc_phase ^= 1u;
        }
      }
      // Every MMA this thread issued has finished before TMEM is released.
      umma_commit(final_bar);
      wait_phase(final_bar, 0, abort_flag, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;  // TMEM lane = channel within the tile
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
      if constexpr (CSA) {
        const CsaPiece pc = csa_piece<TN>(a, u);
        const int64_t ch = static_cast<int64_t>(pc.cg) * kCh + row;
        float ba2[4], bb2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          ba2[k] = __ldg(a.B0 + k * a.c + ch) * kLog2e;
          bb2[k] = __ldg(a.B1 + k * a.c + ch) * kLog2e;
        }
        float carry_l[4], carry_c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          carry_l[k] = -INFINITY;
          carry_c[k] = 0.f;
        }
        for (int t = 0; t < pc.ntiles; ++t) {
          // warp-uniform outcome: tcgen05.ld below needs the whole warp
          if (!__all_sync(0xffffffffu, wait_phase(tmem_full, acc_phase, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int64_t kb_tile = pc.first_block + static_cast<int64_t>(t) * (TN / 4);
#pragma unroll 1
          for (int chunk = 0; chunk < TN / 16; ++chunk) {
            float ca[16], cb[16], za[16], zb[16];
            const uint32_t col = static_cast<uint32_t>(chunk * 16);
            tmem_ld16(lane_addr + 0 * TN + col, ca);
            tmem_ld16(lane_addr + 1 * TN + col, cb);
            tmem_ld16(lane_addr + 2 * TN + col, za);
            tmem_ld16(lane_addr + 3 * TN + col, zb);
            tmem_wait_ld();
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
              const int64_t kb = kb_tile + chunk * 4 + blk;
              float la[4];
              float mx = -INFINITY;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                la[k] = fmaf(za[4 * blk + k], kLog2e, ba2[k]);
                mx = fmaxf(mx, la[k]);
              }
              if (kb >= pc.e0 && kb < pc.e1) {
                // entry kb: a-rows of block kb, b-rows of block kb-1 (the carry); entry
                // 0 has no b-rows (carry holds logit -inf, vector 0).
#pragma unroll
                for (int k = 0; k < 4; ++k) mx = fmaxf(mx, carry_l[k]);
                float s = 0.f, acc = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float w = exp2f(la[k] - mx);
                  s += w;
                  acc = fmaf(w, ca[4 * blk + k], acc);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float w = exp2f(carry_l[k] - mx);
                  s += w;
                  acc = fmaf(w, carry_c[k], acc);
                }
                store_entry<CACHE, OutT>(a, cf, pc.b, kb, ch, __fdividef(acc, s));
              }
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                carry_l[k] = fmaf(zb[4 * blk + k], kLog2e, bb2[k]);
                carry_c[k] = cb[4 * blk + k];
              }
            }
          }
          tc_fence_before();
          mbar_arrive(tmem_empty);
          acc_phase ^= 1u;
        }
      } else {
        const HcaTile h = hca_tile<TN>(a, u);
        const int64_t ch = static_cast<int64_t>(h.cg) * kCh + row;
        if (!__all_sync(0xffffffffu, wait_phase(tmem_full, acc_phase, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int w = 0; w < TN / 128; ++w) {
          const int64_t e = h.j * (TN / 128) + w;
          if (e >= a.ne) break;
          float M = -INFINITY, S = 0.f, A = 0.f;
#pragma unroll 1
          for (int chunk = 0; chunk < 128 / 16; ++chunk) {
            float cv[16], zv[16];
            const uint32_t col = static_cast<uint32_t>(w * 128 + chunk * 16);
            tmem_ld16(lane_addr + col, cv);
            tmem_ld16(lane_addr + TN + col, zv);
            tmem_wait_ld();
            float cm = -INFINITY;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float b2 = __ldg(a.B0 + (chunk * 16 + k) * a.c + ch) * kLog2e;
              zv[k] = fmaf(zv[k], kLog2e, b2);
              cm = fmaxf(cm, zv[k]);
            }
            const float nm = fmaxf(M, cm);
            const float sc = exp2f(M - nm);
            S *= sc;
            A *= sc;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float wgt = exp2f(zv[k] - nm);
              S += wgt;
              A = fmaf(wgt, cv[k], A);
            }
            M = nm;
          }
          store_entry<CACHE, OutT>(a, cf, h.b, e, ch, __fdividef(A, S));
        }
        tc_fence_before();
        mbar_arrive(tmem_empty);
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(512));
  }
}

// ==================================================================================
// CTA-pair kernel (cluster of 2, tcgen05 cta_group::2, M = 256, N <= 256 tokens)
//
// Why: in the single-CTA CSA kernel every token tile of N = 128 re-reads the H tile for
// four MMAs and re-streams the W tiles of four streams, which asks ~206 B/clk of shared
// memory per SM against 128 available.  A pair of CTAs shares each M = 256 MMA: every SM
// reads only its own half of A and of B per MMA and loads W for two streams per 256
// tokens, ~111 B/clk at full tensor rate.
//
// Split of the M = 256 rows over the pair:
//   CSA  the streams: the leader (rank 0) accumulates C^a, Z^a of 128 channels, the peer
//        (rank 1) C^b, Z^b of the same channels, both for the same N tokens.  Entry i needs
//        the a-block i (leader) and the b-block i-1 (peer): the peer reduces each block to
//        a softmax partial per channel, (L, mean) = (max + log2 sum of exp2, weighted
//        mean), and copies them into the leader's shared memory; the leader merges each
//        with its a-block and stores the entry.
//   HCA  the channels: the leader owns channel group 2g, the peer 2g + 1, each with both
//        streams C and Z; windows stay inside each CTA, nothing is exchanged.
// TMEM of each CTA: stream 0 (C) in columns [0, 256), stream 1 (Z) in [256, 512).
//
// Per CTA: warp 0 TMA (its own halves: H rows [y, y + N/2) or [y + N/2, y + N), W tiles of
// its two streams), warp 1 TMEM allocation (both CTAs) and MMA issue (leader only),
// warps 2..17 epilogue.  Stage completion is counted on the leader's barrier; the leader's
// commits arrive on both CTAs' barriers.  Every wait is bounded as in the kernel above,
// and a CTA that gives up also raises the other CTA's abort flag.
//
// Epilogue.  TMEM is full during it (the MMAs of the next tile wait), so its latency is
// what costs: 16 warps in 4 groups, group g taking tokens [64 g, 64 g + 64) of the tile
// (4 warps = the 4 TMEM lane quarters).  CSA tiles advance by 64 blocks (256 rows); the
// b-partial of a tile's first entry is the last block of the tile before, which the
// peer's group 3 hands to its group 0 through shared memory (one 1 KB slot guarded by two
// barriers), so no block is projected twice.  Each CSA group has its own 2-slot ring; a
// slot holds, per channel, the partials of the 4 blocks preceding the chunk's 4 entries
// (the first one the peer group carries from its previous chunk, loads once per tile, or
// takes from the carry), so within a tile the groups never wait on one another.  An HCA
// window is split over two groups whose (max, sum, acc) states merge through shared
// memory.
// ==================================================================================
namespace pair {

constexpr int kGroups = 4;             // epilogue groups of 4 warps
constexpr int kThreads = 64 + kGroups * 128;
constexpr int kSlotsPerGroup = 2;      // CSA exchange ring per group
constexpr int kXFloats = 8;            // per channel and chunk: 4 partials x (L, mean)
constexpr uint32_t kSlotBytes = 128 * kXFloats * 4;  // one exchange slot, 4 KB

struct Cfg {
  static constexpr int BK = 64;
  static constexpr int A_BOX = BK * 64 * 2;          // [64 k x 64 ch] bf16, 8 KB
  static constexpr int A_BYTES = 2 * 2 * A_BOX;      // 2 streams x 128 channels
  static constexpr int B_BYTES = 128 * BK * 2;       // this CTA's 128 H rows
  static constexpr int STAGE = A_BYTES + B_BYTES;    // 48 KB
  static constexpr int STAGES = 4;
  // CSA exchange slots; HCA uses the same space for its half-window states
  static constexpr int XBUF = kGroups * kSlotsPerGroup * static_cast<int>(kSlotBytes);  // 32 KB
  // CSA: the b-partial (L, mean) per channel carried from the last block of a tile to the
  // first entry of the next (peer CTA, epilogue group 3 to group 0)
  static constexpr int CARRY = 128 * 2 * 4;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE + XBUF + CARRY + 512;
  static_assert(STAGE % 1024 == 0 && A_BYTES % 1024 == 0, "1024-byte swizzle atoms");
  static_assert(SMEM <= 232448, "shared memory per CTA");
  static_assert(2 * 2 * 128 * 3 * 4 <= XBUF, "HCA half-window states fit the exchange space");
};

// Bounded wait, as wait_phase, for barriers that the other CTA of the pair may arrive on
// (acquire at cluster scope).  On giving up it raises both CTAs' abort flags.
__device__ __noinline__ bool wait_pair(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                       uint32_t peer_abort, bool honour_abort = true) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      st_cluster_u32(peer_abort, 1u);
      atomicOr(&g_device_error, 1u);
      return false;
    }
  }
}

// One unit of work of a cluster: `ntiles` token tiles, tile t starting at H row
// row0 + t * stride and holding tile_tokens(t) <= 256 tokens; the channel group of this CTA.
struct Unit {
  int b, cg;              // sequence; channel group of this CTA (128 channels)
  int64_t row0;           // first H row of tile 0
  int64_t e0, e1, first_block;  // CSA: entries [e0, e1); blocks from first_block
  int64_t j;              // HCA: token tile index within the sequence
  int64_t rows;           // rows covered by the unit
  int64_t stride;         // rows between tile starts
  int ntiles;
};

// CSA schedule.  With a budget of T tiles per cluster (a tile holds 64 blocks of 4 rows,
// 256 tokens), each sequence is cut into token ranges of T tiles: the first range holds
// entries [0, 64 T), every later one 64 T - 1 entries and starts one block early, at the
// b-block of its first entry (the halo, no entry itself).  A piece is one token range of
// one channel group; pieces are taken in the order (sequence, range, channel group) and
// dealt to the clusters in turn, each cluster taking consecutive pieces while they fit its
// budget (the last range of a sequence is short, and several of its pieces share a
// cluster).  So the clusters that hold the same token range for different channel groups
// are neighbours that run at the same time, and the H rows they all read come from DRAM
// about once.  Within a piece the b-partial of a tile's first entry is carried over from
// the tile before, so no block is projected twice.  The host picks the smallest T for
// which the resident clusters cover every piece (the cost of a tile hardly depends on its
// length: each one streams all of W).
__host__ __device__ inline int64_t csa_ranges(int64_t ne, int64_t T) {
  return ne <= 64 * T ? 1 : 1 + (ne - 64 * T + 64 * T - 2) / (64 * T - 1);
}

__host__ __device__ inline void csa_piece_of(int64_t k, int64_t ne, int ncg, int64_t n, int64_t T,
                                             int64_t R, Unit* q) {
  const int64_t per_seq = R * ncg;
  q->b = static_cast<int>(k / per_seq);
  const int64_t rem = k - static_cast<int64_t>(q->b) * per_seq;
  const int64_t r = rem / ncg;
  q->cg = static_cast<int>(rem - r * ncg);
  q->e0 = r == 0 ? 0 : 64 * T + (r - 1) * (64 * T - 1);
  const int64_t e1 = q->e0 + (r == 0 ? 64 * T : 64 * T - 1);
  q->e1 = e1 < ne ? e1 : ne;
  q->first_block = q->e0 > 0 ? q->e0 - 1 : 0;
  q->rows = 4 * (q->e1 - q->first_block);
  q->stride = 256;
  q->ntiles = static_cast<int>((q->e1 - q->first_block + 63) / 64);
  q->row0 = static_cast<int64_t>(q->b) * n + 4 * q->first_block;
  q->j = 0;
}

struct CsaWalk {
  int64_t k, end;  // pieces [k, end) are this cluster's
};

// The units a cluster works through: CSA pieces from its schedule entry, HCA tiles
// u = cid, cid + ncl, ...
struct Sched {
  int64_t u, step, units;
  CsaWalk w;
};
template <bool CSA>
__device__ __forceinline__ Sched sched_begin(const Args& a, int64_t cid, int64_t ncl) {
  Sched s{cid, ncl, a.units, CsaWalk{0, 0}};
  if constexpr (CSA) {
    if (cid < a.units && cid < kMaxClusters) s.w = CsaWalk{a.start_k[cid], a.start_k[cid + 1]};
  }
  return s;
}
template <bool CSA>
__device__ __forceinline__ bool sched_next(const Args& a, Sched* s, uint32_t rank, Unit* q);

// HCA: unit u = (sequence, 256-token tile, channel-group pair), pair fastest; the leader
// takes group 2p, the peer 2p + 1.  A tile holding one window is 128 tokens.
__device__ __forceinline__ Unit hca_unit(const Args& a, int64_t u, uint32_t rank) {
  Unit h;
  const int npairs = a.ncg / 2;
  const int64_t tiles_per_seq = (a.ne + 1) / 2;
  const int p = static_cast<int>(u % npairs);
  const int64_t r = u / npairs;
  h.b = static_cast<int>(r / tiles_per_seq);
  h.j = r - static_cast<int64_t>(h.b) * tiles_per_seq;
  h.cg = 2 * p + static_cast<int>(rank);
  h.row0 = static_cast<int64_t>(h.b) * a.n + h.j * 256;
  const int64_t wins = a.ne - 2 * h.j < 2 ? a.ne - 2 * h.j : 2;
  h.rows = 128 * wins;
  h.stride = 256;
  h.ntiles = 1;
  h.e0 = h.e1 = h.first_block = 0;
  return h;
}
template <bool CSA>
__device__ __forceinline__ bool sched_next(const Args& a, Sched* s, uint32_t rank, Unit* q) {
  if constexpr (CSA) {
    if (s->w.k >= s->w.end) return false;
    csa_piece_of(s->w.k++, a.ne, a.ncg, a.n, a.tile_budget, a.ranges, q);
    return true;
  } else {
    if (s->u >= s->units) return false;
    *q = hca_unit(a, s->u, rank);
    s->u += s->step;
    return true;
  }
}

// Tokens of tile t (MMA N): 256, or the rest of the unit rounded up to 16.
__device__ __forceinline__ int tile_tokens(const Unit& q, int t) {
  const int64_t left = q.rows - static_cast<int64_t>(t) * q.stride;
  return left >= 256 ? 256 : static_cast<int>((left + 15) & ~int64_t(15));
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Softmax partial of one 4-row b-block for one channel: L = max + log2(sum of exp2) and
// the weighted mean of the C rows (the block's whole contribution to a joint softmax).
__device__ __forceinline__ void block_partial(const float* z, const float* cv, const float* b2,
                                              float* L, float* mean) {
  float l[4], mx = -INFINITY;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    l[k] = fmaf(z[k], kLog2e, b2[k]);
    mx = fmaxf(mx, l[k]);
  }
  float s = 0.f, acc = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float w = ex2_ftz(l[k] - mx);
    s += w;
    acc = fmaf(w, cv[k], acc);
  }
  *L = mx + lg2_approx(s);  // s >= 1: the largest term is exp2(0)
  *mean = __fdividef(acc, s);
}

// Instruction descriptor of the pair MMA: as idesc_bf16 with M = 256.
__host__ __device__ constexpr uint32_t idesc_pair(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(256 >> 4) << 24);
}

}  // namespace pair

// W maps: CSA W0 = W^{KV_a}, W1 = W^{KV_b}, W2 = W^{Z_a}, W3 = W^{Z_b} (the leader loads
// W0/W2, the peer W1/W3); HCA W0 = W^{KV}, W1 = W^{Z} (both CTAs).
template <bool CSA, typename OutT, bool CACHE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::kThreads, 1)
    fused_pair_kernel(const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmW0,
                      const __grid_constant__ CUtensorMap tmW1,
                      const __grid_constant__ CUtensorMap tmW2,
                      const __grid_constant__ CUtensorMap tmW3, const __grid_constant__ Args a,
                      const FusedCacheArg<CACHE> cf) {
  using C = pair::Cfg;
  constexpr int S = C::STAGES;
  constexpr int R = pair::kGroups * pair::kSlotsPerGroup;  // exchange slots (CSA)

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // [R][128][8] CSA partials: the peer stages a slot here, then copies it to the same
  // place in the leader.  HCA: [2 windows][128][3] half-window states.
  float* xbuf = reinterpret_cast<float*>(smem + S * C::STAGE);
  float2* carry = reinterpret_cast<float2*>(smem + S * C::STAGE + C::XBUF);  // [128] (CSA)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE + C::XBUF + C::CARRY);
  uint64_t* full = bars;                   // [S] leader: both CTAs' bytes of a stage
  uint64_t* empty = bars + S;              // [S] each CTA: the leader's MMAs freed the stage
  uint64_t* tmem_full = bars + 2 * S;      // each CTA: accumulators of a tile complete
  uint64_t* tmem_empty = tmem_full + 1;    // leader: every epilogue group drained TMEM
  uint64_t* final_bar = tmem_full + 2;     // each CTA: every MMA of the leader finished
  uint64_t* xfull = tmem_full + 3;         // [R] leader: a slot arrived (1 + its bytes)
  uint64_t* xempty = xfull + R;            // [R] peer: the leader has read a slot (1)
  uint64_t* carry_full = xempty + R;       // peer (CSA): group 3 wrote the carry (1)
  uint64_t* carry_empty = carry_full + 1;  // peer (CSA): group 0 has read it (1)
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(carry_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(carry_empty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = blockIdx.x & 1u;  // clusters of two consecutive CTAs along x
  const uint32_t peer = rank ^ 1u;
  const int64_t cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const uint32_t peer_abort = cluster_addr(smem_u32(const_cast<int*>(abort_flag)), peer);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 2 * pair::kGroups);  // one arrival per epilogue group and CTA
    mbar_init(final_bar, 1);
    for (int r = 0; r < R; ++r) {
      mbar_init(&xfull[r], 1);
      mbar_init(&xempty[r], 1);
    }
    mbar_init(carry_full, 1);
    mbar_init(carry_empty, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  cluster_sync_all();  // barriers and flags of both CTAs exist before any remote arrival
  if (warp == 1) {     // one warp of each CTA allocates the pair's 512 columns
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
      const CUtensorMap* mA0 = CSA ? (rank ? &tmW1 : &tmW0) : &tmW0;
      const CUtensorMap* mA1 = CSA ? (rank ? &tmW3 : &tmW2) : &tmW1;
      // W stays in L2 while H streams past: every pair reads its channel groups' W on every
      // tile (DRAM reads per launch 666 -> 609 MB on the n = 32768 CSA workload)
      const uint64_t wpol = l2_evict_last_policy();
      int stage = 0;
      uint32_t phase = 0;
      int pending_parity[S];
      for (int s = 0; s < S; ++s) pending_parity[s] = -1;
      bool ok = true;
      pair::Sched sc = pair::sched_begin<CSA>(a, cid, ncl);
      pair::Unit q;
      while (ok && pair::sched_next<CSA>(a, &sc, rank, &q)) {
        for (int t = 0; t < q.ntiles && ok; ++t) {
          const int nt = pair::tile_tokens(q, t);
          const int y = static_cast<int>(q.row0 + static_cast<int64_t>(t) * q.stride +
                                         static_cast<int64_t>(rank) * (nt / 2));
          for (int kstep = 0; kstep < a.nk; ++kstep) {
            if (!pair::wait_pair(&empty[stage], phase ^ 1u, abort_flag, peer_abort)) {
              ok = false;
              break;
            }
            if (rank == 0) {  // the leader arms its barrier for both CTAs' bytes
              mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE);
              pending_parity[stage] = static_cast<int>(phase);
            }
            const uint32_t lbar = cluster_addr(smem_u32(&full[stage]), 0);
            uint8_t* st = smem + stage * C::STAGE;
            const int x = kstep * C::BK;
            tma_load_2d_pair(smem_u32(st + C::A_BYTES), &tmH, lbar, x, y);
            tma_load_2d_pair_hint(smem_u32(st + 0 * C::A_BOX), mA0, lbar, q.cg * kCh, x, wpol);
            tma_load_2d_pair_hint(smem_u32(st + 1 * C::A_BOX), mA0, lbar, q.cg * kCh + 64, x, wpol);
            tma_load_2d_pair_hint(smem_u32(st + 2 * C::A_BOX), mA1, lbar, q.cg * kCh, x, wpol);
            tma_load_2d_pair_hint(smem_u32(st + 3 * C::A_BOX), mA1, lbar, q.cg * kCh + 64, x, wpol);
            if (++stage == S) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (!ok && rank == 0) {  // drain the stages this CTA armed before giving up
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
        while (ok && pair::sched_next<CSA>(a, &sc, 0, &q)) {
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
                  // same operand layouts as the single-CTA kernel, per CTA half
                  const uint64_t ad = smem_desc(st + (2 * s) * C::A_BOX + ks * 16 * 128,
                                                C::A_BOX, 1024, 2);
                  const uint64_t bd = smem_desc(st + C::A_BYTES + ks * 32, 16, 1024, 2);
                  umma_bf16_pair(tmem_base + s * 256, ad, bd, idesc, (kstep | ks) != 0 ? 1u : 0u);
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
        // both CTAs learn when every MMA (which reads and writes both) has finished
        umma_commit_pair(cluster_addr(smem_u32(final_bar), 0));
        umma_commit_pair(cluster_addr(smem_u32(final_bar), 1));
      }
      pair::wait_pair(final_bar, 0, abort_flag, peer_abort, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..17)
    const int eg = (warp - 2) >> 2;         // group: tokens [64 eg, 64 eg + 64) of a tile
    const int qw = warp & 3;                // TMEM lane quarter this warp may access
    const int row = qw * 32 + lane;         // TMEM lane = channel within the CTA's group
    const bool elected = ((warp - 2) & 3) == 0 && lane == 0;  // one thread per group
    const int gbar = 1 + eg;                // the group's named barrier (128 threads)
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(qw * 32) << 16);
    const uint32_t leader_tmem_empty = cluster_addr(smem_u32(tmem_empty), 0);
    uint32_t acc_phase = 0;
    uint32_t xcount = 0;  // CSA: exchange chunks of this group so far
    uint32_t ccount = 0;  // CSA peer: carries this group has written (group 3) or read (group 0)
    bool ok = true;
    pair::Sched sc = pair::sched_begin<CSA>(a, cid, ncl);
    pair::Unit unit;
    while (ok && pair::sched_next<CSA>(a, &sc, rank, &unit)) {
      if constexpr (CSA) {
        const pair::Unit& pc = unit;
        const int64_t ch = static_cast<int64_t>(pc.cg) * kCh + row;
        const float* Bsrc = rank == 0 ? a.B0 : a.B1;  // B^a (leader) or B^b (peer)
        float b2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) b2[k] = __ldg(Bsrc + k * a.c + ch) * kLog2e;
        for (int t = 0; t < pc.ntiles && ok; ++t) {
          const int nch = pair::tile_tokens(pc, t) / 16;
          const int c_lo = 4 * eg, c_hi = 4 * eg + 4 < nch ? 4 * eg + 4 : nch;
          // one decision for the group's four warps (they meet at named barriers below)
          if (!bar_and(gbar, 128, pair::wait_pair(tmem_full, acc_phase, abort_flag, peer_abort))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int64_t kb_tile = pc.first_block + static_cast<int64_t>(t) * 64;
          if (rank == 1) {
            // partial of the block before the group's first chunk: block 16 eg - 1 of the
            // tile; for group 0 the last block of the tile before (carried over from group
            // 3), or none in a piece's first tile (its block 0 is the halo, which is no
            // entry, or the sequence's entry 0, which has no b-rows)
            float pL = -INFINITY, pmean = 0.f;
            if (eg > 0 && c_lo < nch) {
              float cv[16], zv[16];
              tmem_ld16(lane_addr + (c_lo - 1) * 16, cv);
              tmem_ld16(lane_addr + 256 + (c_lo - 1) * 16, zv);
              tmem_wait_ld();
              pair::block_partial(zv + 12, cv + 12, b2, &pL, &pmean);
            } else if (eg == 0 && t > 0) {
              if (!bar_and(gbar, 128, pair::wait_pair(carry_full, ccount & 1u, abort_flag,
                                                      peer_abort))) {
                ok = false;
                break;
              }
              const float2 cr = carry[row];
              pL = cr.x;
              pmean = cr.y;
              bar_named(gbar, 128);  // every thread of the group has read the carry
              if (elected) mbar_arrive(carry_empty);
              ++ccount;
            }
#pragma unroll 1
            for (int c = c_lo; c < c_hi; ++c, ++xcount) {
              float cv[16], zv[16];
              tmem_ld16(lane_addr + c * 16, cv);
              tmem_ld16(lane_addr + 256 + c * 16, zv);
              tmem_wait_ld();
              float L[4], mean[4];
#pragma unroll
              for (int blk = 0; blk < 4; ++blk)
                pair::block_partial(zv + 4 * blk, cv + 4 * blk, b2, &L[blk], &mean[blk]);
              const uint32_t slot = eg * pair::kSlotsPerGroup + xcount % pair::kSlotsPerGroup;
              const uint32_t xpar = (xcount / pair::kSlotsPerGroup) & 1u;
              if (!bar_and(gbar, 128, pair::wait_pair(&xempty[slot], xpar ^ 1u, abort_flag,
                                                      peer_abort))) {
                ok = false;
                break;
              }
              // entry 4c + j of the tile takes the partial of block 4c + j - 1
              float4* xs = reinterpret_cast<float4*>(xbuf + (slot * 128 + row) * pair::kXFloats);
              xs[0] = make_float4(pL, pmean, L[0], mean[0]);
              xs[1] = make_float4(L[1], mean[1], L[2], mean[2]);
              fence_proxy_async_smem();
              bar_named(gbar, 128);
              if (elected) {  // one thread moves the slot to the same place in the leader
                const uint32_t src = smem_u32(xbuf + slot * 128 * pair::kXFloats);
                const uint32_t lbar = cluster_addr(smem_u32(&xfull[slot]), 0);
                mbar_arrive_expect_tx_cluster(lbar, pair::kSlotBytes);
                bulk_copy_to_cluster(cluster_addr(src, 0), src, pair::kSlotBytes, lbar);
              }
              pL = L[3];
              pmean = mean[3];
            }
            // the last group hands the partial of the tile's last block to group 0, whose
            // next tile starts with that block's entry
            if (ok && eg == pair::kGroups - 1 && t + 1 < pc.ntiles) {
              if (!bar_and(gbar, 128, pair::wait_pair(carry_empty, (ccount & 1u) ^ 1u, abort_flag,
                                                      peer_abort))) {
                ok = false;
                break;
              }
              carry[row] = make_float2(pL, pmean);
              bar_named(gbar, 128);  // every thread of the group has written
              if (elected) mbar_arrive(carry_full);
              ++ccount;
            }
          } else {
#pragma unroll 1
            for (int c = c_lo; c < c_hi; ++c, ++xcount) {
              float cv[16], zv[16];
              tmem_ld16(lane_addr + c * 16, cv);
              tmem_ld16(lane_addr + 256 + c * 16, zv);
              tmem_wait_ld();
              const uint32_t slot = eg * pair::kSlotsPerGroup + xcount % pair::kSlotsPerGroup;
              const uint32_t xpar = (xcount / pair::kSlotsPerGroup) & 1u;
              if (!bar_and(gbar, 128, pair::wait_pair(&xfull[slot], xpar, abort_flag, peer_abort))) {
                ok = false;
                break;
              }
              const float4* xs =
                  reinterpret_cast<const float4*>(xbuf + (slot * 128 + row) * pair::kXFloats);
              const float4 x0 = xs[0], x1 = xs[1];
              bar_named(gbar, 128);  // every thread of the group has read the slot
              if (elected) mbar_arrive_cluster(cluster_addr(smem_u32(&xempty[slot]), 1));
              const float pl[4] = {x0.x, x0.z, x1.x, x1.z};
              const float pm[4] = {x0.y, x0.w, x1.y, x1.w};
#pragma unroll
              for (int blk = 0; blk < 4; ++blk) {
                const int lb = 4 * c + blk;  // block within the tile
                const int64_t kb = kb_tile + lb;
                // entry kb: a-rows of block kb here, b-rows of block kb - 1 as (L, mean);
                // a piece's halo block (e0 - 1) is no entry
                if (kb >= pc.e0 && kb < pc.e1) {
                  float l[4], mx = pl[blk];
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    l[k] = fmaf(zv[4 * blk + k], kLog2e, b2[k]);
                    mx = fmaxf(mx, l[k]);
                  }
                  float s = 0.f, acc = 0.f;
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const float w = ex2_ftz(l[k] - mx);
                    s += w;
                    acc = fmaf(w, cv[4 * blk + k], acc);
                  }
                  const float f = ex2_ftz(pl[blk] - mx);  // 0 when there are no b-rows
                  s += f;
                  acc = fmaf(pm[blk], f, acc);
                  store_entry<CACHE, OutT>(a, cf, pc.b, kb, ch, __fdividef(acc, s));
                }
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
      } else {
        const pair::Unit& h = unit;
        const int64_t ch = static_cast<int64_t>(h.cg) * kCh + row;
        const int wins = static_cast<int>(h.rows / 128);
        const int w = eg >> 1, half = eg & 1;  // window of the tile, rows [64 half, +64) of it
        const bool active = w < wins;
        const int wbar = 5 + w;  // the window's two groups (256 threads)
        const bool got = pair::wait_pair(tmem_full, acc_phase, abort_flag, peer_abort);
        if (!(active ? bar_and(wbar, 256, got) : bar_and(gbar, 128, got))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (active) {
          float M = -INFINITY, Ssum = 0.f, A = 0.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            const int cc = 4 * half + c;  // chunk within the window
            float cv[16], zv[16];
            const uint32_t col = static_cast<uint32_t>(w * 128 + cc * 16);
            tmem_ld16(lane_addr + col, cv);
            tmem_ld16(lane_addr + 256 + col, zv);
            tmem_wait_ld();
            float cmx = -INFINITY;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float b2 = __ldg(a.B0 + (cc * 16 + k) * a.c + ch) * kLog2e;
              zv[k] = fmaf(zv[k], kLog2e, b2);
              cmx = fmaxf(cmx, zv[k]);
            }
            const float nm = fmaxf(M, cmx);
            const float sc = ex2_ftz(M - nm);
            Ssum *= sc;
            A *= sc;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const float wgt = ex2_ftz(zv[k] - nm);
              Ssum += wgt;
              A = fmaf(wgt, cv[k], A);
            }
            M = nm;
          }
          // the second half's state goes through shared memory to the first half
          float* hs = xbuf + (w * 128 + row) * 3;
          if (half == 1) {
            hs[0] = M;
            hs[1] = Ssum;
            hs[2] = A;
          }
          bar_named(wbar, 256);
          if (half == 0) {
            const float M1 = hs[0], S1 = hs[1], A1 = hs[2];
            const float nm = fmaxf(M, M1);
            const float f0 = ex2_ftz(M - nm), f1 = ex2_ftz(M1 - nm);
            Ssum = fmaf(S1, f1, Ssum * f0);
            A = fmaf(A1, f1, A * f0);
            store_entry<CACHE, OutT>(a, cf, h.b, h.j * 2 + w, ch, __fdividef(A, Ssum));
          }
        }
        tc_fence_before();
        bar_named(gbar, 128);
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

#include "fused_scalar.cuh"

// ------------------------------------------------------------------ host side

// 2-D bf16 row-major [rows, cols] tensor map with a [box_rows, box_cols] box; the
// swizzle span equals the box row (box_cols * 2 bytes: 128 or 64).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool CACHE>
FusedCacheArg<CACHE> fused_cache_arg(const FusedProblem& p) {
  if constexpr (CACHE) {
    return CacheFmt{static_cast<uint8_t*>(p.out_nope), static_cast<__nv_bfloat16*>(p.out_rope),
                    p.inv_freq, p.c - p.r, p.r, p.pos_stride, p.pos_offset, p.fp8_scale};
  } else {
    return NoCache{};
  }
}

template <bool CSA, int BK, typename OutT, bool CACHE>
kvc_status launch_impl(const FusedProblem& p, cudaStream_t st) {
  constexpr int NS = CSA ? 4 : 2;
  using C = Cfg<NS, BK>;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return KVC_ERR_CUDA;
  if (p.batch * p.n > (int64_t(1) << 31) - 1 - C::TN) return KVC_ERR_UNSUPPORTED;  // TMA y: int32
  CUtensorMap mh, mw[4];
  if (!make_map(&mh, p.H, static_cast<uint64_t>(p.batch * p.n), static_cast<uint64_t>(p.d), C::TN,
                BK))
    return KVC_ERR_CUDA;
  for (int s = 0; s < 4; ++s) {
    const void* w = CSA ? p.W[s] : p.W[s < 2 ? s : 0];
    if (!make_map(&mw[s], w, static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.c), BK, 64))
      return KVC_ERR_CUDA;
  }
  Args a{};
  a.B0 = p.B0;
  a.B1 = p.B1;
  a.out = p.out;
  a.batch = p.batch;
  a.n = p.n;
  a.c = p.c;
  a.ne = p.ne;
  a.ncg = static_cast<int>(p.c / kCh);
  a.nk = static_cast<int>(p.d / BK);
  int64_t grid;
  if constexpr (CSA) {
    const int64_t seq_units = p.batch * a.ncg;
    int64_t P = sms / seq_units;
    if (P < 1) P = 1;
    if (P > p.ne) P = p.ne;
    a.pieces_per_unit = static_cast<int>(P);
    a.units = seq_units * P;
  } else {
    a.pieces_per_unit = 1;
    a.units = p.batch * ((p.ne * 128 + C::TN - 1) / C::TN) * a.ncg;
  }
  grid = a.units < sms ? a.units : sms;
  auto kern = fused_pool_kernel<CSA, BK, OutT, CACHE>;
  if (!raise_smem_limit(reinterpret_cast<const void*>(kern))) return KVC_ERR_CUDA;
  kern<<<static_cast<unsigned>(grid), kThreads, C::SMEM, st>>>(mh, mw[0], mw[1], mw[2], mw[3], a,
                                                             fused_cache_arg<CACHE>(p));
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = CSA ? (CACHE ? "fused_pool_kernel/csa/cache" : "fused_pool_kernel/csa")
                      : (CACHE ? "fused_pool_kernel/hca/cache" : "fused_pool_kernel/hca");
  return KVC_OK;
}

// CSA CTA-pair schedule (see csa_piece_of): the smallest tile budget T with which
// `clusters` clusters take every piece, each cluster's first piece, and the number of
// clusters that get work (returned).
int64_t plan_csa(Args* a, int64_t clusters) {
  const int64_t G = a->batch * a->ncg;
  // deal the pieces of budget T to clusters in turn; calls take(k0, k1) per cluster
  auto deal = [&](int64_t T, auto take) {
    const int64_t R = pair::csa_ranges(a->ne, T), total = a->batch * R * a->ncg;
    int64_t k = 0, used = 0;
    pair::Unit q;
    while (k < total) {
      const int64_t k0 = k;
      int64_t left = T;
      while (k < total) {
        pair::csa_piece_of(k, a->ne, a->ncg, a->n, T, R, &q);
        if (q.ntiles > left) break;
        left -= q.ntiles;
        ++k;
      }
      take(used++, k0, k);
    }
    return used;
  };
  auto fits = [&](int64_t T) { return deal(T, [](int64_t, int64_t, int64_t) {}) <= clusters; };
  int64_t lo = (G * ((a->ne + 63) / 64) + clusters - 1) / clusters;
  if (lo < 1) lo = 1;
  int64_t hi = lo;
  while (!fits(hi)) hi *= 2;
  while (lo < hi) {  // the fewest clusters needed does not grow with T
    const int64_t mid = lo + (hi - lo) / 2;
    if (fits(mid)) {
      hi = mid;
    } else {
      lo = mid + 1;
    }
  }
  a->tile_budget = lo;
  a->ranges = pair::csa_ranges(a->ne, lo);
  const int64_t busy = deal(lo, [&](int64_t c, int64_t k0, int64_t k1) {
    a->start_k[c] = static_cast<int32_t>(k0);
    a->start_k[c + 1] = static_cast<int32_t>(k1);
  });
  return busy;
}

// CTA-pair launch (fused_pair_kernel): clusters of two CTAs, as many as can be resident.
template <bool CSA, typename OutT, bool CACHE>
kvc_status launch_pair(const FusedProblem& p, cudaStream_t st) {
  using C = pair::Cfg;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return KVC_ERR_CUDA;
  if (p.batch * p.n > (int64_t(1) << 31) - 1 - 256) return KVC_ERR_UNSUPPORTED;  // TMA y: int32
  CUtensorMap mh, mw[4];
  if (!make_map(&mh, p.H, static_cast<uint64_t>(p.batch * p.n), static_cast<uint64_t>(p.d), 128,
                C::BK))
    return KVC_ERR_CUDA;
  for (int s = 0; s < 4; ++s) {
    const void* w = CSA ? p.W[s] : p.W[s < 2 ? s : 0];
    if (!make_map(&mw[s], w, static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.c), C::BK, 64))
      return KVC_ERR_CUDA;
  }
  auto kern = fused_pair_kernel<CSA, OutT, CACHE>;
  if (!raise_smem_limit(reinterpret_cast<const void*>(kern))) return KVC_ERR_CUDA;
  int clusters = 0;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
    cfg.blockDim = dim3(pair::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
      (void)cudaGetLastError();
      return KVC_ERR_UNSUPPORTED;  // no resident pair: the caller takes the single-CTA kernel
    }
  }
  Args a{};
  a.B0 = p.B0;
  a.B1 = p.B1;
  a.out = p.out;
  a.batch = p.batch;
  a.n = p.n;
  a.c = p.c;
  a.ne = p.ne;
  a.ncg = static_cast<int>(p.c / kCh);
  a.nk = static_cast<int>(p.d / C::BK);
  a.pieces_per_unit = 1;
  if constexpr (CSA) {
    if (clusters > kMaxClusters) clusters = kMaxClusters;
    a.units = plan_csa(&a, clusters);
  } else {
    a.units = p.batch * ((p.ne + 1) / 2) * (a.ncg / 2);
  }
  const int64_t ncl = a.units < clusters ? a.units : clusters;
  kern<<<static_cast<unsigned>(2 * ncl), pair::kThreads, C::SMEM, st>>>(mh, mw[0], mw[1], mw[2], mw[3],
                                                                   a, fused_cache_arg<CACHE>(p));
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = CSA ? (CACHE ? "fused_pair_kernel/csa/cache" : "fused_pair_kernel/csa")
                      : (CACHE ? "fused_pair_kernel/hca/cache" : "fused_pair_kernel/hca");
  return KVC_OK;
}

// Scalar-logit CTA-pair launch (fused_scalar_kernel).  No single-CTA form: without a
// resident pair it returns KVC_ERR_UNSUPPORTED.
template <bool CSA, typename OutT>
kvc_status launch_scalar(const FusedProblem& p, cudaStream_t st) {
  using C = pair::Cfg;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return KVC_ERR_CUDA;
  if (p.batch * p.n > (int64_t(1) << 31) - 1 - 256) return KVC_ERR_UNSUPPORTED;  // TMA y: int32
  CUtensorMap mh, mw0, mw1;
  if (!make_map(&mh, p.H, static_cast<uint64_t>(p.batch * p.n), static_cast<uint64_t>(p.d), 128,
                C::BK) ||
      !make_map(&mw0, p.W[0], static_cast<uint64_t>(p.d), static_cast<uint64_t>(p.c), C::BK, 64) ||
      !make_map(&mw1, CSA ? p.W[1] : p.W[0], static_cast<uint64_t>(p.d),
                static_cast<uint64_t>(p.c), C::BK, 64))
    return KVC_ERR_CUDA;
  auto kern = fused_scalar_kernel<CSA, OutT>;
  if (!raise_smem_limit(reinterpret_cast<const void*>(kern))) return KVC_ERR_CUDA;
  int clusters = 0;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
    cfg.blockDim = dim3(scal::kThreads, 1, 1);
    cfg.dynamicSmemBytes = scal::Cfg::SMEM;
    cfg.stream = st;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
      (void)cudaGetLastError();
      return KVC_ERR_UNSUPPORTED;
    }
  }
  Args a{};
  a.B0 = p.B0;
  a.B1 = p.B1;
  a.out = p.out;
  a.batch = p.batch;
  a.n = p.n;
  a.c = p.c;
  a.ne = p.ne;
  a.nk = static_cast<int>(p.d / C::BK);
  a.wz0 = p.wz[0];
  a.wz1 = p.wz[1];
  const int ncg = static_cast<int>(p.c / kCh);
  if constexpr (CSA) {
    a.ncg = (ncg + 1) / 2;  // channel-group pairs: the leader takes group 2p, the peer 2p + 1
    if (clusters > kMaxClusters) clusters = kMaxClusters;
    a.units = plan_csa(&a, clusters);
  } else {
    a.ncg = (ncg + 3) / 4;  // channel quads: two groups per CTA
    a.units = p.batch * ((p.ne + 1) / 2) * a.ncg;
  }
  const int64_t ncl = a.units < clusters ? a.units : clusters;
  kern<<<static_cast<unsigned>(2 * ncl), scal::kThreads, scal::Cfg::SMEM, st>>>(mh, mw0, mw1, a);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = CSA ? "fused_scalar_kernel/csa" : "fused_scalar_kernel/hca";
  return KVC_OK;
}

}  // namespace fused

// Stage K per mode.  64-deep stages: CSA 80 KB (two fit), HCA 64 KB (three).  32-deep
// stages (CSA: five of 40 KB) measured slower on B200 (0.84 vs 0.79 ms on the n = 32768,
// d = 7168 workload): the CSA tile is bound by shared-memory bandwidth (N = 128 operand
// reads plus TMA writes), not by pipeline depth.
constexpr int kBkCsa = 64;
constexpr int kBkHca = 64;

template <typename OutT, bool CACHE>
kvc_status launch_fused_typed(const FusedProblem& p, cudaStream_t st) {
  if (p.csa) {
    if (p.m != 4 || !p.overlap) return KVC_ERR_UNSUPPORTED;
    const kvc_status r = fused::launch_pair<true, OutT, CACHE>(p, st);
    if (r != KVC_ERR_UNSUPPORTED) return r;
    return fused::launch_impl<true, kBkCsa, OutT, CACHE>(p, st);
  }
  if (p.m != 128) return KVC_ERR_UNSUPPORTED;
  if ((p.c / fused::kCh) % 2 == 0) {  // channel groups pair up over the CTA pair
    const kvc_status r = fused::launch_pair<false, OutT, CACHE>(p, st);
    if (r != KVC_ERR_UNSUPPORTED) return r;
  }
  return fused::launch_impl<false, kBkHca, OutT, CACHE>(p, st);
}

kvc_status launch_fused(const FusedProblem& p, cudaStream_t st) {
  if (p.scalar) {
    if (p.csa ? (p.m != 4 || !p.overlap) : p.m != 128) return KVC_ERR_UNSUPPORTED;
    if (p.csa)
      return p.out_bf16 ? fused::launch_scalar<true, __nv_bfloat16>(p, st)
                        : fused::launch_scalar<true, float>(p, st);
    return p.out_bf16 ? fused::launch_scalar<false, __nv_bfloat16>(p, st)
                      : fused::launch_scalar<false, float>(p, st);
  }
  if (p.cache) return launch_fused_typed<__nv_bfloat16, true>(p, st);
  return p.out_bf16 ? launch_fused_typed<__nv_bfloat16, false>(p, st)
                    : launch_fused_typed<float, false>(p, st);
}

kvc_status read_and_clear_device_error(cudaStream_t st) {
  if (cudaStreamSynchronize(st) != cudaSuccess) return KVC_ERR_CUDA;
  unsigned int v = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return KVC_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return KVC_ERR_CUDA;
  bool failed = false;
  const bool index_error = read_and_clear_index_error(&failed);
  const unsigned int ix = read_and_clear_indexer_error(&failed);
  const unsigned int wx = read_and_clear_window_error(&failed);
  if (failed) return KVC_ERR_CUDA;
  if (v || (ix & 1u) || (wx & 1u)) return KVC_ERR_TIMEOUT;
  if (wx & 2u) return KVC_ERR_WORKSPACE;
  return (index_error || (ix & 2u)) ? KVC_ERR_INDEX : KVC_OK;
}

}  // namespace kvc
