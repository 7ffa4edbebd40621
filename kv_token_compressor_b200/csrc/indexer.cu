// Lightning indexer on sm_100a: scores of queries over compressed indexer keys on the
// tensor cores, and the exact top-k selection over those scores.
//
// What it computes (page "Ch 04 · CSA", §4 Lightning Indexer, the score equation and the
// selected-set equation; §5 for k):
//     I[t, s] = sum_h w[t, h] * max(0, q[t, h] . K[s])      (one key per entry, all heads)
//     selected(t) = the k entries of largest I[t, .]
//
// Scores (indexer_score_kernel).  Per query the work is a [keys x 128] x [128 x H] product
// followed by a per-key reduction over the heads, so the GEMM is arranged with the keys on
// M (128 TMEM lanes) and the heads on N: after tcgen05.ld every epilogue thread owns one
// key's H head dot products and the ReLU-weighted head sum is thread-local.  A decode step
// (one query per sequence) reads every key once: 256 bytes per key against 16 KFLOP on the
// tensor cores, so the kernel is bound by HBM; TMA streams 128-key tiles through a 4-stage
// ring, the accumulators rotate through 4 TMEM buffers so the epilogue of one tile overlaps
// the MMAs and loads of the next, and the queries' q tiles sit in two shared-memory slots.
//
// Top-k (indexer_topk_kernel).  A cluster of 8 CTAs per query holds the query's scores on
// chip (an eighth each, as order-preserving 32-bit keys) and finds the exact k-th largest
// key by a radix select over four 8-bit digits; every CTA pushes its per-digit histogram
// into the others' shared memory (st.async on mbarriers, no cluster-wide barrier per
// digit).  The selected entries (ties at the threshold to the smallest indices) are pushed
// in index order into every CTA's copy of the list, and each CTA places its share of the
// list by counting, for each entry, the entries that sort before it: no sort.
#include "kvc_common.cuh"
#include "kvc_host.h"
#include "kvc_launch.h"
#include "tc_ptx.cuh"

namespace kvc {

// bit 0: a bounded wait gave up; bit 1: a query's candidate window was out of range.
__device__ unsigned int g_indexer_error = 0;

namespace idx {

using namespace tcx;

constexpr int kD = 128;          // key / query width (two 64-wide 128-byte swizzle atoms)
constexpr int kKT = 128;         // keys per tile (MMA M, TMEM lanes)
constexpr int kStages = 4;       // key-tile ring
constexpr int kMaxH = 128;       // heads (MMA N)
constexpr int kAccBufs = 4;      // TMEM accumulators of 128 columns
constexpr int kEpiGroups = 2;    // epilogue groups of 4 warps, taking alternate tiles
constexpr int kThreads = 64 + kEpiGroups * 128;  // warp 0 TMA, warp 1 MMA, then the epilogue
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kHalf = kKT * 64 * 2;            // one [128 rows x 64] bf16 box, 16 KB
constexpr int kTile = 2 * kHalf;               // a key tile, 32 KB
constexpr int kQSlot = 2 * kMaxH * 64 * 2;     // a q tile, two [H x 64] boxes, 32 KB
constexpr size_t kSmem = 1024 + kStages * kTile + 2 * kQSlot + kEpiGroups * 2 * kMaxH * 4 + 256;

struct ScoreArgs {
  const float* w;
  const int64_t* key_start;
  const int64_t* n_visible;
  float* scores;
  int64_t T, key_rows, max_visible, ld, tiles_per_query, units;
  int H;
};

// Instruction descriptor of kind::f16 with both operands K-major: D fp32, A and B bf16,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_kk(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kKT >> 4) << 24);
}

__device__ __noinline__ bool wait_bounded_slow(uint64_t* bar, uint32_t parity,
                                               volatile int* abort_flag, bool honour_abort) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(&g_indexer_error, 1u);
      return false;
    }
  }
}
// Bounded wait; a phase that has already completed costs one try_wait and no call.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bounded_slow(bar, parity, abort_flag, honour_abort);
}

// The candidate window of query t; false (and the error bit) when it is out of range.
struct Window {
  int64_t start, count;
  bool ok;
};
__device__ __forceinline__ Window query_window(const ScoreArgs& a, int64_t t) {
  Window w;
  w.start = a.key_start[t];
  w.count = a.n_visible[t];
  w.ok = w.start >= 0 && w.count >= 0 && w.count <= a.max_visible &&
         w.start <= a.key_rows - w.count;
  return w;
}

// (query t, key tile j) of unit u, advanced one unit at a time (64-bit division once per
// CTA: in every unit it sat on the MMA thread's critical path).
struct UnitCursor {
  int64_t t, j, tiles;
  __device__ UnitCursor(const ScoreArgs& a, int64_t u)
      : t(u / a.tiles_per_query), j(u - (u / a.tiles_per_query) * a.tiles_per_query),
        tiles(a.tiles_per_query) {}
  __device__ __forceinline__ void next() {
    if (++j == tiles) {
      j = 0;
      ++t;
    }
  }
};

// Units u = (query t, key tile j), t-major; each CTA takes one contiguous range so that
// consecutive tiles share the query's q tile.  Every role walks the same units and takes
// the same skip decisions from the same device values.
__global__ void __launch_bounds__(kThreads, 1)
    indexer_score_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK, const ScoreArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ktiles = smem;                                // [kStages][kTile]
  uint8_t* qslots = smem + kStages * kTile;              // [2][kQSlot]
  float* wslots = reinterpret_cast<float*>(qslots + 2 * kQSlot);  // [group][2][kMaxH]
  uint64_t* bars = reinterpret_cast<uint64_t*>(wslots + kEpiGroups * 2 * kMaxH);
  uint64_t* full = bars;                          // [kStages] key tile landed
  uint64_t* empty = bars + kStages;               // [kStages] MMAs done with the key tile
  uint64_t* qfull = bars + 2 * kStages;           // [2] q tile landed
  uint64_t* qempty = qfull + 2;                   // [2] MMAs done with the q tile
  uint64_t* tfull = qempty + 2;                   // [kAccBufs] accumulator complete
  uint64_t* tempty = tfull + kAccBufs;            // [kAccBufs] epilogue drained it
  uint64_t* final_bar = tempty + kAccBufs;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(final_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(final_bar + 2);
  // a top-k launched next on the stream may start launching now (it reads the scores only
  // after this grid has completed)
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = a.H;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"(kAccBufs * 128));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t lo = static_cast<int64_t>(blockIdx.x) * a.units / gridDim.x;
  const int64_t hi = static_cast<int64_t>(blockIdx.x + 1) * a.units / gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int qcount = -1;
      int64_t cur_t = -1;
      Window win{0, 0, false};
      bool ok = true;
      UnitCursor cu(a, lo);
      for (int64_t u = lo; u < hi && ok; ++u, cu.next()) {
        const int64_t t = cu.t, j = cu.j;
        if (t != cur_t) {
          win = query_window(a, t);
          if (!win.ok) atomicOr(&g_indexer_error, 2u);  // the query is skipped
        }
        if (!win.ok || j * kKT >= win.count) {
          cur_t = t;
          continue;
        }
        if (t != cur_t || qcount < 0) {
          ++qcount;
          const int qs = qcount & 1;
          if (!wait_bounded(&qempty[qs], ((qcount >> 1) & 1) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&qfull[qs], 2 * H * 64 * 2);
          uint8_t* qb = qslots + qs * kQSlot;
          tma_load_2d(smem_u32(qb), &tmQ, &qfull[qs], 0, static_cast<int>(t * H));
          tma_load_2d(smem_u32(qb + kQSlot / 2), &tmQ, &qfull[qs], 64, static_cast<int>(t * H));
        }
        cur_t = t;
        if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], kTile);
        uint8_t* kb = ktiles + stage * kTile;
        const int y = static_cast<int>(win.start + j * kKT);
        tma_load_2d(smem_u32(kb), &tmK, &full[stage], 0, y);
        tma_load_2d(smem_u32(kb + kHalf), &tmK, &full[stage], 64, y);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // Copies still in flight finish within microseconds; the final barrier below is
      // reached only after the MMA thread has drained its own work.
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int qcount = -1;
      int64_t cur_t = -1;
      Window win{0, 0, false};
      uint32_t n = 0;  // tiles issued (accumulator rotation)
      const uint32_t idesc = idesc_kk(H);
      // shared memory stays below 256 KB, so address >> 4 fits the 14-bit field with room
      // for every offset added to it
      const uint64_t adesc_base = smem_desc(smem_u32(ktiles), 16, 1024, 2);
      const uint64_t bdesc_base = smem_desc(smem_u32(qslots), 16, 1024, 2);
      bool ok = true;
      UnitCursor cu(a, lo);
      for (int64_t u = lo; u < hi && ok; ++u, cu.next()) {
        const int64_t t = cu.t, j = cu.j;
        if (t != cur_t) win = query_window(a, t);
        if (!win.ok || j * kKT >= win.count) {
          cur_t = t;
          continue;
        }
        if (t != cur_t || qcount < 0) {
          if (qcount >= 0) umma_commit(&qempty[qcount & 1]);  // the last query's q is free
          ++qcount;
          if (!wait_bounded(&qfull[qcount & 1], (qcount >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        cur_t = t;
        const uint32_t buf = n % kAccBufs, bpar = (n / kAccBufs) & 1u;
        if (!wait_bounded(&tempty[buf], bpar ^ 1u, abort_flag) ||
            !wait_bounded(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // both operands K-major, 128-byte swizzle: k-slice ks is 32 bytes into the 128-byte
        // rows of box ks / 4; 8-row groups 1024 bytes apart.  Only the start-address field
        // (address >> 4, low bits) changes between slices, so it is added to a base.
        const uint64_t ad0 = adesc_base + ((stage * kTile) >> 4);
        const uint64_t bd0 = bdesc_base + (((qcount & 1) * kQSlot) >> 4);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t off = ((ks >> 2) * kHalf + (ks & 3) * 32) >> 4;
          const uint32_t offq = ((ks >> 2) * (kQSlot / 2) + (ks & 3) * 32) >> 4;
          umma_bf16(tmem_base + buf * 128, ad0 + off, bd0 + offq, idesc, ks != 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        umma_commit(&tfull[buf]);
        ++n;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      umma_commit(final_bar);  // every MMA issued above has finished before TMEM is freed
      wait_bounded(final_bar, 0, abort_flag, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    // Two groups of four warps (the four TMEM lane quarters each) take alternate tiles, so
    // one group's TMEM round trips and stores overlap the other's.
    const int eg = (warp - 2) >> 2;
    const int qw = warp & 3;
    const int row = qw * 32 + lane;                 // TMEM lane = key within the tile
    const int eid = ((warp - 2) & 3) * 32 + lane;   // 0..127 within the group
    const int gbar = 1 + eg;                        // the group's named barrier
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(qw * 32) << 16);
    float* wg = wslots + eg * 2 * kMaxH;
    int qcount = -1;
    int64_t cur_t = -1;
    Window win{0, 0, false};
    uint32_t n = 0;
    bool ok = true;
    UnitCursor cu(a, lo);
    for (int64_t u = lo; u < hi && ok; ++u, cu.next()) {
      const int64_t t = cu.t, j = cu.j;
      if (t != cur_t) win = query_window(a, t);
      if (!win.ok || j * kKT >= win.count) {
        cur_t = t;
        continue;
      }
      if (t != cur_t || qcount < 0) {
        ++qcount;
        // the query's head weights; the slot's previous user (two queries back) is done
        if (eid < H) wg[(qcount & 1) * kMaxH + eid] = a.w[t * H + eid];
        bar_named(gbar, 128);
      }
      cur_t = t;
      const uint32_t mine = n;
      ++n;
      if ((mine & 1u) != static_cast<uint32_t>(eg)) continue;  // the other group's tile
      const float4* ws = reinterpret_cast<const float4*>(wg + (qcount & 1) * kMaxH);
      const uint32_t buf = mine % kAccBufs, bpar = (mine / kAccBufs) & 1u;
      // one decision for the group's four warps (they meet at the named barrier above)
      if (!bar_and(gbar, 128, wait_bounded(&tfull[buf], bpar, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float acc = 0.f;
      for (int c0 = 0; c0 < H; c0 += 64) {
        float v[64];
#pragma unroll
        for (int c = 0; c < 64; c += 16) {
          float (&vc)[16] = *reinterpret_cast<float(*)[16]>(v + c);
          if (c0 + c < H) tmem_ld16(lane_addr + buf * 128 + c0 + c, vc);
        }
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          if (c0 + c < H) {
            const float4 wq = ws[(c0 + c) >> 2];
            acc = fmaf(wq.x, fmaxf(v[c], 0.f), acc);
            acc = fmaf(wq.y, fmaxf(v[c + 1], 0.f), acc);
            acc = fmaf(wq.z, fmaxf(v[c + 2], 0.f), acc);
            acc = fmaf(wq.w, fmaxf(v[c + 3], 0.f), acc);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
      const int64_t key = j * kKT + row;
      if (key < win.count) a.scores[t * a.ld + key] = acc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kAccBufs * 128));
  }
}

// ---------------------------------------------------------------------------------
// Top-k: one cluster of CL CTAs per query row (launched with the portable 8).
// ---------------------------------------------------------------------------------
constexpr int kCluster = 8;   // portable cluster size: the guaranteed capacity
constexpr int kTkThreads = 1024;
constexpr int kSlice = 40960;    // scores held on chip per CTA
constexpr int kMaxK = 2048;
constexpr int kBins = 256;       // radix digits of 8 bits
constexpr int kWarps = kTkThreads / 32;
constexpr int kCandCap = 64;     // candidate positions a warp keeps after the second digit
constexpr int kRankChunks = kTkThreads / 128;  // threads that share one entry's rank
constexpr int kMaxShare = kMaxK / kCluster;    // list entries one CTA ranks and stores
constexpr int kRankBins = 256;                 // bins of key - threshold for the rank
// u32 offsets in the histogram region once it holds the list: keys [kMaxK + 4], this CTA's
// indices [kMaxShare], then the rank's bin starts, keys by bin and list positions by bin
constexpr int kListIdx = kMaxK + 256;
constexpr int kListAbove = kListIdx + kMaxShare;
constexpr int kListBKey = kListAbove + kRankBins;
constexpr int kListBPos = kListBKey + kMaxK;
// Shared memory (bytes).  The histogram region holds the selected list once the four
// digits are known; the receive region holds the rank sums.
constexpr size_t kTkKeys = 0;                                            // u32 [kSlice]
constexpr size_t kTkHist = kTkKeys + size_t(kSlice) * 4;                 // u32 [kWarps][kBins]
constexpr size_t kTkRecv = kTkHist + size_t(kWarps) * kBins * 4;         // u32 [2][CL][kBins]
constexpr size_t kTkCand = kTkRecv + 2 * size_t(kCluster) * kBins * 4;   // u16 [kWarps][cap]
constexpr size_t kTkBars = kTkCand + size_t(kWarps) * kCandCap * 2;      // 4 mbarriers
constexpr size_t kTkMisc = kTkBars + 4 * 8;
// info [CL][2], wcnt [2][kWarps], wsum [8], per-pass digit and rank [4][2], abort flag
constexpr size_t kTkSmem = kTkMisc + size_t(2 * kCluster + 2 * kWarps + 8 + 8 + 4) * 4;
static_assert(kListBPos + kMaxK / 2 <= kWarps * kBins, "selected list fits the histograms");
static_assert(kMaxShare + kRankBins <= 2 * kCluster * kBins, "rank sums fit the receive buffers");
static_assert(kRankBins == 256, "the rank's bin shift and scan assume 8-bit bins");
static_assert(kTkSmem <= 227 * 1024, "top-k shared memory");

struct TopkArgs {
  const float* scores;
  const int64_t* n_visible;
  int32_t* out_idx;
  float* out_score;
  int64_t T, max_visible, ld;
  int k;
};

// Order-preserving 32-bit key of a score (larger score, larger key; -0.0 as 0.0).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// The same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// A 4- or 8-byte store into a peer CTA's shared memory that counts its bytes on the mbarrier
// `bar` of that CTA (both addresses from peer_addr).
__device__ __forceinline__ void push_u32(uint32_t addr, uint32_t v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(addr),
               "r"(v), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void push_v2(uint32_t addr, uint32_t v0, uint32_t v1, uint32_t bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.u32 [%0], {%1, %2}, [%3];" ::"r"(addr),
      "r"(v0), "r"(v1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
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
__device__ __noinline__ bool tk_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(&g_indexer_error, 1u);
      return false;
    }
  }
}
// Bounded wait for the pushes of the other CTAs (acquire at cluster scope).
__device__ __forceinline__ bool tk_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (try_wait_cluster(bar, parity)) return true;
  return tk_wait_slow(bar, parity, abort_flag);
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait;" ::: "memory");
}
__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ uint32_t warp_inclusive_scan(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// One cluster of CL CTAs per query row; CTA r holds candidates [r * per, r * per + cnt) as
// order keys, warp w of it the contiguous segment [w * seg, (w + 1) * seg) of those.
//  1. Radix select of the ksel-th largest key over four 8-bit digits, high to low.  Each
//     warp counts its segment into its own histogram (the first digit while the scores
//     load); 256 threads sum the CTA's warps and push the sums into every CTA of the
//     cluster (st.async, counted on an mbarrier per buffer, two buffers alternating), so
//     every CTA picks the same digit with no cluster-wide barrier.  While it counts the
//     third digit, a warp keeps the positions of its keys at or above the 16-bit prefix
//     if they fit in kCandCap; the last digit, the warp's counts above and at the
//     threshold and the selection then read those alone (else they scan the segment).
//  2. The copies of the threshold that are taken go to the lowest indices (CTAs, then
//     warps, in index order, from the counts every CTA pushes); each CTA pushes its
//     selected keys, in index order, to their place in every CTA's copy of the list, and
//     each entry's index to the CTA that will store it.
//  3. Every CTA ranks its share of the list: the entry at list position e goes to output
//     place #{keys above it} + #{equal keys before it in the list}: the list is binned by
//     key minus threshold, the keys in higher bins are counted by one warp's scan, those of
//     its own bin one by one.  The list is in index order, so equal scores come out by
//     index.
template <int CL>
__global__ void __launch_bounds__(kTkThreads, 1) indexer_topk_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + kTkKeys);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kTkHist);
  uint32_t* recv = reinterpret_cast<uint32_t*>(smem + kTkRecv);
  uint16_t* cand = reinterpret_cast<uint16_t*>(smem + kTkCand);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTkBars);  // [0,1] digits, [2] counts, [3] list
  uint32_t* info = reinterpret_cast<uint32_t*>(smem + kTkMisc);  // [CL][2] above / at, per CTA
  uint32_t* wcnt = info + 2 * CL;                                 // [2][kWarps]
  uint32_t* wsum = wcnt + 2 * kWarps;                             // [8]
  uint32_t* slot = wsum + 8;                                      // [4][2] digit, rank left
  volatile int* abort_flag = reinterpret_cast<volatile int*>(slot + 8);
  uint32_t* list_key = hist;                   // [kMaxK + 4] selected keys, in index order
  uint32_t* list_idx = hist + kListIdx;        // [kMaxShare] indices of this CTA's share
  uint32_t* rank_acc = recv;                   // [kMaxShare]

  const uint32_t rank = blockIdx.x % CL;
  const int64_t t = blockIdx.x / CL;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  griddep_wait();  // launched early after the score kernel: its scores are complete from here
  const int64_t nv = a.n_visible[t];
  // the same decision in every CTA of the cluster: an out-of-range row is skipped whole
  if (nv < 0 || nv > a.max_visible) {
    if (rank == 0 && tid == 0) atomicOr(&g_indexer_error, 2u);
    return;
  }
  const int k = a.k;
  const int ksel = static_cast<int>(nv < k ? nv : k);
  if (ksel == 0) {  // no candidates: padding only, no exchange
    for (int e = static_cast<int>(rank) * kTkThreads + tid; e < k; e += CL * kTkThreads) {
      a.out_idx[t * k + e] = -1;
      if (a.out_score) a.out_score[t * k + e] = -INFINITY;
    }
    return;
  }
  // list positions [my0, my1) are ranked and stored here
  const int q = (ksel + CL - 1) / CL;
  const int my0 = min(ksel, static_cast<int>(rank) * q), my1 = min(ksel, my0 + q);
  if (tid == 0) {
    *abort_flag = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    mbar_arrive_expect_tx(&bars[0], CL * kBins * 4);
    mbar_arrive_expect_tx(&bars[1], CL * kBins * 4);
    mbar_arrive_expect_tx(&bars[2], CL * 8);
    mbar_arrive_expect_tx(&bars[3], static_cast<uint32_t>(ksel + (my1 - my0)) * 4);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // this CTA's candidates [lo, lo + cnt), a multiple of 4 apart; warp segments of 32s
  const int64_t per = ((nv + CL - 1) / CL + 3) & ~int64_t(3);
  const int64_t lo = rank * per;
  const int cnt = static_cast<int>(lo < nv ? (nv - lo < per ? nv - lo : per) : 0);
  const int seg = ((cnt + kWarps - 1) / kWarps + 31) & ~31;
  const int s0 = min(cnt, warp * seg), s1 = min(cnt, s0 + seg);
  uint32_t* whist = hist + warp * kBins;
  uint16_t* wcand = cand + warp * kCandCap;
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  reinterpret_cast<uint4*>(whist)[lane] = zero4;
  reinterpret_cast<uint4*>(whist)[lane + 32] = zero4;
  __syncwarp();
  cluster_arrive_relaxed();  // the barriers are initialised before any CTA pushes

  // load the segment as order keys, counting the first digit on the way
  const float* row = a.scores + t * a.ld + lo;
  for (int i0 = s0 + 4 * lane; i0 < s1; i0 += 4 * 128) {
    float4 f[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = i0 + 128 * r;
      if (i + 3 < s1) f[r] = __ldg(reinterpret_cast<const float4*>(row + i));
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = i0 + 128 * r;
      if (i + 3 < s1) {
        const uint4 u = make_uint4(order_key(f[r].x), order_key(f[r].y), order_key(f[r].z),
                                   order_key(f[r].w));
        *reinterpret_cast<uint4*>(keys + i) = u;
        atomicAdd(&whist[u.x >> 24], 1u);
        atomicAdd(&whist[u.y >> 24], 1u);
        atomicAdd(&whist[u.z >> 24], 1u);
        atomicAdd(&whist[u.w >> 24], 1u);
      } else {
        for (int e = i; e < s1; ++e) {
          const uint32_t u = order_key(row[e]);
          keys[e] = u;
          atomicAdd(&whist[u >> 24], 1u);
        }
      }
    }
  }
  __syncthreads();
  cluster_wait();

  const uint32_t lt = (1u << lane) - 1u;
  uint32_t prefix = 0, mask = 0;
  uint32_t kk = static_cast<uint32_t>(ksel);  // rank of the wanted key among the matches
  int ncand = 0;
  bool use_cand = false;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const int b = pass & 1;
    if (pass > 0) {
      if (pass == 3 && use_cand) {
        for (int c = lane; c < ncand; c += 32) {
          const uint32_t u = keys[wcand[c]];
          if ((u & mask) == prefix) atomicAdd(&whist[u & 0xFFu], 1u);
        }
      } else if (pass == 2) {
        // count, and keep every key at or above the 16-bit prefix, in index order, while
        // they fit
        int n = 0;
        for (int g0 = s0; g0 < s1; g0 += 128) {  // warp-uniform trip count (ballots)
          uint32_t u[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int i = g0 + 32 * r + lane;
            u[r] = i < s1 ? keys[i] : 0u;
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int i = g0 + 32 * r + lane;
            const bool c = i < s1 && u[r] >= prefix;
            const uint32_t cb = __ballot_sync(0xffffffffu, c);
            if (c) {
              const int at = n + __popc(cb & lt);
              if (at < kCandCap) wcand[at] = static_cast<uint16_t>(i);
              if ((u[r] & mask) == prefix) atomicAdd(&whist[(u[r] >> shift) & 0xFFu], 1u);
            }
            n += __popc(cb);
          }
        }
        ncand = n;
        use_cand = n <= kCandCap;
      } else {
        // 16-byte loads (segments start on multiples of 32 keys), two in flight per thread;
        // lanes of a warp that hit the same bin are serialised by the shared-memory atomics
        auto count4 = [&](uint4 v, int i) {
          if (i < s1 && (v.x & mask) == prefix) atomicAdd(&whist[(v.x >> shift) & 0xFFu], 1u);
          if (i + 1 < s1 && (v.y & mask) == prefix) atomicAdd(&whist[(v.y >> shift) & 0xFFu], 1u);
          if (i + 2 < s1 && (v.z & mask) == prefix) atomicAdd(&whist[(v.z >> shift) & 0xFFu], 1u);
          if (i + 3 < s1 && (v.w & mask) == prefix) atomicAdd(&whist[(v.w >> shift) & 0xFFu], 1u);
        };
        for (int i0 = s0 + 4 * lane; i0 < s1; i0 += 256) {
          const int i1 = i0 + 128;
          const uint4 v0 = *reinterpret_cast<const uint4*>(keys + i0);
          const uint4 v1 = i1 < s1 ? *reinterpret_cast<const uint4*>(keys + i1) : make_uint4(0u, 0u, 0u, 0u);
          count4(v0, i0);
          count4(v1, i1);
        }
      }
      __syncthreads();
    }
    if (tid < kBins) {
      // the CTA's count of bin tid, pushed into every CTA's buffer b
      uint32_t s = 0;
#pragma unroll 8
      for (int w = 0; w < kWarps; ++w) s += hist[w * kBins + tid];
      const uint32_t dst = smem_u32(recv + (b * CL + rank) * kBins + tid);
      const uint32_t bar = smem_u32(&bars[b]);
#pragma unroll
      for (int r = 0; r < CL; ++r) push_u32(peer_addr(dst, r), s, peer_addr(bar, r));
      tk_wait(&bars[b], (pass >> 1) & 1, abort_flag);
      if (tid == 0 && pass < 2) mbar_arrive_expect_tx(&bars[b], CL * kBins * 4);  // pass + 2
      // thread tid takes bin 255 - tid over the cluster, so a thread-order scan counts the
      // keys in higher bins
      uint32_t tot = 0;
      const uint32_t* rb = recv + b * CL * kBins + (kBins - 1 - tid);
#pragma unroll
      for (int r = 0; r < CL; ++r) tot += rb[r * kBins];
      const uint32_t incl = warp_inclusive_scan(tot, lane);
      if (lane == 31) wsum[warp] = incl;
      asm volatile("bar.sync 1, %0;" ::"n"(kBins) : "memory");
      const uint4 w0 = reinterpret_cast<const uint4*>(wsum)[0];
      const uint4 w1 = reinterpret_cast<const uint4*>(wsum)[1];
      const uint32_t above = incl - tot + (warp > 0 ? w0.x : 0u) + (warp > 1 ? w0.y : 0u) +
                             (warp > 2 ? w0.z : 0u) + (warp > 3 ? w0.w : 0u) +
                             (warp > 4 ? w1.x : 0u) + (warp > 5 ? w1.y : 0u) +
                             (warp > 6 ? w1.z : 0u);
      if (tot > 0 && above < kk && kk <= above + tot) {
        slot[2 * pass] = static_cast<uint32_t>(kBins - 1 - tid);
        slot[2 * pass + 1] = kk - above;
      }
    }
    __syncthreads();
    const uint32_t digit = slot[2 * pass] & 0xFFu;
    prefix |= digit << shift;
    mask |= 0xFFu << shift;
    kk = slot[2 * pass + 1];
    if (pass < 3) {
      __syncwarp();
      reinterpret_cast<uint4*>(whist)[lane] = zero4;
      reinterpret_cast<uint4*>(whist)[lane + 32] = zero4;
      __syncwarp();
    }
  }
  const uint32_t thr = prefix;  // the ksel-th largest key; kk of its copies are taken
  uint32_t wgt = 0, weq = 0;    // keys of the warp's segment above / at the threshold
  if (use_cand) {
    for (int c0 = 0; c0 < ncand; c0 += 32) {
      const bool in = c0 + lane < ncand;
      const uint32_t u = in ? keys[wcand[c0 + lane]] : 0u;
      wgt += __popc(__ballot_sync(0xffffffffu, in && u > thr));
      weq += __popc(__ballot_sync(0xffffffffu, in && u == thr));
    }
  } else {
    for (int g0 = s0; g0 < s1; g0 += 128) {
      uint32_t u[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = g0 + 32 * r + lane;
        u[r] = i < s1 ? keys[i] : 0u;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const bool in = g0 + 32 * r + lane < s1;
        wgt += __popc(__ballot_sync(0xffffffffu, in && u[r] > thr));
        weq += __popc(__ballot_sync(0xffffffffu, in && u[r] == thr));
      }
    }
  }
  if (lane == 0) {
    wcnt[warp] = wgt;
    wcnt[kWarps + warp] = weq;
  }
  __syncthreads();  // every warp is done with its histogram: it may now hold the list
  if (warp == 0) {
    const uint32_t g = warp_sum(wcnt[lane]), e = warp_sum(wcnt[kWarps + lane]);
    if (lane < CL)
      push_v2(peer_addr(smem_u32(info + 2 * rank), lane), g, e, peer_addr(smem_u32(&bars[2]), lane));
  }
  if (tid < 4) list_key[ksel + tid] = 0u;  // below every key: the rank loads read up to 3 past
  for (int s = tid; s < kMaxShare; s += kTkThreads) rank_acc[s] = 0u;
  tk_wait(&bars[2], 0, abort_flag);
  // the copies of the threshold go to the lowest indices: CTAs, then warps, in order.
  // Lane r < CL stands for CTA r, then lane w for warp w of this CTA.
  uint32_t base, take, wpos, wtake;
  {
    const uint32_t gr = lane < CL ? info[2 * lane] : 0u, er_ = lane < CL ? info[2 * lane + 1] : 0u;
    const uint32_t ebr = warp_inclusive_scan(er_, lane) - er_;
    const uint32_t tkr = kk > ebr ? min(kk - ebr, er_) : 0u;
    const uint32_t pr = warp_inclusive_scan(gr + tkr, lane) - (gr + tkr);
    base = __shfl_sync(0xffffffffu, pr, rank);
    take = __shfl_sync(0xffffffffu, tkr, rank);
    const uint32_t gl = wcnt[lane], el = wcnt[kWarps + lane];
    const uint32_t eb = warp_inclusive_scan(el, lane) - el;
    const uint32_t tkl = take > eb ? min(take - eb, el) : 0u;
    const uint32_t pl = warp_inclusive_scan(gl + tkl, lane) - (gl + tkl);
    wpos = __shfl_sync(0xffffffffu, pl, warp);
    wtake = __shfl_sync(0xffffffffu, tkl, warp);
  }
  // push the selected entries, in index order, to list position P: the key to every CTA,
  // the index to the CTA whose share holds P
  uint32_t P = base + wpos, er = 0;
  const uint32_t key_dst = smem_u32(list_key), idx_dst = smem_u32(list_idx);
  const uint32_t list_bar = smem_u32(&bars[3]);
  auto push_entry = [&](uint32_t pos, uint32_t u, uint32_t index) {
    if (pos >= static_cast<uint32_t>(ksel)) return;  // only with a wait that gave up
#pragma unroll
    for (int r = 0; r < CL; ++r) push_u32(peer_addr(key_dst + 4 * pos, r), u, peer_addr(list_bar, r));
    const uint32_t owner = pos / static_cast<uint32_t>(q);
    push_u32(peer_addr(idx_dst + 4 * (pos - owner * q), owner), index, peer_addr(list_bar, owner));
  };
  if (use_cand) {
    for (int c0 = 0; c0 < ncand; c0 += 32) {
      const int c = c0 + lane;
      const bool in = c < ncand;
      const int i = in ? wcand[c] : 0;
      const uint32_t u = in ? keys[i] : 0u;
      const uint32_t eb = __ballot_sync(0xffffffffu, in && u == thr);
      const bool sel = in && (u > thr || (u == thr && er + __popc(eb & lt) < wtake));
      const uint32_t sb = __ballot_sync(0xffffffffu, sel);
      if (sel) push_entry(P + __popc(sb & lt), u, static_cast<uint32_t>(lo + i));
      P += __popc(sb);
      er += __popc(eb);
    }
  } else {
    for (int g0 = s0; g0 < s1; g0 += 128) {
      uint32_t u[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = g0 + 32 * r + lane;
        u[r] = i < s1 ? keys[i] : 0u;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = g0 + 32 * r + lane;
        const bool in = i < s1;
        if (!__any_sync(0xffffffffu, in && u[r] >= thr)) continue;  // most groups
        const uint32_t eb = __ballot_sync(0xffffffffu, in && u[r] == thr);
        const bool sel = in && (u[r] > thr || (u[r] == thr && er + __popc(eb & lt) < wtake));
        const uint32_t sb = __ballot_sync(0xffffffffu, sel);
        if (sel) push_entry(P + __popc(sb & lt), u[r], static_cast<uint32_t>(lo + i));
        P += __popc(sb);
        er += __popc(eb);
      }
    }
  }
  cluster_arrive_relaxed();  // no CTA leaves before every CTA is done with the others' memory
  tk_wait(&bars[3], 0, abort_flag);
  __syncthreads();
  // rank.  Every list key is >= thr: bin b holds the keys with (key - thr) >> sh == b, sh
  // the smallest shift that puts the largest key in bin 255.  The list is laid out by bin,
  // highest first, and the entry at list position e goes to output place (keys in higher
  // bins) + (keys of its own bin that sort before it: larger, or equal and earlier in the
  // list, which is index order).  8 threads share each entry's bin.
  {
    uint32_t* bcnt = recv + kMaxShare;                                   // [kRankBins]
    uint32_t* above = hist + kListAbove;                                 // [kRankBins]
    uint32_t* bkey = hist + kListBKey;                                   // [kMaxK]
    uint16_t* bpos = reinterpret_cast<uint16_t*>(hist + kListBPos);      // [kMaxK]
    uint32_t mx = 0;
    for (int o = tid; o < ksel; o += kTkThreads) mx = max(mx, list_key[o]);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) wcnt[warp] = mx;
    if (tid < kRankBins) bcnt[tid] = 0u;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kWarps; w += 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(wcnt + w);
      mx = max(max(mx, v.x), max(v.y, max(v.z, v.w)));
    }
    const uint32_t maxd = mx - thr;
    const int sh = maxd >= kRankBins ? 32 - __clz(maxd) - 8 : 0;
    auto bin_of = [&](uint32_t key) { return min(static_cast<uint32_t>(kRankBins - 1), (key - thr) >> sh); };
    for (int o = tid; o < ksel; o += kTkThreads) atomicAdd(&bcnt[bin_of(list_key[o])], 1u);
    __syncthreads();
    if (warp == 0) {  // lane l: bins 255 - 8l down to 248 - 8l; a lane-order scan counts higher bins
      uint4* c4 = reinterpret_cast<uint4*>(bcnt);
      uint4* a4 = reinterpret_cast<uint4*>(above);
      const uint4 lo4 = c4[62 - 2 * lane], hi4 = c4[63 - 2 * lane];
      const uint32_t sum = lo4.x + lo4.y + lo4.z + lo4.w + hi4.x + hi4.y + hi4.z + hi4.w;
      uint32_t at = warp_inclusive_scan(sum, lane) - sum;
      uint4 ahi, alo;
      ahi.w = at; at += hi4.w;
      ahi.z = at; at += hi4.z;
      ahi.y = at; at += hi4.y;
      ahi.x = at; at += hi4.x;
      alo.w = at; at += lo4.w;
      alo.z = at; at += lo4.z;
      alo.y = at; at += lo4.y;
      alo.x = at;
      a4[63 - 2 * lane] = ahi;  // bin starts, and the bins' fill cursors
      a4[62 - 2 * lane] = alo;
      c4[63 - 2 * lane] = ahi;
      c4[62 - 2 * lane] = alo;
    }
    __syncthreads();
    for (int o = tid; o < ksel; o += kTkThreads) {
      const uint32_t key = list_key[o];
      const uint32_t at = atomicAdd(&bcnt[bin_of(key)], 1u);
      if (at < static_cast<uint32_t>(kMaxK)) {
        bkey[at] = key;
        bpos[at] = static_cast<uint16_t>(o);
      }
    }
    __syncthreads();
    const int j = tid & 127, sub = tid >> 7;
    for (int e0 = my0; e0 < my1; e0 += 128) {
      const int e = e0 + j;
      if (e >= my1) continue;
      const uint32_t ke = list_key[e];
      const uint32_t bin = bin_of(ke);
      const uint32_t lo_ = above[bin], hi_ = min(bcnt[bin], static_cast<uint32_t>(kMaxK));
      uint32_t n = sub == 0 ? lo_ : 0u;
      for (uint32_t p = lo_ + sub; p < hi_; p += kRankChunks) {
        const uint32_t km = bkey[p];
        n += km > ke || (km == ke && bpos[p] < e);
      }
      atomicAdd(&rank_acc[e - my0], n);
    }
  }
  __syncthreads();
  if (!*abort_flag) {
    for (int s = tid; s < my1 - my0; s += kTkThreads) {
      const uint32_t place = rank_acc[s];
      if (place >= static_cast<uint32_t>(ksel)) continue;  // only with a wait that gave up
      a.out_idx[t * k + place] = static_cast<int32_t>(list_idx[s]);
      if (a.out_score) a.out_score[t * k + place] = key_value(list_key[my0 + s]);
    }
  }
  for (int e = ksel + static_cast<int>(rank) * kTkThreads + tid; e < k; e += CL * kTkThreads) {
    a.out_idx[t * k + e] = -1;  // fewer candidates than k: padding
    if (a.out_score) a.out_score[t * k + e] = -INFINITY;
  }
  cluster_wait();
}

}  // namespace idx

// ------------------------------------------------------------------ host side
namespace fused {
// 2-D bf16 row-major tensor map with a [box_rows, box_cols] box (fused_proj.cu).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols);
}  // namespace fused

kvc_status launch_indexer_scores(const IndexerProblem& p, cudaStream_t st) {
  using namespace idx;
  const int64_t tiles = (p.max_visible + kKT - 1) / kKT;
  const int64_t units = p.T * tiles;
  if (units == 0) return KVC_OK;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return KVC_ERR_CUDA;
  CUtensorMap mq, mk;
  // K may have no rows when every window is empty; the map still needs one
  const uint64_t krows = static_cast<uint64_t>(p.key_rows > 0 ? p.key_rows : 1);
  if (!fused::make_map(&mq, p.q, static_cast<uint64_t>(p.T * p.H), kD,
                       static_cast<uint32_t>(p.H), 64) ||
      !fused::make_map(&mk, p.K, krows, kD, kKT, 64))
    return KVC_ERR_CUDA;
  ScoreArgs a{p.w, p.key_start, p.n_visible, p.scores, p.T, p.key_rows, p.max_visible, p.ld,
              tiles, units, p.H};
  if (!raise_smem_limit(reinterpret_cast<const void*>(indexer_score_kernel)))
    return KVC_ERR_CUDA;
  const int64_t grid = units < sms ? units : sms;
  indexer_score_kernel<<<static_cast<unsigned>(grid), kThreads, kSmem, st>>>(mq, mk, a);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = "indexer_score_kernel";
  return KVC_OK;
}

int64_t topk_max_candidates() { return static_cast<int64_t>(idx::kCluster) * idx::kSlice; }

kvc_status launch_indexer_topk(const TopkProblem& p, cudaStream_t st) {
  using namespace idx;
  if (p.T == 0) return KVC_OK;
  if (p.k < 1 || p.k > kMaxK || p.max_visible > topk_max_candidates()) return KVC_ERR_UNSUPPORTED;
  TopkArgs a{p.scores, p.n_visible, p.out_idx, p.out_score, p.T, p.max_visible, p.ld, p.k};
  // Clusters of 8 CTAs (16-CTA clusters were measured slower on the decode step).
  auto try_launch = [&](auto kern, int cl, bool non_portable) -> kvc_status {
    if (!raise_smem_limit(reinterpret_cast<const void*>(kern)) ||
        (non_portable &&
         cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
             cudaSuccess)) {
      (void)cudaGetLastError();
      return KVC_ERR_UNSUPPORTED;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cl), 1, 1);
    cfg.blockDim = dim3(kTkThreads, 1, 1);
    cfg.dynamicSmemBytes = kTkSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
      (void)cudaGetLastError();
      return KVC_ERR_UNSUPPORTED;
    }
    cfg.gridDim = dim3(static_cast<unsigned>(p.T * cl), 1, 1);
    // may launch while the kernel ahead of it (the scores) finishes; the kernel waits for
    // that kernel's completion before its first read
    cudaLaunchAttribute attr2[2] = {attr[0], {}};
    attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr2[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr2;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return KVC_ERR_CUDA;
    last_kernel() = "indexer_topk_kernel";
    return KVC_OK;
  };
  return try_launch(indexer_topk_kernel<kCluster>, kCluster, false);
}

unsigned int read_and_clear_indexer_error(bool* failed) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_indexer_error, sizeof(v)) != cudaSuccess) {
    *failed = true;
    return 0;
  }
  if (v != 0 && cudaMemcpyToSymbol(g_indexer_error, &zero, sizeof(zero)) != cudaSuccess)
    *failed = true;
  return v;
}

}  // namespace kvc
