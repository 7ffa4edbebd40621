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
// chip (an eighth each, as order-preserving 32-bit keys), finds the exact k-th largest key
// by a radix select over four 8-bit digits whose per-pass histograms are summed across the
// cluster through distributed shared memory, gathers the selected entries into one CTA in
// index order (ties at the threshold go to the smallest indices) and sorts them there.
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
constexpr size_t kTkSmem =
    kSlice * 4 + (kWarps + 1) * kBins * 4 + kMaxK * 8 + kTkThreads * 4 + 64 + 2 * kWarps * 4 + 128;

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

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_cluster_u64(uint32_t addr, unsigned long long v) {
  asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}
__device__ __forceinline__ uint32_t cluster_addr_of(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Exclusive prefix sum of v over the block's threads in thread order; total in *total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* scratch,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = lane < kTkThreads / 32 ? scratch[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kTkThreads / 32) scratch[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const uint32_t before = (warp > 0 ? scratch[warp - 1] : 0u) + x - v;
  *total = scratch[kTkThreads / 32 - 1];
  __syncthreads();  // scratch is reused by the next scan
  return before;
}

template <int CL>
__global__ void __launch_bounds__(kTkThreads, 1) indexer_topk_kernel(const TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);                      // [kSlice]
  uint32_t* hist = keys + kSlice;                                  // [kWarps][kBins]
  uint32_t* chist = hist + kWarps * kBins;                         // [kBins] the CTA's sum
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(chist + kBins);  // [kMaxK]
  uint32_t* scratch = reinterpret_cast<uint32_t*>(cand + kMaxK);          // [kTkThreads]
  uint32_t* info = scratch + kTkThreads;                                   // [16]
  uint32_t* wcnt = info + 16;                                              // [2][kWarps]
  uint32_t* runs = wcnt + 2 * kWarps;                                      // [2][16]

  const uint32_t rank = blockIdx.x % CL;
  const int64_t t = blockIdx.x / CL;
  const int tid = threadIdx.x;
  const int64_t nv = a.n_visible[t];
  // the same decision in every CTA of the cluster: an out-of-range row is skipped whole
  if (nv < 0 || nv > a.max_visible) {
    if (rank == 0 && tid == 0) atomicOr(&g_indexer_error, 2u);
    return;
  }
  const int k = a.k;
  const int ksel = static_cast<int>(nv < k ? nv : k);
  // this CTA's candidates [lo, lo + cnt), a multiple of 4 apart
  const int64_t per = ((nv + CL - 1) / CL + 3) & ~int64_t(3);
  const int64_t lo = rank * per;
  const int cnt = static_cast<int>(lo < nv ? (nv - lo < per ? nv - lo : per) : 0);
  const float* row = a.scores + t * a.ld;

  if (ksel > 0) {
    // four 16-byte loads in flight per thread
    constexpr int kStep = kTkThreads * 4;
    for (int i0 = tid * 4; i0 < cnt; i0 += 4 * kStep) {
      float4 f[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = i0 + r * kStep;
        if (i + 3 < cnt) f[r] = *reinterpret_cast<const float4*>(row + lo + i);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = i0 + r * kStep;
        if (i + 3 < cnt) {
          keys[i] = order_key(f[r].x);
          keys[i + 1] = order_key(f[r].y);
          keys[i + 2] = order_key(f[r].z);
          keys[i + 3] = order_key(f[r].w);
        } else {
          for (int e = i; e < cnt; ++e) keys[e] = order_key(row[lo + e]);
        }
      }
    }
    // radix select of the ksel-th largest key: four 8-bit digits, high to low.  Each warp
    // counts into its own histogram (the keys of a query share few leading bits, so one
    // shared histogram would serialise all warps on a handful of bins), the CTA sums its
    // warps', and every CTA sums the cluster's CTA histograms through distributed shared
    // memory.
    const int warp = tid >> 5, lane = tid & 31;
    uint32_t* whist = hist + warp * kBins;
    // Warp w owns candidates [w * seg, (w + 1) * seg) in every pass below, its lanes on
    // consecutive keys (no bank conflicts), so its histogram also gives its own counts of
    // keys above and at the final threshold.
    const int seg = ((cnt + kWarps - 1) / kWarps + 31) & ~31;
    const int s0 = warp * seg;
    const int s1 = s0 + seg < cnt ? s0 + seg : cnt;
    uint32_t wgt = 0;  // keys of the segment above the threshold (summed over the passes)
    uint32_t prefix = 0, mask = 0;
    uint32_t kk = static_cast<uint32_t>(ksel);  // rank of the wanted key among the matches
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int b = tid; b < kWarps * kBins; b += kTkThreads) hist[b] = 0u;
      __syncthreads();
      // four loads in flight per thread; lanes of a warp that hit the same bin are
      // serialised by the shared-memory atomics (measured cheaper than aggregating them
      // with __match_any_sync first)
      for (int i0 = s0 + lane; i0 < s1; i0 += 128) {
        uint32_t u[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = i0 + 32 * r;
          u[r] = i < s1 ? keys[i] : 0u;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = i0 + 32 * r;
          if (i < s1 && (u[r] & mask) == prefix)
            atomicAdd(&whist[(u[r] >> shift) & (kBins - 1)], 1u);
        }
      }
      __syncthreads();
      if (tid < kBins) {
        uint32_t sum = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) sum += hist[w * kBins + tid];
        chist[tid] = sum;
      }
      cluster_sync();  // every CTA's histogram is complete
      // thread tid < 256 takes bin 255 - tid over the cluster, so a thread-order scan
      // counts the keys in higher bins
      uint32_t tot = 0;
      if (tid < kBins) {
        uint32_t rv[CL];
#pragma unroll
        for (int r = 0; r < CL; ++r)  // all remote loads in flight before any use
          rv[r] = ld_cluster_u32(cluster_addr_of(chist + (kBins - 1 - tid), static_cast<uint32_t>(r)));
#pragma unroll
        for (int r = 0; r < CL; ++r) tot += rv[r];
      }
      uint32_t all;
      const uint32_t above = block_exclusive_scan(tot, scratch, &all);
      if (tot > 0 && above < kk && kk <= above + tot) {
        info[0] = static_cast<uint32_t>(kBins - 1 - tid);
        info[1] = kk - above;
      }
      __syncthreads();
      const uint32_t digit = info[0];
      {  // this warp's keys above the chosen digit (they all sort above the threshold)
        uint32_t c = 0;
        for (int b = static_cast<int>(digit) + 1 + lane; b < kBins; b += 32) c += whist[b];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        wgt += c;
      }
      if (pass == 3 && lane == 0) {  // the warp's counts above and at the threshold
        wcnt[warp] = wgt;
        wcnt[kWarps + warp] = whist[digit];
      }
      prefix |= digit << shift;
      mask |= static_cast<uint32_t>(kBins - 1) << shift;
      kk = info[1];
      cluster_sync();  // remote reads are done before the next pass rewrites the histograms
    }
    const uint32_t thr = prefix;  // the ksel-th largest key; kk of its copies are taken
    const uint32_t lt = (1u << lane) - 1u;
    __syncthreads();  // every warp's counts are in wcnt
    if (tid == 0) {
      uint32_t g = 0, e = 0;
      for (int w = 0; w < kWarps; ++w) {
        g += wcnt[w];
        e += wcnt[kWarps + w];
      }
      info[2] = g;
      info[3] = e;
    }
    cluster_sync();
    // the copies of the threshold go to the lowest indices: CTAs, then warps, in order
    uint32_t base = 0, take = 0, eq_before = 0, run_base = 0;
    for (uint32_t r = 0; r < CL; ++r) {
      const uint32_t g = ld_cluster_u32(cluster_addr_of(info + 2, r));
      const uint32_t e = ld_cluster_u32(cluster_addr_of(info + 3, r));
      const uint32_t tk = kk > eq_before ? (kk - eq_before < e ? kk - eq_before : e) : 0u;
      if (r < rank) base += g + tk;
      if (r == rank) take = tk;
      if (tid == 0) {  // every CTA's run of selected entries: [base, base + length)
        runs[2 * r] = run_base;
        runs[2 * r + 1] = g + tk;
      }
      run_base += g + tk;
      eq_before += e;
    }
    uint32_t pos = base, wtake = 0, web = 0;
    for (int w = 0; w <= warp; ++w) {
      const uint32_t e = wcnt[kWarps + w];
      const uint32_t tk = take > web ? (take - web < e ? take - web : e) : 0u;
      if (w < warp) pos += wcnt[w] + tk;
      else wtake = tk;
      web += e;
    }
    // write the selected entries in index order into this CTA's run buffer
    pos -= base;
    uint32_t er = 0;  // threshold copies of this warp already passed
    for (int i0 = s0; i0 < s1; i0 += 128) {
      uint32_t u[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = i0 + 32 * r + lane;
        u[r] = i < s1 ? keys[i] : 0u;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = i0 + 32 * r + lane;
        const bool in = i < s1;
        if (!__any_sync(0xffffffffu, in && u[r] >= thr)) continue;  // most groups
        const uint32_t eb = __ballot_sync(0xffffffffu, in && u[r] == thr);
        const bool sel = in && (u[r] > thr || (u[r] == thr && er + __popc(eb & lt) < wtake));
        const uint32_t sb = __ballot_sync(0xffffffffu, sel);
        if (sel) {
          const uint32_t index = static_cast<uint32_t>(lo + i);
          cand[pos + __popc(sb & lt)] =
              (static_cast<unsigned long long>(u[r]) << 32) | (0xFFFFFFFFu - index);
        }
        pos += __popc(sb);
        er += __popc(eb);
      }
    }
  }
  __syncthreads();
  // Each CTA sorts its own run descending (key, then smaller index first): a bitonic
  // network over P = 2^ceil(log2 n) entries in registers, element e = r * 1024 + tid in
  // x[r]; strides up to 16 are lane exchanges, 32..512 go through shared memory, 1024 is
  // between a thread's two registers.  Threads past n hold 0, below every real entry, and
  // only ever pair with each other.
  const int nsel = ksel > 0 ? static_cast<int>(runs[2 * rank + 1]) : 0;
  int P = 1;
  while (P < nsel) P <<= 1;
  const int E = P > kTkThreads ? 2 : 1;
  unsigned long long x[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int e = r * kTkThreads + tid;
    x[r] = (r < E && e < nsel) ? cand[e] : 0ull;
  }
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= kTkThreads) {  // E == 2: the thread's own two registers
        const bool desc = (tid & size) == 0;
        const unsigned long long hi = x[0] > x[1] ? x[0] : x[1], lo2 = x[0] > x[1] ? x[1] : x[0];
        x[0] = desc ? hi : lo2;
        x[1] = desc ? lo2 : hi;
      } else {
        unsigned long long y[2];
        if (stride >= 32) {
#pragma unroll
          for (int r = 0; r < 2; ++r)
            if (r < E) cand[r * kTkThreads + tid] = x[r];
          __syncthreads();
#pragma unroll
          for (int r = 0; r < 2; ++r)
            if (r < E) y[r] = cand[(r * kTkThreads + tid) ^ stride];
          __syncthreads();
        } else {
          // a warp whose entries are all padding (past P) has nothing to exchange
          if (E == 1 && (tid & ~31) >= P) continue;
#pragma unroll
          for (int r = 0; r < 2; ++r) y[r] = __shfl_xor_sync(0xffffffffu, x[r], stride);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (r < E) {
            const int e = r * kTkThreads + tid;
            const bool lower = (e & stride) == 0, desc = (e & size) == 0;
            const unsigned long long hi = x[r] > y[r] ? x[r] : y[r];
            const unsigned long long lo2 = x[r] > y[r] ? y[r] : x[r];
            x[r] = (desc == lower) ? hi : lo2;
          }
        }
      }
    }
  }
  // the sorted runs go to CTA 0, in its key space (free once every CTA is past this sync)
  cluster_sync();
  unsigned long long* merged = reinterpret_cast<unsigned long long*>(keys);  // [ksel], CTA 0
  if (nsel > 0) {
    const uint32_t mbase = cluster_addr_of(merged, 0) + 8u * runs[2 * rank];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int e = r * kTkThreads + tid;
      if (r < E && e < nsel) st_cluster_u64(mbase + 8u * e, x[r]);
    }
  }
  cluster_sync();
  if (rank != 0) return;
  // CTA 0: each entry's place is its position in its run plus, for every other run, the
  // number of entries there that sort before it (binary search; the entries are distinct)
  for (int e = tid; e < ksel; e += kTkThreads) {
    int r0 = 0;
    while (r0 + 1 < CL && static_cast<uint32_t>(e) >= runs[2 * (r0 + 1)]) ++r0;
    const unsigned long long v = merged[e];
    uint32_t place = static_cast<uint32_t>(e) - runs[2 * r0];
    for (int r = 0; r < CL; ++r) {
      if (r == r0) continue;
      const unsigned long long* run = merged + runs[2 * r];
      int lo_ = 0, hi_ = static_cast<int>(runs[2 * r + 1]);
      while (lo_ < hi_) {
        const int mid = (lo_ + hi_) >> 1;
        if (run[mid] > v) lo_ = mid + 1;
        else hi_ = mid;
      }
      place += static_cast<uint32_t>(lo_);
    }
    a.out_idx[t * k + place] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(v));
    if (a.out_score) a.out_score[t * k + place] = key_value(static_cast<uint32_t>(v >> 32));
  }
  for (int e = ksel + tid; e < k; e += kTkThreads) {  // fewer candidates than k: padding
    a.out_idx[t * k + e] = -1;
    if (a.out_score) a.out_score[t * k + e] = -INFINITY;
  }
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
