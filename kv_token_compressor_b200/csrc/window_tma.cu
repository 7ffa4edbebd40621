// Softmax pools fed by TMA from a shared-memory ring (sm_100a): the single-segment window
// kernel for long windows (HCA, m' = 128) below, and the two-stream CSA kernel (m = 4) for
// small problems further down.
//
// What the window kernel computes ("序列压缩注意力", eq. attn-seqcomp-hca; "Ch 05 · HCA" §2): for every
// entry i and channel ch, the softmax over the window's m rows of Z[i*m + v, ch] + B[v, ch]
// and the weighted sum of C[i*m + v, ch], exactly as the register-staged window kernel.
//
// Why a second kernel.  With loads into registers each warp alternates between waiting on
// memory and computing, and only the warps that happen to be waiting keep bytes in flight.
// Here one producer thread streams the windows into a ring of shared-memory stages with
// 4-D tensor-map copies ([channels, row in window, entry, sequence] boxes), and eight
// consumer warps pool from shared memory; the copies of the next stages are in flight
// while the consumers compute, so every SM keeps about 100 KB of reads outstanding.
//
// Work split.  A task is (channel slab of 16 vectors, sequence, group of E = 16 / RG
// entries).  The 16 consumer thread rows are (entry, row group): with RG row groups an
// entry's rows are dealt round-robin to RG threads, whose partial (max, sum, acc) merge in
// shared memory at the end of the window.  A stage holds UR = 4 RG rows of each of the
// group's E entries, so every consumer thread takes four rows per stage whatever RG is,
// bounds its logits once per two stages (an 8-row chunk), and moves its softmax reference
// (rescaling the running sums) only when a chunk's bound exceeds it by more than 16 log2
// units.  Tasks are ordered slab first, so a CTA's contiguous range of tasks re-stages the
// bias rarely.
//
// Measured limits.  At full clock the consumers just keep up with HBM (the producer waits
// for free stages about 3/4 of the time); under the power cap they set the pace, hence the
// lazy reference and a check-free path for full chunks.  A copy
// engine box row of 256 bytes takes ~6.5 ns, so per-SM TMA throughput with these boxes is
// itself near the SM's share of HBM, and boxes much smaller than 8 KB run far slower (an
// entry-list variant with 1 KB boxes reached ~21 GB/s per SM and was not kept).
#include <cuda.h>

#include "kvc_common.cuh"
#include "kvc_host.h"
#include "kvc_launch.h"
#include "stream_common.cuh"
#include "tc_ptx.cuh"

#include <type_traits>

namespace kvc {

// Bit 0: a bounded wait of the TMA-fed window kernel gave up (outputs undefined).
// Bit 1: a prepared-bias workspace did not belong to the call (nothing was computed).
__device__ unsigned int g_window_error = 0;

namespace wtma {

using namespace tcx;

constexpr int kCG = 16;                       // channel vectors per slab (threads along x)
constexpr int kTY = 16;                       // consumer thread rows
constexpr int kConsumers = kCG * kTY;         // 256
constexpr int kThreads = kConsumers + 32;     // + one producer warp
constexpr int kRowsPerThread = 4;             // rows of each consumer thread per stage
constexpr int kStages = 4;
constexpr int kHalf = kTY * kRowsPerThread * 256;  // one stream's stage: 64 rows x 256 B
constexpr int kStageBytes = 2 * kHalf;             // Z then C
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per wait
constexpr int kMinRows = 32;                       // shorter windows use the other kernels
constexpr float kHeadroom = 16.f;                  // log2 units a chunk may exceed the reference

struct Args {
  const float* B;  // [m, c]
  void* out;       // [batch, ne, c]
  int64_t batch, ne, c;
  int m;
  int64_t groups;  // entry groups per sequence
  int64_t tasks;   // slabs * batch * groups
  int bias_mode;   // how a slab's bias rows arrive: kBiasLoads, kBiasMap or kBiasPrepared
  // kBiasPrepared: the workspace of hca_prepare_bias (its header, and the slabs' rows ready
  // for shared memory, prep_stride floats apart)
  const PrepHeader* hdr;
  const float* prep;
  int64_t prep_stride;
};

template <typename InT>
constexpr int slab() {
  return kCG * VecInfo<InT>::kChannels;
}

constexpr int kBiasLoads = 0;     // plain loads (bias not 16-byte aligned, or too many rows)
constexpr int kBiasMap = 1;       // one 2-D tensor copy of the slab's rows, then scaled here
constexpr int kBiasPrepared = 2;  // one bulk copy of the rows hca_prepare_bias made ready

// Dynamic shared memory: stages, bias rows, per-channel bias maxima, spread partials,
// row-group partials (RG > 1), barriers (stage full / empty, bias full / free) and the
// abort flag; 1 KB slack for alignment.
template <typename InT>
size_t smem_bytes(int m, int rg) {
  constexpr int SC = slab<InT>();
  size_t f = static_cast<size_t>(m) * SC + SC + 2 * kConsumers;
  if (rg > 1) f += 3 * static_cast<size_t>(kTY) * SC;
  return 1024 + static_cast<size_t>(kStages) * kStageBytes + f * sizeof(float) +
         (2 * kStages + 2) * sizeof(uint64_t) + 16;
}

__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                       bool honour_abort) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(&g_window_error, 1u);
      return false;
    }
  }
}
// Bounded wait: true once the phase of `parity` has completed; false after the limit (which
// raises the CTA's abort flag and the error bit) or, when honoured, once another thread of
// the CTA has raised the abort flag.
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                     bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, honour_abort);
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// One contiguous global -> shared copy of `bytes` (16-byte aligned addresses, a multiple of
// 16 bytes), counted on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// (slab, sequence, entry group) of task t, stepped one task at a time (the divisions once
// per CTA, not on every task boundary).
struct Task {
  int64_t x, b, g;
  int64_t batch, groups;
  __device__ Task(int64_t batch_, int64_t groups_, int64_t t) : batch(batch_), groups(groups_) {
    const int64_t per_slab = batch * groups;
    x = t / per_slab;
    const int64_t r = t - x * per_slab;
    b = r / groups;
    g = r - b * groups;
  }
  __device__ __forceinline__ void next() {
    if (++g == groups) {
      g = 0;
      if (++b == batch) {
        b = 0;
        ++x;
      }
    }
  }
};

// Order-preserving map of fp32 to uint32 (larger float, larger key) and its inverse, for
// shared-memory atomic max / min.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <typename InT, typename OutT, int RG>
__global__ void __launch_bounds__(kThreads, 1)
    window_tma_kernel(const __grid_constant__ CUtensorMap mapZ,
                      const __grid_constant__ CUtensorMap mapC,
                      const __grid_constant__ CUtensorMap mapB, const Args a) {
  constexpr int CPT = VecInfo<InT>::kChannels;
  constexpr int SC = slab<InT>();
  constexpr int E = kTY / RG;                 // entries per task
  constexpr int UR = kRowsPerThread * RG;     // rows of each entry per stage
  constexpr int NP = CPT / 2;                 // channel pairs per thread
  static_assert(E * UR * SC * sizeof(InT) == kHalf, "stage geometry");
  const float2 kL2e2 = make_float2(kLog2e, kLog2e);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = base;
  float* sb = reinterpret_cast<float*>(base + kStages * kStageBytes);  // [m][SC] bias * log2 e
  float* bmx = sb + static_cast<size_t>(a.m) * SC;                      // [SC] largest bias
  float* red = bmx + SC;                                                 // [2][256] max / min
  float* pm = red + 2 * kConsumers;                                      // RG > 1: [16][SC]
  float* ps = pm + (RG > 1 ? kTY * SC : 0);
  float* pa = ps + (RG > 1 ? kTY * SC : 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(pa + (RG > 1 ? kTY * SC : 0));
  uint64_t* empty = full + kStages;
  uint64_t* bias_full = empty + kStages;
  uint64_t* bias_free = bias_full + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bias_free + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  uint32_t* kmax = reinterpret_cast<uint32_t*>(red);  // [SC] bias maxima as order keys
  uint32_t* kmin = kmax + SC;                          // [SC] minima
  if (tid < SC && a.bias_mode != kBiasPrepared) {  // (prepared: copies land on these words)
    kmax[tid] = 0u;
    kmin[tid] = 0xFFFFFFFFu;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers / 32);
    }
    mbar_init(bias_full, 1);
    mbar_init(bias_free, kConsumers / 32);
    *abort_flag = 0;
    if (a.bias_mode == kBiasPrepared) {
      // the workspace must have been prepared for this bias shape and stream type
      const PrepHeader h = *a.hdr;
      if (h.magic != kPrepMagic || h.m != a.m || h.c != a.c ||
          h.in_bf16 != (sizeof(InT) == 2 ? 1 : 0) || h.slab_floats != a.prep_stride) {
        *abort_flag = 1;
        atomicOr(&g_window_error, 2u);
      }
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (a.bias_mode == kBiasPrepared && *abort_flag) return;  // nothing issued yet

  const int64_t lo = static_cast<int64_t>(blockIdx.x) * a.tasks / gridDim.x;
  const int64_t hi = static_cast<int64_t>(blockIdx.x + 1) * a.tasks / gridDim.x;
  const int nst = (a.m + UR - 1) / UR;  // stages per window

  if (warp == kConsumers / 32) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t used = 0, last_par = 0;  // stages ever filled; parity of their last fill
      uint32_t nbias = 0;               // bias loads issued
      int64_t px = -1;
      bool ok = true;
      Task k(a.batch, a.groups, lo);
      for (int64_t t = lo; t < hi && ok; ++t, k.next()) {
        if (a.bias_mode != kBiasLoads && k.x != px) {
          // the slab's bias rows, once the consumers are done with the previous slab's
          if (nbias > 0 && !wait(bias_free, (nbias - 1) & 1u, abort_flag)) break;
          if (a.bias_mode == kBiasMap) {
            mbar_arrive_expect_tx(bias_full, static_cast<uint32_t>(a.m) * SC * 4);
            tma_load_2d(smem_u32(sb), &mapB, bias_full, static_cast<int>(k.x * SC), 0);
          } else {  // rows, maxima and spread flag, ready as they are
            const uint32_t bytes = static_cast<uint32_t>(a.prep_stride) * 4;
            mbar_arrive_expect_tx(bias_full, bytes);
            bulk_load(smem_u32(sb), a.prep + k.x * a.prep_stride, bytes, bias_full);
          }
          ++nbias;
          px = k.x;
        }
        for (int st = 0; st < nst; ++st) {
          if (!wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          const uint32_t dst = smem_u32(stages + s * kStageBytes);
          const int x = static_cast<int>(k.x * SC), y = st * UR;
          const int z = static_cast<int>(k.g * E), w = static_cast<int>(k.b);
          tma_load_4d(dst, &mapZ, &full[s], x, y, z, w);
          tma_load_4d(dst + kHalf, &mapC, &full[s], x, y, z, w);
          used |= 1u << s;
          last_par = (last_par & ~(1u << s)) | (ph << s);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // Every copy issued above lands before this thread exits, whatever the consumers did.
      for (int q = 0; q < kStages; ++q)
        if (used & (1u << q)) wait(&full[q], (last_par >> q) & 1u, abort_flag, false);
      if (nbias > 0) wait(bias_full, (nbias - 1) & 1u, abort_flag, false);
    }
    return;
  }

  // -------------------------------------------------------------- consumers (warps 0..7)
  const int tx = tid % kCG, ty = tid / kCG;
  const int e = ty / RG, rg = ty - (ty / RG) * RG;
  const int sc0 = tx * CPT;  // this thread's CPT channels of the slab
  int s = 0;
  uint32_t ph = 0;
  bool dead = false;
  bool fast = false;
  int64_t cur_x = -1;
  uint32_t nb = 0;  // bias loads consumed
  OutT* out = static_cast<OutT*>(a.out);

  Task k(a.batch, a.groups, lo);
  for (int64_t t = lo; t < hi; ++t, k.next()) {
    if (k.x != cur_x) {  // the same in every consumer thread
      bool narrow = true;
      if (a.bias_mode == kBiasPrepared) {
        if (cur_x >= 0) {  // this warp is done with the old slab's bias
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive(bias_free);
        }
        if (!dead && !wait(bias_full, nb & 1u, abort_flag)) dead = true;
        ++nb;
        narrow = red[0] != 0.f;  // the slab's spread flag follows its maxima
      } else if (a.bias_mode == kBiasMap) {
        if (cur_x >= 0) {  // this warp is done with the old slab's bias
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) mbar_arrive(bias_free);
        }
        if (!dead && !wait(bias_full, nb & 1u, abort_flag)) dead = true;
        ++nb;
        // The rows arrive in natural channel order.  Scale them by log2 e and move each
        // float4 to its slot in the consumers' order (whole float4s move: channels 4w..4w+3
        // go to slab_bias_pos(4w)); the SC / 4 float4s of a row are one warp's, or half of
        // one for fp32 (whose order is the identity), so reading the whole row before
        // writing it makes the move safe in place.  This thread always holds float4 w of
        // a row (256 is a multiple of SC / 4): it folds its rows' maxima and minima
        // channel by channel and publishes them with one atomic per channel.
        static_assert(SC / 4 == 32 || SC / 4 == 16, "a row is one warp's (or half)");
        float4* s4 = reinterpret_cast<float4*>(sb);
        float4 mx4 = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        float4 mn4 = make_float4(INFINITY, INFINITY, INFINITY, INFINITY);
        const int w = tid % (SC / 4);
        const int slot = slab_bias_pos<CPT, kCG>(4 * w) / 4;
        for (int f = tid - w; f < a.m * (SC / 4); f += kConsumers) {  // f: the row's start
          float4 v = s4[f + w];
          v.x *= kLog2e;
          v.y *= kLog2e;
          v.z *= kLog2e;
          v.w *= kLog2e;
          if constexpr (CPT == 8) __syncwarp();  // the warp's lanes run this loop alike
          s4[f + slot] = v;
          mx4 = make_float4(fmaxf(mx4.x, v.x), fmaxf(mx4.y, v.y), fmaxf(mx4.z, v.z), fmaxf(mx4.w, v.w));
          mn4 = make_float4(fminf(mn4.x, v.x), fminf(mn4.y, v.y), fminf(mn4.z, v.z), fminf(mn4.w, v.w));
        }
        const int w4 = slot * 4;  // position of this thread's four channels in a staged row
        atomicMax(&kmax[w4], order_key(mx4.x));
        atomicMax(&kmax[w4 + 1], order_key(mx4.y));
        atomicMax(&kmax[w4 + 2], order_key(mx4.z));
        atomicMax(&kmax[w4 + 3], order_key(mx4.w));
        atomicMin(&kmin[w4], order_key(mn4.x));
        atomicMin(&kmin[w4 + 1], order_key(mn4.y));
        atomicMin(&kmin[w4 + 2], order_key(mn4.z));
        atomicMin(&kmin[w4 + 3], order_key(mn4.w));
        bar_named(1, kConsumers);
        if (tid < SC) {  // tid is a position in a staged row here
          const float mx = key_float(kmax[tid]), mn = key_float(kmin[tid]);
          kmax[tid] = 0u;  // ready for the next slab (ordered by the barrier below)
          kmin[tid] = 0xFFFFFFFFu;
          bmx[tid] = mx;
          narrow = mx - mn <= kMaxBiasSpread;  // false for infinite or NaN spreads
        }
      } else {
        if (cur_x >= 0) bar_named(1, kConsumers);  // nobody still reads the old slab's bias
        const float2 mm = stage_bias(sb, a.B, a.B, a.m, a.m, SC, k.x * SC, a.c, tid, kConsumers,
                                     [](int sc) { return slab_bias_pos<CPT, kCG>(sc); });
        red[tid] = mm.x;
        red[kConsumers + tid] = mm.y;
        bar_named(1, kConsumers);
        if (tid < SC) {
          float mx = -INFINITY, mn = INFINITY;
          for (int j = tid; j < kConsumers; j += SC) {
            mx = fmaxf(mx, red[j]);
            mn = fminf(mn, red[kConsumers + j]);
          }
          bmx[slab_bias_pos<CPT, kCG>(tid)] = mx;
          narrow = mx - mn <= kMaxBiasSpread;
        }
      }
      // fast chunk maximum only when every channel's spread is small; also publishes bmx
      fast = bar_and(1, kConsumers, narrow);
      cur_x = k.x;
    }
    const int64_t i = k.g * E + e;  // entry within its sequence
    const int64_t ch0 = k.x * SC + sc0;
    const bool live = i < a.ne && ch0 < a.c;

    float2 M[NP], S[NP], A[NP];  // per channel pair: running max, sum, weighted sum
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      M[p] = make_float2(-INFINITY, -INFINITY);
      S[p] = make_float2(0.f, 0.f);
      A[p] = make_float2(0.f, 0.f);
    }
    for (int st = 0; st < nst; st += 2) {
      const bool two = st + 1 < nst;
      uint4 z[2 * kRowsPerThread], cv[2 * kRowsPerThread];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h == 1 && !two) break;
        if (!dead && !wait(&full[s], ph, abort_flag)) dead = true;
        const uint8_t* sz = stages + s * kStageBytes;
#pragma unroll
        for (int q = 0; q < kRowsPerThread; ++q) {
          const int r = rg + RG * q;  // row within the stage
          const int off = ((e * UR + r) * SC + sc0) * static_cast<int>(sizeof(InT));
          z[h * kRowsPerThread + q] = *reinterpret_cast<const uint4*>(sz + off);
          cv[h * kRowsPerThread + q] = *reinterpret_cast<const uint4*>(sz + kHalf + off);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      // rows of this thread in the two stages: st*UR + rg + RG*q, (st+1)*UR + rg + RG*q
      const int v0 = st * UR + rg;
      if (dead || !live || v0 >= a.m) continue;  // v0 is the smallest row of the chunk
      auto row_of = [&](int u) {
        return v0 + (u / kRowsPerThread) * UR + RG * (u % kRowsPerThread);
      };
      // FULL: every row of the chunk exists (the common case), so no row needs a check; the
      // checks cost about 7% of the consumers' instructions, which set this kernel's pace
      // under the power cap (1000-step runs: 0.351 -> 0.336 ms at n = 2^20)
      auto chunk = [&](auto full_tag) {
        constexpr bool FULL = decltype(full_tag)::value;
        auto valid = [&](int u) {
          return FULL || ((u < kRowsPerThread || two) && row_of(u) < a.m);
        };

        // pass 1: an upper bound of the chunk's largest logit per channel (see the register-
        // staged window kernel: max z * log2 e + max b when the bias spread is small, else the
        // exact per-row maximum)
        float2 cm[NP];
        if (fast) {
          uint4 zm = z[0];
#pragma unroll
          for (int u = 1; u < 2 * kRowsPerThread; ++u)
            if (valid(u)) zm = vec_max<InT>(zm, z[u]);
          const float4* bx = reinterpret_cast<const float4*>(bmx) + tx;
#pragma unroll
          for (int q = 0; q < NP / 2; ++q) {
            const float4 bq = bx[q * kCG];
            cm[2 * q] = f2_fma(vec_pair<InT>(zm, 2 * q), kL2e2, make_float2(bq.x, bq.y));
            cm[2 * q + 1] = f2_fma(vec_pair<InT>(zm, 2 * q + 1), kL2e2, make_float2(bq.z, bq.w));
          }
        } else {
#pragma unroll
          for (int p = 0; p < NP; ++p) cm[p] = make_float2(-INFINITY, -INFINITY);
#pragma unroll
          for (int u = 0; u < 2 * kRowsPerThread; ++u) {
            if (valid(u)) {
              const float4* bp = reinterpret_cast<const float4*>(sb + row_of(u) * SC) + tx;
#pragma unroll
              for (int q = 0; q < NP / 2; ++q) {
                const float4 bq = bp[q * kCG];
                cm[2 * q] = f2_max(cm[2 * q], f2_fma(vec_pair<InT>(z[u], 2 * q), kL2e2,
                                                     make_float2(bq.x, bq.y)));
                cm[2 * q + 1] = f2_max(cm[2 * q + 1], f2_fma(vec_pair<InT>(z[u], 2 * q + 1), kL2e2,
                                                             make_float2(bq.z, bq.w)));
              }
            }
          }
        }
        // M is the reference subtracted from the logits.  It moves (and the running sums
        // are rescaled) only when a chunk's bound exceeds it by more than kHeadroom log2
        // units: the weights then stay <= 2^kHeadroom, far from overflow, and a window's
        // largest weight stays a normal number (the reference never exceeds the window's
        // largest logit by more than the bias spread).  The first chunk always sets it
        // (M = -inf), and most later chunks skip the rescale.
        bool move = false;
#pragma unroll
        for (int p = 0; p < NP; ++p)
          move |= cm[p].x > M[p].x + kHeadroom || cm[p].y > M[p].y + kHeadroom;
        if (move) {
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            const float2 nm = f2_max(M[p], cm[p]);  // finite: row v0 is valid
            const float2 sc = make_float2(ex2_ftz(M[p].x - nm.x), ex2_ftz(M[p].y - nm.y));
            S[p] = f2_mul(S[p], sc);
            A[p] = f2_mul(A[p], sc);
            M[p] = nm;
          }
        }
        // pass 2: one exp2 per element
#pragma unroll
        for (int u = 0; u < 2 * kRowsPerThread; ++u) {
          if (valid(u)) {
            const float4* bp = reinterpret_cast<const float4*>(sb + row_of(u) * SC) + tx;
#pragma unroll
            for (int q = 0; q < NP / 2; ++q) {
              const float4 bq = bp[q * kCG];
              const float2 b2[2] = {make_float2(bq.x, bq.y), make_float2(bq.z, bq.w)};
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int pp = 2 * q + h;
                const float2 l = f2_fma(vec_pair<InT>(z[u], pp), kL2e2, f2_sub(b2[h], M[pp]));
                const float2 w = f2_ex2(l);
                S[pp] = f2_add(S[pp], w);
                A[pp] = f2_fma(w, vec_pair<InT>(cv[u], pp), A[pp]);
              }
            }
          }
        }
      };
      if (two && row_of(2 * kRowsPerThread - 1) < a.m) chunk(std::true_type{});
      else chunk(std::false_type{});
    }

    if constexpr (RG == 1) {
      if (live && !dead) {
        float res[CPT];
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          res[2 * p] = __fdividef(A[p].x, S[p].x);
          res[2 * p + 1] = __fdividef(A[p].y, S[p].y);
        }
        store_out<OutT, CPT>(out + (k.b * a.ne + i) * a.c + ch0, res);
      }
    } else {
      // row-group partials -> shared memory; one thread per (entry, channel vector) merges
#pragma unroll
      for (int q = 0; q < NP / 2; ++q) {
        reinterpret_cast<float4*>(pm + ty * SC + sc0)[q] =
            make_float4(M[2 * q].x, M[2 * q].y, M[2 * q + 1].x, M[2 * q + 1].y);
        reinterpret_cast<float4*>(ps + ty * SC + sc0)[q] =
            make_float4(S[2 * q].x, S[2 * q].y, S[2 * q + 1].x, S[2 * q + 1].y);
        reinterpret_cast<float4*>(pa + ty * SC + sc0)[q] =
            make_float4(A[2 * q].x, A[2 * q].y, A[2 * q + 1].x, A[2 * q + 1].y);
      }
      bar_named(2, kConsumers);
      // one (entry, channel) per thread and item: conflict-free, every consumer busy
      for (int item = tid; item < E * SC; item += kConsumers) {
        const int e2 = item / SC, sc = item - (item / SC) * SC;
        const int64_t i2 = k.g * E + e2;
        const int64_t c2 = k.x * SC + sc;
        if (i2 < a.ne && c2 < a.c && !dead) {
          float gm = -INFINITY;
#pragma unroll 4
          for (int r = 0; r < RG; ++r) gm = fmaxf(gm, pm[(e2 * RG + r) * SC + sc]);
          float sum = 0.f, acc = 0.f;
#pragma unroll 4
          for (int r = 0; r < RG; ++r) {
            const int o = (e2 * RG + r) * SC + sc;
            const float f = ex2_ftz(pm[o] - gm);  // 0 for row groups without rows
            sum = fmaf(ps[o], f, sum);
            acc = fmaf(pa[o], f, acc);
          }
          store_scalar<OutT>(out + (k.b * a.ne + i2) * a.c + c2, __fdividef(acc, sum));
        }
      }
      bar_named(2, kConsumers);
    }
  }
}

// 4-D tensor map of a [batch, n, c] stream viewed as [batch][ne][m][c] (entries of m rows;
// the n mod m tail rows are never addressed), box [1][E][UR][SC], no swizzle, zero fill.
bool make_stream_map(CUtensorMap* map, const void* base, bool bf16, int64_t batch, int64_t n,
                     int64_t ne, int64_t c, int m, int SC, int UR, int E) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const uint64_t es = bf16 ? 2 : 4;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(c), static_cast<cuuint64_t>(m),
                              static_cast<cuuint64_t>(ne), static_cast<cuuint64_t>(batch)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(c) * es,
                                 static_cast<cuuint64_t>(m) * c * es,
                                 static_cast<cuuint64_t>(n) * c * es};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(SC), static_cast<cuuint32_t>(UR),
                             static_cast<cuuint32_t>(E), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D tensor map of the fp32 bias [m, c] with a [m][SC] box (a slab's rows, natural order).
bool make_bias_map(CUtensorMap* map, const float* B, int64_t c, int m, int SC) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc || (reinterpret_cast<uintptr_t>(B) & 15u)) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(c), static_cast<cuuint64_t>(m)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(c) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(SC), static_cast<cuuint32_t>(m)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(B), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename InT, typename OutT, int RG>
kvc_status launch_rg(const StreamProblem& p, cudaStream_t st, const DeviceInfo& di) {
  constexpr int SC = slab<InT>();
  constexpr int E = kTY / RG;
  constexpr int UR = kRowsPerThread * RG;
  const size_t smem = smem_bytes<InT>(p.m, RG);
  if (smem > di.smem_optin) return KVC_ERR_UNSUPPORTED;
  CUtensorMap mz, mc;
  const bool bf = sizeof(InT) == 2;
  if (!make_stream_map(&mz, p.Z0, bf, p.batch, p.n, p.ne, p.c, p.m, SC, UR, E) ||
      !make_stream_map(&mc, p.C0, bf, p.batch, p.n, p.ne, p.c, p.m, SC, UR, E))
    return KVC_ERR_UNSUPPORTED;
  CUtensorMap mb;
  const bool prepared = p.prep_ws != nullptr;
  const bool bias_tma = !prepared && p.m <= 256 && make_bias_map(&mb, p.B0, p.c, p.m, SC);
  if (!bias_tma) mb = mz;  // unused
  auto kern = window_tma_kernel<InT, OutT, RG>;
  if (resident_blocks(kern, kThreads, smem) < 1) return KVC_ERR_UNSUPPORTED;
  Args a{p.B0, p.out, p.batch, p.ne, p.c, p.m, ceil_div(p.ne, E), 0,
         prepared ? kBiasPrepared : bias_tma ? kBiasMap : kBiasLoads, nullptr, nullptr, 0};
  if (prepared) {
    const PrepLayout l = prep_layout(p.c, p.m, bf);
    static_assert(SC == 128 || SC == 64, "prepared slab widths");
    if (l.sc != SC) return KVC_ERR_UNSUPPORTED;
    a.hdr = static_cast<const PrepHeader*>(p.prep_ws);
    a.prep = reinterpret_cast<const float*>(static_cast<const uint8_t*>(p.prep_ws) + l.prep_off);
    a.prep_stride = l.slab_floats;
  }
  a.tasks = ceil_div(p.c, SC) * p.batch * a.groups;
  const int64_t grid = a.tasks < di.sms ? a.tasks : di.sms;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(mz, mc, mb, a);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = prepared ? "window_tma_kernel/prepared" : "window_tma_kernel";
  return KVC_OK;
}

// Share of the SMs' task rounds that do work when `tasks` tasks are split into contiguous
// ranges over `sms` CTAs.
double balance(int64_t tasks, int sms) {
  const int64_t rounds = ceil_div(tasks, sms);
  return static_cast<double>(tasks) / (static_cast<double>(rounds) * sms);
}

template <typename InT, typename OutT>
kvc_status launch_typed(const StreamProblem& p, cudaStream_t st) {
  constexpr int SC = slab<InT>();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (di.sms == 0) return KVC_ERR_CUDA;
  // The fewest row groups whose task count keeps the SMs at least 90% busy (else the
  // best balance); one row group needs no merge.
  const int64_t per_group = ceil_div(p.c, SC) * p.batch;
  int best = 16;
  double best_bal = -1.0;
  for (int rg = 1; rg <= 16; rg *= 2) {
    const double bal = balance(per_group * ceil_div(p.ne, kTY / rg), di.sms);
    if (bal >= 0.9) {
      best = rg;
      break;
    }
    if (bal > best_bal + 1e-9) {
      best_bal = bal;
      best = rg;
    }
  }
  switch (best) {
    case 1: return launch_rg<InT, OutT, 1>(p, st, di);
    case 2: return launch_rg<InT, OutT, 2>(p, st, di);
    case 4: return launch_rg<InT, OutT, 4>(p, st, di);
    case 8: return launch_rg<InT, OutT, 8>(p, st, di);
    default: return launch_rg<InT, OutT, 16>(p, st, di);
  }
}


// ---------------------------------------------------------------------------------
// CSA, m = 4, two overlapping streams ("序列压缩注意力", eqs. attn-seqcomp-csa-softmax,
// attn-seqcomp-csa-pool, attn-seqcomp-overlap-bound; "Ch 04 · CSA" §3): entry i pools the
// a-block, rows [4i, 4i + 4) of Z^a / C^a, and the b-block, rows [4i - 4, 4i) of Z^b / C^b,
// under one softmax over the 8 rows; entry 0 has no b-block (logit -inf, vector 0).
//
// A stage holds kCsaE entries: the [1][8][4][SC] boxes of Z^a and C^a at entry coordinate
// g * 8 and of Z^b and C^b at g * 8 - 1 (the b-block of entry i is the a-row block of
// entry i - 1 in the b streams; for the first group the coordinate is -1 and the copy
// fills zeros, which entry 0 never reads).  Consumer thread rows pair up: ty = 2 e + h
// takes entry e's a-block (h = 0) or b-block (h = 1), lanes l and l ^ 16 of one warp, and
// the pair combines its maxima, sums and weighted sums with two shuffles per value.
// Each window is short, so a warp's work per stage is one serial chain (loads, logits,
// maximum, shuffle, exp2, sums, shuffle, divide); two independent groups of eight consumer
// warps take alternate stages (each with its own copy of the bias) so that the SM always
// has another chain to issue from.
// ---------------------------------------------------------------------------------
constexpr int kCsaE = 8;                                // entries per stage
constexpr int kCsaStages = 6;                           // 6 x 32 KB, even: groups alternate
constexpr int kCsaBox = kCsaE * 4 * 256;                // one stream's box: 8 KB
constexpr int kCsaStageBytes = 4 * kCsaBox;             // Za, Ca, Zb, Cb
constexpr int kCsaGroups = 2;
constexpr int kCsaConsumers = kCsaGroups * kConsumers;  // 512
constexpr int kCsaThreads = kCsaConsumers + 32;         // + one producer warp

struct CsaArgs {
  const float* Ba;  // [4, c]
  const float* Bb;  // [4, c]
  void* out;        // [batch, ne, c]
  int64_t batch, ne, c;
  int64_t groups;   // entry groups of kCsaE per sequence
  int64_t tasks;    // slabs * batch * groups
};

template <typename InT>
size_t csa_smem_bytes() {
  constexpr int SC = slab<InT>();
  return 1024 + static_cast<size_t>(kCsaStages) * kCsaStageBytes +
         kCsaGroups * 8 * SC * sizeof(float) + 2 * kCsaStages * sizeof(uint64_t) + 16;
}

template <typename InT, typename OutT>
__global__ void __launch_bounds__(kCsaThreads, 1)
    csa_tma_kernel(const __grid_constant__ CUtensorMap mapZa,
                   const __grid_constant__ CUtensorMap mapCa,
                   const __grid_constant__ CUtensorMap mapZb,
                   const __grid_constant__ CUtensorMap mapCb, const CsaArgs a) {
  constexpr int CPT = VecInfo<InT>::kChannels;
  constexpr int SC = slab<InT>();
  constexpr int NP = CPT / 2;
  static_assert(kCsaE * 4 * SC * sizeof(InT) == kCsaBox, "box geometry");
  const float2 kL2e2 = make_float2(kLog2e, kLog2e);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = base;
  float* sb_all = reinterpret_cast<float*>(base + kCsaStages * kCsaStageBytes);  // [2][8][SC]
  uint64_t* full = reinterpret_cast<uint64_t*>(sb_all + kCsaGroups * 8 * SC);
  uint64_t* empty = full + kCsaStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kCsaStages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kCsaStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers / 32);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  const int64_t lo = static_cast<int64_t>(blockIdx.x) * a.tasks / gridDim.x;
  const int64_t hi = static_cast<int64_t>(blockIdx.x + 1) * a.tasks / gridDim.x;

  if (warp == kCsaConsumers / 32) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, used = 0, last_par = 0;
      Task k(a.batch, a.groups, lo);
      for (int64_t t = lo; t < hi; ++t, k.next()) {
        if (!wait(&empty[s], ph ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], kCsaStageBytes);
        const uint32_t dst = smem_u32(stages + s * kCsaStageBytes);
        const int x = static_cast<int>(k.x * SC), z = static_cast<int>(k.g * kCsaE);
        const int w = static_cast<int>(k.b);
        tma_load_4d(dst, &mapZa, &full[s], x, 0, z, w);
        tma_load_4d(dst + kCsaBox, &mapCa, &full[s], x, 0, z, w);
        tma_load_4d(dst + 2 * kCsaBox, &mapZb, &full[s], x, 0, z - 1, w);
        tma_load_4d(dst + 3 * kCsaBox, &mapCb, &full[s], x, 0, z - 1, w);
        used |= 1u << s;
        last_par = (last_par & ~(1u << s)) | (ph << s);
        if (++s == kCsaStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      for (int q = 0; q < kCsaStages; ++q)
        if (used & (1u << q)) wait(&full[q], (last_par >> q) & 1u, abort_flag, false);
    }
    return;
  }

  // ------------------------------------------------- consumers (warps 0..15, two groups)
  const int grp = tid / kConsumers;  // takes the group's alternate tasks and stages
  const int ct = tid - grp * kConsumers;
  const int tx = ct % kCG, ty = ct / kCG;
  const int e = ty >> 1, h = ty & 1;  // entry within the stage; a-block (0) or b-block (1)
  const int sc0 = tx * CPT;
  float* sb = sb_all + grp * 8 * SC;  // this group's bias rows
  int s = grp;
  uint32_t ph = 0;
  bool dead = false;
  int64_t cur_x = -1;
  OutT* out = static_cast<OutT*>(a.out);

  Task k(a.batch, a.groups, lo);
  if (grp == 1) k.next();
  for (int64_t t = lo + grp; t < hi; t += kCsaGroups, k.next(), k.next()) {
    if (k.x != cur_x) {  // the same in every thread of the group
      if (cur_x >= 0) bar_named(1 + grp, kConsumers);  // nobody still reads the old bias
      stage_bias(sb, a.Ba, a.Bb, 4, 8, SC, k.x * SC, a.c, ct, kConsumers,
                 [](int sc) { return slab_bias_pos<CPT, kCG>(sc); });
      bar_named(1 + grp, kConsumers);
      cur_x = k.x;
    }
    const int64_t i = k.g * kCsaE + e;
    const int64_t ch0 = k.x * SC + sc0;
    const bool live = i < a.ne && ch0 < a.c;
    const bool none = h == 1 && i == 0;  // entry 0 has no b-block

    uint4 z[4], cv[4];
    if (!dead && !wait(&full[s], ph, abort_flag)) dead = true;
    {
      const uint8_t* sz = stages + s * kCsaStageBytes + h * 2 * kCsaBox;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int off = ((e * 4 + r) * SC + sc0) * static_cast<int>(sizeof(InT));
        z[r] = *reinterpret_cast<const uint4*>(sz + off);
        cv[r] = *reinterpret_cast<const uint4*>(sz + kCsaBox + off);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    s += kCsaGroups;
    if (s >= kCsaStages) {
      s -= kCsaStages;
      ph ^= 1u;
    }

    // logits of this thread's four rows (bias rows h*4 .. h*4+3), their maximum, then the
    // pair's maximum
    float2 l[4][NP], mx[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) mx[p] = make_float2(-INFINITY, -INFINITY);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4* bp = reinterpret_cast<const float4*>(sb + (h * 4 + r) * SC) + tx;
#pragma unroll
      for (int q = 0; q < NP / 2; ++q) {
        const float4 bq = bp[q * kCG];
        l[r][2 * q] = f2_fma(vec_pair<InT>(z[r], 2 * q), kL2e2, make_float2(bq.x, bq.y));
        l[r][2 * q + 1] = f2_fma(vec_pair<InT>(z[r], 2 * q + 1), kL2e2, make_float2(bq.z, bq.w));
        mx[2 * q] = f2_max(mx[2 * q], l[r][2 * q]);
        mx[2 * q + 1] = f2_max(mx[2 * q + 1], l[r][2 * q + 1]);
      }
    }
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      if (none) mx[p] = make_float2(-INFINITY, -INFINITY);
      mx[p].x = fmaxf(mx[p].x, __shfl_xor_sync(0xffffffffu, mx[p].x, 16));
      mx[p].y = fmaxf(mx[p].y, __shfl_xor_sync(0xffffffffu, mx[p].y, 16));
    }
    float res[CPT];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const float2 negm = make_float2(-mx[p].x, -mx[p].y);
      float2 sum = make_float2(0.f, 0.f), acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2 w = f2_ex2(f2_add(l[r][p], negm));
        sum = f2_add(sum, w);
        acc = f2_fma(w, vec_pair<InT>(cv[r], p), acc);
      }
      if (none) {
        sum = make_float2(0.f, 0.f);
        acc = make_float2(0.f, 0.f);
      }
      sum.x += __shfl_xor_sync(0xffffffffu, sum.x, 16);
      sum.y += __shfl_xor_sync(0xffffffffu, sum.y, 16);
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, 16);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, 16);
      res[2 * p] = __fdividef(acc.x, sum.x);
      res[2 * p + 1] = __fdividef(acc.y, sum.y);
    }
    if (h == 0 && live && !dead) store_out<OutT, CPT>(out + (k.b * a.ne + i) * a.c + ch0, res);
  }
}

template <typename InT, typename OutT>
kvc_status launch_csa_typed(const StreamProblem& p, cudaStream_t st) {
  constexpr int SC = slab<InT>();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (di.sms == 0) return KVC_ERR_CUDA;
  CsaArgs a{p.B0, p.B1, p.out, p.batch, p.ne, p.c, ceil_div(p.ne, kCsaE), 0};
  a.tasks = ceil_div(p.c, SC) * p.batch * a.groups;
  // Measured against the register-staged kernel (L2 flushed, B200): faster up to ~16 tasks
  // per SM (c = 512 bf16: n = 1024 10.2 vs 16.4 us, n = 16384 24.6 vs 28.7 us; c = 128,
  // n = 32768: 16.4 vs 18.5 us), then equal or slower (n = 2^18: 206 vs 197 us), where the
  // loads-in-registers kernel already streams at ~0.97 of HBM.
  if (a.tasks > 16 * static_cast<int64_t>(di.sms)) return KVC_ERR_UNSUPPORTED;
  const size_t smem = csa_smem_bytes<InT>();
  if (smem > di.smem_optin) return KVC_ERR_UNSUPPORTED;
  const bool bf = sizeof(InT) == 2;
  CUtensorMap m0, m1, m2, m3;
  if (!make_stream_map(&m0, p.Z0, bf, p.batch, p.n, p.ne, p.c, 4, SC, 4, kCsaE) ||
      !make_stream_map(&m1, p.C0, bf, p.batch, p.n, p.ne, p.c, 4, SC, 4, kCsaE) ||
      !make_stream_map(&m2, p.Z1, bf, p.batch, p.n, p.ne, p.c, 4, SC, 4, kCsaE) ||
      !make_stream_map(&m3, p.C1, bf, p.batch, p.n, p.ne, p.c, 4, SC, 4, kCsaE))
    return KVC_ERR_UNSUPPORTED;
  auto kern = csa_tma_kernel<InT, OutT>;
  if (resident_blocks(kern, kCsaThreads, smem) < 1) return KVC_ERR_UNSUPPORTED;
  const int64_t grid = a.tasks < di.sms ? a.tasks : di.sms;
  kern<<<static_cast<unsigned>(grid), kCsaThreads, smem, st>>>(m0, m1, m2, m3, a);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = "csa_tma_kernel";
  return KVC_OK;
}


// ---------------------------------------------------------------------------------
// Self-test of the bounded waits (failure detection without a GPU fault): warp 0 waits on
// an mbarrier that nothing completes until the limit, raises the CTA's abort flag and the
// error bit; warp 1 waits on the same barrier honouring the abort flag and must leave
// once it is raised.  out[0] = 1 if warp 0 gave up, out[1] = 1 if warp 1 left on the flag.
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(64, 1) wait_selftest_kernel(int32_t* out) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  volatile int* abort_flag = &abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival would complete phase 0; none comes
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    out[0] = wait(&bar, 0, abort_flag, false) ? 0 : 1;
  } else if (threadIdx.x == 32) {
    // start a quarter of the limit later, so that it is warp 0's wait that runs out first
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < kWaitLimitNs / 4) {
    }
    const uint64_t t1 = global_timer_ns();
    const bool done = wait(&bar, 0, abort_flag, true);
    out[1] = (!done && global_timer_ns() - t1 < kWaitLimitNs) ? 1 : 0;  // left on the flag
  }
}

// hca_prepare_bias: block x writes the block of channel slab x (the rows scaled by log2 e
// at their positions in the consumers' order, with 0 past c; the per-position maxima; the
// spread flag) and slab x's columns of the raw copy; block 0 writes the header.  The values
// are the ones the kernel above would stage itself (the same fp32 products), so a prepared
// call gives bit for bit the result of an unprepared one.
template <int SC, int CPT>
__global__ void __launch_bounds__(256) prepare_bias_kernel(const float* __restrict__ B, int64_t c,
                                                           int m, int in_bf16, uint8_t* ws,
                                                           PrepLayout l) {
  const int64_t x = blockIdx.x;
  float* raw = reinterpret_cast<float*>(ws + l.raw_off);
  float* blk = reinterpret_cast<float*>(ws + l.prep_off) + x * l.slab_floats;
  float* bmx = blk + static_cast<int64_t>(m) * SC;
  bool narrow = true;
  for (int p = threadIdx.x; p < SC; p += blockDim.x) {
    const int64_t ch = x * SC + p;
    const int pos = slab_bias_pos<CPT, kCG>(p);
    float mx = -INFINITY, mn = INFINITY;
    for (int k = 0; k < m; ++k) {
      float v = 0.f;
      if (ch < c) {
        v = B[static_cast<int64_t>(k) * c + ch];
        raw[static_cast<int64_t>(k) * c + ch] = v;
      }
      const float sv = v * kLog2e;
      blk[k * SC + pos] = sv;
      mx = fmaxf(mx, sv);
      mn = fminf(mn, sv);
    }
    bmx[pos] = mx;
    narrow = narrow && (mx - mn <= kMaxBiasSpread);  // false for infinite or NaN spreads
  }
  narrow = __syncthreads_and(narrow) != 0;
  if (threadIdx.x < 4) bmx[SC + threadIdx.x] = (threadIdx.x == 0 && narrow) ? 1.f : 0.f;
  if (x == 0 && threadIdx.x == 0) {
    PrepHeader h;
    h.magic = kPrepMagic;
    h.version = 1;
    h.m = m;
    h.in_bf16 = in_bf16;
    h.c = c;
    h.slabs = l.slabs;
    h.slab_floats = l.slab_floats;
    h.raw_off = l.raw_off;
    h.prep_off = l.prep_off;
    *reinterpret_cast<PrepHeader*>(ws) = h;
  }
}

}  // namespace wtma

kvc_status launch_prepare_bias(const float* B, int64_t c, int m, bool in_bf16, void* ws,
                               cudaStream_t st) {
  const PrepLayout l = prep_layout(c, m, in_bf16);
  static_assert(wtma::slab<__nv_bfloat16>() == 128 && wtma::slab<float>() == 64,
                "prep_layout's slab widths are the window kernel's");
  if (in_bf16) {
    wtma::prepare_bias_kernel<128, 8><<<static_cast<unsigned>(l.slabs), 256, 0, st>>>(
        B, c, m, 1, static_cast<uint8_t*>(ws), l);
  } else {
    wtma::prepare_bias_kernel<64, 4><<<static_cast<unsigned>(l.slabs), 256, 0, st>>>(
        B, c, m, 0, static_cast<uint8_t*>(ws), l);
  }
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = "prepare_bias_kernel";
  return KVC_OK;
}

kvc_status launch_window_tma(const StreamProblem& p, cudaStream_t st) {
  if (p.two_segments || p.listed || p.cache || p.m < wtma::kMinRows || p.ne <= 0 ||
      p.ne > INT32_MAX || p.batch > INT32_MAX || p.c > INT32_MAX)
    return KVC_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(p.C0) | reinterpret_cast<uintptr_t>(p.Z0);
  if (al & 15u) return KVC_ERR_UNSUPPORTED;
  if (p.in_bf16)
    return p.out_bf16 ? wtma::launch_typed<__nv_bfloat16, __nv_bfloat16>(p, st)
                      : wtma::launch_typed<__nv_bfloat16, float>(p, st);
  return p.out_bf16 ? wtma::launch_typed<float, __nv_bfloat16>(p, st)
                    : wtma::launch_typed<float, float>(p, st);
}

kvc_status launch_csa_tma(const StreamProblem& p, cudaStream_t st) {
  if (!p.two_segments || p.m != 4 || p.listed || p.cache || p.ne <= 0 || p.ne > INT32_MAX ||
      p.batch > INT32_MAX || p.c > INT32_MAX)
    return KVC_ERR_UNSUPPORTED;
  const uintptr_t al = reinterpret_cast<uintptr_t>(p.C0) | reinterpret_cast<uintptr_t>(p.Z0) |
                       reinterpret_cast<uintptr_t>(p.C1) | reinterpret_cast<uintptr_t>(p.Z1);
  if (al & 15u) return KVC_ERR_UNSUPPORTED;
  if (p.in_bf16)
    return p.out_bf16 ? wtma::launch_csa_typed<__nv_bfloat16, __nv_bfloat16>(p, st)
                      : wtma::launch_csa_typed<__nv_bfloat16, float>(p, st);
  return p.out_bf16 ? wtma::launch_csa_typed<float, __nv_bfloat16>(p, st)
                    : wtma::launch_csa_typed<float, float>(p, st);
}

kvc_status launch_wait_selftest(int32_t* out, cudaStream_t st) {
  wtma::wait_selftest_kernel<<<1, 64, 0, st>>>(out);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = "wait_selftest_kernel";
  return KVC_OK;
}

unsigned int read_and_clear_window_error(bool* failed) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_window_error, sizeof(v)) != cudaSuccess) {
    *failed = true;
    return 0;
  }
  if (v != 0 && cudaMemcpyToSymbol(g_window_error, &zero, sizeof(zero)) != cudaSuccess)
    *failed = true;
  return v;
}

}  // namespace kvc
