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
// Per CTA (persistent, one per SM, 192 threads):
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
#include "kvc_launch.h"

#include <mutex>

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

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

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

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format: start >> 4 at [0,14), leading byte
// offset >> 4 at [16,30), stride byte offset >> 4 at [32,46), version 1 at [46,48),
// layout type at [61,64): 2 = SWIZZLE_128B, 4 = SWIZZLE_64B).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint64_t layout) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= layout << 61;
  return d;
}

// Instruction descriptor of kind::f16: D fp32, A and B bf16, A MN-major, B K-major,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kCh >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ work schedules

struct Args {
  const float* B0;  // CSA: B^a [m, c]; HCA: B [m, c]
  const float* B1;  // CSA: B^b [m, c]
  void* out;
  int64_t batch, n, c, ne;
  int ncg;          // channel groups of 128
  int nk;           // K steps of 64
  int pieces_per_unit;  // CSA: entry ranges per (sequence, channel group)
  int64_t units;        // CSA: pieces; HCA: tiles
};

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

template <bool CSA, int BK, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    fused_pool_kernel(const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmW0,
                      const __grid_constant__ CUtensorMap tmW1,
                      const __grid_constant__ CUtensorMap tmW2,
                      const __grid_constant__ CUtensorMap tmW3, const Args a) {
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
              tma_load_2d(smem_u32(st + (2 * s) * C::A_BOX), maps[s], &full[stage], cg * kCh, x);
              tma_load_2d(smem_u32(st + (2 * s + 1) * C::A_BOX), maps[s], &full[stage],
                          cg * kCh + 64, x);
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
    OutT* out = static_cast<OutT*>(a.out);
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
                store_scalar<OutT>(out + (static_cast<int64_t>(pc.b) * a.ne + kb) * a.c + ch,
                                   __fdividef(acc, s));
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
          store_scalar<OutT>(out + (static_cast<int64_t>(h.b) * a.ne + e) * a.c + ch,
                             __fdividef(A, S));
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

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] tensor map with a [box_rows, box_cols] box; the
// swizzle span equals the box row (box_cols * 2 bytes: 128 or 64).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
              uint32_t box_cols) {
  EncodeTiledFn enc = encode_fn();
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

template <bool CSA, int BK, typename OutT>
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
  auto kern = fused_pool_kernel<CSA, BK, OutT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(C::SMEM)) != cudaSuccess)
    return KVC_ERR_CUDA;
  kern<<<static_cast<unsigned>(grid), kThreads, C::SMEM, st>>>(mh, mw[0], mw[1], mw[2], mw[3], a);
  return cudaGetLastError() == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

}  // namespace fused

// Stage K per mode.  64-deep stages: CSA 80 KB (two fit), HCA 64 KB (three).  32-deep
// stages (CSA: five of 40 KB) measured slower on B200 (0.84 vs 0.79 ms on the n = 32768,
// d = 7168 workload): the CSA tile is bound by shared-memory bandwidth (N = 128 operand
// reads plus TMA writes), not by pipeline depth.
constexpr int kBkCsa = 64;
constexpr int kBkHca = 64;

kvc_status launch_fused(const FusedProblem& p, cudaStream_t st) {
  if (p.csa) {
    if (p.m != 4 || !p.overlap) return KVC_ERR_UNSUPPORTED;
    return p.out_bf16 ? fused::launch_impl<true, kBkCsa, __nv_bfloat16>(p, st)
                      : fused::launch_impl<true, kBkCsa, float>(p, st);
  }
  if (p.m != 128) return KVC_ERR_UNSUPPORTED;
  return p.out_bf16 ? fused::launch_impl<false, kBkHca, __nv_bfloat16>(p, st)
                    : fused::launch_impl<false, kBkHca, float>(p, st);
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
  if (failed) return KVC_ERR_CUDA;
  if (v) return KVC_ERR_TIMEOUT;
  return index_error ? KVC_ERR_INDEX : KVC_OK;
}

}  // namespace kvc
