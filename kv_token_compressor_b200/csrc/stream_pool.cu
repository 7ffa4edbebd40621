// Streaming softmax-pool kernels over precomputed C/Z streams (sm_100a).
//
// What they compute ("序列压缩注意力", eqs. attn-seqcomp-csa-softmax, attn-seqcomp-csa-pool,
// attn-seqcomp-overlap-bound, attn-seqcomp-hca; "Ch 04 · CSA" §3; "Ch 05 · HCA" §2):
// for every entry i and channel ch, a softmax over the window's logit rows
// (Z + B per channel) and the weighted sum of the matching C rows.
//
// Memory behaviour.  The work is HBM-bound: every stream byte is needed exactly once
// (CSA: the a-block of entry i is read only by entry i, the b-block of entry i-1 only
// by entry i; HCA: segments are disjoint).  Both kernels therefore stream the inputs
// with 16-byte read-once loads straight into registers, issue all loads of a window
// before using any, and keep the biases (pre-scaled by log2 e) in shared memory.
// Softmax is exact two-pass per window in registers for the small CSA windows
// (one exp2 per element), and chunked online (max, sum, acc) with a shared-memory
// merge across row groups for long windows (HCA m' = 128).
#include "kvc_common.cuh"
#include "kvc_host.h"
#include "kvc_launch.h"
#include "stream_common.cuh"

#include <math.h>

#include <type_traits>


namespace kvc {

// ---------------------------------------------------------------------------------
// CSA, small m (1, 2, 4): one thread = one entry x one 16-byte channel vector.
// ---------------------------------------------------------------------------------
// Set when an entry list read from device memory names a window outside its sequence or
// the streams (that entry is skipped); read and cleared by kvc_device_status().
__device__ unsigned int g_index_error = 0;

// Entry lists (decode / ragged batches): entry k reads the sequence whose rows start at
// seq_start[k] (seq_len[k] rows) and is that sequence's entry entry[k]; its output row is k.
struct EntryList {
  const int64_t* seq_start;
  const int64_t* seq_len;
  const int64_t* entry;
  int64_t num, total_rows;
};

// Checks one listed entry against its sequence and the streams; on success gives the first
// a-row and whether it is the sequence's entry 0.
__device__ __forceinline__ bool listed_entry(const EntryList& L, int64_t k, int m, int64_t* rowA,
                                             bool* first, int64_t* e_out) {
  const int64_t s0 = L.seq_start[k], len = L.seq_len[k], e = L.entry[k];
  if (!(s0 >= 0 && len >= 0 && s0 <= L.total_rows - len && e >= 0 && e < len / m)) return false;
  *rowA = s0 + static_cast<int64_t>(m) * e;
  *first = e == 0;
  *e_out = e;
  return true;
}

// Extra kernel argument of the cache-layout instantiations (empty otherwise).
template <bool CACHE>
using CacheArg = typename std::conditional<CACHE, CacheFmt, NoCache>::type;

struct CsaSmallArgs {
  const void* Ca;
  const void* Cb;
  const void* Za;
  const void* Zb;
  const float* Ba;
  const float* Bb;
  int64_t batch, n, c, ne;
  void* out;
};

// CK: the channel count as a compile-time row stride (0: a.c at run time).  With a
// run-time stride each of the 16 row addresses of a window needs registers of its own; a
// constant one folds into the load offsets, which took the bf16 CSA kernel from 88 bytes
// of spills to 16 and 2% off the long-context launch.
template <typename InT, typename OutT, int M, bool OVERLAP, bool LISTED, bool CACHE, int CK = 0>
__global__ void __launch_bounds__(256, 2) csa_small_m_kernel(CsaSmallArgs a, const EntryList list,
                                                             const CacheArg<CACHE> cf) {
  constexpr int CPT = VecInfo<InT>::kChannels;
  constexpr int NP = CPT / 2;              // channel pairs per thread
  constexpr int NB = OVERLAP ? 2 * M : M;  // bias rows: B^a rows then B^b rows
  const float2 kL2e2 = make_float2(kLog2e, kLog2e);
  extern __shared__ float4 smem_f4[];
  float* sb = reinterpret_cast<float*>(smem_f4);  // [NB][SC], pre-scaled by log2 e

  const int SC = blockDim.x * CPT;
  const int64_t ch_base = static_cast<int64_t>(blockIdx.x) * SC;
  const int tid = threadIdx.y * blockDim.x + threadIdx.x;
  const int nthr = blockDim.x * blockDim.y;
  stage_bias(sb, a.Ba, a.Bb, M, NB, SC, ch_base, a.c, tid, nthr, [](int sc) { return sc; });
  __syncthreads();

  const int sc0 = threadIdx.x * CPT;
  const int64_t ch0 = ch_base + sc0;
  if (ch0 >= a.c) return;
  const int64_t cs = CK ? static_cast<int64_t>(CK) : a.c;  // row stride in elements

  const InT* Ca = static_cast<const InT*>(a.Ca);
  const InT* Za = static_cast<const InT*>(a.Za);
  const InT* Cb = static_cast<const InT*>(a.Cb);
  const InT* Zb = static_cast<const InT*>(a.Zb);
  OutT* out = static_cast<OutT*>(a.out);
  // Boundary rows of entry 0 (eq. attn-seqcomp-overlap-bound): logit -inf, vector 0.
  const uint32_t neg_inf_bits = sizeof(InT) == 2 ? 0xFF80FF80u : 0xFF800000u;
  const uint4 z_boundary = make_uint4(neg_inf_bits, neg_inf_bits, neg_inf_bits, neg_inf_bits);
  const uint4 c_boundary = make_uint4(0u, 0u, 0u, 0u);

  const int64_t istep = static_cast<int64_t>(gridDim.y) * blockDim.y;
  const int64_t lim = LISTED ? list.num : a.ne;
  for (int64_t b = blockIdx.z; b < a.batch; b += gridDim.z) {
    for (int64_t i = static_cast<int64_t>(blockIdx.y) * blockDim.y + threadIdx.y; i < lim;
         i += istep) {
      int64_t rowA;  // a-range start of the entry
      bool first;    // entry 0 of its sequence: no b-rows
      int64_t orow;  // output row
      int64_t eidx;  // entry index within its sequence
      if constexpr (LISTED) {
        if (!listed_entry(list, i, M, &rowA, &first, &eidx)) {
          if (threadIdx.x == 0) atomicOr(&g_index_error, 1u);
          continue;
        }
        orow = i;
      } else {
        rowA = b * a.n + static_cast<int64_t>(M) * i;
        first = i == 0;
        orow = b * a.ne + i;
        eidx = i;
      }
      uint4 za[M], ca[M], zb[M], cb[M];
#pragma unroll
      for (int k = 0; k < M; ++k) {
        za[k] = ld_stream16(Za + (rowA + k) * cs + ch0);
        ca[k] = ld_stream16(Ca + (rowA + k) * cs + ch0);
      }
      if constexpr (OVERLAP) {
        if (!first) {  // b-range(i) = a-range(i-1)
#pragma unroll
          for (int k = 0; k < M; ++k) {
            zb[k] = ld_stream16(Zb + (rowA - M + k) * cs + ch0);
            cb[k] = ld_stream16(Cb + (rowA - M + k) * cs + ch0);
          }
        } else {
#pragma unroll
          for (int k = 0; k < M; ++k) {
            zb[k] = z_boundary;
            cb[k] = c_boundary;
          }
        }
      }
      float res[CPT];
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float2 ba_k0 = *reinterpret_cast<const float2*>(sb + sc0 + 2 * p);  // row 0
        float2 la[M], lb[M];
        float2 mx = make_float2(-INFINITY, -INFINITY);
#pragma unroll
        for (int k = 0; k < M; ++k) {
          const float2 bk = k == 0 ? ba_k0 : *reinterpret_cast<const float2*>(sb + k * SC + sc0 + 2 * p);
          la[k] = f2_fma(vec_pair<InT>(za[k], p), kL2e2, bk);
          mx = f2_max(mx, la[k]);
        }
        if constexpr (OVERLAP) {
#pragma unroll
          for (int k = 0; k < M; ++k) {
            const float2 bk = *reinterpret_cast<const float2*>(sb + (M + k) * SC + sc0 + 2 * p);
            lb[k] = f2_fma(vec_pair<InT>(zb[k], p), kL2e2, bk);
            mx = f2_max(mx, lb[k]);
          }
        }
        const float2 negm = make_float2(-mx.x, -mx.y);
        float2 s = make_float2(0.f, 0.f), acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < M; ++k) {
          const float2 w = f2_ex2(f2_add(la[k], negm));
          s = f2_add(s, w);
          acc = f2_fma(w, vec_pair<InT>(ca[k], p), acc);
        }
        if constexpr (OVERLAP) {
#pragma unroll
          for (int k = 0; k < M; ++k) {
            const float2 w = f2_ex2(f2_add(lb[k], negm));
            s = f2_add(s, w);
            acc = f2_fma(w, vec_pair<InT>(cb[k], p), acc);
          }
        }
        res[2 * p] = __fdividef(acc.x, s.x);
        res[2 * p + 1] = __fdividef(acc.y, s.y);
      }
      if constexpr (CACHE) {
        store_cache<CPT>(cf, orow, ch0, eidx, res);
      } else {
        store_out<OutT, CPT>(out + orow * cs + ch0, res);
      }
    }
  }
}

// ---------------------------------------------------------------------------------
// Any window length: HCA (one segment of m rows), CSA with overlap for other m (the
// a-segment then the b-segment), CSA without overlap.  A CTA covers a slab of SC
// channels (16 vectors of 16 bytes) and 16 thread rows; thread row ty = (entry es, row
// group rg) with RG row groups per entry.  Each thread walks rows rg, rg+RG, ... of its
// entry in chunks of U rows (all 2U loads in flight), keeping an online (max, sum, acc)
// per channel: per chunk one exp2 per element plus one rescale.  With RG = 1 a thread
// owns a whole window and stores its result directly; with RG > 1 (few entries) the
// row-group partials merge through shared memory.
// ---------------------------------------------------------------------------------
struct WinArgs {
  const void* C0;  // segment 0 streams (a-range / the HCA segment)
  const void* Z0;
  const void* C1;  // segment 1 streams (b-range), TWO_SEG only
  const void* Z1;
  const float* B0;  // [m, c]
  const float* B1;  // [m, c], TWO_SEG only
  int64_t batch, n, c, ne;
  int m;
  void* out;
};

constexpr int kWinCG = 16;  // channel vectors per CTA
constexpr int kWinTY = 16;  // thread rows per CTA
constexpr int kWinU = 8;    // rows per thread per chunk

template <typename InT>
constexpr int win_slab() {
  return kWinCG * VecInfo<InT>::kChannels;
}

template <typename InT, bool TWO_SEG>
size_t win_smem_bytes(int m, int rg) {
  const int rows = TWO_SEG ? 2 * m : m;
  const size_t partial = rg > 1 ? 3 * kWinTY * win_slab<InT>() : 0;
  const size_t extra = win_slab<InT>() + 2 * kWinCG * kWinTY;  // bias maxima, spread partials
  return sizeof(float) * (static_cast<size_t>(rows) * win_slab<InT>() + extra + partial);
}

template <typename InT, typename OutT, bool TWO_SEG, int RG, bool LISTED, bool CACHE>
__global__ void __launch_bounds__(256, 2) window_pool_kernel(WinArgs a, const EntryList list,
                                                             const CacheArg<CACHE> cf) {
  static_assert(!(LISTED || CACHE) || RG == 1, "entry lists and the cache layout use one window per thread");
  constexpr int CPT = VecInfo<InT>::kChannels;
  constexpr int SC = win_slab<InT>();
  constexpr int EY = kWinTY / RG;  // entries per CTA iteration
  constexpr int U = kWinU;
  constexpr int NP = CPT / 2;      // channel pairs per thread
  const float2 kL2e2 = make_float2(kLog2e, kLog2e);
  extern __shared__ float4 smem_f4[];
  const int nb = TWO_SEG ? 2 * a.m : a.m;
  // Bias rows pre-scaled by log2 e, as [nb][CPT/4][kWinCG] float4: the q-th float4 of
  // every thread group of a row is contiguous, so a warp's reads of it hit no bank twice.
  float* sb = reinterpret_cast<float*>(smem_f4);
  float* bmx = sb + static_cast<size_t>(nb) * SC;  // [SC] per-channel largest bias, same order
  float* red = bmx + SC;                           // [2][256] bias max / min partials
  float* pm = red + 2 * kWinCG * kWinTY;           // RG > 1: [16][SC] partial max
  float* ps = pm + kWinTY * SC;                    //         partial sum
  float* pa = ps + kWinTY * SC;                    //         partial weighted sum

  const int tx = threadIdx.x, ty = threadIdx.y;
  const int tid = ty * kWinCG + tx;
  const int es = ty / RG, rg = ty - (ty / RG) * RG;
  const int64_t ch_base = static_cast<int64_t>(blockIdx.x) * SC;
  // 256 is a multiple of SC, so each thread stages one channel's rows tid/SC, tid/SC + 256/SC, ...
  const float2 mm = stage_bias(sb, a.B0, a.B1, a.m, nb, SC, ch_base, a.c, tid, kWinCG * kWinTY,
                               [](int sc) { return slab_bias_pos<CPT, kWinCG>(sc); });
  red[tid] = mm.x;
  red[kWinCG * kWinTY + tid] = mm.y;
  __syncthreads();
  // Fast chunk maximum (see pass 1 below) when every channel's bias spread is at most
  // kMaxBiasSpread; a CTA-uniform choice.
  bool wide = false;
  if (tid < SC) {
    float mx = -INFINITY, mn = INFINITY;
    for (int j = tid; j < kWinCG * kWinTY; j += SC) {
      mx = fmaxf(mx, red[j]);
      mn = fminf(mn, red[kWinCG * kWinTY + j]);
    }
    bmx[slab_bias_pos<CPT, kWinCG>(tid)] = mx;
    wide = !(mx - mn <= kMaxBiasSpread);  // also true for infinite or NaN spreads
  }
  const bool fast = !__syncthreads_or(wide);

  const int sc0 = tx * CPT;
  const int64_t ch0 = ch_base + sc0;
  const bool active = ch0 < a.c;
  const InT* C0 = static_cast<const InT*>(a.C0);
  const InT* Z0 = static_cast<const InT*>(a.Z0);
  const InT* C1 = static_cast<const InT*>(a.C1);
  const InT* Z1 = static_cast<const InT*>(a.Z1);
  OutT* out = static_cast<OutT*>(a.out);
  const int m = a.m;

  for (int64_t b = blockIdx.z; b < a.batch; b += gridDim.z) {
    const int64_t lim = LISTED ? list.num : a.ne;
    for (int64_t i0 = static_cast<int64_t>(blockIdx.y) * EY; i0 < lim;
         i0 += static_cast<int64_t>(gridDim.y) * EY) {
      const int64_t i = i0 + es;
      int64_t row0 = b * a.n + static_cast<int64_t>(m) * i;  // first row of its own segment
      bool first = i == 0;                                      // no b-rows
      bool ok = true;
      int64_t eidx = i;                                         // index within its sequence
      if constexpr (LISTED) {
        ok = i < lim && listed_entry(list, i, m, &row0, &first, &eidx);
        if (i < lim && !ok && tx == 0) atomicOr(&g_index_error, 1u);
      }
      const bool live = active && i < lim && ok;
      const int rows_i = (TWO_SEG && !first) ? 2 * m : m;
      float2 M[NP], S[NP], A[NP];  // per channel pair: running max, sum, weighted sum
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        M[p] = make_float2(-INFINITY, -INFINITY);
        S[p] = make_float2(0.f, 0.f);
        A[p] = make_float2(0.f, 0.f);
      }
      if (live) {
        for (int v0 = rg; v0 < rows_i; v0 += RG * U) {
          uint4 z[U], cv[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int v = v0 + u * RG;
            if (v < rows_i) {
              const bool seg1 = TWO_SEG && v >= m;
              const int64_t row = seg1 ? row0 - m + (v - m) : row0 + v;
              z[u] = ld_stream16((seg1 ? Z1 : Z0) + row * a.c + ch0);
              cv[u] = ld_stream16((seg1 ? C1 : C0) + row * a.c + ch0);
            }
          }
          // pass 1: an upper bound M' of the chunk's largest logit per channel.  Fast form:
          // max_k z_k * log2 e + max_k b_k, the maximum taken in the input type (exact).
          // M' exceeds the true maximum by at most the bias spread, so the largest weight
          // exp2(l* - M') stays >= 2^-kMaxBiasSpread: the softmax is unchanged and nothing
          // underflows.  Otherwise the exact per-row maximum of z * log2 e + b.
          float2 cm[NP];
          if (fast) {
            uint4 zm = z[0];
#pragma unroll
            for (int u = 1; u < U; ++u)
              if (v0 + u * RG < rows_i) zm = vec_max<InT>(zm, z[u]);
            const float4* bx = reinterpret_cast<const float4*>(bmx) + tx;
#pragma unroll
            for (int q = 0; q < NP / 2; ++q) {
              const float4 bq = bx[q * kWinCG];
              cm[2 * q] = f2_fma(vec_pair<InT>(zm, 2 * q), kL2e2, make_float2(bq.x, bq.y));
              cm[2 * q + 1] = f2_fma(vec_pair<InT>(zm, 2 * q + 1), kL2e2, make_float2(bq.z, bq.w));
            }
          } else {
#pragma unroll
            for (int p = 0; p < NP; ++p) cm[p] = make_float2(-INFINITY, -INFINITY);
#pragma unroll
            for (int u = 0; u < U; ++u) {
              const int v = v0 + u * RG;
              if (v < rows_i) {
                const float4* bp = reinterpret_cast<const float4*>(sb + v * SC) + tx;
#pragma unroll
                for (int q = 0; q < NP / 2; ++q) {
                  const float4 bq = bp[q * kWinCG];
                  cm[2 * q] = f2_max(cm[2 * q], f2_fma(vec_pair<InT>(z[u], 2 * q), kL2e2,
                                                       make_float2(bq.x, bq.y)));
                  cm[2 * q + 1] = f2_max(cm[2 * q + 1], f2_fma(vec_pair<InT>(z[u], 2 * q + 1),
                                                               kL2e2, make_float2(bq.z, bq.w)));
                }
              }
            }
          }
          // rescale the running state once per chunk
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            const float2 nm = f2_max(M[p], cm[p]);  // finite: row v0 < rows_i is valid
            const float2 sc = make_float2(ex2_ftz(M[p].x - nm.x), ex2_ftz(M[p].y - nm.y));
            S[p] = f2_mul(S[p], sc);
            A[p] = f2_mul(A[p], sc);
            M[p] = nm;
          }
          // pass 2: one exp2 per element, packed pair arithmetic
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int v = v0 + u * RG;
            if (v < rows_i) {
              const float4* bp = reinterpret_cast<const float4*>(sb + v * SC) + tx;
#pragma unroll
              for (int q = 0; q < NP / 2; ++q) {
                const float4 bq = bp[q * kWinCG];
                const float2 b2[2] = {make_float2(bq.x, bq.y), make_float2(bq.z, bq.w)};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int pp = 2 * q + e;
                  const float2 l = f2_fma(vec_pair<InT>(z[u], pp), kL2e2, f2_sub(b2[e], M[pp]));
                  const float2 w = f2_ex2(l);
                  S[pp] = f2_add(S[pp], w);
                  A[pp] = f2_fma(w, vec_pair<InT>(cv[u], pp), A[pp]);
                }
              }
            }
          }
        }
      }
      if constexpr (RG == 1) {
        if (live) {
          float res[CPT];
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            res[2 * p] = __fdividef(A[p].x, S[p].x);
            res[2 * p + 1] = __fdividef(A[p].y, S[p].y);
          }
          if constexpr (CACHE) {
            store_cache<CPT>(cf, LISTED ? i : b * a.ne + i, ch0, eidx, res);
          } else {
            store_out<OutT, CPT>(out + (LISTED ? i : b * a.ne + i) * a.c + ch0, res);
          }
        }
      } else {
#pragma unroll
        for (int q = 0; q < NP / 2; ++q) {
          reinterpret_cast<float4*>(pm + ty * SC + sc0)[q] =
              make_float4(M[2 * q].x, M[2 * q].y, M[2 * q + 1].x, M[2 * q + 1].y);
          reinterpret_cast<float4*>(ps + ty * SC + sc0)[q] =
              make_float4(S[2 * q].x, S[2 * q].y, S[2 * q + 1].x, S[2 * q + 1].y);
          reinterpret_cast<float4*>(pa + ty * SC + sc0)[q] =
              make_float4(A[2 * q].x, A[2 * q].y, A[2 * q + 1].x, A[2 * q + 1].y);
        }
        __syncthreads();
        for (int item = tid; item < EY * SC; item += kWinCG * kWinTY) {
          const int e2 = item / SC, sc = item - (item / SC) * SC;
          const int64_t i2 = i0 + e2;
          const int64_t ch = ch_base + sc;
          if (i2 < a.ne && ch < a.c) {
            float gm = -INFINITY;
#pragma unroll
            for (int r = 0; r < RG; ++r) gm = fmaxf(gm, pm[(e2 * RG + r) * SC + sc]);
            float s = 0.f, acc = 0.f;
#pragma unroll
            for (int r = 0; r < RG; ++r) {
              const float f = ex2_ftz(pm[(e2 * RG + r) * SC + sc] - gm);  // 0 for empty groups
              s = fmaf(ps[(e2 * RG + r) * SC + sc], f, s);
              acc = fmaf(pa[(e2 * RG + r) * SC + sc], f, acc);
            }
            store_scalar<OutT>(out + (b * a.ne + i2) * a.c + ch, __fdividef(acc, s));
          }
        }
        __syncthreads();
      }
    }
  }
}

// ---------------------------------------------------------------------------------
// Few long windows in one segment (HCA with few entries): the row-group split of the
// window kernel (RG row groups per window, partials merged in shared memory), software
// pipelined.  Each thread walks its rows of a window in steps of kPipeU rows and issues
// the loads of its next step (in this window or the next) before computing the current
// one, so the CTA's loads stay in flight while it computes and merges.  With one chunk
// per thread and window (the kernel above) a CTA alternates between waiting on memory
// and computing, and with few windows nothing else covers the wait.
// ---------------------------------------------------------------------------------
constexpr int kPipeU = 4;

struct PipeBuf {
  uint4 z[kPipeU], c[kPipeU];
};

template <typename InT, int RG>
__device__ __forceinline__ void pipe_load(PipeBuf& buf, const InT* C0, const InT* Z0, int64_t row0,
                                          int v0, int m, int64_t c, int64_t ch0, bool live) {
#pragma unroll
  for (int u = 0; u < kPipeU; ++u) {
    const int v = v0 + u * RG;
    if (live && v < m) {
      buf.z[u] = ld_stream16(Z0 + (row0 + v) * c + ch0);
      buf.c[u] = ld_stream16(C0 + (row0 + v) * c + ch0);
    }
  }
}

// One step of rows v0, v0 + RG, ... (v0 < m) into the running (max, sum, acc) per channel
// pair; `fast` as in the window kernel (chunk maximum bounded by max z + max bias).
template <typename InT, int RG>
__device__ __forceinline__ void pipe_compute(const PipeBuf& buf, int v0, int m, bool fast,
                                             const float* sb, const float* bmx, int tx,
                                             float2 (&M)[VecInfo<InT>::kChannels / 2],
                                             float2 (&S)[VecInfo<InT>::kChannels / 2],
                                             float2 (&A)[VecInfo<InT>::kChannels / 2]) {
  constexpr int NP = VecInfo<InT>::kChannels / 2;
  constexpr int SC = win_slab<InT>();
  const float2 kL2e2 = make_float2(kLog2e, kLog2e);
  float2 cm[NP];
  if (fast) {
    uint4 zm = buf.z[0];
#pragma unroll
    for (int u = 1; u < kPipeU; ++u)
      if (v0 + u * RG < m) zm = vec_max<InT>(zm, buf.z[u]);
    const float4* bx = reinterpret_cast<const float4*>(bmx) + tx;
#pragma unroll
    for (int q = 0; q < NP / 2; ++q) {
      const float4 bq = bx[q * kWinCG];
      cm[2 * q] = f2_fma(vec_pair<InT>(zm, 2 * q), kL2e2, make_float2(bq.x, bq.y));
      cm[2 * q + 1] = f2_fma(vec_pair<InT>(zm, 2 * q + 1), kL2e2, make_float2(bq.z, bq.w));
    }
  } else {
#pragma unroll
    for (int p = 0; p < NP; ++p) cm[p] = make_float2(-INFINITY, -INFINITY);
#pragma unroll
    for (int u = 0; u < kPipeU; ++u) {
      const int v = v0 + u * RG;
      if (v < m) {
        const float4* bp = reinterpret_cast<const float4*>(sb + v * SC) + tx;
#pragma unroll
        for (int q = 0; q < NP / 2; ++q) {
          const float4 bq = bp[q * kWinCG];
          cm[2 * q] = f2_max(cm[2 * q], f2_fma(vec_pair<InT>(buf.z[u], 2 * q), kL2e2,
                                               make_float2(bq.x, bq.y)));
          cm[2 * q + 1] = f2_max(cm[2 * q + 1], f2_fma(vec_pair<InT>(buf.z[u], 2 * q + 1), kL2e2,
                                                       make_float2(bq.z, bq.w)));
        }
      }
    }
  }
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const float2 nm = f2_max(M[p], cm[p]);  // finite: row v0 < m is valid
    const float2 sc = make_float2(ex2_ftz(M[p].x - nm.x), ex2_ftz(M[p].y - nm.y));
    S[p] = f2_mul(S[p], sc);
    A[p] = f2_mul(A[p], sc);
    M[p] = nm;
  }
#pragma unroll
  for (int u = 0; u < kPipeU; ++u) {
    const int v = v0 + u * RG;
    if (v < m) {
      const float4* bp = reinterpret_cast<const float4*>(sb + v * SC) + tx;
#pragma unroll
      for (int q = 0; q < NP / 2; ++q) {
        const float4 bq = bp[q * kWinCG];
        const float2 b2[2] = {make_float2(bq.x, bq.y), make_float2(bq.z, bq.w)};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int pp = 2 * q + e;
          const float2 l = f2_fma(vec_pair<InT>(buf.z[u], pp), kL2e2, f2_sub(b2[e], M[pp]));
          const float2 w = f2_ex2(l);
          S[pp] = f2_add(S[pp], w);
          A[pp] = f2_fma(w, vec_pair<InT>(buf.c[u], pp), A[pp]);
        }
      }
    }
  }
}

template <typename InT, typename OutT, int RG>
__global__ void __launch_bounds__(256, 2) window_pipe_kernel(WinArgs a) {
  static_assert(RG > 1, "row groups merge in shared memory");
  constexpr int CPT = VecInfo<InT>::kChannels;
  constexpr int SC = win_slab<InT>();
  constexpr int EY = kWinTY / RG;  // windows per CTA iteration
  constexpr int NP = CPT / 2;
  extern __shared__ float4 smem_f4[];
  const int m = a.m;
  float* sb = reinterpret_cast<float*>(smem_f4);   // [m] bias rows, float4-major
  float* bmx = sb + static_cast<size_t>(m) * SC;   // [SC] per-channel largest bias
  float* red = bmx + SC;                           // [2][256] bias max / min partials
  float* pm = red + 2 * kWinCG * kWinTY;           // [16][SC] partial max
  float* ps = pm + kWinTY * SC;                    //          partial sum
  float* pa = ps + kWinTY * SC;                    //          partial weighted sum

  const int tx = threadIdx.x, ty = threadIdx.y;
  const int tid = ty * kWinCG + tx;
  const int es = ty / RG, rg = ty - (ty / RG) * RG;
  const int64_t ch_base = static_cast<int64_t>(blockIdx.x) * SC;
  const float2 mm = stage_bias(sb, a.B0, a.B0, m, m, SC, ch_base, a.c, tid, kWinCG * kWinTY,
                               [](int sc) { return slab_bias_pos<CPT, kWinCG>(sc); });
  red[tid] = mm.x;
  red[kWinCG * kWinTY + tid] = mm.y;
  __syncthreads();
  bool wide = false;
  if (tid < SC) {
    float mx = -INFINITY, mn = INFINITY;
    for (int j = tid; j < kWinCG * kWinTY; j += SC) {
      mx = fmaxf(mx, red[j]);
      mn = fminf(mn, red[kWinCG * kWinTY + j]);
    }
    bmx[slab_bias_pos<CPT, kWinCG>(tid)] = mx;
    wide = !(mx - mn <= kMaxBiasSpread);
  }
  const bool fast = !__syncthreads_or(wide);

  const int sc0 = tx * CPT;
  const int64_t ch0 = ch_base + sc0;
  const bool active = ch0 < a.c;
  const InT* C0 = static_cast<const InT*>(a.C0);
  const InT* Z0 = static_cast<const InT*>(a.Z0);
  OutT* out = static_cast<OutT*>(a.out);

  // This CTA's windows: w = (batch step jb, entry step jy); entry i = y0 + jy * ystep + es.
  const int64_t y0 = static_cast<int64_t>(blockIdx.y) * EY;
  const int64_t ystep = static_cast<int64_t>(gridDim.y) * EY;
  const int64_t ny = y0 < a.ne ? (a.ne - y0 + ystep - 1) / ystep : 0;
  const int64_t nbat = blockIdx.z < a.batch ? (a.batch - blockIdx.z + gridDim.z - 1) / gridDim.z : 0;
  const int64_t W = ny * nbat;
  // Steps of rows per window for this thread (rows rg, rg + RG, ... < m, kPipeU per step).
  const int K = rg < m ? (m - rg + RG * kPipeU - 1) / (RG * kPipeU) : 0;
  auto window = [&](int64_t w, int64_t* b, int64_t* i, int64_t* row0, bool* live) {
    const int64_t jb = w / ny, jy = w - (w / ny) * ny;
    *b = blockIdx.z + jb * gridDim.z;
    *i = y0 + jy * ystep + es;
    *row0 = *b * a.n + static_cast<int64_t>(m) * *i;
    *live = active && *i < a.ne;
  };

  PipeBuf b0, b1;
  // step cursor of the next load: window wn, step kn
  int64_t wn = 0;
  int kn = 0;
  if (K > 0 && W > 0) {
    int64_t bb, ii, r0;
    bool lv;
    window(0, &bb, &ii, &r0, &lv);
    pipe_load<InT, RG>(b0, C0, Z0, r0, rg, m, a.c, ch0, lv);
    kn = 1;
    if (kn == K) { kn = 0; wn = 1; }
  }
  int64_t s = 0;  // steps computed so far (buffer parity)
  for (int64_t w = 0; w < W; ++w) {
    int64_t b, i, row0;
    bool live;
    window(w, &b, &i, &row0, &live);
    float2 M[NP], S[NP], A[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      M[p] = make_float2(-INFINITY, -INFINITY);
      S[p] = make_float2(0.f, 0.f);
      A[p] = make_float2(0.f, 0.f);
    }
    for (int k = 0; k < K; ++k, ++s) {
      // prefetch the next step (possibly in the next window) into the other buffer
      const bool more = wn < W;
      int64_t nb_, ni, nrow0;
      bool nlive = false;
      if (more) window(wn, &nb_, &ni, &nrow0, &nlive);
      const int nv0 = rg + kn * RG * kPipeU;
      if ((s & 1) == 0) {
        if (more) pipe_load<InT, RG>(b1, C0, Z0, nrow0, nv0, m, a.c, ch0, nlive);
        if (live) pipe_compute<InT, RG>(b0, rg + k * RG * kPipeU, m, fast, sb, bmx, tx, M, S, A);
      } else {
        if (more) pipe_load<InT, RG>(b0, C0, Z0, nrow0, nv0, m, a.c, ch0, nlive);
        if (live) pipe_compute<InT, RG>(b1, rg + k * RG * kPipeU, m, fast, sb, bmx, tx, M, S, A);
      }
      if (more && ++kn == K) {
        kn = 0;
        ++wn;
      }
    }
    // merge the row groups of each of the EY windows through shared memory
#pragma unroll
    for (int q = 0; q < NP / 2; ++q) {
      reinterpret_cast<float4*>(pm + ty * SC + sc0)[q] =
          make_float4(M[2 * q].x, M[2 * q].y, M[2 * q + 1].x, M[2 * q + 1].y);
      reinterpret_cast<float4*>(ps + ty * SC + sc0)[q] =
          make_float4(S[2 * q].x, S[2 * q].y, S[2 * q + 1].x, S[2 * q + 1].y);
      reinterpret_cast<float4*>(pa + ty * SC + sc0)[q] =
          make_float4(A[2 * q].x, A[2 * q].y, A[2 * q + 1].x, A[2 * q + 1].y);
    }
    __syncthreads();
    const int64_t i0 = i - es;
    for (int item = tid; item < EY * SC; item += kWinCG * kWinTY) {
      const int e2 = item / SC, sc = item - (item / SC) * SC;
      const int64_t i2 = i0 + e2;
      const int64_t ch = ch_base + sc;
      if (i2 < a.ne && ch < a.c) {
        float gm = -INFINITY;
#pragma unroll
        for (int r = 0; r < RG; ++r) gm = fmaxf(gm, pm[(e2 * RG + r) * SC + sc]);
        float sum = 0.f, acc = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) {
          const float f = ex2_ftz(pm[(e2 * RG + r) * SC + sc] - gm);  // 0 for empty groups
          sum = fmaf(ps[(e2 * RG + r) * SC + sc], f, sum);
          acc = fmaf(pa[(e2 * RG + r) * SC + sc], f, acc);
        }
        store_scalar<OutT>(out + (b * a.ne + i2) * a.c + ch, __fdividef(acc, sum));
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------------
namespace {

EntryList entry_list(const StreamProblem& p) {
  return EntryList{p.seq_start, p.seq_len, p.entry, p.num, p.total_rows};
}

template <bool CACHE>
CacheArg<CACHE> cache_arg(const StreamProblem& p) {
  if constexpr (CACHE) {
    return CacheFmt{static_cast<uint8_t*>(p.out_nope), static_cast<__nv_bfloat16*>(p.out_rope),
                    p.inv_freq, p.c - p.r, p.r, p.pos_stride, p.pos_offset, p.fp8_scale};
  } else {
    return NoCache{};
  }
}

template <typename InT, typename OutT, int M, bool OVERLAP, bool LISTED, bool CACHE, int CK = 0>
kvc_status launch_csa_small_ck(const StreamProblem& p, cudaStream_t st) {
  constexpr int CPT = VecInfo<InT>::kChannels;
  const int64_t G = p.c / CPT;  // channel vectors
  const int cg = static_cast<int>(G < 64 ? G : 64);
  const int ey = 256 / cg;
  const dim3 block(cg, ey);
  const size_t smem = sizeof(float) * (OVERLAP ? 2 * M : M) * cg * CPT;
  auto kern = csa_small_m_kernel<InT, OutT, M, OVERLAP, LISTED, CACHE, CK>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  const int occ = resident_blocks(kern, cg * ey, smem);
  if (di.sms == 0 || occ == 0) return KVC_ERR_CUDA;
  const int64_t gx = ceil_div(G, cg);
  const int64_t batch = LISTED ? 1 : p.batch;
  const int64_t gz = batch < 65535 ? batch : 65535;
  int64_t want = static_cast<int64_t>(di.sms) * occ;  // one resident wave
  int64_t gy = want / (gx * gz);
  if (gy < 1) gy = 1;
  const int64_t need = ceil_div(LISTED ? p.num : p.ne, ey);
  if (gy > need) gy = need;
  if (gy > 65535) gy = 65535;
  // Balance: every CTA row gets the same number of entry iterations (+-1).
  gy = ceil_div(need, ceil_div(need, gy));
  CsaSmallArgs args{p.C0, p.C1, p.Z0, p.Z1, p.B0, p.B1, batch, p.n, p.c, p.ne, p.out};
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), static_cast<unsigned>(gz)),
         block, smem, st>>>(args, entry_list(p), cache_arg<CACHE>(p));
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = CK == 512   ? "csa_small_m_kernel/c512"
                  : CK == 128 ? "csa_small_m_kernel/c128"
                              : "csa_small_m_kernel";
  return KVC_OK;
}

// The dense CSA (m = 4, overlap; plain outputs) at the channel counts of the workloads
// (c = 512 compressed KV, c = 128 indexer keys) with the row stride as a constant.
template <typename InT, typename OutT, int M, bool OVERLAP, bool LISTED, bool CACHE>
kvc_status launch_csa_small(const StreamProblem& p, cudaStream_t st) {
  if constexpr (M == 4 && OVERLAP && !LISTED && !CACHE) {
    if (p.c == 512) return launch_csa_small_ck<InT, OutT, M, OVERLAP, LISTED, CACHE, 512>(p, st);
    if (p.c == 128) return launch_csa_small_ck<InT, OutT, M, OVERLAP, LISTED, CACHE, 128>(p, st);
  }
  return launch_csa_small_ck<InT, OutT, M, OVERLAP, LISTED, CACHE>(p, st);
}

template <typename InT, typename OutT, bool TWO_SEG, int RG, bool LISTED, bool CACHE>
kvc_status launch_window_rg(const StreamProblem& p, cudaStream_t st, const DeviceInfo& di) {
  constexpr int SC = win_slab<InT>();
  constexpr int EY = kWinTY / RG;
  const size_t smem = win_smem_bytes<InT, TWO_SEG>(p.m, RG);
  if (smem > di.smem_optin) return KVC_ERR_UNSUPPORTED;
  auto kern = window_pool_kernel<InT, OutT, TWO_SEG, RG, LISTED, CACHE>;
  const int occ = resident_blocks(kern, kWinCG * kWinTY, smem);
  if (occ == 0) return KVC_ERR_CUDA;
  const int64_t gx = ceil_div(p.c, SC);
  const int64_t batch = LISTED ? 1 : p.batch;
  const int64_t gz = batch < 65535 ? batch : 65535;
  const int64_t need = ceil_div(LISTED ? p.num : p.ne, EY);
  int64_t gy = static_cast<int64_t>(di.sms) * occ / (gx * gz);
  if (gy < 1) gy = 1;
  if (gy > need) gy = need;
  if (gy > 65535) gy = 65535;
  gy = ceil_div(need, ceil_div(need, gy));
  // The entry list is its own parameter: inside WinArgs it made ptxas spill the dense path.
  WinArgs args{p.C0, p.Z0, p.C1, p.Z1, p.B0, p.B1, batch, p.n, p.c, p.ne, p.m, p.out};
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), static_cast<unsigned>(gz)),
         dim3(kWinCG, kWinTY), smem, st>>>(args, entry_list(p), cache_arg<CACHE>(p));
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = RG == 1 ? "window_pool_kernel/rg1" : RG == 4 ? "window_pool_kernel/rg4"
                                                               : "window_pool_kernel/rg16";
  return KVC_OK;
}

// The pipelined few-window kernel (one segment, dense streams), same grid as above.
template <typename InT, typename OutT, int RG>
kvc_status launch_window_pipe(const StreamProblem& p, cudaStream_t st, const DeviceInfo& di) {
  constexpr int SC = win_slab<InT>();
  constexpr int EY = kWinTY / RG;
  const size_t smem = win_smem_bytes<InT, false>(p.m, RG);
  if (smem > di.smem_optin) return KVC_ERR_UNSUPPORTED;
  auto kern = window_pipe_kernel<InT, OutT, RG>;
  const int occ = resident_blocks(kern, kWinCG * kWinTY, smem);
  if (occ == 0) return KVC_ERR_CUDA;
  const int64_t gx = ceil_div(p.c, SC);
  const int64_t gz = p.batch < 65535 ? p.batch : 65535;
  const int64_t need = ceil_div(p.ne, EY);
  int64_t gy = static_cast<int64_t>(di.sms) * occ / (gx * gz);
  if (gy < 1) gy = 1;
  if (gy > need) gy = need;
  if (gy > 65535) gy = 65535;
  gy = ceil_div(need, ceil_div(need, gy));
  WinArgs args{p.C0, p.Z0, p.C1, p.Z1, p.B0, p.B1, p.batch, p.n, p.c, p.ne, p.m, p.out};
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), static_cast<unsigned>(gz)),
         dim3(kWinCG, kWinTY), smem, st>>>(args);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = RG == 4 ? "window_pipe_kernel/rg4" : RG == 8 ? "window_pipe_kernel/rg8"
                                                               : "window_pipe_kernel/rg16";
  return KVC_OK;
}

// Row groups per entry: the fewest that still give every resident CTA slot a few
// iterations (one window per thread needs no merge at all).
template <typename InT, typename OutT, bool TWO_SEG, bool LISTED, bool CACHE>
kvc_status launch_window(const StreamProblem& p, cudaStream_t st) {
  constexpr int SC = win_slab<InT>();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (di.sms == 0) return KVC_ERR_CUDA;
  if constexpr (LISTED || CACHE) {
    return launch_window_rg<InT, OutT, TWO_SEG, 1, LISTED, CACHE>(p, st, di);
  } else {
    if constexpr (!TWO_SEG) {
      const kvc_status r = launch_window_tma(p, st);
      if (r != KVC_ERR_UNSUPPORTED) return r;
    }
    const int64_t tasks = p.batch * p.ne * ceil_div(p.c, SC);  // (entry, slab) pairs
    const int64_t slots = static_cast<int64_t>(di.sms) * 2;
    const int rows = TWO_SEG ? 2 * p.m : p.m;
    if (tasks >= 3 * slots * kWinTY || rows <= kWinU)
      return launch_window_rg<InT, OutT, TWO_SEG, 1, false, false>(p, st, di);
    if (tasks >= 3 * slots * (kWinTY / 4)) {
      if constexpr (!TWO_SEG) return launch_window_pipe<InT, OutT, 4>(p, st, di);
      return launch_window_rg<InT, OutT, TWO_SEG, 4, false, false>(p, st, di);
    }
    if constexpr (!TWO_SEG) {
      // measured on HCA n = 65536 (2048 tasks): 8 row groups 46.5 us, 16: 50.7, 4: 54.8
      if (tasks >= 2 * slots) return launch_window_pipe<InT, OutT, 8>(p, st, di);
      return launch_window_pipe<InT, OutT, 16>(p, st, di);
    }
    return launch_window_rg<InT, OutT, TWO_SEG, 16, false, false>(p, st, di);
  }
}

template <typename InT, typename OutT, bool LISTED, bool CACHE>
kvc_status dispatch_stream(const StreamProblem& p, cudaStream_t st) {
  if (p.two_segments) {
    if constexpr (!LISTED && !CACHE) {
      if (p.m == 4) {
        const kvc_status r = launch_csa_tma(p, st);
        if (r != KVC_ERR_UNSUPPORTED) return r;
      }
    }
    switch (p.m) {
      case 1: return launch_csa_small<InT, OutT, 1, true, LISTED, CACHE>(p, st);
      case 2: return launch_csa_small<InT, OutT, 2, true, LISTED, CACHE>(p, st);
      case 4: return launch_csa_small<InT, OutT, 4, true, LISTED, CACHE>(p, st);
      default: return launch_window<InT, OutT, true, LISTED, CACHE>(p, st);
    }
  }
  if (p.small_window_kernel) {
    switch (p.m) {
      case 1: return launch_csa_small<InT, OutT, 1, false, LISTED, CACHE>(p, st);
      case 2: return launch_csa_small<InT, OutT, 2, false, LISTED, CACHE>(p, st);
      case 4: return launch_csa_small<InT, OutT, 4, false, LISTED, CACHE>(p, st);
      default: break;
    }
  }
  return launch_window<InT, OutT, false, LISTED, CACHE>(p, st);
}

template <typename InT, typename OutT>
kvc_status dispatch_listed(const StreamProblem& p, cudaStream_t st) {
  return p.listed ? dispatch_stream<InT, OutT, true, false>(p, st)
                  : dispatch_stream<InT, OutT, false, false>(p, st);
}

// Cache layout: the output type is fixed by the layout (E4M3 + bf16).
template <typename InT>
kvc_status dispatch_cache(const StreamProblem& p, cudaStream_t st) {
  return p.listed ? dispatch_stream<InT, __nv_bfloat16, true, true>(p, st)
                  : dispatch_stream<InT, __nv_bfloat16, false, true>(p, st);
}

}  // namespace

size_t window_kernel_smem_bytes(bool bf16_in, bool two_segments, int m) {
  if (bf16_in)
    return two_segments ? win_smem_bytes<__nv_bfloat16, true>(m, 16)
                        : win_smem_bytes<__nv_bfloat16, false>(m, 16);
  return two_segments ? win_smem_bytes<float, true>(m, 16) : win_smem_bytes<float, false>(m, 16);
}

kvc_status launch_stream_pool(const StreamProblem& p, cudaStream_t st) {
  if (p.cache)
    return p.in_bf16 ? dispatch_cache<__nv_bfloat16>(p, st) : dispatch_cache<float>(p, st);
  if (p.in_bf16) {
    return p.out_bf16 ? dispatch_listed<__nv_bfloat16, __nv_bfloat16>(p, st)
                      : dispatch_listed<__nv_bfloat16, float>(p, st);
  }
  return p.out_bf16 ? dispatch_listed<float, __nv_bfloat16>(p, st)
                    : dispatch_listed<float, float>(p, st);
}

bool read_and_clear_index_error(bool* failed) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  *failed = cudaMemcpyFromSymbol(&v, g_index_error, sizeof(v)) != cudaSuccess;
  if (!*failed && v != 0)
    *failed = cudaMemcpyToSymbol(g_index_error, &zero, sizeof(zero)) != cudaSuccess;
  return v != 0;
}

}  // namespace kvc
