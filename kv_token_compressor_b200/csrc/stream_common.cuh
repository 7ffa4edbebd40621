// Device helpers shared by the streaming softmax-pool kernels: bias staging in shared
// memory and the bias-spread rule of the fast chunk maximum.
#pragma once

#include "kvc_common.cuh"

namespace kvc {

// Stages `nrows` bias rows of a channel slab, pre-scaled by log2 e, into shared memory:
// row k comes from B0 row k (k < m0) or B1 row k - m0, slab channel sc goes to
// dst[k * SC + pos(sc)] (channels past c read 0).  The loads are issued kBiasBatch at a
// time per thread so that they overlap: this stage sits at the start of every CTA, and
// one dependent L2 round trip per value made it a sizeable part of short launches.
// Returns this thread's (max, min) over the values it staged.
constexpr int kBiasBatch = 16;

template <typename PosFn>
__device__ __forceinline__ float2 stage_bias(float* dst, const float* B0, const float* B1, int m0,
                                             int nrows, int SC, int64_t ch_base, int64_t c,
                                             int tid, int nthr, PosFn pos) {
  float lmax = -INFINITY, lmin = INFINITY;
  const int total = nrows * SC;
  for (int base = tid; base < total; base += nthr * kBiasBatch) {
    float v[kBiasBatch];
#pragma unroll
    for (int r = 0; r < kBiasBatch; ++r) {
      const int idx = base + r * nthr;
      v[r] = 0.f;
      if (idx < total) {
        const int k = idx / SC;
        const int64_t ch = ch_base + (idx - k * SC);
        if (ch < c) v[r] = __ldg(k < m0 ? B0 + k * c + ch : B1 + (k - m0) * c + ch);
      }
    }
#pragma unroll
    for (int r = 0; r < kBiasBatch; ++r) {
      const int idx = base + r * nthr;
      if (idx < total) {
        const int k = idx / SC;
        const float x = v[r] * kLog2e;
        dst[k * SC + pos(idx - k * SC)] = x;
        lmax = fmaxf(lmax, x);
        lmin = fminf(lmin, x);
      }
    }
  }
  return make_float2(lmax, lmin);
}

// Largest per-channel spread of the (log2 e-scaled) bias rows for which a chunk's maximum
// logit may be bounded by max(z) * log2 e + max(b) instead of taken row by row.
constexpr float kMaxBiasSpread = 64.f;

// Position of slab channel sc in a shared-memory bias row when CG thread groups of CPT
// channels share the slab: float4 q of thread group g sits at (q * CG + g) * 4, so a warp's
// reads of one float4 per thread group are contiguous and hit no bank twice.
template <int CPT, int CG>
__device__ __forceinline__ int slab_bias_pos(int sc) {
  const int g = sc / CPT, j = sc - (sc / CPT) * CPT;
  return ((j >> 2) * CG + g) * 4 + (j & 3);
}

}  // namespace kvc
