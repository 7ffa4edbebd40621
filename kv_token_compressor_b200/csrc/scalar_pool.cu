// Scalar-logit compressor kernels (sm_100a).
//
// What they compute ("Ch 04 · CSA" §3, symbol table: one score per token and stream,
// an m-dimensional position bias, S_j a scalar weight on the whole vector C_j; "Ch 05 ·
// HCA" §2 likewise with an m'-dimensional bias): for entry i the window's logits are
// [z^a_{mi..m(i+1)-1} + b^a ; z^b_{m(i-1)..mi-1} + b^b] (HCA: z + b over the segment),
// one softmax over them, and C^Comp_i = sum_j S_j C_j with the same weights for every
// channel.  Entry 0 has no b-rows (eq. attn-seqcomp-overlap-bound of "序列压缩注意力").
//
// Small CSA windows (m <= 4): one thread per entry and 16-byte channel vector (below).
// Other windows: one warp = one entry x a slab of 32 channel vectors (256 bf16 / 128 fp32).
// The warp first turns the window's scalar logits into weights (lanes split the rows;
// shuffle max and sum; one exp2 per row), keeps them in shared memory, then every lane
// streams its 16-byte vector of each window row (8 rows in flight) and accumulates the
// weighted sum with packed f32x2 FMAs.  HBM-bound: the value streams are read once.
#include "kvc_common.cuh"
#include "kvc_host.h"
#include "kvc_launch.h"

namespace kvc {

namespace {

struct ScalarArgs {
  const void* C0;  // value stream of segment 0 (C^a / the HCA stream)
  const void* Z0;  // scalar logits of segment 0 [batch, n]
  const void* C1;  // segment 1 (b-rows), TWO_SEG only
  const void* Z1;
  const float* B0;  // [m]
  const float* B1;  // [m], TWO_SEG only
  int64_t batch, n, c, ne;
  int m;
  void* out;
};

constexpr int kScWarps = 8;  // warps per CTA
constexpr int kScU = 8;      // rows in flight per lane

template <typename T>
__device__ __forceinline__ float load_scalar(const T* p);
template <>
__device__ __forceinline__ float load_scalar<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float load_scalar<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename InT, typename OutT, bool TWO_SEG>
__global__ void __launch_bounds__(kScWarps * 32) scalar_pool_kernel(ScalarArgs a) {
  constexpr int CPT = VecInfo<InT>::kChannels;
  constexpr int NP = CPT / 2;
  extern __shared__ float smem_w[];  // [kScWarps][window rows] weights
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = a.m;
  const int wmax = TWO_SEG ? 2 * m : m;
  float* wts = smem_w + warp * wmax;
  const InT* C0 = static_cast<const InT*>(a.C0);
  const InT* Z0 = static_cast<const InT*>(a.Z0);
  const InT* C1 = static_cast<const InT*>(a.C1);
  const InT* Z1 = static_cast<const InT*>(a.Z1);
  OutT* out = static_cast<OutT*>(a.out);
  const int64_t G = a.c / CPT;               // channel vectors per row
  const int64_t slabs = (G + 31) / 32;
  const int64_t tasks = a.batch * a.ne * slabs;

  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kScWarps + warp; t < tasks;
       t += static_cast<int64_t>(gridDim.x) * kScWarps) {
    const int64_t slab = t % slabs;
    const int64_t e = t / slabs;
    const int64_t b = e / a.ne, i = e - (e / a.ne) * a.ne;
    const int64_t row0 = b * a.n + static_cast<int64_t>(m) * i;  // a-range(i) start
    const int rows = (TWO_SEG && i > 0) ? 2 * m : m;

    // weights of the window's rows (row v < m: segment 0; v >= m: segment 1)
    float mx = -INFINITY;
    for (int v = lane; v < rows; v += 32) {
      const bool seg1 = TWO_SEG && v >= m;
      const float z = seg1 ? load_scalar<InT>(Z1 + row0 - m + (v - m)) : load_scalar<InT>(Z0 + row0 + v);
      const float l = fmaf(z, kLog2e, (seg1 ? a.B1[v - m] : a.B0[v]) * kLog2e);
      wts[v] = l;
      mx = fmaxf(mx, l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int v = lane; v < rows; v += 32) {
      const float w = ex2_ftz(wts[v] - mx);
      wts[v] = w;
      sum += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.0f / sum;
    __syncwarp();

    const int64_t vec = slab * 32 + lane;
    if (vec < G) {
      const int64_t ch0 = vec * CPT;
      float2 A[NP];
#pragma unroll
      for (int p = 0; p < NP; ++p) A[p] = make_float2(0.f, 0.f);
      for (int v0 = 0; v0 < rows; v0 += kScU) {
        uint4 cv[kScU];
#pragma unroll
        for (int u = 0; u < kScU; ++u) {
          const int v = v0 + u;
          if (v < rows) {
            const bool seg1 = TWO_SEG && v >= m;
            const int64_t row = seg1 ? row0 - m + (v - m) : row0 + v;
            cv[u] = ld_stream16((seg1 ? C1 : C0) + row * a.c + ch0);
          }
        }
#pragma unroll
        for (int u = 0; u < kScU; ++u) {
          const int v = v0 + u;
          if (v < rows) {
            const float w = wts[v];
            const float2 w2 = make_float2(w, w);
#pragma unroll
            for (int p = 0; p < NP; ++p) A[p] = f2_fma(w2, vec_pair<InT>(cv[u], p), A[p]);
          }
        }
      }
      float res[CPT];
      const float2 inv2 = make_float2(inv, inv);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float2 r = f2_mul(A[p], inv2);
        res[2 * p] = r.x;
        res[2 * p + 1] = r.y;
      }
      store_out<OutT, CPT>(out + (b * a.ne + i) * a.c + ch0, res);
    }
    __syncwarp();  // the next task overwrites this warp's weights
  }
}

// Small windows (m in {1, 2, 4}): one thread = one entry x one 16-byte channel vector,
// the same shape as the per-channel CSA kernel.  The thread loads its window's 2m scalar
// logits (the same addresses for every thread of the entry, served by broadcast), forms
// the 2m weights itself, issues all value loads before using any, and pools.
template <typename InT, typename OutT, int M, bool OVERLAP>
__global__ void __launch_bounds__(256) scalar_small_m_kernel(ScalarArgs a) {
  constexpr int CPT = VecInfo<InT>::kChannels;
  constexpr int NP = CPT / 2;
  constexpr int NR = OVERLAP ? 2 * M : M;
  const InT* C0 = static_cast<const InT*>(a.C0);
  const InT* Z0 = static_cast<const InT*>(a.Z0);
  const InT* C1 = static_cast<const InT*>(a.C1);
  const InT* Z1 = static_cast<const InT*>(a.Z1);
  OutT* out = static_cast<OutT*>(a.out);
  float b2[NR];
#pragma unroll
  for (int k = 0; k < NR; ++k) b2[k] = (k < M ? a.B0[k] : a.B1[k - M]) * kLog2e;
  const int64_t ch0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * CPT;
  if (ch0 >= a.c) return;
  const int64_t istep = static_cast<int64_t>(gridDim.y) * blockDim.y;
  for (int64_t b = blockIdx.z; b < a.batch; b += gridDim.z) {
    for (int64_t i = static_cast<int64_t>(blockIdx.y) * blockDim.y + threadIdx.y; i < a.ne;
         i += istep) {
      const int64_t rowA = b * a.n + static_cast<int64_t>(M) * i;
      const bool has_b = OVERLAP && i > 0;
      uint4 cv[NR];
      float l[NR];
#pragma unroll
      for (int k = 0; k < M; ++k) {
        cv[k] = ld_stream16(C0 + (rowA + k) * a.c + ch0);
        l[k] = fmaf(load_scalar<InT>(Z0 + rowA + k), kLog2e, b2[k]);
      }
      if constexpr (OVERLAP) {
#pragma unroll
        for (int k = 0; k < M; ++k) {
          if (has_b) {
            cv[M + k] = ld_stream16(C1 + (rowA - M + k) * a.c + ch0);
            l[M + k] = fmaf(load_scalar<InT>(Z1 + rowA - M + k), kLog2e, b2[M + k]);
          } else {
            cv[M + k] = make_uint4(0u, 0u, 0u, 0u);  // entry 0: vector 0, logit -inf
            l[M + k] = -INFINITY;
          }
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < NR; ++k) mx = fmaxf(mx, l[k]);
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        l[k] = ex2_ftz(l[k] - mx);
        sum += l[k];
      }
      const float inv = 1.0f / sum;
      float2 A[NP];
#pragma unroll
      for (int p = 0; p < NP; ++p) A[p] = make_float2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const float2 w2 = make_float2(l[k] * inv, l[k] * inv);
#pragma unroll
        for (int p = 0; p < NP; ++p) A[p] = f2_fma(w2, vec_pair<InT>(cv[k], p), A[p]);
      }
      float res[CPT];
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        res[2 * p] = A[p].x;
        res[2 * p + 1] = A[p].y;
      }
      store_out<OutT, CPT>(out + (b * a.ne + i) * a.c + ch0, res);
    }
  }
}

template <typename InT, typename OutT, int M, bool OVERLAP>
kvc_status launch_small(const StreamProblem& p, cudaStream_t st) {
  constexpr int CPT = VecInfo<InT>::kChannels;
  const int64_t G = p.c / CPT;
  const int cg = static_cast<int>(G < 64 ? G : 64);
  const int ey = 256 / cg;
  auto kern = scalar_small_m_kernel<InT, OutT, M, OVERLAP>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  const int occ = resident_blocks(kern, cg * ey, 0);
  if (di.sms == 0 || occ == 0) return KVC_ERR_CUDA;
  const int64_t gx = ceil_div(G, cg);
  const int64_t gz = p.batch < 65535 ? p.batch : 65535;
  int64_t gy = static_cast<int64_t>(di.sms) * occ / (gx * gz);
  if (gy < 1) gy = 1;
  const int64_t need = ceil_div(p.ne, ey);
  if (gy > need) gy = need;
  if (gy > 65535) gy = 65535;
  gy = ceil_div(need, ceil_div(need, gy));
  ScalarArgs args{p.C0, p.Z0, p.C1, p.Z1, p.B0, p.B1, p.batch, p.n, p.c, p.ne, p.m, p.out};
  kern<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), static_cast<unsigned>(gz)),
         dim3(cg, ey), 0, st>>>(args);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = "scalar_small_m_kernel";
  return KVC_OK;
}

template <typename InT, typename OutT, bool TWO_SEG>
kvc_status launch(const StreamProblem& p, cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  const DeviceInfo di = device_info(dev);
  if (di.sms == 0) return KVC_ERR_CUDA;
  const size_t smem = sizeof(float) * kScWarps * (TWO_SEG ? 2 * p.m : p.m);
  auto kern = scalar_pool_kernel<InT, OutT, TWO_SEG>;
  const int occ = resident_blocks(kern, kScWarps * 32, smem);
  if (occ == 0) return KVC_ERR_CUDA;
  constexpr int CPT = VecInfo<InT>::kChannels;
  const int64_t tasks = p.batch * p.ne * ceil_div(p.c / CPT, 32);
  int64_t grid = static_cast<int64_t>(di.sms) * occ;
  const int64_t need = ceil_div(tasks, kScWarps);
  if (grid > need) grid = need;
  ScalarArgs args{p.C0, p.Z0, p.C1, p.Z1, p.B0, p.B1, p.batch, p.n, p.c, p.ne, p.m, p.out};
  kern<<<static_cast<unsigned>(grid), kScWarps * 32, smem, st>>>(args);
  if (cudaGetLastError() != cudaSuccess) return KVC_ERR_CUDA;
  last_kernel() = "scalar_pool_kernel";
  return KVC_OK;
}

template <typename InT, typename OutT>
kvc_status dispatch(const StreamProblem& p, cudaStream_t st) {
  if (p.two_segments) {
    switch (p.m) {
      case 1: return launch_small<InT, OutT, 1, true>(p, st);
      case 2: return launch_small<InT, OutT, 2, true>(p, st);
      case 4: return launch_small<InT, OutT, 4, true>(p, st);
      default: return launch<InT, OutT, true>(p, st);
    }
  }
  return launch<InT, OutT, false>(p, st);
}

}  // namespace

kvc_status launch_scalar_pool(const StreamProblem& p, cudaStream_t st) {
  if (p.in_bf16) {
    return p.out_bf16 ? dispatch<__nv_bfloat16, __nv_bfloat16>(p, st)
                      : dispatch<__nv_bfloat16, float>(p, st);
  }
  return p.out_bf16 ? dispatch<float, __nv_bfloat16>(p, st) : dispatch<float, float>(p, st);
}

}  // namespace kvc
