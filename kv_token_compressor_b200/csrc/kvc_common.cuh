// Shared device helpers of the sm_100a compressor kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/kvc.h"

namespace kvc {

constexpr float kLog2e = 1.4426950408889634f;

// 16-byte streaming load: read once, no L1 allocation, 256-byte L2 prefetch.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// Streaming (evict-first) stores.
__device__ __forceinline__ void st_stream16(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_stream8(void* p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// Element j of a 16-byte vector holding 8 bf16 or 4 fp32 values, widened to fp32.
template <typename T>
__device__ __forceinline__ float vec_elem(const uint4& v, int j);

template <>
__device__ __forceinline__ float vec_elem<__nv_bfloat16>(const uint4& v, int j) {
  const uint32_t w = (j >> 1) == 0 ? v.x : (j >> 1) == 1 ? v.y : (j >> 1) == 2 ? v.z : v.w;
  return __uint_as_float((j & 1) ? (w & 0xffff0000u) : (w << 16));
}
template <>
__device__ __forceinline__ float vec_elem<float>(const uint4& v, int j) {
  const uint32_t w = j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
  return __uint_as_float(w);
}

// 2^x on the special-function unit, flushing subnormal results to zero (weights below
// 2^-126 of the window maximum are negligible next to the maximum's weight of 1;
// 2^-inf = +0, which the entry-0 boundary relies on).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction for two lanes of math).
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2_max(float2 a, float2 b) {
  return make_float2(fmaxf(a.x, b.x), fmaxf(a.y, b.y));
}
__device__ __forceinline__ float2 f2_ex2(float2 a) { return make_float2(ex2_ftz(a.x), ex2_ftz(a.y)); }

// Channel pair p (channels 2p, 2p+1) of a 16-byte vector of T, widened to fp32.
template <typename T>
__device__ __forceinline__ float2 vec_pair(const uint4& v, int p);
template <>
__device__ __forceinline__ float2 vec_pair<__nv_bfloat16>(const uint4& v, int p) {
  const uint32_t w = p == 0 ? v.x : p == 1 ? v.y : p == 2 ? v.z : v.w;
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
template <>
__device__ __forceinline__ float2 vec_pair<float>(const uint4& v, int p) {
  return p == 0 ? make_float2(__uint_as_float(v.x), __uint_as_float(v.y))
                : make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}

// Lane-wise maximum of two 16-byte vectors of T, in T (bf16: max.bf16x2, two lanes per
// instruction; exact, since a maximum only selects).
template <typename T>
__device__ __forceinline__ uint4 vec_max(const uint4& a, const uint4& b);
template <>
__device__ __forceinline__ uint4 vec_max<__nv_bfloat16>(const uint4& a, const uint4& b) {
  uint4 r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r.x) : "r"(a.x), "r"(b.x));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r.y) : "r"(a.y), "r"(b.y));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r.z) : "r"(a.z), "r"(b.z));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r.w) : "r"(a.w), "r"(b.w));
  return r;
}
template <>
__device__ __forceinline__ uint4 vec_max<float>(const uint4& a, const uint4& b) {
  return make_uint4(__float_as_uint(fmaxf(__uint_as_float(a.x), __uint_as_float(b.x))),
                    __float_as_uint(fmaxf(__uint_as_float(a.y), __uint_as_float(b.y))),
                    __float_as_uint(fmaxf(__uint_as_float(a.z), __uint_as_float(b.z))),
                    __float_as_uint(fmaxf(__uint_as_float(a.w), __uint_as_float(b.w))));
}

// Channels carried by one 16-byte vector of T.
template <typename T>
struct VecInfo {
  static constexpr int kChannels = 16 / sizeof(T);
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Store CPT consecutive fp32 results as OutT (fp32 or bf16, RNE) with streaming stores.
template <typename OutT, int CPT>
__device__ __forceinline__ void store_out(OutT* dst, const float (&v)[CPT]) {
  if constexpr (sizeof(OutT) == 2) {
    static_assert(CPT == 8 || CPT == 4, "bf16 output vector");
    if constexpr (CPT == 8) {
      st_stream16(dst, make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                  pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7])));
    } else {
      st_stream8(dst, make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3])));
    }
  } else {
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q)
      st_stream16(dst + 4 * q, make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                          __float_as_uint(v[4 * q + 2]),
                                          __float_as_uint(v[4 * q + 3])));
  }
}

// Store one fp32 result as OutT.
template <typename OutT>
__device__ __forceinline__ void store_scalar(OutT* dst, float v) {
  if constexpr (sizeof(OutT) == 2) {
    *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(v);
  } else {
    *dst = v;
  }
}

// Cache layout of an entry ("Ch 05 · HCA" §4 (2): RoPE on the last r dimensions only,
// rotating adjacent pairs; the comparison article's storage split: BF16 for the RoPE part,
// FP8 for the rest).  nope: [rows, c - r] E4M3 bytes = entry[:c-r] * scale, round to
// nearest even, saturating; rope: [rows, r] bf16 = entry[c-r:] with pair j rotated by
// (pos_offset + pos_stride * i) * inv_freq[j], i = the entry's index in its sequence.
struct CacheFmt {
  uint8_t* nope;
  __nv_bfloat16* rope;
  const float* inv_freq;  // [r / 2]
  int64_t cn, r;          // c - r, r
  double pos_stride, pos_offset;
  float scale;
};
struct NoCache {};

// Sine and cosine of the RoPE angle of pair j of entry `entry`: the angle is formed in
// fp64 and reduced by a multiple of 2 pi in fp64, then the fp32 sine and cosine of the
// remainder (|red| <= pi) are taken.  pos is exact for the usual integer or half-integer
// offsets and strides; the product with inv_freq and the reduction each add at most a few
// units of 2^-53 relative to |ang| (about 1e-10 rad at |ang| = 1e6), far below the fp32
// rounding of the remainder (about 2e-7 rad near pi).
__device__ __forceinline__ void rope_sincos(const CacheFmt& cf, int64_t entry, int64_t j,
                                            float* sn, float* cs) {
  const double pos = cf.pos_offset + cf.pos_stride * static_cast<double>(entry);
  const double ang = pos * static_cast<double>(cf.inv_freq[j]);
  const double turns = rint(ang * 0.15915494309189535);
  const float red = static_cast<float>(fma(-turns, 6.283185307179586, ang));
  sincosf(red, sn, cs);
}

// One result per lane of a full warp whose lanes hold consecutive channels (ch has the
// lane's parity), stored in the cache layout: a channel below c - r as one E4M3 byte of
// v * scale; a RoPE channel as bf16, rotated together with its pair partner, which is the
// adjacent lane (exchanged by a shuffle, so every lane of the warp must make the call;
// lanes with live == false store nothing).
__device__ __forceinline__ void store_cache_lane(const CacheFmt& cf, int64_t orow, int64_t ch,
                                                 int64_t entry, float v, bool live) {
  const float partner = __shfl_xor_sync(0xffffffffu, v, 1);
  if (!live) return;
  if (ch < cf.cn) {
    cf.nope[orow * cf.cn + ch] =
        static_cast<uint8_t>(__nv_cvt_float_to_fp8(v * cf.scale, __NV_SATFINITE, __NV_E4M3));
  } else {
    const int64_t off = ch - cf.cn;
    float sn, cs;
    rope_sincos(cf, entry, off >> 1, &sn, &cs);
    const bool odd = (off & 1) != 0;
    const float x = odd ? partner : v, y = odd ? v : partner;
    const float res = odd ? fmaf(x, sn, y * cs) : fmaf(x, cs, -y * sn);
    cf.rope[orow * cf.r + off] = __float2bfloat16_rn(res);
  }
}

// Store the CPT results of channels [ch0, ch0 + CPT) of entry `entry` (output row orow)
// in the cache layout.  A thread's vector lies wholly in one part (r % 8 == 0).
template <int CPT>
__device__ __forceinline__ void store_cache(const CacheFmt& cf, int64_t orow, int64_t ch0,
                                            int64_t entry, const float (&v)[CPT]) {
  if (ch0 < cf.cn) {
    uint32_t w[CPT / 4];
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q) {
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(
          make_float2(v[4 * q] * cf.scale, v[4 * q + 1] * cf.scale), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(
          make_float2(v[4 * q + 2] * cf.scale, v[4 * q + 3] * cf.scale), __NV_SATFINITE, __NV_E4M3);
      w[q] = lo | (hi << 16);
    }
    uint8_t* dst = cf.nope + orow * cf.cn + ch0;
    if constexpr (CPT == 8) {
      st_stream8(dst, make_uint2(w[0], w[1]));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = w[0];
    }
  } else {
    const int64_t off = ch0 - cf.cn;  // channel offset inside the rope part (even)
    float rot[CPT];
#pragma unroll
    for (int p = 0; p < CPT / 2; ++p) {
      float sn, cs;
      rope_sincos(cf, entry, off / 2 + p, &sn, &cs);
      const float x = v[2 * p], y = v[2 * p + 1];
      rot[2 * p] = fmaf(x, cs, -y * sn);
      rot[2 * p + 1] = fmaf(x, sn, y * cs);
    }
    store_out<__nv_bfloat16, CPT>(cf.rope + orow * cf.r + off, rot);
  }
}

}  // namespace kvc
