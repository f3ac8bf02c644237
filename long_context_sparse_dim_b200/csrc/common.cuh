// Shared device helpers for the RTPurbo sm_100a kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rtp.h"

#define RTP_DEVICE __device__ __forceinline__

namespace rtp {

constexpr int kHeadDim = 128;  // full head dimension
constexpr int kIdxDim = 16;    // indexer dimension

// Strided 4-D view [B, H, N, D] passed to kernels (element strides; D contiguous).
struct View4 {
  const void* data;
  int64_t sb, sh, sn;
};
struct MutView4 {
  void* data;
  int64_t sb, sh, sn;
};

// ---- scalar conversions --------------------------------------------------
RTP_DEVICE float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
RTP_DEVICE float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

RTP_DEVICE uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&r);
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key).
// Scores are canonicalised first so that -0 and +0 map to one key.
RTP_DEVICE uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
RTP_DEVICE float key_score(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// ---- the indexer score ----------------------------------------------------
// s = (q_idx . k_idx) / 4 in fp32 with one fixed summation order: the products
// of two bf16 values are exact in fp32; each step is one fused multiply-add in
// index order; the final scale is exact (power of two); adding +0 maps -0 to +0.
// Every CUDA-core consumer of a score uses this one function.
RTP_DEVICE float indexer_dot16(const float (&q)[kIdxDim], const float (&k)[kIdxDim]) {
  float acc = __fmul_rn(q[0], k[0]);
#pragma unroll
  for (int t = 1; t < kIdxDim; ++t) acc = __fmaf_rn(q[t], k[t], acc);
  return __fadd_rn(__fmul_rn(acc, 0.25f), 0.0f);
}

template <typename T>
RTP_DEVICE void load_idx_row(const T* row, float (&k)[kIdxDim]);

template <>
RTP_DEVICE void load_idx_row<__nv_bfloat16>(const __nv_bfloat16* row, float (&k)[kIdxDim]) {
  const uint4* p = reinterpret_cast<const uint4*>(row);
  uint4 a = __ldg(p), b = __ldg(p + 1);
  uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    k[2 * i] = bf16_lo(w[i]);
    k[2 * i + 1] = bf16_hi(w[i]);
  }
}

template <>
RTP_DEVICE void load_idx_row<float>(const float* row, float (&k)[kIdxDim]) {
  const float4* p = reinterpret_cast<const float4*>(row);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 v = __ldg(p + i);
    k[4 * i] = v.x;
    k[4 * i + 1] = v.y;
    k[4 * i + 2] = v.z;
    k[4 * i + 3] = v.w;
  }
}

// A projected-key row as raw 16-byte vectors (2 for bf16, 4 for fp32), so that
// several rows can be in flight per thread before any conversion.
template <typename T>
struct IdxRaw {
  static constexpr int kVec = sizeof(T) == 2 ? 2 : 4;
  uint4 v[kVec];
};

template <typename T>
RTP_DEVICE void load_idx_raw(const T* row, IdxRaw<T>& r) {
  const uint4* p = reinterpret_cast<const uint4*>(row);
#pragma unroll
  for (int i = 0; i < IdxRaw<T>::kVec; ++i) r.v[i] = __ldg(p + i);
}

template <typename T>
RTP_DEVICE void idx_raw_to_float(const IdxRaw<T>& r, float (&k)[kIdxDim]) {
  if constexpr (sizeof(T) == 2) {
    const uint32_t w[8] = {r.v[0].x, r.v[0].y, r.v[0].z, r.v[0].w, r.v[1].x, r.v[1].y, r.v[1].z, r.v[1].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      k[2 * i] = bf16_lo(w[i]);
      k[2 * i + 1] = bf16_hi(w[i]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      k[4 * i] = __uint_as_float(r.v[i].x);
      k[4 * i + 1] = __uint_as_float(r.v[i].y);
      k[4 * i + 2] = __uint_as_float(r.v[i].z);
      k[4 * i + 3] = __uint_as_float(r.v[i].w);
    }
  }
}

// Fixed-point top-p weight: round(exp(s - m) * 2^frac) as an unsigned 64-bit
// integer.  With frac = 63 - ceil(log2 n) a sum over n keys cannot overflow,
// and integer sums do not depend on the order of accumulation.
RTP_DEVICE uint64_t fixed_weight(float s, float m, float two_pow_frac) {
  float e = expf(__fsub_rn(s, m));
  return __float2ull_rn(__fmul_rn(e, two_pow_frac));
}

// ---- programmatic dependent launch -----------------------------------------
// A kernel launched with programmatic stream serialization may start while the
// previous kernel of its stream is still finishing; pdl_wait() blocks until that
// kernel has completed and its writes are visible (a no-op otherwise), and
// pdl_release() lets the next kernel of the stream be launched early.
RTP_DEVICE void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
RTP_DEVICE void pdl_release() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---- warp helpers ----------------------------------------------------------
RTP_DEVICE float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
RTP_DEVICE float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace rtp
