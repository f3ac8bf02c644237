// The per-row arithmetic of the 16-dim indexer projection x_idx = P x, shared
// by rtp_index_project and the cache append (rtp_kv_append) so that both give
// bit-identical projected keys.
//
// One warp per row: lane l holds dims 4l..4l+3 of the row and the matching
// 16x4 block of P in registers; each lane forms 16 partial sums, and a
// reduce-scatter over the warp (16 shuffles) leaves output j on lane pair
// (2j', 2j'+1).  fp32 throughout (one fixed tree order), rounded once to the
// output type.  With P a coordinate selection every output is a single exact
// product plus exact zeros, so the result is exact.
#pragma once

#include "common.cuh"

namespace rtp {

template <typename Tin>
RTP_DEVICE void load4(const Tin* p, float (&x)[4]);

template <>
RTP_DEVICE void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
  x[0] = bf16_lo(a.x);
  x[1] = bf16_hi(a.x);
  x[2] = bf16_lo(a.y);
  x[3] = bf16_hi(a.y);
}

template <>
RTP_DEVICE void load4<float>(const float* p, float (&x)[4]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  x[0] = a.x;
  x[1] = a.y;
  x[2] = a.z;
  x[3] = a.w;
}

template <typename Tout>
RTP_DEVICE void store1(Tout* p, float y);
template <>
RTP_DEVICE void store1<__nv_bfloat16>(__nv_bfloat16* p, float y) { *p = __float2bfloat16_rn(y); }
template <>
RTP_DEVICE void store1<float>(float* p, float y) { *p = y; }

// Halving step of the reduce-scatter: lanes with `bit` set keep the upper half
// of the n live values, the others the lower half, and add the partner's copy.
template <int n>
RTP_DEVICE void halve(float (&v)[kIdxDim], int lane, int bit) {
  const bool up = (lane & bit) != 0;
#pragma unroll
  for (int t = 0; t < n / 2; ++t) {
    const float keep = up ? v[t + n / 2] : v[t];
    const float give = up ? v[t] : v[t + n / 2];
    v[t] = keep + __shfl_xor_sync(0xffffffffu, give, bit);
  }
}

// Lane l holds x[4l .. 4l+3] in xv and reads P[j][4l .. 4l+3] as pl(j) (a float4:
// registers, or a load); the warp writes the 16 outputs of the row to out[0 .. 15].
template <typename Tout, typename PL>
RTP_DEVICE void project_row_with(PL pl, const float (&xv)[4], int lane, Tout* out) {
  float acc[kIdxDim];
#pragma unroll
  for (int j = 0; j < kIdxDim; ++j) {
    const float4 pj = pl(j);
    float a = __fmul_rn(pj.x, xv[0]);
    a = __fmaf_rn(pj.y, xv[1], a);
    a = __fmaf_rn(pj.z, xv[2], a);
    acc[j] = __fmaf_rn(pj.w, xv[3], a);
  }
  halve<16>(acc, lane, 16);
  halve<8>(acc, lane, 8);
  halve<4>(acc, lane, 4);
  halve<2>(acc, lane, 2);
  const float y = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
  if ((lane & 1) == 0) {
    const int j = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
    store1<Tout>(out + j, y);
  }
}

// The same with P's block held in registers: Pl[j] = P[j][4l .. 4l+3].
template <typename Tout>
RTP_DEVICE void project_row(const float (&Pl)[kIdxDim][4], const float (&xv)[4], int lane, Tout* out) {
  project_row_with<Tout>([&](int j) { return make_float4(Pl[j][0], Pl[j][1], Pl[j][2], Pl[j][3]); }, xv, lane,
                         out);
}

}  // namespace rtp
