// a1: the 16-dim token indexer projection, x_idx = P x per row.
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 2: a 16-dimensional projection
// of the (post-rotary) key and query ranks tokens for retrieval heads.
//
// One thread per row: the row (128 values) streams through registers in
// 16-byte pieces while P^T sits in shared memory and is read as broadcasts.
// fp32 products summed in dimension order, then rounded once to the output
// type (round to nearest even).  With P a coordinate selection every output
// is one exact product, so the result is exact.
#include "common.cuh"
#include "launch.h"

namespace rtp {

constexpr int kProjThreads = 128;

template <typename Tin>
RTP_DEVICE void load8(const Tin* p, float (&x)[8]);

template <>
RTP_DEVICE void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8]) {
  uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = bf16_lo(w[i]);
    x[2 * i + 1] = bf16_hi(w[i]);
  }
}

template <>
RTP_DEVICE void load8<float>(const float* p, float (&x)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <typename Tout>
RTP_DEVICE void store16(Tout* p, const float (&y)[kIdxDim]);

template <>
RTP_DEVICE void store16<__nv_bfloat16>(__nv_bfloat16* p, const float (&y)[kIdxDim]) {
  uint4 a, b;
  a.x = pack_bf16x2(y[0], y[1]);   a.y = pack_bf16x2(y[2], y[3]);
  a.z = pack_bf16x2(y[4], y[5]);   a.w = pack_bf16x2(y[6], y[7]);
  b.x = pack_bf16x2(y[8], y[9]);   b.y = pack_bf16x2(y[10], y[11]);
  b.z = pack_bf16x2(y[12], y[13]); b.w = pack_bf16x2(y[14], y[15]);
  reinterpret_cast<uint4*>(p)[0] = a;
  reinterpret_cast<uint4*>(p)[1] = b;
}

template <>
RTP_DEVICE void store16<float>(float* p, const float (&y)[kIdxDim]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    reinterpret_cast<float4*>(p)[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kProjThreads)
index_project_kernel(View4 x, const float* __restrict__ P, int H, int heads_per_p, int N, MutView4 out) {
  __shared__ __align__(16) float Pt[kHeadDim][kIdxDim];  // Pt[d][j] = P[j][d]
  const int bh = blockIdx.y;
  const int b = bh / H, h = bh % H;
  const float* Ph = P + (int64_t)(h / heads_per_p) * kIdxDim * kHeadDim;
  for (int i = threadIdx.x; i < kIdxDim * kHeadDim; i += kProjThreads) {
    int j = i / kHeadDim, d = i % kHeadDim;
    Pt[d][j] = Ph[i];
  }
  __syncthreads();
  const int n = blockIdx.x * kProjThreads + threadIdx.x;
  if (n >= N) return;
  const Tin* row = static_cast<const Tin*>(x.data) + b * x.sb + h * x.sh + (int64_t)n * x.sn;
  float acc[kIdxDim];
#pragma unroll
  for (int j = 0; j < kIdxDim; ++j) acc[j] = 0.f;
#pragma unroll 2
  for (int c = 0; c < kHeadDim / 8; ++c) {
    float xv[8];
    load8<Tin>(row + c * 8, xv);
#pragma unroll
    for (int dd = 0; dd < 8; ++dd) {
      const float4* pr = reinterpret_cast<const float4*>(&Pt[c * 8 + dd][0]);
#pragma unroll
      for (int j4 = 0; j4 < 4; ++j4) {
        float4 pv = pr[j4];
        acc[4 * j4 + 0] = __fmaf_rn(pv.x, xv[dd], acc[4 * j4 + 0]);
        acc[4 * j4 + 1] = __fmaf_rn(pv.y, xv[dd], acc[4 * j4 + 1]);
        acc[4 * j4 + 2] = __fmaf_rn(pv.z, xv[dd], acc[4 * j4 + 2]);
        acc[4 * j4 + 3] = __fmaf_rn(pv.w, xv[dd], acc[4 * j4 + 3]);
      }
    }
  }
  Tout* orow = static_cast<Tout*>(out.data) + b * out.sb + h * out.sh + (int64_t)n * out.sn;
  store16<Tout>(orow, acc);
}

cudaError_t launch_index_project(const LaunchIndexProject& a, cudaStream_t stream) {
  if (a.B == 0 || a.H == 0 || a.N == 0) return cudaSuccess;
  dim3 grid((unsigned)((a.N + kProjThreads - 1) / kProjThreads), (unsigned)(a.B * a.H));
  const int hpp = a.H / a.HP;
  if (a.in_bf16 && a.out_bf16)
    index_project_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, kProjThreads, 0, stream>>>(a.x, a.P, a.H, hpp, a.N, a.out);
  else if (a.in_bf16)
    index_project_kernel<__nv_bfloat16, float><<<grid, kProjThreads, 0, stream>>>(a.x, a.P, a.H, hpp, a.N, a.out);
  else if (a.out_bf16)
    index_project_kernel<float, __nv_bfloat16><<<grid, kProjThreads, 0, stream>>>(a.x, a.P, a.H, hpp, a.N, a.out);
  else
    index_project_kernel<float, float><<<grid, kProjThreads, 0, stream>>>(a.x, a.P, a.H, hpp, a.N, a.out);
  return cudaGetLastError();
}

}  // namespace rtp
