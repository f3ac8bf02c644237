// a1: the 16-dim token indexer projection, x_idx = P x per row.
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 2: a 16-dimensional projection
// of the (post-rotary) key and query ranks tokens for retrieval heads.
//
// One warp per row: lane l holds dims 4l..4l+3 of the row and the matching
// 16x4 block of P in registers; each lane forms 16 partial sums, and a
// reduce-scatter over the warp (16 shuffles) leaves output j on lane pair
// (2j', 2j'+1).  fp32 throughout (one fixed tree order), rounded once to the
// output type.  With P a coordinate selection every output is a single exact
// product plus exact zeros, so the result is exact.
#include "common.cuh"
#include "launch.h"

namespace rtp {

constexpr int kProjThreads = 256;

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

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kProjThreads)
index_project_kernel(View4 x, const float* __restrict__ P, int H, int heads_per_p, int N, int64_t rows,
                     MutView4 out) {
  pdl_wait();
  pdl_release();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * kProjThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kProjThreads) >> 5;
  int cur_hp = -1;
  float Pl[kIdxDim][4];
  for (int64_t row = warp0; row < rows; row += nwarps) {
    const int n = (int)(row % N);
    const int64_t bh = row / N;
    const int h = (int)(bh % H), b = (int)(bh / H);
    const int hp = h / heads_per_p;
    if (hp != cur_hp) {  // warp-uniform
      const float* Ph = P + (int64_t)hp * kIdxDim * kHeadDim + 4 * lane;
#pragma unroll
      for (int j = 0; j < kIdxDim; ++j) {
        const float4 pv = __ldg(reinterpret_cast<const float4*>(Ph + j * kHeadDim));
        Pl[j][0] = pv.x;
        Pl[j][1] = pv.y;
        Pl[j][2] = pv.z;
        Pl[j][3] = pv.w;
      }
      cur_hp = hp;
    }
    float xv[4];
    load4<Tin>(static_cast<const Tin*>(x.data) + b * x.sb + h * x.sh + (int64_t)n * x.sn + 4 * lane, xv);
    float acc[kIdxDim];
#pragma unroll
    for (int j = 0; j < kIdxDim; ++j) {
      float a = __fmul_rn(Pl[j][0], xv[0]);
      a = __fmaf_rn(Pl[j][1], xv[1], a);
      a = __fmaf_rn(Pl[j][2], xv[2], a);
      acc[j] = __fmaf_rn(Pl[j][3], xv[3], a);
    }
    halve<16>(acc, lane, 16);
    halve<8>(acc, lane, 8);
    halve<4>(acc, lane, 4);
    halve<2>(acc, lane, 2);
    const float y = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
    if ((lane & 1) == 0) {
      const int j = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
      store1<Tout>(static_cast<Tout*>(out.data) + b * out.sb + h * out.sh + (int64_t)n * out.sn + j, y);
    }
  }
}

cudaError_t launch_index_project(const LaunchIndexProject& a, cudaStream_t stream) {
  const int64_t rows = a.B * a.H * a.N;
  if (rows == 0) return cudaSuccess;
  const int warps_per_block = kProjThreads / 32;
  int64_t blocks = (rows + warps_per_block - 1) / warps_per_block;
  if (blocks > 148 * 16) blocks = 148 * 16;
  const dim3 grid((unsigned)blocks);
  const int hpp = (int)(a.H / a.HP);
  const int H = (int)a.H, N = (int)a.N;
  const dim3 block(kProjThreads);
  if (a.in_bf16 && a.out_bf16)
    return launch_pdl(index_project_kernel<__nv_bfloat16, __nv_bfloat16>, grid, block, 0, stream, 1, a.x, a.P, H, hpp,
                      N, rows, a.out);
  if (a.in_bf16)
    return launch_pdl(index_project_kernel<__nv_bfloat16, float>, grid, block, 0, stream, 1, a.x, a.P, H, hpp, N, rows,
                      a.out);
  if (a.out_bf16)
    return launch_pdl(index_project_kernel<float, __nv_bfloat16>, grid, block, 0, stream, 1, a.x, a.P, H, hpp, N, rows,
                      a.out);
  return launch_pdl(index_project_kernel<float, float>, grid, block, 0, stream, 1, a.x, a.P, H, hpp, N, rows, a.out);
}

}  // namespace rtp
