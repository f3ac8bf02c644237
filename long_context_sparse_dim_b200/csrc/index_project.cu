// a1: the 16-dim token indexer projection, x_idx = P x per row.
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 2: a 16-dimensional projection
// of the (post-rotary) key and query ranks tokens for retrieval heads.
//
// One warp per row (the arithmetic is project_row in project.cuh, shared with
// the cache append so that both give bit-identical projected keys).
#include "common.cuh"
#include "launch.h"
#include "project.cuh"

namespace rtp {

constexpr int kProjThreads = 256;

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
    project_row<Tout>(Pl, xv, lane, static_cast<Tout*>(out.data) + b * out.sb + h * out.sh + (int64_t)n * out.sn);
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
