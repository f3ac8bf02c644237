// Merge of attention partials computed over disjoint key ranges of the same
// queries (a sequence's keys split across devices, each attending its own
// range of the selected keys).
//
// Softmax attention over a union of disjoint key sets is the weighted mean of
// the per-set attention outputs, each weighted by its share of the softmax
// denominator: with lse_s = ln sum_{j in set s} exp(score_j) and o_s the
// attention output over set s,
//     o = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M),   M = max_s lse_s.
// A set with no key has lse = -inf and weight 0; a row whose sets are all
// empty gets o = 0 (what the decode attention writes for an empty selection).
//
// One warp per (sequence, query head) row; lane l handles dims 4l .. 4l+3.
// The partials are a few hundred bytes per row: the kernel is latency-bound.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace rtp {

namespace {

constexpr int kCombThreads = 256;

__global__ void __launch_bounds__(kCombThreads) attn_combine_kernel(AttnCombineArgs A) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * kCombThreads + threadIdx.x) >> 5;
  const int64_t rows = (int64_t)A.B * A.Hq;
  if (row >= rows) return;
  const int b = (int)(row / A.Hq), h = (int)(row % A.Hq);
  float M = -INFINITY;
  for (int s = 0; s < A.S; ++s) M = fmaxf(M, __ldg(A.lse + s * A.ls + b * A.lb + h));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < A.S; ++s) {
      const float ls = __ldg(A.lse + s * A.ls + b * A.lb + h);
      if (ls == -INFINITY) continue;
      const float w = expf(ls - M);
      const float4 x =
          __ldg(reinterpret_cast<const float4*>(A.o_parts + s * A.ps + b * A.pb + h * A.ph) + lane);
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
      den += w;
    }
  }
  const float r = den > 0.f ? 1.f / den : 0.f;
  const float y0 = acc.x * r, y1 = acc.y * r, y2 = acc.z * r, y3 = acc.w * r;
  if (A.o_bf16) {
    __nv_bfloat16* op = static_cast<__nv_bfloat16*>(A.o.data) + b * A.o.sb + h * A.o.sh + 4 * lane;
    op[0] = __float2bfloat16_rn(y0);
    op[1] = __float2bfloat16_rn(y1);
    op[2] = __float2bfloat16_rn(y2);
    op[3] = __float2bfloat16_rn(y3);
  } else {
    *reinterpret_cast<float4*>(static_cast<float*>(A.o.data) + b * A.o.sb + h * A.o.sh + 4 * lane) =
        make_float4(y0, y1, y2, y3);
  }
}

}  // namespace

cudaError_t launch_attn_combine(const AttnCombineArgs& a, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.B * a.Hq;
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows * 32 + kCombThreads - 1) / kCombThreads;
  attn_combine_kernel<<<(unsigned)blocks, kCombThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rtp
