// Cache maintenance around the path: appending the new tokens of a sequence.
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 1: retrieval heads keep the
// full KV cache, local heads only a local window; "Full Attention Strikes Back
// ... (RTPurbo)", TL;DR: the lightweight token indexer keeps a projected key
// per cached token of the retrieval heads.
//
// One warp per new (sequence, KV head, token) row, in one pass over the row:
//   retrieval head (kv head < R): the K and V rows go to the full cache at the
//     token's position, and the projected key P k to the projected-key cache
//     (the arithmetic of rtp_index_project, so both give identical bits);
//   local head: the K and V rows go to a ring of W rows at position mod W, so
//     the ring always holds the last W tokens (every key a local query of the
//     newest token attends) in O(W) memory.
// Attention over a set of keys does not depend on their order, so the window
// attention of the newest token is the ordinary window attention over the
// min(n, W) stored ring rows; the kernel writes that length per sequence, and
// the sequence length after the append (the next append's position).
#include "common.cuh"
#include "launch.h"
#include "project.cuh"

#include <type_traits>

namespace rtp {

namespace {

constexpr int kAppThreads = 256;

constexpr int kAppUnroll = 2;  // rows per warp in flight (their loads issued together)

// 128 elements of a row: 4 per lane, 8 bytes (bf16) or 16 bytes (f32).
template <typename T>
struct Row4 {
  using V = typename std::conditional<sizeof(T) == 2, uint2, float4>::type;
  V x;
  RTP_DEVICE void load(const T* row, int lane) { x = __ldg(reinterpret_cast<const V*>(row + 4 * lane)); }
  RTP_DEVICE void store(T* row, int lane) const { *reinterpret_cast<V*>(row + 4 * lane) = x; }
  RTP_DEVICE void to_float(float (&f)[4]) const {
    if constexpr (sizeof(T) == 2) {
      f[0] = bf16_lo(x.x);
      f[1] = bf16_hi(x.x);
      f[2] = bf16_lo(x.y);
      f[3] = bf16_hi(x.y);
    } else {
      f[0] = x.x;
      f[1] = x.y;
      f[2] = x.z;
      f[3] = x.w;
    }
  }
};

constexpr int kAppSmemHeads = 8;  // P of up to this many retrieval heads is staged in shared memory

template <typename T>
__global__ void __launch_bounds__(kAppThreads, 3)
kv_append_kernel(KvAppendArgs A) {
  // P [R, 16, 128] f32 in shared memory (32 KB per 4 heads), read there by every projection
  extern __shared__ float4 p_smem[];
  const bool p_in_smem = A.R <= kAppSmemHeads;
  if (p_in_smem)
    for (int i = threadIdx.x; i < A.R * kIdxDim * kHeadDim / 4; i += kAppThreads)
      p_smem[i] = __ldg(reinterpret_cast<const float4*>(A.P) + i);
  __syncthreads();
  const float4* P4 = p_in_smem ? p_smem : reinterpret_cast<const float4*>(A.P);
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = ((int64_t)blockIdx.x * kAppThreads + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * kAppThreads) >> 5;
  const int64_t rows = (int64_t)A.B * A.H * A.T;
  for (int64_t r0 = warp0; r0 < rows; r0 += kAppUnroll * nwarps) {
    // up to kAppUnroll rows of this warp: every load first, then the writes
    Row4<T> kx[kAppUnroll], vx[kAppUnroll];
    T* kdst[kAppUnroll];
    T* vdst[kAppUnroll];
    T* idst[kAppUnroll];
    int hrow[kAppUnroll];
#pragma unroll
    for (int u = 0; u < kAppUnroll; ++u) {
      const int64_t r = r0 + u * nwarps;
      kdst[u] = nullptr;
      if (r >= rows) continue;
      const int t = (int)(r % A.T);
      const int64_t bh = r / A.T;
      const int h = (int)(bh % A.H), b = (int)(bh / A.H);
      const int p = A.pos[b] + t;  // position of this token in its sequence
      hrow[u] = h;
      idst[u] = nullptr;
      if (h < A.R) {
        if (p < 0 || p >= A.N) continue;  // outside the cache: nothing written
        kdst[u] = static_cast<T*>(A.k_cache.data) + b * A.k_cache.sb + h * A.k_cache.sh + (int64_t)p * A.k_cache.sn;
        vdst[u] = static_cast<T*>(A.v_cache.data) + b * A.v_cache.sb + h * A.v_cache.sh + (int64_t)p * A.v_cache.sn;
        idst[u] = static_cast<T*>(A.k_idx.data) + b * A.k_idx.sb + h * A.k_idx.sh + (int64_t)p * A.k_idx.sn;
      } else {
        // only the last W tokens of the append are kept (two tokens W apart share a slot)
        if (p < 0 || t < A.T - A.W) continue;
        const int l = h - A.R;
        const int slot = p % A.W;
        kdst[u] = static_cast<T*>(A.k_ring.data) + b * A.k_ring.sb + l * A.k_ring.sh + (int64_t)slot * A.k_ring.sn;
        vdst[u] = static_cast<T*>(A.v_ring.data) + b * A.v_ring.sb + l * A.v_ring.sh + (int64_t)slot * A.v_ring.sn;
      }
      kx[u].load(static_cast<const T*>(A.k_new.data) + b * A.k_new.sb + h * A.k_new.sh + (int64_t)t * A.k_new.sn,
                 lane);
      vx[u].load(static_cast<const T*>(A.v_new.data) + b * A.v_new.sb + h * A.v_new.sh + (int64_t)t * A.v_new.sn,
                 lane);
    }
#pragma unroll
    for (int u = 0; u < kAppUnroll; ++u) {
      if (!kdst[u]) continue;  // warp-uniform
      kx[u].store(kdst[u], lane);
      vx[u].store(vdst[u], lane);
      if (idst[u]) {
        // P[h][j][4 lane .. 4 lane + 3] is float4 number (h * 16 + j) * 32 + lane
        const float4* Ph = P4 + (int64_t)hrow[u] * kIdxDim * (kHeadDim / 4) + lane;
        float xv[4];
        kx[u].to_float(xv);  // the loaded key row: the inputs of rtp_index_project, bit for bit
        project_row_with<T>([&](int j) { return Ph[j * (kHeadDim / 4)]; }, xv, lane, idst[u]);
      }
    }
  }
  if (blockIdx.x == 0) {
    for (int b = threadIdx.x; b < A.B; b += kAppThreads) {
      const int end = A.pos[b] + A.T;  // one past the last appended position
      if (A.lens_out) A.lens_out[b] = A.R > 0 ? max(min(end, A.N), 0) : max(end, 0);
      if (A.ring_lens) A.ring_lens[b] = max(min(end, A.W), 0);
    }
  }
}

}  // namespace

cudaError_t launch_kv_append(const KvAppendArgs& a, bool bf16, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.B * a.H * a.T;
  if (a.B == 0 || (rows == 0 && !a.lens_out && !a.ring_lens)) return cudaSuccess;
  int64_t blocks = (rows + kAppUnroll * (kAppThreads / 32) - 1) / (kAppUnroll * (kAppThreads / 32));
  if (blocks < 1) blocks = 1;  // an empty append still writes the lengths
  if (blocks > 148 * 16) blocks = 148 * 16;
  const size_t smem = a.R <= kAppSmemHeads ? (size_t)a.R * kIdxDim * kHeadDim * sizeof(float) : 0;
  if (bf16) {
    cudaFuncSetAttribute(kv_append_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kv_append_kernel<__nv_bfloat16><<<(unsigned)blocks, kAppThreads, smem, stream>>>(a);
  } else {
    cudaFuncSetAttribute(kv_append_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kv_append_kernel<float><<<(unsigned)blocks, kAppThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace rtp
