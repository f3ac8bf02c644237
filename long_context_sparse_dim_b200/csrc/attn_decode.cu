// a4 / a5 (decode): attention of one new token per sequence over
//   - its selected keys (retrieval heads; the top-p mask from rtp_topp_select), or
//   - the last W keys (local heads, sliding window).
//
// "Full Attention Strikes Back ... (RTPurbo)", TL;DR: retrieval heads keep the
// full KV cache and attend the tokens the indexer picks; "RTPurbo: Turning
// Dense LLMs into Sparse Attention Models ...", "Three Key Insights" 1: local
// heads keep only a local window.
//
// Design (B200): decode attention is an HBM stream, so the kernel is built
// around moving each needed K/V row exactly once:
//   * one CTA per (sequence, KV head, key chunk): the whole GQA group of query
//     heads is served from one read of every K/V row that ANY head of the group
//     selected (the union of the group's masks); rows nobody selected are never
//     loaded and 64-key tiles nobody selected are skipped;
//   * rows are gathered with 16-byte cp.async into a shared-memory ring of 3
//     stages (2 for the window, so that its CTAs fit beside the selection's on
//     an SM; both kernels ask for the largest shared-memory carveout)
//     (XOR-swizzled 256-byte rows so ldmatrix is conflict-free);
//   * bf16 tensor-core math (mma.sync m16n8k16) with the KEYS on the M side and
//     the query heads of the group on N (8 columns; G <= 8), so a GQA group of
//     4 wastes half a column tile instead of 3/4 of a row tile; the score
//     fragment is turned into the P^T operand in registers with movmatrix;
//   * P is fed to the PV product as a bf16 hi + lo pair (two MMAs), so the
//     probabilities keep ~16 bits instead of bf16's 8;
//   * split-K partials (max, sum, unnormalised output) go to the caller's
//     workspace; the last CTA of each group to finish (atomic ticket, no
//     waiting) merges them and resets its ticket.
// The fp32 variant (CUDA cores) serves fp32 caches.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace rtp {

constexpr int kAttnThreads = 128;  // 4 warps
constexpr int kTileKeys = 64;      // keys per pipeline stage (16 per warp)
constexpr int kStagesSparse = 3;  // pipeline depth of the gather (retrieval heads)
constexpr int kStagesWindow = 2;  // and of the window (local heads): a smaller footprint lets its CTAs share
                                  // SMs with the selection kernel, which runs concurrently
constexpr int kRowBytes = kHeadDim * 2;  // 256 B per bf16 row
constexpr int kTileBytes = kTileKeys * kRowBytes;
constexpr int kMaxGroup = 8;
constexpr int kMaxChunk = 8192;                 // keys per CTA at most
constexpr int kMaxChunkWords = kMaxChunk / 32;  // mask words per head per CTA
constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
  View4 q, k, v;
  const int32_t* lens;
  const uint32_t* mask;
  int64_t mask_words;
  int Hq, Hk, G, N, W;
  int chunk, splits;
  float scale_log2;
  MutView4 o;
  int o_bf16;
  int key_lo;     // global position of key row 0 (a key range of a longer sequence)
  float* lse;     // [B, Hq] (row stride lse_sb) or null: natural-log sum of exp(scaled scores)
  int64_t lse_sb; //   over the keys attended
  float* ws_o;    // [groups][splits][kMaxGroup][128]
  float* ws_ml;   // [groups][splits][kMaxGroup][2]
  uint32_t* tickets;  // [groups]
};

// ---- PTX wrappers ---------------------------------------------------------
RTP_DEVICE uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

RTP_DEVICE void cp_async16(uint32_t dst, const void* src, bool pred) {
  const int n = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
RTP_DEVICE void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
RTP_DEVICE void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

RTP_DEVICE void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
RTP_DEVICE void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
RTP_DEVICE uint32_t movm_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}
RTP_DEVICE void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
RTP_DEVICE float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Offset of 16-byte chunk `c` of tile row `r` (rows of 256 B, chunk index XOR row%8).
RTP_DEVICE uint32_t swz(int r, int c) { return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4)); }

struct KeyRange {
  int lo, hi;  // keys of the group: [lo, hi)
  int c0, c1;  // this CTA's chunk
};

RTP_DEVICE KeyRange key_range(const AttnArgs& A, int b, int split) {
  int n_b = A.N;  // rows of this call's K/V: keys key_lo .. key_lo + n_b - 1 of the sequence
  if (A.lens) n_b = min(max(A.lens[b] - A.key_lo, 0), A.N);
  // a key range may run past the keys the selection covers: those are not selected
  if (A.W <= 0) n_b = (int)min((int64_t)n_b, max(A.mask_words * 32 - A.key_lo, (int64_t)0));
  KeyRange r;
  r.hi = n_b;
  r.lo = A.W > 0 ? max(0, n_b - A.W) : 0;
  r.c0 = r.lo + split * A.chunk;
  r.c1 = min(r.hi, r.c0 + A.chunk);
  if (r.c1 < r.c0) r.c1 = r.c0;
  return r;
}

// ---- split partial write + last-CTA merge (shared by both variants) --------
// part_o[h][d] (unnormalised), part_m[h] (log2 domain), part_l[h] are in smem;
// `scratch` holds at least 2 * kMaxSplits * kMaxGroup + 2 * kMaxGroup floats.
constexpr int kMaxSplits = 256;  // >= one split per SM for a single (sequence, KV head) group

__device__ void finish_split(const AttnArgs& A, int grp, int split, const float* part_o,
                             const float* part_m, const float* part_l, int* flag_smem, float* scratch) {
  const int tid = threadIdx.x;
  const int G = A.G;
  float* wo = A.ws_o + ((int64_t)grp * A.splits + split) * kMaxGroup * kHeadDim;
  float* wml = A.ws_ml + ((int64_t)grp * A.splits + split) * kMaxGroup * 2;
  for (int i = tid; i < G * kHeadDim; i += blockDim.x) wo[i] = part_o[i];
  if (tid < G) {
    wml[2 * tid] = part_m[tid];
    wml[2 * tid + 1] = part_l[tid];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t t = atomicAdd(&A.tickets[grp], 1u);
    *flag_smem = (t == (uint32_t)(A.splits - 1));
  }
  __syncthreads();
  if (!*flag_smem) return;
  __threadfence();
  const int S = A.splits;
  const int b = grp / A.Hk, kvh = grp % A.Hk;
  const float* go = A.ws_o + (int64_t)grp * S * kMaxGroup * kHeadDim;
  const float* gml = A.ws_ml + (int64_t)grp * S * kMaxGroup * 2;
  float* fm = scratch;                       // [S][G]: split max, then its weight
  float* fl = scratch + kMaxSplits * kMaxGroup;  // [S][G]: split sum
  float* Mh = fl + kMaxSplits * kMaxGroup;   // [G]
  float* Lh = Mh + kMaxGroup;                // [G]
  for (int i = tid; i < S * G; i += blockDim.x) {
    const int s = i / G, h = i % G;
    fm[i] = __ldcg(gml + (s * kMaxGroup + h) * 2);
    fl[i] = __ldcg(gml + (s * kMaxGroup + h) * 2 + 1);
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, fm[s * G + tid]);
    float L = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < S; ++s) {
        const float ms = fm[s * G + tid];
        if (ms != -INFINITY) L += ex2(ms - M) * fl[s * G + tid];
      }
    Mh[tid] = M;
    Lh[tid] = L;
  }
  __syncthreads();
  for (int i = tid; i < S * G; i += blockDim.x) {
    const float ms = fm[i], M = Mh[i % G];
    fm[i] = (ms == -INFINITY || M == -INFINITY) ? 0.f : ex2(ms - M);
  }
  __syncthreads();
  for (int i = tid; i < G * kHeadDim; i += blockDim.x) {
    const int h = i / kHeadDim, d = i % kHeadDim;
    const float* src = go + h * kHeadDim + d;
    float num = 0.f;
    int s = 0;
    for (; s + 8 <= S; s += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (int64_t)(s + u) * kMaxGroup * kHeadDim);
#pragma unroll
      for (int u = 0; u < 8; ++u) num += fm[(s + u) * G + h] * v[u];
    }
    for (; s < S; ++s) num += fm[s * G + h] * __ldcg(src + (int64_t)s * kMaxGroup * kHeadDim);
    const float den = Lh[h];
    const float val = den > 0.f ? num / den : 0.f;
    const int hq = kvh * G + h;
    if (A.lse && d == 0)  // scores are kept in the log2 domain: ln sum = (M + log2 L) ln 2
      A.lse[b * A.lse_sb + hq] = den > 0.f ? (Mh[h] + log2f(den)) * 0.69314718055994531f : -INFINITY;
    if (A.o_bf16) {
      __nv_bfloat16* op = static_cast<__nv_bfloat16*>(A.o.data) + b * A.o.sb + hq * A.o.sh;
      op[d] = __float2bfloat16_rn(val);
    } else {
      float* op = static_cast<float*>(A.o.data) + b * A.o.sb + hq * A.o.sh;
      op[d] = val;
    }
  }
  if (tid == 0) A.tickets[grp] = 0u;  // leave the workspace ready for the next call
}

// ---- bf16 tensor-core variant ---------------------------------------------
template <int kStages>
__global__ void __launch_bounds__(kAttnThreads)
attn_decode_bf16_kernel(AttnArgs A) {
  pdl_wait();
  pdl_release();
  extern __shared__ __align__(128) unsigned char smem[];
  const int split = blockIdx.x, grp = blockIdx.y;
  const int b = grp / A.Hk, kvh = grp % A.Hk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = A.G;
  const KeyRange R = key_range(A, b, split);
  const int ntiles = (R.c1 - R.c0 + kTileKeys - 1) / kTileKeys;
  const bool sparse = A.W <= 0;

  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(A.k.data) + b * A.k.sb + kvh * A.k.sh;
  const __nv_bfloat16* vbase = static_cast<const __nv_bfloat16*>(A.v.data) + b * A.v.sb + kvh * A.v.sh;
  const uint32_t* mrow0 =
      sparse ? A.mask + (int64_t)(b * A.Hq + kvh * G) * A.mask_words + (A.key_lo >> 5) : nullptr;

  // Q^T as the B operand: column n = head g (zero for g >= G), rows = dims.
  uint32_t qb[8][2];
  {
    const uint32_t* qrow = nullptr;
    if (g < G)
      qrow = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(A.q.data) + b * A.q.sb +
                                               (kvh * G + g) * A.q.sh);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qb[kk][0] = qrow ? __ldg(qrow + (16 * kk + 2 * c) / 2) : 0u;
      qb[kk][1] = qrow ? __ldg(qrow + (16 * kk + 2 * c + 8) / 2) : 0u;
    }
  }

  const uint32_t sbase = smem_u32(smem);
  auto stageK = [&](int st) { return sbase + st * 2 * kTileBytes; };
  auto stageV = [&](int st) { return sbase + st * 2 * kTileBytes + kTileBytes; };

  // Sparse mode: the chunk's mask words (per head, and their union over the
  // group) are staged once; R.c0 is a multiple of 64 there.
  uint32_t* umask = reinterpret_cast<uint32_t*>(smem + kStages * 2 * kTileBytes);
  uint32_t* hmask = umask + kMaxChunkWords;  // [G][kMaxChunkWords]
  const int nw = (R.c1 - R.c0 + 31) >> 5;
  if (sparse) {
    const int w0 = R.c0 >> 5;
    for (int i = tid; i < nw; i += kAttnThreads) {
      uint32_t u = 0;
      for (int hh = 0; hh < G; ++hh) {
        const uint32_t x = __ldg(mrow0 + (int64_t)hh * A.mask_words + w0 + i);
        hmask[hh * kMaxChunkWords + i] = x;
        u |= x;
      }
      umask[i] = u;
    }
    __syncthreads();
  }

  // Load tile t into stage st: 64 rows x 16 chunks for K and for V, 8 + 8 per thread.
  auto load_tile = [&](int t, int st) {
    const int tb = R.c0 + t * kTileKeys;
    uint64_t uni = ~0ull;
    if (sparse) {
      const int wl = (tb - R.c0) >> 5;
      const uint32_t lo = umask[wl];
      const uint32_t hi = (wl + 1 < nw) ? umask[wl + 1] : 0u;
      uni = (uint64_t)lo | ((uint64_t)hi << 32);
    }
    const int ch = tid & 15;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (tid >> 4) + 8 * i;
      const int key = tb + r;
      const bool ok = key < R.c1 && ((uni >> r) & 1ull);
      const int kk = ok ? key : R.c0;
      cp_async16(stageK(st) + swz(r, ch), kbase + (int64_t)kk * A.k.sn + ch * 8, ok);
      cp_async16(stageV(st) + swz(r, ch), vbase + (int64_t)kk * A.v.sn + ch * 8, ok);
    }
  };

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float acc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  const int h0 = 2 * c, h1 = 2 * c + 1;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < ntiles) load_tile(s, s);
    cp_async_commit();
  }
  for (int t = 0; t < ntiles; ++t) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (t + kStages - 1 < ntiles) load_tile(t + kStages - 1, (t + kStages - 1) % kStages);
    cp_async_commit();
    const int st = t % kStages;
    const int tb = R.c0 + t * kTileKeys;
    const int kw = tb + 16 * warp;  // first key of this warp's 16

    // which of this thread's 4 score entries are admitted
    bool a00, a01, a10, a11;  // [key g / g+8][head h0 / h1]
    {
      const int kg0 = kw + g, kg1 = kw + g + 8;
      const bool v0 = kg0 < R.c1, v1 = kg1 < R.c1;
      if (sparse) {
        const int wi = (kw - R.c0) >> 5, sh = (kw & 31) + g;
        const bool wv = kw < R.c1;  // the word is inside the chunk
        const uint32_t w0 = (wv && h0 < G) ? hmask[h0 * kMaxChunkWords + wi] : 0u;
        const uint32_t w1 = (wv && h1 < G) ? hmask[h1 * kMaxChunkWords + wi] : 0u;
        a00 = v0 && ((w0 >> sh) & 1u);
        a01 = v0 && ((w1 >> sh) & 1u);
        a10 = v1 && ((w0 >> (sh + 8)) & 1u);
        a11 = v1 && ((w1 >> (sh + 8)) & 1u);
      } else {
        a00 = v0 && h0 < G;
        a01 = v0 && h1 < G;
        a10 = v1 && h0 < G;
        a11 = v1 && h1 < G;
      }
    }
    const bool any = __any_sync(0xffffffffu, a00 | a01 | a10 | a11);
    if (!any) continue;

    // S^T[16 keys][8 heads] = K_w . Q^T
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int r = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
      const uint32_t kst = stageK(st);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t a[4];
        ldsm_x4(kst + swz(r, 2 * kk + (lane >> 4)), a);
        mma_bf16(sc, a, qb[kk][0], qb[kk][1]);
      }
    }
    float x00 = a00 ? sc[0] * A.scale_log2 : -INFINITY;
    float x01 = a01 ? sc[1] * A.scale_log2 : -INFINITY;
    float x10 = a10 ? sc[2] * A.scale_log2 : -INFINITY;
    float x11 = a11 ? sc[3] * A.scale_log2 : -INFINITY;
    float mx0 = fmaxf(x00, x10), mx1 = fmaxf(x01, x11);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = mn0 == -INFINITY ? 1.f : ex2(m0 - mn0);
    const float al1 = mn1 == -INFINITY ? 1.f : ex2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const float p00 = a00 ? ex2(x00 - mn0) : 0.f;
    const float p01 = a01 ? ex2(x01 - mn1) : 0.f;
    const float p10 = a10 ? ex2(x10 - mn0) : 0.f;
    const float p11 = a11 ? ex2(x11 - mn1) : 0.f;
    l0 = l0 * al0 + p00 + p10;
    l1 = l1 * al1 + p01 + p11;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      acc[mt][0] *= al0;
      acc[mt][1] *= al1;
      acc[mt][2] *= al0;
      acc[mt][3] *= al1;
    }
    // P^T operand (keys x heads), as a bf16 hi + lo pair
    const uint32_t X0h = pack_bf16x2(p00, p01), X1h = pack_bf16x2(p10, p11);
    const uint32_t X0l = pack_bf16x2(p00 - bf16_lo(X0h), p01 - bf16_hi(X0h));
    const uint32_t X1l = pack_bf16x2(p10 - bf16_lo(X1h), p11 - bf16_hi(X1h));
    const uint32_t b0h = movm_t(X0h), b1h = movm_t(X1h);
    const uint32_t b0l = movm_t(X0l), b1l = movm_t(X1l);
    {
      const int r = 16 * warp + (lane & 7) + 8 * (lane >> 4);
      const uint32_t vst = stageV(st);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a[4];
        ldsm_x4_t(vst + swz(r, 2 * mt + ((lane >> 3) & 1)), a);
        mma_bf16(acc[mt], a, b0h, b1h);
        mma_bf16(acc[mt], a, b0l, b1l);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- merge the 4 warps (smem reuses the pipeline ring) ----
  float* wm = reinterpret_cast<float*>(smem);                 // [4][8]
  float* wl = wm + 4 * kMaxGroup;                             // [4][8]
  float* wo = wl + 4 * kMaxGroup;                             // [4][8][128]
  float* part_o = wo + 4 * kMaxGroup * kHeadDim;              // [8][128]
  float* part_m = part_o + kMaxGroup * kHeadDim;              // [8]
  float* part_l = part_m + kMaxGroup;                         // [8]
  int* flag = reinterpret_cast<int*>(part_l + kMaxGroup);
  float* scratch = reinterpret_cast<float*>(flag + 4);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (g == 0) {
    wm[warp * kMaxGroup + h0] = m0;
    wm[warp * kMaxGroup + h1] = m1;
    wl[warp * kMaxGroup + h0] = l0;
    wl[warp * kMaxGroup + h1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    float* o0 = wo + (warp * kMaxGroup) * kHeadDim;
    o0[h0 * kHeadDim + 16 * mt + g] = acc[mt][0];
    o0[h1 * kHeadDim + 16 * mt + g] = acc[mt][1];
    o0[h0 * kHeadDim + 16 * mt + g + 8] = acc[mt][2];
    o0[h1 * kHeadDim + 16 * mt + g + 8] = acc[mt][3];
  }
  __syncthreads();
  for (int i = tid; i < G * kHeadDim; i += kAttnThreads) {
    const int h = i / kHeadDim, d = i % kHeadDim;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * kMaxGroup + h]);
    float sum = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < 4; ++w) {
        const float mw = wm[w * kMaxGroup + h];
        if (mw == -INFINITY) continue;
        const float f = ex2(mw - M);
        sum += f * wo[(w * kMaxGroup + h) * kHeadDim + d];
        lsum += f * wl[w * kMaxGroup + h];
      }
    }
    part_o[h * kHeadDim + d] = sum;
    if (d == 0) {
      part_m[h] = M;
      part_l[h] = lsum;
    }
  }
  __syncthreads();
  finish_split(A, grp, split, part_o, part_m, part_l, flag, scratch);
}

// ---- fp32 CUDA-core variant -----------------------------------------------
__global__ void __launch_bounds__(kAttnThreads)
attn_decode_f32_kernel(AttnArgs A) {
  pdl_wait();
  pdl_release();
  __shared__ float wm[4][kMaxGroup], wl[4][kMaxGroup];
  __shared__ __align__(16) float wo[4][kMaxGroup][kHeadDim];
  __shared__ __align__(16) float part_o[kMaxGroup * kHeadDim];
  __shared__ float part_m[kMaxGroup], part_l[kMaxGroup];
  __shared__ int flag;
  __shared__ float scratch[2 * kMaxSplits * kMaxGroup + 2 * kMaxGroup];
  const int split = blockIdx.x, grp = blockIdx.y;
  const int b = grp / A.Hk, kvh = grp % A.Hk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = A.G;
  const KeyRange R = key_range(A, b, split);
  const bool sparse = A.W <= 0;
  const float* kbase = static_cast<const float*>(A.k.data) + b * A.k.sb + kvh * A.k.sh;
  const float* vbase = static_cast<const float*>(A.v.data) + b * A.v.sb + kvh * A.v.sh;
  const uint32_t* mrow0 =
      sparse ? A.mask + (int64_t)(b * A.Hq + kvh * G) * A.mask_words + (A.key_lo >> 5) : nullptr;

  float4 qv[kMaxGroup];
  float m[kMaxGroup], l[kMaxGroup];
  float4 o[kMaxGroup];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    qv[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (h < G) {
      const float* qr = static_cast<const float*>(A.q.data) + b * A.q.sb + (kvh * G + h) * A.q.sh;
      qv[h] = __ldg(reinterpret_cast<const float4*>(qr) + lane);
    }
    m[h] = -INFINITY;
    l[h] = 0.f;
    o[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int key = R.c0 + warp; key < R.c1; key += 4) {
    uint32_t adm = 0;
    if (sparse) {
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h)
        if (h < G) adm |= ((__ldg(mrow0 + (int64_t)h * A.mask_words + (key >> 5)) >> (key & 31)) & 1u) << h;
    } else {
      adm = (1u << G) - 1u;
    }
    if (!adm) continue;
    const float4 kx = __ldg(reinterpret_cast<const float4*>(kbase + (int64_t)key * A.k.sn) + lane);
    const float4 vx = __ldg(reinterpret_cast<const float4*>(vbase + (int64_t)key * A.v.sn) + lane);
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (!((adm >> h) & 1u)) continue;
      float s = qv[h].x * kx.x + qv[h].y * kx.y + qv[h].z * kx.z + qv[h].w * kx.w;
      s = warp_sum(s) * A.scale_log2;
      const float mn = fmaxf(m[h], s);
      const float al = ex2(m[h] - mn);
      const float pp = ex2(s - mn);
      m[h] = mn;
      l[h] = l[h] * al + pp;
      o[h].x = o[h].x * al + pp * vx.x;
      o[h].y = o[h].y * al + pp * vx.y;
      o[h].z = o[h].z * al + pp * vx.z;
      o[h].w = o[h].w * al + pp * vx.w;
    }
  }
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    if (h >= G) continue;
    if (lane == 0) {
      wm[warp][h] = m[h];
      wl[warp][h] = l[h];
    }
    reinterpret_cast<float4*>(&wo[warp][h][0])[lane] = o[h];
  }
  __syncthreads();
  for (int i = tid; i < G * kHeadDim; i += kAttnThreads) {
    const int h = i / kHeadDim, d = i % kHeadDim;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w][h]);
    float sum = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < 4; ++w) {
        if (wm[w][h] == -INFINITY) continue;
        const float f = ex2(wm[w][h] - M);
        sum += f * wo[w][h][d];
        lsum += f * wl[w][h];
      }
    }
    part_o[h * kHeadDim + d] = sum;
    if (d == 0) {
      part_m[h] = M;
      part_l[h] = lsum;
    }
  }
  __syncthreads();
  finish_split(A, grp, split, part_o, part_m, part_l, &flag, scratch);
}

// ---- host side ---------------------------------------------------------------
// One wave: about two CTAs per SM over all (sequence, KV head) groups; chunks a
// multiple of the tile, between 256 and kMaxChunk keys, at most kMaxSplits.
static void attn_layout(int64_t B, int64_t Hk, int64_t N, int32_t W, int sms, int* chunk, int* splits) {
  int64_t range = W > 0 ? (W < N ? W : N) : N;
  if (range < 1) range = 1;
  const int64_t groups = B * Hk > 0 ? B * Hk : 1;
  int64_t want = (2 * (int64_t)sms) / groups;
  if (want < 1) want = 1;
  int64_t c = (range + want - 1) / want;
  c = (c + kTileKeys - 1) / kTileKeys * kTileKeys;
  if (c < 256) c = 256;
  if (c > kMaxChunk) c = kMaxChunk;
  int64_t s = (range + c - 1) / c;
  if (s > kMaxSplits) {  // very long ranges: the smallest tile-multiple chunk that needs at most kMaxSplits
    c = (range + kMaxSplits - 1) / kMaxSplits;
    c = (c + kTileKeys - 1) / kTileKeys * kTileKeys;
    s = (range + c - 1) / c;
  }
  *chunk = (int)c;
  *splits = (int)s;
}

size_t attn_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t Hk, int64_t N, int32_t W) {
  (void)Hq;
  int chunk = 0, splits = 0;
  attn_layout(B, Hk, N, W, 148, &chunk, &splits);
  // sized for the smallest SM count this build targets, so it never under-reports
  const int64_t groups = B * Hk;
  const size_t o_bytes = (size_t)groups * splits * kMaxGroup * kHeadDim * sizeof(float);
  const size_t ml_bytes = (size_t)groups * splits * kMaxGroup * 2 * sizeof(float);
  const size_t t_bytes = (size_t)groups * sizeof(uint32_t);
  return ((o_bytes + 255) / 256 * 256) + ((ml_bytes + 255) / 256 * 256) + ((t_bytes + 255) / 256 * 256);
}

void attn_decode_ticket_range(int64_t B, int64_t Hk, int64_t N, int32_t W, size_t* offset, size_t* bytes) {
  int chunk = 0, splits = 0;
  attn_layout(B, Hk, N, W, 148, &chunk, &splits);
  const int64_t groups = B * Hk;
  const size_t o_bytes = (size_t)groups * splits * kMaxGroup * kHeadDim * sizeof(float);
  const size_t ml_bytes = (size_t)groups * splits * kMaxGroup * 2 * sizeof(float);
  *offset = (o_bytes + 255) / 256 * 256 + (ml_bytes + 255) / 256 * 256;
  *bytes = (size_t)(groups > 0 ? groups : 0) * sizeof(uint32_t);
}

bool attn_decode_supported(int64_t B, int64_t Hk, int64_t N, int32_t W) {
  int chunk = 0, splits = 0;
  attn_layout(B, Hk, N, W, 148, &chunk, &splits);
  return W > 0 || chunk <= kMaxChunk;  // the sparse form stages a chunk's masks on chip
}

cudaError_t launch_attn_decode(const LaunchAttnDecode& a, cudaStream_t stream) {
  const int64_t groups = a.B * a.Hk;
  if (groups == 0) return cudaSuccess;
  int chunk = 0, splits = 0;
  attn_layout(a.B, a.Hk, a.N, a.W, 148, &chunk, &splits);
  if (a.W <= 0 && chunk > kMaxChunk) return cudaErrorInvalidValue;
  AttnArgs A;
  A.q = a.q;
  A.k = a.k;
  A.v = a.v;
  A.lens = a.lens;
  A.mask = a.mask;
  A.mask_words = a.mask_words;
  A.Hq = (int)a.Hq;
  A.Hk = (int)a.Hk;
  A.G = (int)(a.Hq / a.Hk);
  A.N = (int)a.N;
  A.W = a.W;
  A.chunk = chunk;
  A.splits = splits;
  A.scale_log2 = a.scale * kLog2e;
  A.o = a.o;
  A.o_bf16 = a.o_bf16 ? 1 : 0;
  A.key_lo = (int)a.key_lo;
  A.lse = a.lse;
  A.lse_sb = a.lse_sb;
  const size_t o_bytes = (size_t)groups * splits * kMaxGroup * kHeadDim * sizeof(float);
  const size_t ml_bytes = (size_t)groups * splits * kMaxGroup * 2 * sizeof(float);
  char* ws = static_cast<char*>(a.ws);
  A.ws_o = reinterpret_cast<float*>(ws);
  A.ws_ml = reinterpret_cast<float*>(ws + (o_bytes + 255) / 256 * 256);
  A.tickets = reinterpret_cast<uint32_t*>(ws + (o_bytes + 255) / 256 * 256 + (ml_bytes + 255) / 256 * 256);
  dim3 grid((unsigned)splits, (unsigned)groups);
  if (a.bf16) {
    if (a.W > 0) {  // window: no mask staging
      const size_t smem = (size_t)kStagesWindow * 2 * kTileBytes;
      cudaFuncSetAttribute(attn_decode_bf16_kernel<kStagesWindow>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      cudaFuncSetAttribute(attn_decode_bf16_kernel<kStagesWindow>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           100);
      return launch_pdl(attn_decode_bf16_kernel<kStagesWindow>, grid, dim3(kAttnThreads), smem, stream, 1, A);
    }
    const size_t smem = (size_t)kStagesSparse * 2 * kTileBytes + (size_t)(kMaxGroup + 1) * kMaxChunkWords * 4;
    cudaFuncSetAttribute(attn_decode_bf16_kernel<kStagesSparse>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    cudaFuncSetAttribute(attn_decode_bf16_kernel<kStagesSparse>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return launch_pdl(attn_decode_bf16_kernel<kStagesSparse>, grid, dim3(kAttnThreads), smem, stream, 1, A);
  }
  return launch_pdl(attn_decode_f32_kernel, grid, dim3(kAttnThreads), 0, stream, 1, A);
}

}  // namespace rtp
