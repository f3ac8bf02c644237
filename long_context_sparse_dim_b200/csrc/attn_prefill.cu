// a4 / a5 (prefill): causal attention of T query tokens per sequence over
//   - their selected keys (retrieval heads: threshold form tau, tiepos from
//     rtp_topp_select), or
//   - the last W keys up to their own position (local heads).
//
// "Full Attention Strikes Back ... (RTPurbo)", TL;DR (sparse attention over the
// tokens the indexer picks); "RTPurbo: Turning Dense LLMs into Sparse Attention
// Models ...", "Three Key Insights" 1 (local heads keep a window) and 3.
//
// Design (B200, tcgen05): a CTA takes one query head and 128 query tokens
// (TMEM lane r = token r) and streams 128-key K/V tiles through a two-stage
// TMA ring (128-byte swizzle, no multicast).  Per tile:
//   S = Q K^T       tcgen05.mma M=128 N=128, eight K=16 slices over the head
//                   dim, into one of two TMEM buffers (double-buffered)
//   softmax         warps 0-3, one query row per thread: pass 1 takes the
//                   row maximum over the admitted keys, pass 2 writes
//                   P = 2^(s * scale * log2 e - m) over S in place as a bf16
//                   hi + lo pair (so P V keeps fp32-level precision)
//   O = P V         tcgen05.mma with A = P read from TMEM and B = V as an
//                   MN-major operand, hi and lo parts, into a TMEM O tile
//   fold            warps 4-7 (same TMEM lane quadrants, one row per thread)
//                   add O into fp32 registers with the online-softmax
//                   rescaling 2^(m_old - m_new), rounding to nearest every
//                   tile (no drift over a million keys); the softmax hands
//                   them each tile's row maximum and sum through shared memory
// Warp 8 issues the TMA loads, warp 9 the MMAs; every hand-off is an mbarrier
// and every wait is time-bounded.  For the sparse form, key j is admitted for
// token i iff s_ij > tau_i or (s_ij == tau_i and j <= tiepos_i): the indexer
// tile s is recomputed with exactly the instruction the selection used
// (tcgen05.mma kind::f16, M=128, N=128, K=16 over 128-key tiles aligned as in
// the selection), so the predicate sees bit-identical scores.
#include <math.h>

#include "launch.h"
#include "tc05.cuh"

namespace rtp {

namespace {

constexpr int kAtRows = 128;                          // query rows per CTA (MMA M, TMEM lanes)
constexpr int kAtKeys = 128;                          // keys per tile
constexpr int kAtStages = 2;                          // K/V ring
constexpr int kAtSoftWarps = 4;                       // warps 0-3: softmax
constexpr int kAtCorrWarps = 4;                       // warps 4-7: O fold and output
constexpr int kAtProducerWarp = 8, kAtMmaWarp = 9;
constexpr int kAtThreads = 10 * 32;
constexpr int kAtHalfBytes = kAtKeys * 128;           // 128 rows x 64 bf16 (one 128-byte-swizzled half)
constexpr int kAtTileBytes = 2 * kAtHalfBytes;        // one Q, K or V tile: 32 KB
constexpr int kAtIdxBytes = kAtKeys * kIdxDim * 2;    // 4 KB
constexpr uint32_t kTmemS = 0, kTmemO = 256, kTmemIdx = 384, kAtTmemCols = 512;
constexpr float kLog2eF = 1.4426950408889634f;

struct AtSmem {
  alignas(1024) uint8_t q[kAtTileBytes];
  alignas(1024) uint8_t k[kAtStages][kAtTileBytes];
  alignas(1024) uint8_t v[kAtStages][kAtTileBytes];
  alignas(1024) uint8_t qidx[kAtRows * kIdxDim * 2];  // sparse form
  alignas(1024) uint8_t kidx[kAtStages][kAtIdxBytes];
  uint64_t q_full;
  uint64_t k_full[kAtStages], v_full[kAtStages], kv_empty[kAtStages];
  uint64_t s_full[2], p_full[2], s_free[2];
  uint64_t idx_full, idx_free;
  uint64_t o_full, o_free;
  uint64_t stat_full[2], stat_free[2];
  float2 stat[2][kAtRows];  // per tile (double-buffered): the row's maximum and sum of P
  uint32_t tmem_base;
};

struct AtArgs {
  const int32_t* lens;
  const uint32_t* tau_bits;
  const int32_t* tiepos;
  int Hq, Hk, G, T, N, W;
  float scale_log2;
  MutView4 o;
  int o_bf16;
  int* err;
  long long budget;
};

RTP_DEVICE float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Bits j of a 32-key chunk with lo <= j <= hi.
RTP_DEVICE uint32_t band32(int lo, int hi) {
  if (hi < 0 || lo > 31 || hi < lo) return 0u;
  const int l = max(lo, 0), r = min(hi, 31);
  const uint32_t upto = r >= 31 ? 0xffffffffu : ((1u << (r + 1)) - 1u);
  return upto & ~((1u << l) - 1u);
}

}  // namespace

template <bool SPARSE>
__global__ void __launch_bounds__(kAtThreads, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap qimap,
                    const __grid_constant__ CUtensorMap kimap, AtArgs A) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AtSmem& S = *reinterpret_cast<AtSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // heaviest (latest) query blocks first
  const int t0 = ((int)gridDim.x - 1 - (int)blockIdx.x) * kAtRows;
  const int bh = blockIdx.y;
  const int b = bh / A.Hq, h = bh % A.Hq, kvh = h / A.G;
  int n_b = A.N;
  if (A.lens) n_b = min(max(A.lens[b], 0), A.N);
  const int qbase = n_b - A.T;
  const int t_last = min(t0 + kAtRows, A.T) - 1;
  const int kmax = min(qbase + t_last, n_b - 1);  // last key any row of the block sees
  const int klo = SPARSE ? 0 : max(0, qbase + t0 - A.W + 1);
  const int tile0 = klo / kAtKeys;
  const int ntiles = kmax >= klo ? (kmax / kAtKeys) - tile0 + 1 : 0;

  if (tid == 0) {
    mbar_init(&S.q_full, 1);
    for (int i = 0; i < kAtStages; ++i) {
      mbar_init(&S.k_full[i], 1);
      mbar_init(&S.v_full[i], 1);
      mbar_init(&S.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.p_full[i], kAtSoftWarps);
      mbar_init(&S.s_free[i], 1);
    }
    mbar_init(&S.idx_full, 1);
    mbar_init(&S.idx_free, kAtSoftWarps);
    mbar_init(&S.o_full, 1);
    mbar_init(&S.o_free, kAtCorrWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.stat_full[i], kAtSoftWarps);
      mbar_init(&S.stat_free[i], kAtCorrWarps);
    }
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, kAtTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  bool alive = true;
  uint32_t loads = 0, pvs = 0, qks = 0;
  bool q_issued = false;

  if (warp == kAtProducerWarp) {
    // ---------------- TMA producer (one elected lane) ----------------
    if (lane == 0 && ntiles > 0) {
      mbar_expect_tx(&S.q_full, kAtTileBytes + (SPARSE ? kAtRows * kIdxDim * 2 : 0));
      tma_load_4d(S.q, &qmap, &S.q_full, 0, t0, h, b);
      tma_load_4d(S.q + kAtHalfBytes, &qmap, &S.q_full, 64, t0, h, b);
      if (SPARSE) tma_load_4d(S.qidx, &qimap, &S.q_full, 0, t0, h, b);
      q_issued = true;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kAtStages;
        const uint32_t ph = (uint32_t)(i / kAtStages) & 1u;
        if (!mbar_wait(&S.kv_empty[st], ph ^ 1u, alive, A.err, A.budget)) break;
        const int key0 = (tile0 + i) * kAtKeys;
        mbar_expect_tx(&S.k_full[st], kAtTileBytes + (SPARSE ? kAtIdxBytes : 0));
        tma_load_4d(S.k[st], &kmap, &S.k_full[st], 0, key0, kvh, b);
        tma_load_4d(S.k[st] + kAtHalfBytes, &kmap, &S.k_full[st], 64, key0, kvh, b);
        if (SPARSE) tma_load_4d(S.kidx[st], &kimap, &S.k_full[st], 0, key0, kvh, b);
        mbar_expect_tx(&S.v_full[st], kAtTileBytes);
        tma_load_4d(S.v[st], &vmap, &S.v_full[st], 0, key0, kvh, b);
        tma_load_4d(S.v[st] + kAtHalfBytes, &vmap, &S.v_full[st], 64, key0, kvh, b);
        loads = (uint32_t)i + 1u;
      }
    }
  } else if (warp == kAtMmaWarp) {
    // ---------------- MMA issuer (one elected lane) ----------------
    if (lane == 0 && ntiles > 0) {
      mbar_wait(&S.q_full, 0, alive, A.err, A.budget);
      constexpr uint32_t idesc_qk = umma_idesc_bf16_f32(kAtRows, kAtKeys);
      constexpr uint32_t idesc_pv = umma_idesc_bf16_f32(kAtRows, kHeadDim) | (1u << 16);  // V is MN-major
      const uint32_t qa = smem_addr(S.q);
      // O = P_j V_j: A = the P tile (bf16 hi + lo) in TMEM, B = V_j in shared memory
      auto issue_pv = [&](int j) -> bool {
        const int st = j % kAtStages, bj = j & 1;
        if (!mbar_wait(&S.p_full[bj], (uint32_t)(j >> 1) & 1u, alive, A.err, A.budget)) return false;
        if (!mbar_wait(&S.o_free, ((uint32_t)j & 1u) ^ 1u, alive, A.err, A.budget)) return false;
        if (!mbar_wait(&S.v_full[st], (uint32_t)(j / kAtStages) & 1u, alive, A.err, A.budget)) return false;
        tc_fence_after();
        const uint32_t va = smem_addr(S.v[st]);
#pragma unroll
        for (int kk = 0; kk < kAtKeys / 16; ++kk) {
          const uint64_t bdesc = umma_desc_sw128(va + (uint32_t)kk * 16u * 128u, kAtHalfBytes);
          const uint32_t a_hi =
              tmem + kTmemS + (uint32_t)bj * kAtKeys + 32u * (uint32_t)(kk >> 1) + 8u * (uint32_t)(kk & 1);
          umma_f16_tmem_a(tmem + kTmemO, a_hi, bdesc, idesc_pv, kk > 0 ? 1u : 0u);
          umma_f16_tmem_a(tmem + kTmemO, a_hi + 16u, bdesc, idesc_pv, 1u);
        }
        umma_commit(&S.o_full);
        umma_commit(&S.s_free[bj]);
        umma_commit(&S.kv_empty[st]);
        pvs = (uint32_t)j + 1u;
        return true;
      };
      bool ok = alive;
      for (int i = 0; i < ntiles && ok; ++i) {
        const int st = i % kAtStages, bi = i & 1;
        if (!mbar_wait(&S.k_full[st], (uint32_t)(i / kAtStages) & 1u, alive, A.err, A.budget)) break;
        if (!mbar_wait(&S.s_free[bi], ((uint32_t)(i >> 1) & 1u) ^ 1u, alive, A.err, A.budget)) break;
        tc_fence_after();
        const uint32_t ka = smem_addr(S.k[st]);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kAtHalfBytes + 32u * (uint32_t)(kk & 3);
          umma_f16(tmem + kTmemS + (uint32_t)bi * kAtKeys, umma_desc_sw128(qa + off, 16),
                   umma_desc_sw128(ka + off, 16), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&S.s_full[bi]);
        qks = (uint32_t)i + 1u;
        if (SPARSE) {
          if (!mbar_wait(&S.idx_free, ((uint32_t)i & 1u) ^ 1u, alive, A.err, A.budget)) break;
          tc_fence_after();
          umma_f16(tmem + kTmemIdx, umma_desc_k_sw32(S.qidx), umma_desc_k_sw32(S.kidx[st]), idesc_qk, 0u);
          umma_commit(&S.idx_full);
        }
        if (i > 0) ok = issue_pv(i - 1);
      }
      if (ok && alive && qks == (uint32_t)ntiles) issue_pv(ntiles - 1);
    }
  } else if (warp < kAtSoftWarps) {
    // ---------------- softmax: one query row per thread ----------------
    const int row = tid;
    const int t = t0 + row;
    const int pos = t < A.T ? qbase + t : -1;  // -1: no keys
    float tau = 0.f;
    int tpos = -1;
    if (SPARSE && pos >= 0) {
      const int64_t qrow = (int64_t)bh * A.T + t;
      tau = __uint_as_float(A.tau_bits[qrow]);
      tpos = A.tiepos[qrow];
    }
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    float m_run = -INFINITY;  // running maximum of the scaled logits (log2 units)
    for (int i = 0; i < ntiles; ++i) {
      const int bi = i & 1;
      const int key0 = (tile0 + i) * kAtKeys;
      // admission bits of this row over the tile's 128 keys
      uint32_t adm[4];
      if (SPARSE) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&S.idx_full, (uint32_t)i & 1u, alive, A.err, A.budget));
        if (!ok) {
          alive = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + kTmemIdx + 32u * (uint32_t)c, v);
          tmem_ld_wait();
          uint32_t bits = 0u;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float s = __fadd_rn(__fmul_rn(__uint_as_float(v[jj]), 0.25f), 0.0f);
            bits |= (uint32_t)(s > tau || (s == tau && key0 + 32 * c + jj <= tpos)) << jj;
          }
          adm[c] = bits & band32(0, pos - key0 - 32 * c);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.idx_free);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          adm[c] = pos < 0 ? 0u : band32(max(pos - A.W + 1, 0) - key0 - 32 * c, pos - key0 - 32 * c);
      }
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait(&S.s_full[bi], (uint32_t)(i >> 1) & 1u, alive, A.err, A.budget));
      if (!ok) {
        alive = false;
        break;
      }
      tc_fence_after();
      const uint32_t sb = lane_base + kTmemS + (uint32_t)bi * kAtKeys;
      // pass 1: the tile maximum of the admitted logits
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(sb + 32u * (uint32_t)c, v);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
          tmax = fmaxf(tmax, ((adm[c] >> jj) & 1u) ? __uint_as_float(v[jj]) : -INFINITY);
      }
      const float m_new = fmaxf(m_run, tmax * A.scale_log2);
      // pass 2: P = 2^(s * scale * log2 e - m_new) as bf16 hi + lo, written over S
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(sb + 32u * (uint32_t)c, v);
        tmem_ld_wait();
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const float e0 = ex2a(__fmaf_rn(__uint_as_float(v[2 * jj]), A.scale_log2, -m_new));
          const float e1 = ex2a(__fmaf_rn(__uint_as_float(v[2 * jj + 1]), A.scale_log2, -m_new));
          const float p0 = ((adm[c] >> (2 * jj)) & 1u) ? e0 : 0.f;
          const float p1 = ((adm[c] >> (2 * jj + 1)) & 1u) ? e1 : 0.f;
          lsum += p0 + p1;
          hi[jj] = pack_bf16x2(p0, p1);
          lo[jj] = pack_bf16x2(p0 - bf16_lo(hi[jj]), p1 - bf16_hi(hi[jj]));
        }
        tmem_st16(sb + 32u * (uint32_t)c, hi);
        tmem_st16(sb + 32u * (uint32_t)c + 16u, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full[bi]);
      m_run = m_new;
      // hand the tile's (maximum, sum) to the fold
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&S.stat_free[bi], ((uint32_t)(i >> 1) & 1u) ^ 1u, alive, A.err, A.budget))) {
        alive = false;
        break;
      }
      S.stat[bi][row] = make_float2(m_new, lsum);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.stat_full[bi]);
    }
  } else if (warp < kAtSoftWarps + kAtCorrWarps) {
    // ---------------- fold and output: one query row per thread ----------------
    const int row = tid - kAtSoftWarps * 32;
    const int t = t0 + row;
    const uint32_t lane_base = tmem + ((uint32_t)((warp - kAtSoftWarps) * 32) << 16);
    float o[kHeadDim];
#pragma unroll
    for (int d = 0; d < kHeadDim; ++d) o[d] = 0.f;
    float m_t = -INFINITY, l_t = 0.f;  // reference maximum and denominator of o
    for (int j = 0; j < ntiles; ++j) {
      const int bj = j & 1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&S.stat_full[bj], (uint32_t)(j >> 1) & 1u, alive, A.err, A.budget))) {
        alive = false;
        break;
      }
      const float2 st = S.stat[bj][row];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.stat_free[bj]);
      if (!__all_sync(0xffffffffu, mbar_wait(&S.o_full, (uint32_t)j & 1u, alive, A.err, A.budget))) {
        alive = false;
        break;
      }
      tc_fence_after();
      // O_j was computed relative to st.x; rescale the running sum to it
      const float alpha = st.x == -INFINITY ? 1.f : ex2a(m_t - st.x);
#pragma unroll
      for (int c = 0; c < kHeadDim / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_base + kTmemO + 32u * (uint32_t)c, v);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) o[32 * c + jj] = __fmaf_rn(o[32 * c + jj], alpha, __uint_as_float(v[jj]));
      }
      l_t = __fmaf_rn(l_t, alpha, st.y);
      if (st.x != -INFINITY) m_t = st.x;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.o_free);
    }

    // ---- normalise and store ----
    if (t < A.T) {
      const float inv = l_t > 0.f ? 1.f / l_t : 0.f;
      if (A.o_bf16) {
        __nv_bfloat16* orow =
            static_cast<__nv_bfloat16*>(A.o.data) + b * A.o.sb + h * A.o.sh + (int64_t)t * A.o.sn;
#pragma unroll
        for (int d = 0; d < kHeadDim; d += 8) {
          uint4 w;
          w.x = pack_bf16x2(o[d] * inv, o[d + 1] * inv);
          w.y = pack_bf16x2(o[d + 2] * inv, o[d + 3] * inv);
          w.z = pack_bf16x2(o[d + 4] * inv, o[d + 5] * inv);
          w.w = pack_bf16x2(o[d + 6] * inv, o[d + 7] * inv);
          *reinterpret_cast<uint4*>(orow + d) = w;
        }
      } else {
        float* orow = static_cast<float*>(A.o.data) + b * A.o.sb + h * A.o.sh + (int64_t)t * A.o.sn;
#pragma unroll
        for (int d = 0; d < kHeadDim; d += 4)
          *reinterpret_cast<float4*>(orow + d) =
              make_float4(o[d] * inv, o[d + 1] * inv, o[d + 2] * inv, o[d + 3] * inv);
      }
    }
  }

  // ---- wind down: every copy and MMA issued lands before TMEM is freed, even
  // after a wait gave up (the last commit of this thread covers all earlier MMAs)
  if (warp == kAtMmaWarp && lane == 0) {
    if (pvs > 0 && pvs >= qks) {
      mbar_drain(&S.o_full, (pvs - 1u) & 1u, A.err);
    } else if (qks > 0) {
      const uint32_t last = qks - 1u;
      if (SPARSE && qks > 0) mbar_drain(&S.idx_full, last & 1u, A.err);
      mbar_drain(&S.s_full[last & 1u], (last >> 1) & 1u, A.err);
    }
  }
  if (warp == kAtProducerWarp && lane == 0) {
    if (q_issued) mbar_drain(&S.q_full, 0, A.err);
    for (uint32_t i = loads > (uint32_t)kAtStages ? loads - kAtStages : 0u; i < loads; ++i) {
      mbar_drain(&S.k_full[i % kAtStages], (i / kAtStages) & 1u, A.err);
      mbar_drain(&S.v_full[i % kAtStages], (i / kAtStages) & 1u, A.err);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, kAtTmemCols);
}

// ---- host side ------------------------------------------------------------------

cudaError_t launch_attn_prefill(const LaunchAttnPrefill& a, cudaStream_t stream) {
  if (a.B * a.Hq * a.T == 0) return cudaSuccess;
  AtArgs A;
  A.lens = a.lens;
  A.tau_bits = a.tau_bits;
  A.tiepos = a.tiepos;
  A.Hq = (int)a.Hq;
  A.Hk = (int)a.Hk;
  A.G = (int)(a.Hq / a.Hk);
  A.T = (int)a.T;
  A.N = (int)a.N;
  A.W = a.W;
  A.scale_log2 = a.scale * kLog2eF;
  A.o = a.o;
  A.o_bf16 = a.o_bf16 ? 1 : 0;
  A.err = a.err;
  A.budget = wait_budget_cycles();
  CUtensorMap qmap, kmap, vmap, qimap{}, kimap{};
  if (!make_row_map(&qmap, a.q, a.B, a.Hq, a.T, kAtRows)) return cudaErrorInvalidValue;
  if (!make_row_map(&kmap, a.k, a.B, a.Hk, a.N, kAtKeys)) return cudaErrorInvalidValue;
  if (!make_row_map(&vmap, a.v, a.B, a.Hk, a.N, kAtKeys)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(AtSmem) + 1024;
  const dim3 grid((unsigned)((a.T + kAtRows - 1) / kAtRows), (unsigned)(a.B * a.Hq));
  if (a.W > 0) {
    cudaFuncSetAttribute(attn_prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_prefill_kernel<false><<<grid, kAtThreads, smem, stream>>>(qmap, kmap, vmap, qimap, kimap, A);
  } else {
    if (!make_idx_map(&qimap, a.q_idx, a.B, a.Hq, a.T, kAtRows)) return cudaErrorInvalidValue;
    if (!make_idx_map(&kimap, a.k_idx, a.B, a.Hk, a.N, kAtKeys)) return cudaErrorInvalidValue;
    cudaFuncSetAttribute(attn_prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_prefill_kernel<true><<<grid, kAtThreads, smem, stream>>>(qmap, kmap, vmap, qimap, kimap, A);
  }
  return cudaGetLastError();
}

}  // namespace rtp
