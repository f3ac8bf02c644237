// a4 / a5 (prefill): causal attention of T query tokens per sequence over
//   - their selected keys (retrieval heads: threshold form tau, tiepos from
//     rtp_topp_select), or
//   - the last W keys up to their own position (local heads).
//
// "Full Attention Strikes Back ... (RTPurbo)", TL;DR (sparse attention over the
// tokens the indexer picks); "RTPurbo: Turning Dense LLMs into Sparse Attention
// Models ...", "Three Key Insights" 1 (local heads keep a window) and 3.
//
// Design (B200, tcgen05): a CTA takes the G query heads of one KV head x 128/G
// query tokens, 128 rows in all (TMEM lane r = row r), and streams 128-key K/V
// tiles of that KV head through a two-stage TMA ring (128-byte swizzle, no
// multicast); each tile is read once for the whole GQA group.  Per tile:
//   S = Q K^T       tcgen05.mma M=128 N=128, eight K=16 slices over the head
//                   dim, into one of two TMEM buffers (double-buffered)
//   softmax         warps 0-7, two threads per query row (warps w and w+4
//                   share TMEM lane quadrant w % 4, each takes 64 of the
//                   tile's keys): pass 1 takes the row maximum over the
//                   admitted keys (the halves meet at a 64-thread named
//                   barrier), pass 2 writes P = 2^(s * scale * log2 e - m)
//                   over S in place as a bf16 hi + lo pair (so P V keeps
//                   fp32-level precision): the 16 keys of MMA slice k keep
//                   their hi words in columns 16k .. 16k+7, lo in 16k+8 ..
//   O = P V         tcgen05.mma with A = P read from TMEM and B = V as an
//                   MN-major operand, hi and lo parts, into a TMEM O tile
//   fold            warps 8-15 (two threads per row, 64 head dims each) add O
//                   into fp32 registers with the online-softmax rescaling
//                   2^(m_old - m_new), rounding to nearest every tile (no
//                   drift over a million keys); the softmax hands them each
//                   tile's row maximum and sums through shared memory
// Warp 16 issues the TMA loads, warp 17 the MMAs; every hand-off is an
// mbarrier and every wait is time-bounded.  Eighteen warps put five on two of
// the SM's four sub-partitions (16K registers each), so a thread may hold at
// most 96 registers.  For the sparse form, key j is admitted for
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
constexpr int kAtSoftWarps = 8;                       // warps 0-7: softmax, two threads per row
constexpr int kAtCorrWarps = 8;                       // warps 8-15: O fold and output, two threads per row
constexpr int kAtProducerWarp = 16, kAtMmaWarp = 17;
constexpr int kAtThreads = 18 * 32;
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
  float2 stat[2][2][kAtRows];  // per tile (double-buffered) and column half: the row's maximum, sum of P
  float pmax[2][2][kAtRows];   // per tile (double-buffered) and column half: the row's partial maximum
  uint32_t tmem_base;
};

struct AtArgs {
  const int32_t* lens;
  const uint32_t* tau_bits;
  const int32_t* tiepos;
  int Hq, Hk, G, T, N, W;
  int TB;  // tokens per block (the block holds G heads x TB tokens)
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

RTP_DEVICE float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// (a * s + c, b * s + c) in one packed fp32x2 fused multiply-add.
RTP_DEVICE void fma2(float a, float b, float sc, float c, float& ra, float& rb) {
  uint64_t x, y, z, r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(x) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(y) : "f"(sc), "f"(sc));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(z) : "f"(c), "f"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(r) : "l"(x), "l"(y), "l"(z));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(ra), "=f"(rb) : "l"(r));
}

// (acc0, acc1) += (a, b) in one packed fp32x2 add.
RTP_DEVICE void add2(float& acc0, float& acc1, float a, float b) {
  uint64_t x, y, r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(x) : "f"(acc0), "f"(acc1));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(y) : "f"(a), "f"(b));
  asm("add.rn.f32x2 %0, %1, %2;\n" : "=l"(r) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(acc0), "=f"(acc1) : "l"(r));
}

// (a - c, b - d) in one packed fp32x2 subtract.
RTP_DEVICE void sub2p(float a, float b, float c, float d, float& ra, float& rb) {
  uint64_t x, y, r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(x) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(y) : "f"(c), "f"(d));
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(r) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(ra), "=f"(rb) : "l"(r));
}

RTP_DEVICE void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory"); }

}  // namespace

template <bool SPARSE>
__global__ void __maxnreg__(96)
attn_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap qimap,
                    const __grid_constant__ CUtensorMap kimap, AtArgs A) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  AtSmem& S = *reinterpret_cast<AtSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // A block holds the G query heads of one KV head x TB consecutive tokens (row
  // r: head r / TB of the group, token t0 + r % TB), so every K/V tile it loads
  // serves all G heads.  Heaviest (latest) token blocks first.
  const int TB = A.TB;
  const int t0 = ((int)gridDim.x - 1 - (int)blockIdx.x) * TB;
  const int bk = blockIdx.y;
  const int b = bk / A.Hk, kvh = bk % A.Hk;
  int n_b = A.N;
  if (A.lens) n_b = min(max(A.lens[b], 0), A.N);
  const int qbase = n_b - A.T;
  const int t_last = min(t0 + TB, A.T) - 1;
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
      // one box of TB rows per head of the group (and per 64-column half)
      mbar_expect_tx(&S.q_full, A.G * TB * (kHeadDim + (SPARSE ? kIdxDim : 0)) * 2);
      for (int g = 0; g < A.G; ++g) {
        const int hq = kvh * A.G + g;
        tma_load_4d(S.q + g * TB * 128, &qmap, &S.q_full, 0, t0, hq, b);
        tma_load_4d(S.q + kAtHalfBytes + g * TB * 128, &qmap, &S.q_full, 64, t0, hq, b);
        if (SPARSE) tma_load_4d(S.qidx + g * TB * kIdxDim * 2, &qimap, &S.q_full, 0, t0, hq, b);
      }
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
          const uint32_t a_hi = tmem + kTmemS + (uint32_t)bj * kAtKeys + 16u * (uint32_t)kk;
          umma_f16_tmem_a(tmem + kTmemO, a_hi, bdesc, idesc_pv, kk > 0 ? 1u : 0u);
          umma_f16_tmem_a(tmem + kTmemO, a_hi + 8u, bdesc, idesc_pv, 1u);
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
    // ---------------- softmax: two threads per query row, 64 keys each ----------------
    const int quad = warp & 3, hf = warp >> 2;
    const int row = quad * 32 + lane;
    const bool in_block = row < A.G * TB;
    const int h = kvh * A.G + (in_block ? row / TB : 0);
    const int t = in_block ? t0 + row % TB : A.T;
    const int pos = t < A.T ? qbase + t : -1;  // -1: no keys
    float vtau = 0.f;     // raw indexer accumulator of the cut score (4 tau, an exact scaling)
    float vtau_lo = 0.f;  // the float just below it: x >= vtau  <=>  x > vtau_lo
    int tpos = -1;
    if (SPARSE && pos >= 0) {
      const int64_t qrow = ((int64_t)b * A.Hq + h) * A.T + t;
      vtau = __fmul_rn(__uint_as_float(A.tau_bits[qrow]), 4.f);
      vtau_lo = nextafterf(vtau, -INFINITY);
      tpos = A.tiepos[qrow];
    }
    const int wlo = pos - A.W + 1;  // window: first key a local row sees (may be negative)
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16) + 64u * (uint32_t)hf;
    float m_run = -INFINITY;  // running maximum of the scaled logits (log2 units)
    // The logits of 16 keys from k0 on, with the keys the row does not attend set to -inf.
    // Sparse: key k is attended iff k <= pos and (x > vtau or (x == vtau and k <= tpos)), x
    // its indexer accumulator; inside the causal prefix and away from the tie position that
    // is one compare against vtau or vtau_lo.  Window: wlo <= k <= pos.
    // Returns whether any of the 16 was masked.
    auto admit16 = [&](uint32_t (&v)[16], const uint32_t (&x)[16], int k0) -> bool {
      uint32_t any = 0u;
      if (SPARSE) {
        if (k0 + 15 <= pos && (k0 > tpos || k0 + 15 <= tpos)) {
          const float th = k0 > tpos ? vtau : vtau_lo;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const bool out = !(__uint_as_float(x[j]) > th);
            any |= (uint32_t)out;
            v[j] = out ? 0xff800000u : v[j];
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float xf = __uint_as_float(x[j]);
            const int k = k0 + j;
            const bool out = !(k <= pos && (xf > vtau || (xf == vtau && k <= tpos)));
            any |= (uint32_t)out;
            v[j] = out ? 0xff800000u : v[j];
          }
        }
      } else if (!(k0 >= wlo && k0 + 15 <= pos)) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const bool out = !(k0 + j >= wlo && k0 + j <= pos);
          any |= (uint32_t)out;
          v[j] = out ? 0xff800000u : v[j];
        }
      }
      return any != 0u;
    };
    for (int i = 0; i < ntiles; ++i) {
      const int bi = i & 1;
      const int kh = (tile0 + i) * kAtKeys + 64 * hf;  // first key of this thread's half
      if (SPARSE) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&S.idx_full, (uint32_t)i & 1u, alive, A.err, A.budget));
        if (!ok) {
          alive = false;
          break;
        }
      }
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait(&S.s_full[bi], (uint32_t)(i >> 1) & 1u, alive, A.err, A.budget));
      if (!ok) {
        alive = false;
        break;
      }
      tc_fence_after();
      const uint32_t sb = lane_base + kTmemS + (uint32_t)bi * kAtKeys;
      const uint32_t ib = lane_base + kTmemIdx;
      // pass 1: the logits the row does not attend are overwritten with -inf in place (so
      // that pass 2 needs no admission test and the indexer tile is free for the next one),
      // and the maximum of the rest is taken over both halves of the row
      float tmax = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t v[16], x[16];
        tmem_ld16(sb + 16u * (uint32_t)q, v);
        if (SPARSE) tmem_ld16(ib + 16u * (uint32_t)q, x);
        tmem_ld_wait();
        // (the store is warp-collective: taken by every lane when any lane masked a logit)
        if (__any_sync(0xffffffffu, admit16(v, x, kh + 16 * q))) tmem_st16(sb + 16u * (uint32_t)q, v);
#pragma unroll
        for (int jj = 0; jj < 16; jj += 2)
          tmax = max3f(tmax, __uint_as_float(v[jj]), __uint_as_float(v[jj + 1]));
      }
      tmem_st_wait();
      if (SPARSE) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.idx_free);
      }
      S.pmax[bi][hf][row] = tmax;
      named_sync(1 + quad, 64);  // warps quad and quad + 4
      tmax = fmaxf(S.pmax[bi][0][row], S.pmax[bi][1][row]);
      const float m_new = fmaxf(m_run, tmax * A.scale_log2);
      // reference of the exponentials; masked logits are -inf, so while no key of
      // the row is admitted yet (m_new = -inf) any finite reference gives P = 0
      const float m_ref = m_new == -INFINITY ? 0.f : m_new;
      // pass 2: P = 2^(s * scale * log2 e - m_new) as bf16 hi + lo, written over S
      // (16 keys at a time: slice q of 16 keys, which occupied columns
      // 16q .. 16q+15 as S, keeps its 8 hi words in 16q .. 16q+7 and its 8 lo
      // words in 16q+8 .. 16q+15, so a store only overwrites what was just read).
      // Pairs of keys go through packed fp32x2 instructions.
      float l0 = 0.f, l1 = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t v[16];
        tmem_ld16(sb + 16u * (uint32_t)q, v);
        tmem_ld_wait();
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          float y0, y1, p0, p1, r0, r1;
          fma2(__uint_as_float(v[2 * jj]), __uint_as_float(v[2 * jj + 1]), A.scale_log2, -m_ref, y0, y1);
          p0 = ex2a(y0);
          p1 = ex2a(y1);
          add2(l0, l1, p0, p1);
          hi[jj] = pack_bf16x2(p0, p1);
          sub2p(p0, p1, bf16_lo(hi[jj]), bf16_hi(hi[jj]), r0, r1);
          lo[jj] = pack_bf16x2(r0, r1);
        }
        tmem_st8(sb + 16u * (uint32_t)q, hi);
        tmem_st8(sb + 16u * (uint32_t)q + 8u, lo);
      }
      const float lsum = l0 + l1;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full[bi]);
      m_run = m_new;
      // hand the tile's (maximum, partial sum) to the fold
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&S.stat_free[bi], ((uint32_t)(i >> 1) & 1u) ^ 1u, alive, A.err, A.budget))) {
        alive = false;
        break;
      }
      S.stat[bi][hf][row] = make_float2(m_new, lsum);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.stat_full[bi]);
    }
  } else if (warp < kAtSoftWarps + kAtCorrWarps) {
    // ---------------- fold and output: two threads per query row, 64 head dims each ----------------
    const int cw = warp - kAtSoftWarps;
    const int quad = cw & 3, hf = cw >> 2;
    const int row = quad * 32 + lane;
    const bool in_block = row < A.G * TB;
    const int h = kvh * A.G + (in_block ? row / TB : 0);
    const int t = in_block ? t0 + row % TB : A.T;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16) + kTmemO + 64u * (uint32_t)hf;
    float o[64];
#pragma unroll
    for (int d = 0; d < 64; ++d) o[d] = 0.f;
    float m_t = -INFINITY, l_t = 0.f;  // reference maximum and denominator of o
    for (int j = 0; j < ntiles; ++j) {
      const int bj = j & 1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&S.stat_full[bj], (uint32_t)(j >> 1) & 1u, alive, A.err, A.budget))) {
        alive = false;
        break;
      }
      const float2 s0 = S.stat[bj][0][row], s1 = S.stat[bj][1][row];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.stat_free[bj]);
      if (!__all_sync(0xffffffffu, mbar_wait(&S.o_full, (uint32_t)j & 1u, alive, A.err, A.budget))) {
        alive = false;
        break;
      }
      tc_fence_after();
      // O_j was computed relative to s0.x (= s1.x); rescale the running sum to it
      const float mj = s0.x;
      const float alpha = mj == -INFINITY ? 1.f : ex2a(m_t - mj);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[16];
        tmem_ld16(lane_base + 16u * (uint32_t)c, v);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) o[16 * c + jj] = __fmaf_rn(o[16 * c + jj], alpha, __uint_as_float(v[jj]));
      }
      l_t = __fmaf_rn(l_t, alpha, s0.y + s1.y);
      if (mj != -INFINITY) m_t = mj;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.o_free);
    }

    // ---- normalise and store this thread's 64 head dims ----
    if (t < A.T) {
      const float inv = l_t > 0.f ? 1.f / l_t : 0.f;
      const int d0 = 64 * hf;
      if (A.o_bf16) {
        __nv_bfloat16* orow =
            static_cast<__nv_bfloat16*>(A.o.data) + b * A.o.sb + h * A.o.sh + (int64_t)t * A.o.sn + d0;
#pragma unroll
        for (int d = 0; d < 64; d += 8) {
          uint4 w;
          w.x = pack_bf16x2(o[d] * inv, o[d + 1] * inv);
          w.y = pack_bf16x2(o[d + 2] * inv, o[d + 3] * inv);
          w.z = pack_bf16x2(o[d + 4] * inv, o[d + 5] * inv);
          w.w = pack_bf16x2(o[d + 6] * inv, o[d + 7] * inv);
          *reinterpret_cast<uint4*>(orow + d) = w;
        }
      } else {
        float* orow = static_cast<float*>(A.o.data) + b * A.o.sb + h * A.o.sh + (int64_t)t * A.o.sn + d0;
#pragma unroll
        for (int d = 0; d < 64; d += 4)
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
  A.TB = prefill_tokens_per_block(A.G);
  CUtensorMap qmap, kmap, vmap, qimap{}, kimap{};
  if (!make_row_map(&qmap, a.q, a.B, a.Hq, a.T, A.TB)) return cudaErrorInvalidValue;
  if (!make_row_map(&kmap, a.k, a.B, a.Hk, a.N, kAtKeys)) return cudaErrorInvalidValue;
  if (!make_row_map(&vmap, a.v, a.B, a.Hk, a.N, kAtKeys)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(AtSmem) + 1024;
  const dim3 grid((unsigned)((a.T + A.TB - 1) / A.TB), (unsigned)(a.B * a.Hk));
  if (a.W > 0) {
    cudaFuncSetAttribute(attn_prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_prefill_kernel<false><<<grid, kAtThreads, smem, stream>>>(qmap, kmap, vmap, qimap, kimap, A);
  } else {
    if (!make_idx_map(&qimap, a.q_idx, a.B, a.Hq, a.T, A.TB)) return cudaErrorInvalidValue;
    if (!make_idx_map(&kimap, a.k_idx, a.B, a.Hk, a.N, kAtKeys)) return cudaErrorInvalidValue;
    cudaFuncSetAttribute(attn_prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_prefill_kernel<true><<<grid, kAtThreads, smem, stream>>>(qmap, kmap, vmap, qimap, kimap, A);
  }
  return cudaGetLastError();
}

}  // namespace rtp
