// a2 + a3 (prefill): indexer scores of every (query, earlier key) pair on the
// tcgen05 tensor cores, and the dynamic top-p cut of every query over its
// causal prefix, in threshold form (tau, tiepos, count) and optionally as a
// selection mask.
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 2-3: a 16-dim indexer ranks the
// tokens and each query keeps the cumulative top-p of that ranking.
//
// Design (B200): a CTA takes the G query heads of one KV head x 128/G
// consecutive query tokens (128 rows, row r = TMEM lane r), so every key tile
// it streams serves the whole GQA group.  A score tile of 128 rows x 128 keys
// is ONE tcgen05.mma (kind::f16, M=128, N=128, K=16): the projected queries
// (A) stay in shared memory, 128-key tiles of the projected-key cache (B) are
// streamed by TMA (32-byte swizzle, no multicast) through a 2-stage ring, and
// the fp32 accumulators alternate between two TMEM buffers so the next MMA
// runs while the epilogue reads the previous tile.  Warp roles (two CTAs per
// SM):
//   warps 0-7  epilogue: warp w reads TMEM lane quadrant w % 4; warps 0-3
//              take columns 0-63 of every tile, warps 4-7 columns 64-127, so
//              each query row is served by two threads ("halves"); the half-0
//              thread owns the row's decisions
//   warp 8     TMA producer (one elected lane)
//   warp 9     MMA issuer (one elected lane)
// The cut of every row is found by sweeps over its causal prefix; each sweep
// recomputes the score tiles (depth-16 MMAs are cheap) and narrows a bracket
// around the cut score.  All arithmetic is on the raw accumulator v = 4 s (the
// score scaling is exact), with u = m - v for the row maximum m:
//   MAX      row maximum m (3-input max, two independent halves)
//   LIN0     32 bins of u, 1/4 nat each (1/2 nat for caches longer than 2^17
//            keys, whose cut can lie deeper), the last one the tail, with
//            64-bit fixed-point masses; Z is their sum
//   TAIL     a cut in the last (tail) bin: the next 31 bins of the same width
//            further out, the last one again the rest (repeated up to 5 times,
//            far past the depth where a 64-bit fixed-point weight is still > 0)
//   LIN 1-3  32 sub-bins of the previous cut bin (each level 32 times finer;
//            power-of-two rescaling of u is exact), masses; a cut bin whose mass
//            is at most 32 times the least weight a key of it can have holds at
//            most 32 keys
//   COLLECT  once the cut bin holds <= 32 keys, their (v, position) pairs are
//            kept and sorted by (score desc, position asc) to finish the cut
//   MASK     (only when a mask is requested) one more sweep writes it
// Fallbacks: a cut past the last TAIL level, or a bin still too full after
// LIN 3, continue with 5-bit digits of the order-preserving uint32 image of the score
// (KEY) until one value is left; a TIE sweep then counts the keys above it and
// locates the ties in position order.
// Every bracket is an interval (vlo, vhi] of raw accumulators, precomputed
// once per row and sweep, so testing a key costs two compares; each thread
// then walks its own keys inside the bracket.  Masses are integers, so the cut does not depend on the order in
// which threads add them.
#include <math.h>

#include "launch.h"
#include "tc05.cuh"

namespace rtp {

namespace {

constexpr int kPfRows = 128;      // query rows per CTA (TMEM lanes)
constexpr int kPfKeys = 128;      // keys per score tile (MMA N)
constexpr int kPfStages = 2;      // K_idx tile ring (a tile's epilogue takes far longer than its load)
constexpr int kPfBins = 32;       // histogram bins per row (also the candidate capacity)
constexpr int kPfEpiWarps = 8;    // two per TMEM lane quadrant (column halves)
constexpr int kPfProducerWarp = kPfEpiWarps;
constexpr int kPfMmaWarp = kPfEpiWarps + 1;
constexpr int kPfThreads = (kPfEpiWarps + 2) * 32;
constexpr int kPfTileBytes = kPfKeys * kIdxDim * 2;  // 4 KB
constexpr int kPfTmemCols = 2 * kPfKeys;             // two accumulator buffers
constexpr int kPfMaxSweeps = 24;

enum PfLevel : int { kLvMax, kLvLin0, kLvTail, kLvLin, kLvKey, kLvCollect, kLvTie, kLvMask, kLvDone };

// A cut past the first level's 31 bins of u is binned again at the same width (TAIL), 31 bins further
// each time, up to this offset in first-level bins; past it the exact score-key digits take over.
constexpr int kPfMaxTailOff = 5 * 31;

// The part of a row's state that its half-1 thread needs in the next sweep
// (written by the row's half-0 thread after every sweep).
struct PfRowState {
  int level;
  float m;         // raw row maximum
  float vlo, vhi;  // bracket: raw accumulators v with vlo < v <= vhi
  float dscale;    // LIN: c0 * 32^lin
  int prefix;      // LIN: full bin index of the bracket at the previous level; TAIL: first-level bin of bin 0
  uint32_t kbase;  // KEY: lowest score key of the digit range
  int shift;       // KEY: digit shift
  uint64_t kend;   // KEY: one past the highest score key
  float vtau;      // MASK: raw accumulator of the cut score
  int tiepos;      // MASK: last selected position among keys equal to the cut score
};

struct PfSmem {
  alignas(1024) uint8_t qtile[kPfRows * kIdxDim * 2];  // A operand, 4 KB
  alignas(1024) uint8_t ktile[kPfStages][kPfTileBytes];  // B operand ring
  uint64_t hist[2][kPfBins][kPfRows];  // per half: bin masses, or candidates (COLLECT)
  PfRowState rs[kPfRows];
  float xs[16][kPfEpiWarps * 32];  // per epilogue thread: 16 keys of a chunk, for picking keys by column
  float pmax[kPfRows];  // half 1's partial maximum
  int pn[kPfRows];      // half 1's candidate count
  int pgt[kPfRows];     // half 1's count of keys above the bracket
  uint64_t q_full;
  uint64_t k_full[kPfStages];
  uint64_t k_empty[kPfStages];
  uint64_t t_full[2];
  uint64_t t_empty[2];
  uint32_t tmem_base;
};

struct PfArgs {
  const int32_t* lens;
  int Hq, Hk, G, T, N;
  int TB;  // tokens per block
  int GP;  // query heads per block (TB * GP <= 128 rows)
  float c0;  // level-0 bins per raw unit (1, or 1/2 for long caches: a 16-nat range before the tail)
  float p;
  float two_pow_frac;
  uint32_t* tau_bits;
  int32_t* tiepos;
  int32_t* count;
  uint32_t* mask;
  int64_t mask_words;
  int* err;
  long long budget;
};

// Fixed-point weight of a key at raw distance u = m - v from the row maximum:
// round(2^(u * wmul) * 2^frac) with wmul = -log2(e) / 4, i.e. exp(s - max s).
RTP_DEVICE uint64_t pf_weight_u(float u, float wmul, float two_pow_frac) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(e) : "f"(__fmul_rn(u, wmul)));
  return __float2ull_rn(__fmul_rn(e, two_pow_frac));
}

RTP_DEVICE float canon_score(float v) { return __fadd_rn(__fmul_rn(v, 0.25f), 0.0f); }

RTP_DEVICE float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// (a - c, b - c) in one packed fp32x2 instruction.
RTP_DEVICE void sub2(float a, float b, float c, float& ra, float& rb) {
  uint64_t x, y, z;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(x) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(y) : "f"(c), "f"(c));
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(z) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(ra), "=f"(rb) : "l"(z));
}

// (c - a·s, c - b·s) in one packed fp32x2 fused multiply-add.
RTP_DEVICE void cms2(float a, float b, float s, float c, float& ra, float& rb) {
  uint64_t x, y, z, r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(x) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(y) : "f"(-s), "f"(-s));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(z) : "f"(c), "f"(c));
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(r) : "l"(x), "l"(y), "l"(z));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(ra), "=f"(rb) : "l"(r));
}

// (a·s, b·s) in one packed fp32x2 multiply.
RTP_DEVICE void mul2(float a, float b, float s, float& ra, float& rb) {
  uint64_t x, y, r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(x) : "f"(a), "f"(b));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(y) : "f"(s), "f"(s));
  asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(r) : "l"(x), "l"(y));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(ra), "=f"(rb) : "l"(r));
}

RTP_DEVICE float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Level-0 bin of u: floor(u) clamped to [0, 31] (31 is the tail; NaN -> 0),
// by rounding u + 2^23 down, which leaves floor(u) in the low mantissa bits.
RTP_DEVICE int lin0_bin(float u) {
  const float x = __fadd_rd(fminf(fmaxf(u, 0.f), 31.f), 8388608.f);
  return __float_as_int(x) - 0x4B000000;
}

// The largest v with fsub_rn(m, v) >= u.  fsub_rn(m, v) does not increase
// with v, so {v : lo <= fsub_rn(m, v) < hi} = (vmax(hi), vmax(lo)]; binary
// search over the order-preserving integer image of the floats.
RTP_DEVICE float vmax_u_ge(float m, float u) {
  uint32_t lo = score_key(-INFINITY), hi = score_key(INFINITY);  // predicate true at lo, false at hi
  while (hi - lo > 1u) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    if (__fsub_rn(m, key_score(mid)) >= u)
      lo = mid;
    else
      hi = mid;
  }
  return key_score(lo);
}

RTP_DEVICE void hist_add(uint64_t* h, uint64_t w) { *h += w; }

}  // namespace

__global__ void __launch_bounds__(kPfThreads, 2)
topp_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, PfArgs A) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PfSmem& S = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // A block holds GP query heads of one KV head x TB consecutive tokens (row r:
  // head hq0 + r / TB, token t0 + r % TB), so the projected-key tiles it
  // streams serve all GP heads.  1-D grid ordered longest causal prefix
  // first across all KV heads, so every SM receives a mix of long and short blocks.
  const int TB = A.TB, GP = A.GP;  // GP query heads per block (all G of the group, or 1)
  const int nb = (A.T + TB - 1) / TB;
  const int hblocks = (int)(gridDim.x / nb);
  const int t0 = (nb - 1 - (int)blockIdx.x / hblocks) * TB;
  const int bg = (int)blockIdx.x % hblocks;
  const int b = bg / (A.Hq / GP), hq0 = (bg % (A.Hq / GP)) * GP, kvh = hq0 / A.G;
  int n_b = A.N;
  if (A.lens) n_b = min(max(A.lens[b], 0), A.N);
  const int qbase = n_b - A.T;  // position of query token 0
  // keys needed by the block: 0 .. position of its last token
  const int t_last = min(t0 + TB, A.T) - 1;
  const int kmax = min(qbase + t_last, n_b - 1);
  const int ntiles = kmax >= 0 ? kmax / kPfKeys + 1 : 0;
  const int64_t words = (A.N + 31) / 32;

  if (tid == 0) {
    mbar_init(&S.q_full, 1);
    for (int i = 0; i < kPfStages; ++i) {
      mbar_init(&S.k_full[i], 1);
      mbar_init(&S.k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.t_full[i], 1);
      mbar_init(&S.t_empty[i], kPfEpiWarps);
    }
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, kPfTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  bool alive = true;

  // ---- per-row state (epilogue threads) ---------------------------------------
  const bool epi = warp < kPfEpiWarps;
  const int quad = warp & 3, half = (warp >> 2) & 1;
  const int row = quad * 32 + lane;
  const bool in_block = row < GP * TB;
  const int h = hq0 + (in_block ? row / TB : 0);
  const int t = in_block ? t0 + row % TB : A.T;
  const int pos = qbase + t;
  const bool owner = epi && half == 0;
  const int64_t qrow = ((int64_t)b * A.Hq + h) * A.T + t;
  int level = (epi && t < A.T && pos >= 0) ? kLvMax : kLvDone;
  uint32_t* mrow = (A.mask && epi && t < A.T) ? A.mask + qrow * A.mask_words : nullptr;
  if (owner && t < A.T && pos < 0) {  // a token before the sequence: no keys
    A.tau_bits[qrow] = 0x7f800000u;
    A.tiepos[qrow] = -1;
    A.count[qrow] = 0;
    if (mrow)
      for (int64_t w = 0; w < words; ++w) mrow[w] = 0u;
  }
  float m = -INFINITY, vlo = 0.f, vhi = 0.f, dscale = A.c0, vtau = 0.f;
  int prefix = 0, shift = 0, tiepos = -1, ngt = 0, neq = 0, ncand = 0;
  uint32_t kbase = 0;
  uint64_t kend = 0;
  // owner-only state
  uint64_t target = 0, mass_above = 0;
  int lin = 0, n_tau = 0;
  uint32_t tau_key = 0;
  const float wmul = -0.25f * 1.4426950408889634f;  // weight 2^(u * wmul) = exp(-(m - v) / 4)

  uint32_t g = 0;      // tiles consumed so far, over all sweeps (drives every ring phase)
  uint32_t loads = 0;  // producer: K tiles issued
  uint32_t mmas = 0;   // MMA issuer: MMAs issued
  bool q_issued = false;
  for (int sweep = 0; sweep < kPfMaxSweeps; ++sweep) {
    const int more = __syncthreads_or(level != kLvDone);
    const int abort = __syncthreads_or(!alive);
    if (!more || abort || ntiles == 0) break;
    if (epi && (level == kLvLin0 || level == kLvTail || level == kLvLin || level == kLvKey)) {
#pragma unroll 4
      for (int i = 0; i < kPfBins; ++i) {
        S.hist[half][i][row] = 0;
      }
    }
    ncand = 0;
    if (level != kLvTie) ngt = 0;
    if (level == kLvMax) m = -INFINITY;

    if (warp == kPfProducerWarp) {
      // ---------------- TMA producer ----------------
      if (lane == 0) {
        if (sweep == 0) {
          // one box of TB rows per head of the group; rows past G * TB stay unused
          mbar_expect_tx(&S.q_full, GP * TB * kIdxDim * 2);
          for (int g = 0; g < GP; ++g)
            tma_load_4d(S.qtile + g * TB * kIdxDim * 2, &qmap, &S.q_full, 0, t0, hq0 + g, b);
          q_issued = true;
        }
        for (int i = 0; i < ntiles; ++i) {
          const uint32_t gi = g + i, st = gi % kPfStages, ph = (gi / kPfStages) & 1;
          if (!mbar_wait(&S.k_empty[st], ph ^ 1, alive, A.err, A.budget)) break;
          mbar_expect_tx(&S.k_full[st], kPfTileBytes);
          tma_load_4d(S.ktile[st], &kmap, &S.k_full[st], 0, i * kPfKeys, kvh, b);
          loads = gi + 1;
        }
      }
    } else if (warp == kPfMmaWarp) {
      // ---------------- MMA issuer ----------------
      if (lane == 0) {
        if (sweep == 0) mbar_wait(&S.q_full, 0, alive, A.err, A.budget);
        const uint64_t adesc = umma_desc_k_sw32(S.qtile);
        constexpr uint32_t idesc = umma_idesc_bf16_f32(kPfRows, kPfKeys);
        for (int i = 0; i < ntiles; ++i) {
          const uint32_t gi = g + i, st = gi % kPfStages, buf = gi & 1;
          if (!mbar_wait(&S.k_full[st], (gi / kPfStages) & 1, alive, A.err, A.budget)) break;
          if (!mbar_wait(&S.t_empty[buf], ((gi >> 1) & 1) ^ 1, alive, A.err, A.budget)) break;
          tc_fence_after();
          umma_f16(tmem + buf * kPfKeys, adesc, umma_desc_k_sw32(S.ktile[st]), idesc, 0);
          umma_commit(&S.k_empty[st]);
          umma_commit(&S.t_full[buf]);
          mmas = gi + 1;
        }
      }
    } else {
      // ---------------- epilogue: two threads per query row ----------------
      const float mh = m;
      const bool bracket = level == kLvLin || level == kLvTail || level == kLvKey || level == kLvCollect;
      // the screen: past the first linear level (a bracket 1/32 as wide or less) and with
      // finite bounds; bhw is the half width plus a margin for the rounding of x - c
      const bool screen = (level == kLvCollect || (level == kLvLin && dscale > 32.f * A.c0)) &&
                          vlo > -INFINITY && vhi < INFINITY;
      const float bc = __fmaf_rn(0.5f, vlo, 0.5f * vhi);
      const float bhw = 0.5f * (vhi - vlo) + 1e-6f * fmaxf(fabsf(vlo), fabsf(vhi)) + 1e-30f;
      for (int i = 0; i < ntiles; ++i) {
        const uint32_t gi = g + i, buf = gi & 1;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&S.t_full[buf], (gi >> 1) & 1, alive, A.err, A.budget));
        if (!ok) {
          alive = false;
          break;
        }
        tc_fence_after();
        const uint32_t tb = tmem + ((uint32_t)(quad * 32) << 16) + buf * kPfKeys;
        // a TIE row is finished by its half-0 thread alone, over all 128 columns in position order
        const bool tie_warp = half == 0 && __any_sync(0xffffffffu, level == kLvTie);
        const int nch = tie_warp ? 4 : 2;
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          const int col = tie_warp ? 32 * c : 64 * half + 32 * c;
          uint32_t v[32];
          tmem_ld32(tb + col, v);
          tmem_ld_wait();
          if (c == nch - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.t_empty[buf]);
          }
          const int kb = i * kPfKeys + col;
          const int nv = pos - kb + 1;  // keys of this chunk inside the row's causal prefix
          const bool own = (col >> 6) == half;
          const uint32_t vmask = nv >= 32 ? 0xffffffffu : (nv > 0 ? (1u << nv) - 1u : 0u);
          if (level == kLvMax) {
            if (own && nv > 0) {
              float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
              if (nv >= 32) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  a0 = max3f(a0, __uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                  a1 = max3f(a1, __uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                  a2 = max3f(a2, __uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                  a3 = max3f(a3, __uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                }
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nv) a0 = fmaxf(a0, __uint_as_float(v[j]));
              }
              m = max3f(m, max3f(a0, a1, a2), a3);
            }
          } else if (level == kLvLin0) {
            if (own && nv >= 32) {
              // the whole chunk is inside the prefix, so every u = m - v is >= 0: per pair of keys
              // c0 u in one packed multiply-add (c0 a power of two: the same bits as c0 (m - v)),
              // the weights' scalings in packed multiplies, and the two read-modify-writes
              // overlapped (a pair in one bin is added as one update)
              uint64_t* H = &S.hist[half][0][row];
              const float mc = __fmul_rn(mh, A.c0), wmc = __fdiv_rn(wmul, A.c0);
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                float u0, u1, x0, x1, e0, e1, y0, y1;
                cms2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), A.c0, mc, u0, u1);
                const int d0 = __float_as_int(__fadd_rd(fminf(u0, 31.f), 8388608.f)) - 0x4B000000;
                const int d1 = __float_as_int(__fadd_rd(fminf(u1, 31.f), 8388608.f)) - 0x4B000000;
                mul2(u0, u1, wmc, x0, x1);
                asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(e0) : "f"(x0));
                asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(e1) : "f"(x1));
                y0 = __fmul_rn(e0, A.two_pow_frac);
                y1 = __fmul_rn(e1, A.two_pow_frac);
                const uint64_t w0 = __float2ull_rn(y0), w1 = __float2ull_rn(y1);
                const uint64_t h0 = H[d0 * kPfRows], h1 = H[d1 * kPfRows];
                const uint64_t s0 = h0 + w0;
                const uint64_t s1 = (d0 == d1 ? s0 : h1) + w1;
                H[d0 * kPfRows] = s0;
                H[d1 * kPfRows] = s1;  // after s0: a pair in one bin ends as h + w0 + w1
              }
            } else if (own && nv > 0) {
              // every key lands in a bin; consecutive keys are taken in pairs so that the two
              // read-modify-writes overlap (a pair in one bin is added as one update)
              uint64_t* H = &S.hist[half][0][row];
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                const float u0 = __fsub_rn(mh, __uint_as_float(v[j]));
                const float u1 = __fsub_rn(mh, __uint_as_float(v[j + 1]));
                const int d0 = lin0_bin(__fmul_rn(u0, A.c0)), d1 = lin0_bin(__fmul_rn(u1, A.c0));
                const uint64_t w0 = j < nv ? pf_weight_u(u0, wmul, A.two_pow_frac) : 0ull;
                const uint64_t w1 = j + 1 < nv ? pf_weight_u(u1, wmul, A.two_pow_frac) : 0ull;
                const uint64_t h0 = H[d0 * kPfRows], h1 = H[d1 * kPfRows];
                const bool same = d0 == d1;
                const uint64_t s0 = h0 + w0 + (same ? w1 : 0ull);
                const uint64_t s1 = same ? s0 : h1 + w1;
                H[d0 * kPfRows] = s0;
                H[d1 * kPfRows] = s1;
              }
            }
          }
          {
            // bracket levels: the keys inside are found by two compares each, then handled one
            // by one.  Past the first linear level a chunk rarely holds one, so a cheap screen
            // (the least |x - c| over the chunk, c the bracket's centre) skips the compares.
            uint32_t inb = 0u;
            if (bracket && own) {
              bool maybe = true;
              if (screen) {
                float mn = INFINITY;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                  float d0, d1;
                  sub2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), bc, d0, d1);
                  mn = min3f(mn, fabsf(d0), fabsf(d1));
                }
                maybe = mn <= bhw;
              }
              if (maybe) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  const float x = __uint_as_float(v[j]);
                  inb |= (uint32_t)(x > vlo && x <= vhi) << j;
                }
                inb &= vmask;
              }
              if (level == kLvCollect) {  // keys above the bracket
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                  a0 += (j < nv && __uint_as_float(v[j]) > vhi) ? 1.f : 0.f;
                  a1 += (j + 1 < nv && __uint_as_float(v[j + 1]) > vhi) ? 1.f : 0.f;
                }
                ngt += (int)(a0 + a1);
              }
            }
            // each lane walks its own keys inside the bracket (about one in twelve at the first
            // linear level, far fewer later): each half chunk holding one goes to the thread's
            // column of a shared array, so that a key can be picked by its index
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t hb = (inb >> (16 * hh)) & 0xFFFFu;
              if (!hb) continue;
#pragma unroll
              for (int j = 0; j < 16; ++j) S.xs[j][tid] = __uint_as_float(v[16 * hh + j]);
              while (hb) {
                const int j = 16 * hh + __ffs(hb) - 1;
                hb &= hb - 1u;
                const float x = S.xs[j - 16 * hh][tid];
                const float u = __fsub_rn(mh, x);
                if (level == kLvLin || level == kLvTail) {
                  const int d = min(max((int)__fmul_rn(u, dscale) - (level == kLvTail ? prefix : 32 * prefix), 0),
                                    kPfBins - 1);
                  hist_add(&S.hist[half][d][row], pf_weight_u(u, wmul, A.two_pow_frac));
                } else if (level == kLvKey) {
                  const uint32_t k = score_key(canon_score(x));
                  if (k >= kbase && (uint64_t)k < kend) {
                    const int d = (int)((k - kbase) >> shift);
                    hist_add(&S.hist[half][d][row], pf_weight_u(u, wmul, A.two_pow_frac));
                  }
                } else {  // COLLECT
                  if (ncand < kPfBins)
                    S.hist[half][ncand][row] = ((uint64_t)(uint32_t)(kb + j) << 32) | __float_as_uint(x);
                  ++ncand;
                }
              }
            }
            if (level == kLvMask && own) {
              uint32_t bits = 0u;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float x = __uint_as_float(v[j]);
                bits |= (uint32_t)(x > vtau || (x == vtau && kb + j <= tiepos)) << j;
              }
              bits &= vmask;
              if ((kb >> 5) < A.mask_words) mrow[kb >> 5] = bits;
            } else if (level == kLvTie && half == 0) {
              uint32_t bits = 0u;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (j < nv) {
                  const float x = __uint_as_float(v[j]);
                  const bool gt = x > vtau;
                  bool sel = gt;
                  ngt += gt;
                  if (x == vtau) {
                    ++neq;
                    sel = neq <= n_tau;
                    if (neq == n_tau) tiepos = kb + j;
                  }
                  bits |= (uint32_t)sel << j;
                }
              }
              if (mrow && (kb >> 5) < A.mask_words) mrow[kb >> 5] = bits;
            }
          }
        }
      }
      if (half == 1) {
        S.pmax[row] = m;
        S.pn[row] = ncand;
        S.pgt[row] = ngt;
      }
    }
    g += ntiles;
    __syncthreads();  // both halves' partial results are in shared memory

    // ---- end of sweep: the row's half-0 thread advances its bracket ----
    if (owner && level != kLvDone && alive) {
      if (level == kLvMax) {
        m = fmaxf(m, S.pmax[row]);  // m is the raw maximum
        level = kLvLin0;
      } else if (level == kLvTie) {
        const int64_t w_end = 4 * (int64_t)ntiles;
        if (mrow)  // words past the block's last tile
          for (int64_t w = w_end; w < words; ++w) mrow[w] = 0u;
        A.tau_bits[qrow] = __float_as_uint(key_score(tau_key));
        A.tiepos[qrow] = tiepos;
        A.count[qrow] = ngt + min(n_tau, neq);
        level = kLvDone;
      } else if (level == kLvMask) {
        if (mrow)
          for (int64_t w = 4 * (int64_t)ntiles; w < words; ++w) mrow[w] = 0u;
        level = kLvDone;
      } else if (level == kLvCollect) {
        // both halves' candidates, sorted by (score desc, position asc), taken in order
        const int n0 = min(ncand, kPfBins);
        const int n1 = min(S.pn[row], kPfBins - n0);
        for (int a = 0; a < n1; ++a) S.hist[0][n0 + a][row] = S.hist[1][a][row];
        const int n = n0 + n1;
        const int gt_all = ngt + S.pgt[row];
        for (int a = 1; a < n; ++a) {
          const uint64_t x = S.hist[0][a][row];
          const float xv = __uint_as_float((uint32_t)x);
          const uint32_t xp = (uint32_t)(x >> 32);
          int bI = a - 1;
          while (bI >= 0) {
            const uint64_t y = S.hist[0][bI][row];
            const float yv = __uint_as_float((uint32_t)y);
            if (yv > xv || (yv == xv && (uint32_t)(y >> 32) < xp)) break;
            S.hist[0][bI + 1][row] = y;
            --bI;
          }
          S.hist[0][bI + 1][row] = x;
        }
        const uint64_t need = target - mass_above;
        uint64_t cum = 0;
        int taken = n;
        for (int a = 0; a < n; ++a) {
          cum += pf_weight_u(__fsub_rn(m, __uint_as_float((uint32_t)S.hist[0][a][row])), wmul, A.two_pow_frac);
          if (cum >= need) {
            taken = a + 1;
            break;
          }
        }
        if (taken < 1) taken = 1;
        const uint64_t last = S.hist[0][taken - 1][row];
        vtau = __uint_as_float((uint32_t)last);
        tiepos = (int)(last >> 32);
        A.tau_bits[qrow] = __float_as_uint(canon_score(vtau));
        A.tiepos[qrow] = tiepos;
        A.count[qrow] = gt_all + taken;
        level = mrow ? kLvMask : kLvDone;  // the selection mask needs one more sweep
      } else {  // LIN0, TAIL, LIN or KEY: find the cut bin
        if (level == kLvLin0) {
          uint64_t Z = 0;
          for (int i = 0; i < kPfBins; ++i) {
            const uint64_t hv = S.hist[0][i][row] + S.hist[1][i][row];
            S.hist[0][i][row] = hv;
            Z += hv;
          }
          const double tt = ceil((double)A.p * (double)Z);
          const uint64_t tg = tt >= (double)Z ? Z : (uint64_t)tt;
          target = tg < 1 ? 1 : tg;
        } else {
          for (int i = 0; i < kPfBins; ++i) S.hist[0][i][row] += S.hist[1][i][row];
        }
        // the first bin (in score order) where the cumulative mass reaches the target; should
        // rounding ever leave it short, the last non-empty bin
        const uint64_t need = target - mass_above;
        uint64_t cum = 0, cum_nz = 0;
        int cut = -1, last_nz = level == kLvKey ? kPfBins - 1 : 0;
        for (int r = 0; r < kPfBins; ++r) {
          const int bin = level == kLvKey ? kPfBins - 1 - r : r;
          const uint64_t hv = S.hist[0][bin][row];
          if (hv) {
            last_nz = bin;
            cum_nz = cum;
          }
          if (cum + hv >= need) {
            cut = bin;
            break;
          }
          cum += hv;
        }
        if (cut < 0) {
          cut = last_nz;
          cum = cum_nz;
        }
        mass_above += cum;
        if (level == kLvLin0 || level == kLvTail || level == kLvLin) {
          const int off = level == kLvTail ? prefix : 0;  // first-level bin of this level's bin 0
          if (level != kLvLin && cut == kPfBins - 1 && off + 31 <= kPfMaxTailOff) {
            // the cut lies past this level's 31 bins (c0 u >= off + 31): the next 31 bins of the same
            // width, over the keys from there on (the last bin again holds the rest)
            prefix = off + 31;
            vlo = -INFINITY;
            vhi = vmax_u_ge(m, (float)prefix / A.c0);  // exact: c0 is a power of two
            level = kLvTail;
          } else if (level != kLvLin && cut == kPfBins - 1) {
            // still further out: exact digits over the keys past the last binned range
            const float u_tail = (float)(off + 31) / A.c0;
            const float hi_s = __fmul_rn(__fsub_rn(m, u_tail), 0.25f);
            const float mg = 1e-5f * (fabsf(hi_s) + 8.f) + 1e-30f;
            kbase = 0u;
            kend = (uint64_t)score_key(__fadd_rn(hi_s + mg, 0.0f)) + 1;
            shift = 0;
            while (((kend - kbase - 1) >> shift) >= (uint64_t)kPfBins) ++shift;
            vlo = -INFINITY;
            vhi = vmax_u_ge(m, u_tail);
            level = kLvKey;
          } else {
            prefix = level == kLvLin ? 32 * prefix + cut : off + cut;  // full bin index at level `lin`
            const float ulo = (float)prefix / dscale;             // exact: dscale is a power of two
            const float uhi = (float)(prefix + 1) / dscale;
            vlo = vmax_u_ge(m, uhi);
            vhi = vmax_u_ge(m, ulo);
            // every key of the cut bin has u < uhi, so weighs at least the weight at uhi: the bin's
            // mass bounds how many keys it holds (2^-20 covers the rounding of the exponential)
            const uint64_t w_lo = pf_weight_u(uhi, wmul, A.two_pow_frac);
            const bool few = w_lo > 0 && (double)S.hist[0][cut][row] <=
                                             (double)kPfBins * (double)w_lo * (1.0 - 9.5367431640625e-07);
            if (few) {
              level = kLvCollect;
            } else if (lin < 3) {
              ++lin;
              dscale *= 32.f;
              level = kLvLin;
            } else {
              // still too many keys: exact digits inside this bracket of u
              const float hi_s = __fmul_rn(__fsub_rn(m, ulo), 0.25f);
              const float lo_s = __fmul_rn(__fsub_rn(m, uhi), 0.25f);
              const float mg = 1e-5f * (fabsf(hi_s) + fabsf(lo_s) + uhi) + 1e-30f;
              kbase = score_key(__fadd_rn(lo_s - mg, 0.0f));
              kend = (uint64_t)score_key(__fadd_rn(hi_s + mg, 0.0f)) + 1;
              shift = 0;
              while (((kend - kbase - 1) >> shift) >= (uint64_t)kPfBins) ++shift;
              level = kLvKey;
            }
          }
        } else {  // KEY
          kbase += (uint32_t)cut << shift;
          const uint64_t e = (uint64_t)kbase + (uint64_t(1) << shift);
          kend = e < kend ? e : kend;
          if (shift == 0) {
            tau_key = kbase;
            const float st = key_score(tau_key);
            const uint64_t w_tau = pf_weight_u(__fsub_rn(m, __fmul_rn(st, 4.f)), wmul, A.two_pow_frac);
            const uint64_t rem = target - mass_above;
            const uint64_t nt = w_tau ? (rem + w_tau - 1) / w_tau : 1;
            n_tau = (int)(nt < 1 ? 1 : (nt > 0x7fffffffull ? 0x7fffffffull : nt));
            vtau = __fmul_rn(st, 4.f);
            ngt = 0;
            neq = 0;
            tiepos = -1;
            level = kLvTie;
          } else {
            shift = shift >= 5 ? shift - 5 : 0;
          }
        }
      }
    }
    if (owner) {
      PfRowState& R = S.rs[row];
      R.level = level;
      R.m = m;
      R.vlo = vlo;
      R.vhi = vhi;
      R.dscale = dscale;
      R.prefix = prefix;
      R.kbase = kbase;
      R.shift = shift;
      R.kend = kend;
      R.vtau = vtau;
      R.tiepos = tiepos;
    }
    __syncthreads();
    if (epi && half == 1) {
      const PfRowState& R = S.rs[row];
      level = R.level;
      m = R.m;
      vlo = R.vlo;
      vhi = R.vhi;
      dscale = R.dscale;
      prefix = R.prefix;
      kbase = R.kbase;
      shift = R.shift;
      kend = R.kend;
      vtau = R.vtau;
      tiepos = R.tiepos;
    }
  }

  // ---- wind down: every copy and MMA this CTA issued lands before its tensor
  // memory is freed and it exits, even after a wait gave up
  if (warp == kPfMmaWarp && lane == 0 && mmas > 0) {
    const uint32_t last = mmas - 1;
    mbar_drain(&S.t_full[last & 1], (last >> 1) & 1, A.err);
  }
  if (warp == kPfProducerWarp && lane == 0) {
    if (q_issued) mbar_drain(&S.q_full, 0, A.err);
    for (uint32_t i = loads > (uint32_t)kPfStages ? loads - kPfStages : 0u; i < loads; ++i)
      mbar_drain(&S.k_full[i % kPfStages], (i / kPfStages) & 1, A.err);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_free(tmem, kPfTmemCols);
}

// p >= 1: every candidate is selected.
__global__ void topp_prefill_all_kernel(PfArgs A, int rows) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const int t = (int)(r % A.T);
  const int bh = (int)(r / A.T);
  const int b = bh / A.Hq;
  int n_b = A.N;
  if (A.lens) n_b = min(max(A.lens[b], 0), A.N);
  const int pos = n_b - A.T + t;
  A.tau_bits[r] = pos >= 0 ? 0xff800000u : 0x7f800000u;
  A.tiepos[r] = pos >= 0 ? pos : -1;
  A.count[r] = pos >= 0 ? pos + 1 : 0;
  if (A.mask) {
    uint32_t* mrow = A.mask + r * A.mask_words;
    for (int w = 0; w < (A.N + 31) / 32; ++w) {
      const int nv = min(max(pos + 1 - w * 32, 0), 32);
      mrow[w] = nv >= 32 ? 0xffffffffu : ((1u << nv) - 1u);
    }
  }
}

// ---- host side ------------------------------------------------------------------

cudaError_t launch_topp_prefill(const LaunchToppPrefill& a, cudaStream_t stream) {
  const int64_t rows = a.B * a.Hq * a.T;
  if (rows == 0) return cudaSuccess;
  PfArgs A;
  A.lens = a.lens;
  A.Hq = (int)a.Hq;
  A.Hk = (int)a.Hk;
  A.G = (int)(a.Hq / a.Hk);
  A.T = (int)a.T;
  A.N = (int)a.N;
  A.p = a.p;
  int lg = 0;
  while ((int64_t(1) << lg) < a.N) ++lg;
  A.two_pow_frac = ldexpf(1.f, 63 - lg);
  A.tau_bits = a.tau_bits;
  A.tiepos = a.tiepos;
  A.count = a.count;
  A.mask = a.mask;
  A.mask_words = a.mask_words;
  A.err = a.err;
  A.budget = wait_budget_cycles();
  if (a.p >= 1.f) {
    topp_prefill_all_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(A, (int)rows);
    return cudaGetLastError();
  }
  A.c0 = a.N > (int64_t(1) << 17) ? 0.5f : 1.f;
  A.GP = A.G;
  A.TB = prefill_tokens_per_block(A.GP);
  CUtensorMap qmap, kmap;
  if (!make_idx_map(&qmap, a.q_idx, a.B, a.Hq, a.T, A.TB)) return cudaErrorInvalidValue;
  if (!make_idx_map(&kmap, a.k_idx, a.B, a.Hk, a.N, kPfKeys)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(PfSmem) + 1024;
  cudaFuncSetAttribute(topp_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(topp_prefill_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  const dim3 grid((unsigned)(((a.T + A.TB - 1) / A.TB) * a.B * (a.Hq / A.GP)));
  topp_prefill_kernel<<<grid, kPfThreads, smem, stream>>>(qmap, kmap, A);
  return cudaGetLastError();
}

}  // namespace rtp
