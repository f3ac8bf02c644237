// a2 + a3 (prefill): indexer scores of every (query, earlier key) pair on the
// tcgen05 tensor cores, and the dynamic top-p cut of every query over its
// causal prefix, in threshold form (tau, tiepos, count).
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 2-3: a 16-dim indexer ranks the
// tokens and each query keeps the cumulative top-p of that ranking.
//
// Design (B200): a CTA takes one query head and 128 consecutive query tokens;
// token r of the block is TMEM lane r.  The score tile of 128 tokens x 64 keys
// is ONE tcgen05.mma (kind::f16, M=128, N=64, K=16): the projected queries
// (A) stay in shared memory, 64-key tiles of the projected-key cache (B) are
// streamed by TMA (32-byte swizzle, each CTA loading its own) through a 2-stage ring, and
// the fp32 accumulators alternate between two TMEM buffers so the next MMA
// runs while four epilogue warps read the previous tile.  Warp roles:
//   warps 0-3  epilogue: thread r owns query row r (its TMEM lane)
//   warp 4     TMA producer (one elected lane)
//   warp 5     MMA issuer (one elected lane)
// The cut of every row is found by sweeps over its causal prefix; each sweep
// recomputes the score tiles (depth-16 MMAs are cheap) and narrows a bracket
// around the cut score, every row on the same schedule:
//   MAX      row maximum m
//   LIN 0-3  32 bins of u = m - s, 1/4, 1/128, 1/4096, 1/131072 nat wide (each
//            level splits the previous cut bin; power-of-two rescaling of u is
//            exact), with 64-bit fixed-point masses (Z on level 0) and counts
//   COLLECT  once the cut bin holds <= 32 keys, their (score, position) pairs
//            are kept and an in-thread sort by (score desc, position asc)
//            finishes the cut: tau, the number taken, tiepos, count
// Fallbacks: the tail bin of level 0, or a bin still too full after level 3,
// continue with 5-bit digits of the order-preserving uint32 image of the score
// (KEY) until one value is left, then a TIE sweep counts and locates the ties;
// the TIE sweep also writes the optional selection mask.
// A row owns its 32-bin histogram columns in shared memory (no atomics); the
// candidate list reuses the row's mass column.
#include <cudaTypedefs.h>

#include <math.h>

#include "launch.h"
#include "tc05.cuh"

namespace rtp {

constexpr int kPfRows = 128;      // query rows per CTA (TMEM lanes)
constexpr int kPfKeys = 64;       // keys per score tile (MMA N)
constexpr int kPfStages = 2;      // K_idx tile ring
constexpr int kPfBins = 32;       // histogram bins per row (also the candidate capacity)
constexpr int kPfThreads = 192;   // 4 epilogue warps + producer + MMA
constexpr int kPfTileBytes = kPfKeys * kIdxDim * 2;  // 2 KB
constexpr int kPfTmemCols = 2 * kPfKeys;             // two accumulator buffers

enum PfLevel : int { kLvMax = 0, kLvLin = 1, kLvCollect = 2, kLvKey = 3, kLvTie = 4, kLvDone = 5 };

struct PfSmem {
  alignas(256) uint8_t qtile[kPfRows * kIdxDim * 2];             // A operand, 4 KB
  alignas(256) uint8_t ktile[kPfStages][kPfTileBytes];            // B operand ring
  uint64_t hist[kPfBins][kPfRows];                                // per-row masses / candidates
  uint16_t hcnt[kPfBins][kPfRows];                                // per-row counts (saturating)
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
  float p;
  float two_pow_frac;
  uint32_t* tau_bits;
  int32_t* tiepos;
  int32_t* count;
  uint32_t* mask;
  int64_t mask_words;
  int* err;
};

// Fixed-point weight of a key at raw distance u = m - v from the row maximum:
// round(2^(u * wmul) * 2^frac) with wmul = -log2(e) / 4, i.e. exp(s - max s).
RTP_DEVICE uint64_t pf_weight_u(float u, float wmul, float two_pow_frac) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(e) : "f"(__fmul_rn(u, wmul)));
  return __float2ull_rn(__fmul_rn(e, two_pow_frac));
}

__global__ void __launch_bounds__(kPfThreads, 2)
topp_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, PfArgs A) {
  extern __shared__ __align__(256) unsigned char smem_raw[];
  PfSmem& S = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 255) & ~uintptr_t(255));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // 1-D grid ordered longest causal prefix first across all heads, so every SM
  // receives a mix of long and short blocks
  const int nb = (A.T + kPfRows - 1) / kPfRows;
  const int heads = (int)(gridDim.x / nb);
  const int t0 = (nb - 1 - (int)blockIdx.x / heads) * kPfRows;
  const int bh = (int)blockIdx.x % heads;
  const int b = bh / A.Hq, h = bh % A.Hq, kvh = h / A.G;
  int n_b = A.N;
  if (A.lens) n_b = min(max(A.lens[b], 0), A.N);
  const int qbase = n_b - A.T;  // position of query token 0
  // keys needed by the block: 0 .. position of its last token
  const int t_last = min(t0 + kPfRows, A.T) - 1;
  const int kmax = min(qbase + t_last, n_b - 1);
  const int ntiles = kmax >= 0 ? (kmax + kPfKeys) / kPfKeys : 0;

  if (tid == 0) {
    mbar_init(&S.q_full, 1);
    for (int i = 0; i < kPfStages; ++i) {
      mbar_init(&S.k_full[i], 1);
      mbar_init(&S.k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.t_full[i], 1);
      mbar_init(&S.t_empty[i], kPfRows);
    }
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, kPfTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  bool alive = true;

  // ---- per-row state (epilogue threads) -------------------------------------
  const int row = tid;  // valid for tid < 128
  const int t = t0 + row;
  const int pos = qbase + t;
  const bool is_row = tid < kPfRows;
  int level = (is_row && t < A.T && pos >= 0) ? kLvMax : kLvDone;
  if (is_row && t < A.T && pos < 0) {  // a token before the sequence: no keys
    const int64_t qrow = (int64_t)bh * A.T + t;
    A.tau_bits[qrow] = 0x7f800000u;
    A.tiepos[qrow] = -1;
    A.count[qrow] = 0;
  }
  // Everything below works on raw accumulators v (the score is s = v / 4, an
  // exact scaling): u = m - v with m the row's raw maximum.  Level-k bins are
  // floor(u * 32^k) (level 0: floor(u), the tail folded into bin 31), so a
  // level-k bin P is the interval [P / 32^k, (P + 1) / 32^k) of u, exactly.
  float m = -INFINITY;
  uint64_t target = 0, mass_above = 0;
  int lin = 0, prefix = 0, tail = 0, shift = 0, n_tau = 0, ngt = 0, neq = 0, tiepos = -1, ncand = 0;
  float ulo = 0.f, uhi = 0.f, dscale = 1.f;  // current bracket of u, and 32^lin
  uint32_t kbase = 0, tau_key = 0;
  uint64_t kend = 0;
  const float wmul = -0.25f * 1.4426950408889634f;  // weight 2^(u * wmul) = exp(-(m - v) / 4)
  uint32_t* mrow = (A.mask && is_row && t < A.T) ? A.mask + ((int64_t)bh * A.T + t) * A.mask_words : nullptr;

  uint32_t g = 0;  // global tile counter across sweeps (drives every ring phase)
  for (int sweep = 0; sweep < 16; ++sweep) {
    const int more = __syncthreads_or(is_row && level != kLvDone);
    const int abort = __syncthreads_or(!alive);
    if (!more || abort || ntiles == 0) break;
    if (is_row && level == kLvLin && lin == 0) dscale = 1.f;
    if (is_row && (level == kLvLin || level == kLvKey))
      for (int i = 0; i < kPfBins; ++i) {
        S.hist[i][row] = 0;
        S.hcnt[i][row] = 0;
      }
    if (is_row) {
      ncand = 0;
      if (level == kLvCollect) ngt = 0;
    }

    if (warp == 4) {
      // ---------------- TMA producer ----------------
      if (lane == 0) {
        if (sweep == 0) {
          mbar_expect_tx(&S.q_full, kPfRows * kIdxDim * 2);
          tma_load_4d(S.qtile, &qmap, &S.q_full, 0, t0, h, b);
        }
        for (int i = 0; i < ntiles; ++i) {
          const uint32_t gi = g + i, st = gi % kPfStages, ph = (gi / kPfStages) & 1;
          if (!mbar_wait(&S.k_empty[st], ph ^ 1, alive, A.err)) break;
          mbar_expect_tx(&S.k_full[st], kPfTileBytes);
          tma_load_4d(S.ktile[st], &kmap, &S.k_full[st], 0, i * kPfKeys, kvh, b);
        }
      }
    } else if (warp == 5) {
      // ---------------- MMA issuer ----------------
      if (lane == 0) {
        if (sweep == 0) mbar_wait(&S.q_full, 0, alive, A.err);
        const uint64_t adesc = umma_desc_k_sw32(S.qtile);
        constexpr uint32_t idesc = umma_idesc_bf16_f32(kPfRows, kPfKeys);
        for (int i = 0; i < ntiles; ++i) {
          const uint32_t gi = g + i, st = gi % kPfStages, buf = gi & 1;
          if (!mbar_wait(&S.k_full[st], (gi / kPfStages) & 1, alive, A.err)) break;
          if (!mbar_wait(&S.t_empty[buf], ((gi >> 1) & 1) ^ 1, alive, A.err)) break;
          tc_fence_after();
          umma_f16(tmem + buf * kPfKeys, adesc, umma_desc_k_sw32(S.ktile[st]), idesc, 0);
          umma_commit(&S.k_empty[st]);
          umma_commit(&S.t_full[buf]);
        }
      }
    } else {
      // ---------------- epilogue: one query row per thread ----------------
      const float mh = m;
      for (int i = 0; i < ntiles; ++i) {
        const uint32_t gi = g + i, buf = gi & 1;
        if (!mbar_wait(&S.t_full[buf], (gi >> 1) & 1, alive, A.err)) break;
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + buf * kPfKeys;
        const int key0 = i * kPfKeys;
        uint64_t mbits = 0ull;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {  // two chunks of 32 columns
          uint32_t v[32];
          tmem_ld32(taddr + half * 32, v);
          tmem_ld_wait();
          if (half == 1) {
            tc_fence_before();
            mbar_arrive(&S.t_empty[buf]);
          }
          if (level == kLvDone) continue;
          const int kb = key0 + half * 32;
          const int nv = pos - kb + 1;  // keys of this chunk inside the row's causal prefix
          if (nv <= 0) continue;
          if (level == kLvMax) {
            if (nv >= 32) {
#pragma unroll
              for (int j = 0; j < 32; ++j) m = fmaxf(m, __uint_as_float(v[j]));
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < nv) m = fmaxf(m, __uint_as_float(v[j]));
            }
          } else if (level == kLvTie) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nv) {
                const float sv = __fadd_rn(__fmul_rn(__uint_as_float(v[j]), 0.25f), 0.0f);
                const uint32_t k = score_key(sv);
                const bool gt = k > tau_key;
                bool sel = gt;
                ngt += gt;
                if (k == tau_key) {
                  ++neq;
                  sel = neq <= n_tau;
                  if (neq == n_tau) tiepos = kb + j;
                }
                mbits |= (uint64_t)sel << (half * 32 + j);
              }
            }
          } else if (level == kLvLin && lin == 0) {
            // every key lands in a bin; Z is the sum of the bins afterwards
            const int nvc = nv < 32 ? nv : 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nvc) {
                const float u = __fsub_rn(mh, __uint_as_float(v[j]));
                const int d = u >= 31.f ? 31 : (u > 0.f ? (int)u : 0);  // also 0 for a NaN input
                S.hist[d][row] += pf_weight_u(u, wmul, A.two_pow_frac);
              }
            }
          } else if (level == kLvLin || level == kLvCollect) {
            // keys inside the bracket [ulo, uhi) of u (two compares each); most chunks have none
            uint32_t in = 0u;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float u = __fsub_rn(mh, __uint_as_float(v[j]));
              const bool ok = j < nv;
              in |= (uint32_t)(ok && u >= ulo && u < uhi) << j;
              if (level == kLvCollect) ngt += ok && u < ulo;  // keys above the bracket
            }
            if (in) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if ((in >> j) & 1u) {
                  const float u = __fsub_rn(mh, __uint_as_float(v[j]));
                  if (level == kLvLin) {
                    const int d = (int)__fmul_rn(u, dscale) - 32 * prefix;
                    S.hist[d][row] += pf_weight_u(u, wmul, A.two_pow_frac);
                    const uint16_t cc = S.hcnt[d][row];
                    S.hcnt[d][row] = cc == 0xFFFFu ? cc : (uint16_t)(cc + 1u);
                  } else if (ncand < kPfBins) {
                    const float sv = __fadd_rn(__fmul_rn(__uint_as_float(v[j]), 0.25f), 0.0f);
                    S.hist[ncand][row] = ((uint64_t)(uint32_t)(kb + j) << 32) | __float_as_uint(sv);
                    ++ncand;
                  }
                }
              }
            }
          } else {  // KEY fallback: exact digits of the score key inside the bracket
            const int nvc = nv < 32 ? nv : 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nvc) {
                const float u = __fsub_rn(mh, __uint_as_float(v[j]));
                const bool inb = tail ? u >= 31.f : (u >= ulo && u < uhi);
                const float sv = __fadd_rn(__fmul_rn(__uint_as_float(v[j]), 0.25f), 0.0f);
                const uint32_t k = score_key(sv);
                if (inb && k >= kbase && (uint64_t)k < kend) {
                  const int d = (int)((k - kbase) >> shift);
                  S.hist[d][row] += pf_weight_u(u, wmul, A.two_pow_frac);
                }
              }
            }
          }
        }
        if (level == kLvTie && mrow) {
          const int w0 = key0 >> 5;
          if (w0 < A.mask_words) mrow[w0] = (uint32_t)mbits;
          if (w0 + 1 < A.mask_words) mrow[w0 + 1] = (uint32_t)(mbits >> 32);
        }
      }
      // ---- end of sweep: advance this row's bracket ----
      if (is_row && level != kLvDone && alive) {
        if (level == kLvMax) {
          level = kLvLin;  // m is the raw maximum
          lin = 0;
          prefix = 0;
        } else if (level == kLvTie) {
          if (mrow)  // words past the block's last tile
            for (int64_t w = 2 * (int64_t)ntiles; w < (A.N + 31) / 32; ++w) mrow[w] = 0u;
          const int64_t qrow = (int64_t)bh * A.T + t;
          A.tau_bits[qrow] = __float_as_uint(key_score(tau_key));
          A.tiepos[qrow] = tiepos;
          A.count[qrow] = ngt + n_tau;
          level = kLvDone;
        } else if (level == kLvCollect) {
          // sort the candidates by (score desc, position asc), then take them in order
          for (int a = 1; a < ncand; ++a) {
            const uint64_t x = S.hist[a][row];
            const uint32_t xk = score_key(__uint_as_float((uint32_t)x));
            const uint32_t xp = (uint32_t)(x >> 32);
            int bI = a - 1;
            while (bI >= 0) {
              const uint64_t y = S.hist[bI][row];
              const uint32_t yk = score_key(__uint_as_float((uint32_t)y));
              if (yk > xk || (yk == xk && (uint32_t)(y >> 32) < xp)) break;
              S.hist[bI + 1][row] = y;
              --bI;
            }
            S.hist[bI + 1][row] = x;
          }
          const uint64_t need = target - mass_above;
          uint64_t cum = 0;
          int taken = ncand;
          for (int a = 0; a < ncand; ++a) {
            const float sa = __uint_as_float((uint32_t)S.hist[a][row]);
            cum += pf_weight_u(__fsub_rn(mh, __fmul_rn(sa, 4.f)), wmul, A.two_pow_frac);
            if (cum >= need) {
              taken = a + 1;
              break;
            }
          }
          if (taken < 1) taken = 1;
          const uint64_t last = S.hist[taken - 1][row];
          tau_key = score_key(__uint_as_float((uint32_t)last));
          n_tau = 0;
          for (int a = 0; a < taken; ++a) n_tau += score_key(__uint_as_float((uint32_t)S.hist[a][row])) == tau_key;
          const int cnt = ngt + taken;
          if (mrow) {  // the selection mask needs one more sweep
            ngt = 0;
            neq = 0;
            tiepos = -1;
            level = kLvTie;
          } else {
            const int64_t qrow = (int64_t)bh * A.T + t;
            A.tau_bits[qrow] = __float_as_uint(key_score(tau_key));
            A.tiepos[qrow] = (int)(last >> 32);
            A.count[qrow] = cnt;
            level = kLvDone;
          }
        } else {  // LIN or KEY: find the cut bin
          if (level == kLvLin && lin == 0) {
            uint64_t Z = 0;
            for (int i = 0; i < kPfBins; ++i) Z += S.hist[i][row];
            const double tt = ceil((double)A.p * (double)Z);
            uint64_t tg = tt >= (double)Z ? Z : (uint64_t)tt;
            target = tg < 1 ? 1 : tg;
          }
          const uint64_t need = target - mass_above;
          uint64_t cum = 0;
          int cut = 0;
          for (int r = 0; r < kPfBins; ++r) {
            const int bin = level == kLvKey ? kPfBins - 1 - r : r;
            const uint64_t hv = S.hist[bin][row];
            if (cum + hv >= need) {
              cut = bin;
              break;
            }
            cum += hv;
          }
          mass_above += cum;
          if (level == kLvLin) {
            if (lin == 0 && cut == 31) {
              // tail bin (u >= 31, i.e. s <= max s - 7.75): exact digits over its keys
              tail = 1;
              const float hi_s = __fmul_rn(__fsub_rn(mh, 31.f), 0.25f);
              const float mg = 1e-5f * (fabsf(hi_s) + 8.f) + 1e-30f;
              kbase = 0u;
              kend = (uint64_t)score_key(__fadd_rn(hi_s + mg, 0.0f)) + 1;
              shift = 0;
              while (((kend - kbase - 1) >> shift) >= (uint64_t)kPfBins) ++shift;
              level = kLvKey;
            } else {
              const uint32_t in_bin = lin == 0 ? 0xFFFFu : S.hcnt[cut][row];  // level 0 keeps no counts
              prefix = lin == 0 ? cut : 32 * prefix + cut;  // full bin index at level `lin`
              ulo = (float)prefix / dscale;                  // exact: dscale is a power of two
              uhi = (float)(prefix + 1) / dscale;
              if (in_bin <= (uint32_t)kPfBins) {
                level = kLvCollect;
              } else if (lin < 3) {
                ++lin;
                dscale *= 32.f;
              } else {
                // still too many keys: exact digits inside this bracket of u
                const float hi_s = __fmul_rn(__fsub_rn(mh, ulo), 0.25f);
                const float lo_s = __fmul_rn(__fsub_rn(mh, uhi), 0.25f);
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
              const uint64_t w_tau = pf_weight_u(__fsub_rn(mh, __fmul_rn(st, 4.f)), wmul, A.two_pow_frac);
              const uint64_t rem = target - mass_above;
              uint64_t nt = w_tau ? (rem + w_tau - 1) / w_tau : 1;
              n_tau = (int)(nt < 1 ? 1 : nt);
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
    }
    g += ntiles;
  }

  // ---- wind down: the last accumulator commit has landed before TMEM is freed
  if (warp == 5 && lane == 0 && g > 0) {
    const uint32_t last = g - 1;
    mbar_wait(&S.t_full[last & 1], (last >> 1) & 1, alive, A.err);
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

// ---- host ---------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Tensor map over a [B, H, R, 16] bf16 view, box of `box_rows` rows, 32-byte swizzle.
bool make_idx_map(CUtensorMap* map, const View4& v, int64_t B, int64_t H, int64_t R, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {16, (cuuint64_t)R, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t st1 = (cuuint64_t)v.sn * 2, st2 = (cuuint64_t)v.sh * 2, st3 = (cuuint64_t)v.sb * 2;
  if (R <= 1) st1 = 32;
  if (H <= 1) st2 = st1 * (cuuint64_t)(R > 0 ? R : 1);
  if (B <= 1) st3 = st2 * (cuuint64_t)(H > 0 ? H : 1);
  cuuint64_t strides[3] = {st1, st2, st3};
  cuuint32_t box[4] = {16, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(v.data), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

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
  if (a.p >= 1.f) {
    topp_prefill_all_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(A, (int)rows);
    return cudaGetLastError();
  }
  CUtensorMap qmap, kmap;
  if (!make_idx_map(&qmap, a.q_idx, a.B, a.Hq, a.T, kPfRows)) return cudaErrorInvalidValue;
  if (!make_idx_map(&kmap, a.k_idx, a.B, a.Hk, a.N, kPfKeys)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(PfSmem) + 256;
  cudaFuncSetAttribute(topp_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const dim3 grid((unsigned)(((a.T + kPfRows - 1) / kPfRows) * a.B * a.Hq));
  topp_prefill_kernel<<<grid, kPfThreads, smem, stream>>>(qmap, kmap, A);
  return cudaGetLastError();
}

}  // namespace rtp
