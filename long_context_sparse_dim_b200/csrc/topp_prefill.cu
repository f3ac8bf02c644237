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
// streamed by TMA (32-byte swizzle, no multicast) through a 4-stage ring, and
// the fp32 accumulators alternate between two TMEM buffers so the next MMA
// runs while four epilogue warps read the previous tile.  Warp roles:
//   warps 0-3  epilogue: thread r owns query row r (its TMEM lane)
//   warp 4     TMA producer (one elected lane)
//   warp 5     MMA issuer (one elected lane)
// The cut of every row is found by sweeps over its causal prefix; each sweep
// recomputes the score tiles (depth-16 MMAs are cheap) and narrows a bracket
// around the cut score:
//   MAX   row maximum m
//   L0    Z = sum of 64-bit fixed-point weights; 32 bins of (m - s) 1/4 nat wide
//   L1    32 sub-bins of the L0 cut bin (1/128 nat)
//   KEY   5-bit digits of the order-preserving uint32 image of s inside the
//         bracket, until the bracket is one score value tau
//   TIE   keys above tau are counted, the n-th key equal to tau (position
//         order) gives tiepos, and the optional selection mask is written
// A row owns its 32-bin histogram column in shared memory, so no atomics are
// needed.  Sweeps continue while any row of the block is unresolved.
#include <cudaTypedefs.h>

#include <math.h>

#include "launch.h"
#include "tc05.cuh"

namespace rtp {

constexpr int kPfRows = 128;      // query rows per CTA (TMEM lanes)
constexpr int kPfKeys = 64;       // keys per score tile (MMA N)
constexpr int kPfStages = 4;      // K_idx tile ring
constexpr int kPfBins = 32;       // histogram bins per row
constexpr int kPfThreads = 192;   // 4 epilogue warps + producer + MMA
constexpr int kPfTileBytes = kPfKeys * kIdxDim * 2;  // 2 KB
constexpr int kPfTmemCols = 2 * kPfKeys;             // two accumulator buffers

enum PfLevel : int { kLvMax = 0, kLvL0 = 1, kLvL1 = 2, kLvKey = 3, kLvTie = 4, kLvDone = 5 };

struct PfSmem {
  alignas(1024) uint8_t qtile[kPfRows * kIdxDim * 2];            // A operand, 4 KB
  alignas(1024) uint8_t ktile[kPfStages][kPfTileBytes];           // B operand ring
  uint64_t hist[kPfBins][kPfRows];                                // per-row mass histograms
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

RTP_DEVICE uint64_t pf_weight(float s, float m, float two_pow_frac) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(e) : "f"(__fmul_rn(__fsub_rn(s, m), 1.4426950408889634f)));
  return __float2ull_rn(__fmul_rn(e, two_pow_frac));
}

__global__ void __launch_bounds__(kPfThreads)
topp_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, PfArgs A) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  PfSmem& S = *reinterpret_cast<PfSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kPfRows;
  const int bh = blockIdx.y;
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
  float m = -INFINITY;
  uint64_t Z = 0, target = 0, mass_above = 0;
  int b0 = 0, b1 = 0, shift = 0, n_tau = 0, ngt = 0, neq = 0, tiepos = -1;
  uint32_t kbase = 0, tau_key = 0;
  uint64_t kend = 0;
  uint32_t* mrow = (A.mask && is_row && t < A.T) ? A.mask + ((int64_t)bh * A.T + t) * A.mask_words : nullptr;

  uint32_t g = 0;  // global tile counter across sweeps (drives every ring phase)
  for (int sweep = 0; sweep < 16; ++sweep) {
    const int more = __syncthreads_or(is_row && level != kLvDone);
    const int abort = __syncthreads_or(!alive);
    if (!more || abort || ntiles == 0) break;
    if (is_row && (level == kLvL0 || level == kLvL1 || level == kLvKey))
      for (int i = 0; i < kPfBins; ++i) S.hist[i][row] = 0;

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
        uint32_t v[2][32];
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + buf * kPfKeys;
        tmem_ld32(taddr, v[0]);
        tmem_ld32(taddr + 32, v[1]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&S.t_empty[buf]);
        if (level == kLvDone) continue;
        const int key0 = i * kPfKeys;
        const int nv = pos - key0 + 1;  // keys of this tile inside the row's causal prefix
        uint32_t mbits[2] = {0u, 0u};
        if (level == kLvMax) {
#pragma unroll
          for (int j = 0; j < kPfKeys; ++j)
            if (j < nv) m = fmaxf(m, __fadd_rn(__fmul_rn(__uint_as_float(v[j >> 5][j & 31]), 0.25f), 0.0f));
        } else if (level == kLvTie) {
#pragma unroll
          for (int j = 0; j < kPfKeys; ++j) {
            if (j < nv) {
              const float s = __fadd_rn(__fmul_rn(__uint_as_float(v[j >> 5][j & 31]), 0.25f), 0.0f);
              const uint32_t k = score_key(s);
              const bool gt = k > tau_key;
              bool sel = gt;
              ngt += gt;
              if (k == tau_key) {
                ++neq;
                sel = neq <= n_tau;
                if (neq == n_tau) tiepos = key0 + j;
              }
              mbits[j >> 5] |= (uint32_t)sel << (j & 31);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < kPfKeys; ++j) {
            if (j < nv) {
              const float s = __fadd_rn(__fmul_rn(__uint_as_float(v[j >> 5][j & 31]), 0.25f), 0.0f);
              const float u = __fsub_rn(mh, s);
              const float u4 = __fmul_rn(u, 4.f);
              const int l0 = u4 >= 31.f ? 31 : (int)u4;
              int d = -1;
              if (level == kLvL0) {
                d = l0;
              } else if (l0 == b0) {
                if (level == kLvL1) {
                  d = (int)__fmul_rn(u, 128.f) - 32 * b0;
                } else {
                  bool in = true;
                  if (b0 < 31) in = ((int)__fmul_rn(u, 128.f) - 32 * b0) == b1;
                  const uint32_t k = score_key(s);
                  if (in && k >= kbase && (uint64_t)k < kend) d = (int)((k - kbase) >> shift);
                }
              }
              if (d >= 0) {
                const uint64_t w = pf_weight(s, mh, A.two_pow_frac);
                if (level == kLvL0) Z += w;
                S.hist[d][row] += w;
              }
            }
          }
        }
        if (level == kLvTie && mrow) {
          const int w0 = key0 >> 5;
          if (w0 < A.mask_words) mrow[w0] = mbits[0];
          if (w0 + 1 < A.mask_words) mrow[w0 + 1] = mbits[1];
        }
      }
      // ---- end of sweep: advance this row's bracket ----
      if (is_row && level != kLvDone && alive) {
        if (level == kLvMax) {
          level = kLvL0;
        } else if (level == kLvTie) {
          if (mrow)  // words past the block's last tile
            for (int64_t w = 2 * (int64_t)ntiles; w < (A.N + 31) / 32; ++w) mrow[w] = 0u;
          const int64_t qrow = (int64_t)bh * A.T + t;
          A.tau_bits[qrow] = __float_as_uint(key_score(tau_key));
          A.tiepos[qrow] = tiepos;
          A.count[qrow] = ngt + n_tau;
          level = kLvDone;
        } else {
          if (level == kLvL0) {
            const double tt = ceil((double)A.p * (double)Z);
            uint64_t tg = tt >= (double)Z ? Z : (uint64_t)tt;
            target = tg < 1 ? 1 : tg;
          }
          const uint64_t need = target - mass_above;
          // bins in descending score order: L0/L1 bin 0 first; KEY bin 31 first
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
          if (level == kLvL0) {
            b0 = cut;
            if (b0 < 31) {
              level = kLvL1;
            } else {  // the tail bin: key window from the lowest key up to m - 7.75
              const float hi_s = mh - 7.75f;
              const float mg = 1e-5f * (fabsf(mh) + 8.f) + 1e-30f;
              kbase = 0u;
              kend = (uint64_t)score_key(__fadd_rn(hi_s + mg, 0.0f)) + 1;
              shift = 0;
              while (((kend - kbase - 1) >> shift) >= (uint64_t)kPfBins) ++shift;
              level = kLvKey;
            }
          } else if (level == kLvL1) {
            b1 = cut;
            const int fine = 32 * b0 + b1;  // u in [fine/128, (fine+1)/128)
            const float hi_s = mh - (float)fine / 128.f;
            const float lo_s = mh - (float)(fine + 1) / 128.f;
            const float mg = 1e-5f * (fabsf(mh) + (float)(fine + 1) / 128.f) + 1e-30f;
            kbase = score_key(__fadd_rn(lo_s - mg, 0.0f));
            kend = (uint64_t)score_key(__fadd_rn(hi_s + mg, 0.0f)) + 1;
            shift = 0;
            while (((kend - kbase - 1) >> shift) >= (uint64_t)kPfBins) ++shift;
            level = kLvKey;
          } else {  // KEY
            kbase += (uint32_t)cut << shift;
            const uint64_t e = (uint64_t)kbase + (uint64_t(1) << shift);
            kend = e < kend ? e : kend;
            if (shift == 0) {
              tau_key = kbase;
              const uint64_t w_tau = pf_weight(key_score(tau_key), mh, A.two_pow_frac);
              const uint64_t rem = target - mass_above;
              uint64_t nt = w_tau ? (rem + w_tau - 1) / w_tau : 1;
              n_tau = (int)(nt < 1 ? 1 : nt);
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
  const size_t smem = sizeof(PfSmem) + 1024;
  cudaFuncSetAttribute(topp_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const dim3 grid((unsigned)((a.T + kPfRows - 1) / kPfRows), (unsigned)(a.B * a.Hq));
  topp_prefill_kernel<<<grid, kPfThreads, smem, stream>>>(qmap, kmap, A);
  return cudaGetLastError();
}

}  // namespace rtp
