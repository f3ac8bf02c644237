// a2 + a3 (decode): indexer scores of every cached key and the dynamic top-p cut.
//
// "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
// Hundred Training Steps", "Three Key Insights" 3: per query, cumulative top-p
// over the ranked tokens instead of a fixed top-k.  Read here as: the shortest
// prefix of the keys ordered by (score desc, position asc) whose weight
// exp(s - max s) reaches p * Z.
//
// Design (B200): one thread-block CLUSTER per query.  Each CTA of the cluster
// owns a contiguous slice of the keys, computes their scores once from the
// projected-key cache (32-byte rows, 16-byte vector loads) and keeps them in
// shared memory.  The cut is found without sorting, by narrowing a bracket:
//   pass 0   256 bins linear in (max - s) (1/16 nat wide; the last bin holds
//            the tail) -- scores spread over many bins, so the per-warp
//            shared-memory histograms see few same-bin collisions;
//   pass 1.. 256 bins over the order-preserving uint32 image of the fp32
//            score (8-bit digits of the offset inside the bracket), only for
//            keys still inside the bracket, until the bracket is one score
//            value tau.
// Every pass accumulates 64-bit fixed-point masses (integer sums, so the
// result does not depend on thread order).  After each pass every CTA reads
// all CTAs' 256 bins through distributed shared memory and finds the same cut
// bin by itself, so a pass costs one cluster barrier.  Ties at tau are
// resolved by position with a prefix count over the cluster; then every CTA
// writes its bits of the selection mask.  No global-memory atomics and no spin
// waits: all synchronisation is the hardware cluster barrier.
#include <cooperative_groups.h>

#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace rtp {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 256;
constexpr int kMaxCluster = 16;
constexpr int kMaxKeysPerCta = 32768;  // scores of one CTA held in shared memory (128 KB)
constexpr float kLinBinsPerNat = 16.f; // pass 0 bin width 1/16 nat
static_assert(kSelThreads == kBins, "one thread per histogram bin");

struct SelSmem {
  uint32_t whlo[kSelWarps][kBins];   // per-warp private histograms (64-bit masses as lo/hi words)
  uint32_t whhi[kSelWarps][kBins];
  uint64_t hist[2][kBins];           // this CTA's histogram, double-buffered by pass parity
  uint64_t red[kBins];               // cluster-wide histogram (each CTA holds a copy)
  uint64_t wsum[kSelWarps];
  uint32_t tcount[kMaxCluster];      // keys equal to tau, per CTA
  uint32_t gcount[kMaxCluster];      // keys above tau, per CTA
  float cmax_self;
  float wmax[kSelWarps];
  uint32_t wcnt[kSelWarps];
  uint32_t wcnt2[kSelWarps];
  int cut_bin;
  uint64_t cut_above;
};

// Exact 64-bit add into a (lo, hi) pair of 32-bit shared-memory words: native
// 32-bit atomics, the carry out of the low word is added to the high word by the
// one thread whose addition wrapped it.  (64-bit shared-memory atomics are far
// slower on this part, more so under contention.)
RTP_DEVICE void add_u64_pair(uint32_t* lo, uint32_t* hi, uint64_t w) {
  const uint32_t l = (uint32_t)w;
  uint32_t h = (uint32_t)(w >> 32);
  const uint32_t old = atomicAdd(lo, l);
  if (old + l < old) ++h;
  if (h) atomicAdd(hi, h);
}
RTP_DEVICE uint64_t pair_value(uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; }

RTP_DEVICE float ex2f_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Fixed-point top-p weight round(2^((s - m) log2 e) * 2^frac).  Every use of a
// weight in the cut goes through this one function.
RTP_DEVICE uint64_t sel_weight(float s, float m, float two_pow_frac) {
  const float e = ex2f_fast(__fmul_rn(__fsub_rn(s, m), 1.4426950408889634f));
  return __float2ull_rn(__fmul_rn(e, two_pow_frac));
}

// pass-0 bin of a score: floor((m - s) * 16), the tail folded into the last bin
RTP_DEVICE int lin_bin(float s, float m) {
  const float t = __fmul_rn(__fsub_rn(m, s), kLinBinsPerNat);
  return t >= (float)(kBins - 1) ? kBins - 1 : (int)t;
}

template <typename T>
__global__ void __launch_bounds__(kSelThreads)
topp_query_kernel(View4 qv, View4 kv, const int32_t* __restrict__ lens, int Hq, int G, int N,
                   int n_chunk, float p, float two_pow_frac, uint32_t* __restrict__ tau_bits,
                   int32_t* __restrict__ tiepos, int32_t* __restrict__ count,
                   uint32_t* __restrict__ mask, int64_t mask_words) {
  pdl_wait();
  pdl_release();
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qrow = blockIdx.x / C;
  const int b = qrow / Hq, h = qrow % Hq, kvh = h / G;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelSmem& S = *reinterpret_cast<SelSmem*>(smem_raw);
  float* scores = reinterpret_cast<float*>(smem_raw + sizeof(SelSmem));

  int n_b = N;
  if (lens) n_b = min(max(lens[b], 0), N);
  const int c0 = rank * n_chunk;
  const int c1 = min(c0 + n_chunk, n_b);
  const int nloc = max(c1 - c0, 0);
  const int n_words_total = (N + 31) / 32;
  uint32_t* mrow = mask ? mask + (int64_t)qrow * mask_words : nullptr;

  // Trivial cuts: no candidates, or p >= 1 (every candidate).  Uniform over the
  // cluster, taken before any distributed-shared-memory access.
  if (n_b == 0 || p >= 1.f) {
    const bool all = n_b > 0;
    for (int wi = tid; wi * 32 < n_chunk; wi += kSelThreads) {
      const int w = (c0 >> 5) + wi;
      if (w >= n_words_total || !mrow) continue;
      const int j0 = w * 32;
      uint32_t bits = 0;
      if (all) {
        const int nv = min(max(n_b - j0, 0), 32);
        bits = nv >= 32 ? 0xffffffffu : ((1u << nv) - 1u);
      }
      mrow[w] = bits;
    }
    if (rank == 0 && tid == 0) {
      tau_bits[qrow] = all ? 0xff800000u : 0x7f800000u;  // -inf: everything passes; +inf: nothing
      tiepos[qrow] = n_b - 1;
      count[qrow] = n_b;
    }
    return;
  }

  // ---- scores of this CTA's keys (eight independent row loads in flight per thread)
  float qf[kIdxDim];
  load_idx_row<T>(static_cast<const T*>(qv.data) + b * qv.sb + h * qv.sh, qf);
  const T* kb = static_cast<const T*>(kv.data) + b * kv.sb + kvh * kv.sh;
  float lmax = -INFINITY;
  constexpr int U = sizeof(T) == 2 ? 8 : 4;
  for (int base = 0; base < nloc; base += U * kSelThreads) {
    IdxRaw<T> raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * kSelThreads + tid;
      if (i < nloc) load_idx_raw<T>(kb + (int64_t)(c0 + i) * kv.sn, raw[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * kSelThreads + tid;
      if (i < nloc) {
        float kf[kIdxDim];
        idx_raw_to_float<T>(raw[u], kf);
        const float sc = indexer_dot16(qf, kf);
        scores[i] = sc;
        lmax = fmaxf(lmax, sc);
      }
    }
  }
  lmax = warp_max(lmax);
  if (lane == 0) S.wmax[warp] = lmax;
  __syncthreads();
  if (tid == 0) {
    float mm = S.wmax[0];
    for (int w = 1; w < kSelWarps; ++w) mm = fmaxf(mm, S.wmax[w]);
    S.cmax_self = mm;
  }
  cluster.sync();
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r)
    if (r < C) m = fmaxf(m, *cluster.map_shared_rank(&S.cmax_self, r));

  // ---- bracket narrowing --------------------------------------------------------
  // pass 0: linear bins; then key-window bins [base, base + 256 << shift).
  uint64_t target = 0, mass_above = 0;
  int lin = -1;               // cut bin of pass 0
  uint32_t kbase = 0;         // key window [kbase, kend) of the refinement passes
  uint64_t kend = 0;
  int shift = 0;
  for (int pass = 0;; ++pass) {
    uint32_t* wlo = S.whlo[warp];
    uint32_t* whi = S.whhi[warp];
    for (int i = lane; i < kBins; i += 32) {
      wlo[i] = 0;
      whi[i] = 0;
    }
    __syncwarp();
    for (int i = tid; i < nloc; i += kSelThreads) {
      const float sc = scores[i];
      int d = -1;
      if (pass == 0) {
        d = lin_bin(sc, m);
      } else if (lin_bin(sc, m) == lin) {
        const uint32_t k = score_key(sc);
        if (k >= kbase && (uint64_t)k < kend) d = (int)((uint64_t)(k - kbase) >> shift);
      }
      if (d >= 0) add_u64_pair(&wlo[d], &whi[d], sel_weight(sc, m, two_pow_frac));
    }
    __syncthreads();
    uint64_t* hb = S.hist[pass & 1];
    {
      uint64_t a = 0;
#pragma unroll
      for (int w = 0; w < kSelWarps; ++w) a += pair_value(S.whlo[w][tid], S.whhi[w][tid]);
      hb[tid] = a;
    }
    cluster.sync();  // every CTA's histogram of this pass is complete
    // cluster-wide histogram, computed identically by every CTA
    {
      uint64_t a = 0;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r)
        if (r < C) a += cluster.map_shared_rank(hb, r)[tid];
      S.red[tid] = a;
    }
    __syncthreads();
    if (pass == 0) {
      // Z = total mass; target = ceil(p Z)
      uint64_t a = S.red[tid];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) S.wsum[warp] = a;
      __syncthreads();
      uint64_t Z = 0;
      for (int w = 0; w < kSelWarps; ++w) Z += S.wsum[w];
      const double t = ceil((double)p * (double)Z);
      const uint64_t tt = t >= (double)Z ? Z : (uint64_t)t;
      target = tt < 1 ? 1 : tt;
      __syncthreads();  // S.wsum is reused by the scan below
    }
    const uint64_t need = target - mass_above;  // >= 1
    // Bins in descending score order: pass 0 bin 0 is the highest scores;
    // refinement bin 255 is the highest key.  Position r in that order:
    const int bin_of_r = pass == 0 ? tid : (kBins - 1 - tid);
    const uint64_t mine = S.red[bin_of_r];
    // inclusive prefix of the mass over the descending order (block scan)
    uint64_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) S.wsum[warp] = incl;
    __syncthreads();
    uint64_t off = 0;
    for (int w = 0; w < warp; ++w) off += S.wsum[w];
    incl += off;
    const uint64_t excl = incl - mine;
    if (excl < need && need <= incl) {  // exactly one position holds the cut
      S.cut_bin = bin_of_r;
      S.cut_above = excl;
    }
    __syncthreads();
    mass_above += S.cut_above;
    const int cb = S.cut_bin;
    __syncthreads();
    if (pass == 0) {
      lin = cb;
      // key window holding every score of linear bin `lin` (with a margin)
      const float hi_s = m - (float)lin / kLinBinsPerNat;
      const float lo_s = m - (float)(lin + 1) / kLinBinsPerNat;
      const float mg = 1e-5f * (fabsf(m) + (float)(lin + 1) / kLinBinsPerNat) + 1e-30f;
      const uint32_t khi = score_key(__fadd_rn(hi_s + mg, 0.0f));
      const uint32_t klo = lin == kBins - 1 ? 0u : score_key(__fadd_rn(lo_s - mg, 0.0f));
      kbase = klo;
      kend = (uint64_t)khi + 1;
      const uint64_t range = kend - klo;
      shift = 0;
      while (((range - 1) >> shift) >= (uint64_t)kBins) ++shift;
    } else {
      kbase += (uint32_t)cb << shift;
      const uint64_t e = (uint64_t)kbase + (uint64_t(1) << shift);
      kend = e < kend ? e : kend;
      if (shift == 0) break;            // the bracket is one score value
      shift = shift >= 8 ? shift - 8 : 0;
    }
  }

  // ---- counts at tau: keys above and equal, per CTA, then over the cluster ----
  const uint32_t tau_key = kbase;
  const float tau = key_score(tau_key);
  uint32_t ngt = 0, neq = 0;
  for (int i = tid; i < nloc; i += kSelThreads) {
    const uint32_t k = score_key(scores[i]);
    ngt += k > tau_key;
    neq += k == tau_key;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ngt += __shfl_xor_sync(0xffffffffu, ngt, o);
    neq += __shfl_xor_sync(0xffffffffu, neq, o);
  }
  if (lane == 0) {
    S.wcnt[warp] = ngt;
    S.wcnt2[warp] = neq;
  }
  __syncthreads();
  if (tid < C) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      g += S.wcnt[w];
      e += S.wcnt2[w];
    }
    cluster.map_shared_rank(S.gcount, tid)[rank] = g;
    cluster.map_shared_rank(S.tcount, tid)[rank] = e;
  }
  cluster.sync();  // last distributed access
  uint32_t cnt_above = 0, tau_cnt = 0;
  int before = 0;
  for (int r = 0; r < C; ++r) {
    cnt_above += S.gcount[r];
    tau_cnt += S.tcount[r];
    if (r < rank) before += (int)S.tcount[r];
  }
  const uint64_t w_tau = sel_weight(tau, m, two_pow_frac);
  const uint64_t rem = target - mass_above;
  uint64_t n_tau64 = w_tau ? (rem + w_tau - 1) / w_tau : (uint64_t)tau_cnt;
  if (n_tau64 < 1) n_tau64 = 1;
  if (n_tau64 > tau_cnt) n_tau64 = tau_cnt;
  const int n_tau = (int)n_tau64;
  const int want = n_tau - before;           // how many of this CTA's tau keys are taken
  const bool my_ties = S.tcount[rank] != 0;  // uniform over the CTA

  // ---- mask bits and the tie position ---------------------------------------
  int running = 0;
  for (int base = 0; base < n_chunk; base += kSelThreads) {
    const int i = base + tid;
    const bool valid = i < nloc;
    const uint32_t k = valid ? score_key(scores[i]) : 0u;
    const bool gt = valid && k > tau_key;
    bool sel = gt;
    if (my_ties) {
      const bool eq = valid && k == tau_key;
      const uint32_t beq = __ballot_sync(0xffffffffu, eq);
      const int wpre = __popc(beq & ((1u << lane) - 1u));
      if (lane == 0) S.wcnt[warp] = __popc(beq);
      __syncthreads();
      int woff = 0, rtot = 0;
      for (int w = 0; w < kSelWarps; ++w) {
        const int t = (int)S.wcnt[w];
        woff += w < warp ? t : 0;
        rtot += t;
      }
      __syncthreads();
      const int r_eq = running + woff + wpre;
      sel = gt || (eq && r_eq < want);
      if (eq && r_eq == want - 1) tiepos[qrow] = c0 + i;
      running += rtot;
    }
    const uint32_t word = __ballot_sync(0xffffffffu, sel);
    const int wpos = base + warp * 32;
    const int w = (c0 + wpos) >> 5;
    if (lane == 0 && mrow && wpos < n_chunk && w < n_words_total) mrow[w] = word;
  }
  if (rank == 0 && tid == 0) {
    tau_bits[qrow] = __float_as_uint(tau);
    count[qrow] = (int)(cnt_above + (uint32_t)n_tau);
  }
}

bool topp_decode_supported(int64_t N) { return N <= (int64_t)kMaxKeysPerCta * kMaxCluster; }

static int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <typename K, typename... Args>
static cudaError_t launch_cluster(K kern, int grid, int C, size_t smem, cudaStream_t stream, Args... args) {
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (C > 8) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kSelThreads), smem, stream, (unsigned)C, args...);
}

cudaError_t launch_topp_decode(const LaunchToppDecode& a, cudaStream_t stream) {
  const int64_t Q = a.B * a.Hq;
  if (Q == 0) return cudaSuccess;
  const int sms = sm_count();
  int lg = 0;
  while ((int64_t(1) << lg) < a.N) ++lg;
  const float two_pow_frac = ldexpf(1.f, 63 - lg);
  const int G = (int)(a.Hq / a.Hk);

  // Query form: one cluster per query.
  int C = 1;
  while (C < 8 && Q * C < sms) C <<= 1;
  while ((a.N + C - 1) / C > kMaxKeysPerCta && C < kMaxCluster) C <<= 1;
  int64_t n_chunk = (a.N + C - 1) / C;
  n_chunk = (n_chunk + 31) / 32 * 32;
  if (n_chunk == 0) n_chunk = 32;
  if (n_chunk > kMaxKeysPerCta) return cudaErrorInvalidValue;
  const size_t smem = sizeof(SelSmem) + (size_t)n_chunk * sizeof(float);
  if (a.bf16)
    return launch_cluster(topp_query_kernel<__nv_bfloat16>, (int)(Q * C), C, smem, stream, a.q_idx, a.k_idx, a.lens,
                          (int)a.Hq, G, (int)a.N, (int)n_chunk, a.p, two_pow_frac, a.tau_bits, a.tiepos, a.count,
                          a.mask, a.mask_words);
  return launch_cluster(topp_query_kernel<float>, (int)(Q * C), C, smem, stream, a.q_idx, a.k_idx, a.lens, (int)a.Hq,
                        G, (int)a.N, (int)n_chunk, a.p, two_pow_frac, a.tau_bits, a.tiepos, a.count, a.mask,
                        a.mask_words);
}

}  // namespace rtp
