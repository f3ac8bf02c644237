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
constexpr int kListCap = kSelWarps * kBins;  // members of the cut bin one CTA can list
constexpr int kCandCap = kSelThreads;        // candidates rank 0 orders (one per thread)
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
  // candidate path (pass-0 cut bin -> 256 sub-bins -> candidates at rank 0)
  uint32_t l1lo[kBins];              // sub-bin masses of this CTA (lo/hi words)
  uint32_t l1hi[kBins];
  uint32_t l1cnt[kBins];             // sub-bin key counts of this CTA
  uint64_t h1[kBins];                // sub-bin masses of this CTA as 64-bit values
  uint32_t nlist, nabove, novf;      // members listed, keys above the cut bin, list overflow
  uint32_t tot_above, tot_ovf, cut_cnt, cut_cnt_above;
  uint32_t ncand;                    // rank 0: candidates received
  float cand_s[kCandCap];            // rank 0: candidates (score, position) in arrival order
  int32_t cand_p[kCandCap];
  float sort_s[kCandCap];            // rank 0: candidates in (score desc, position asc) order
  int32_t sort_p[kCandCap];
  int bc_t;
  float bc_tau;                      // the cut, written into every CTA by rank 0
  int32_t bc_tiepos;
  uint32_t bc_count;
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

// Sub-bin of a score inside pass-0 bin `lin` (lin < 255): floor((m - s) * 4096)
// - 256 lin.  (m - s) is the same rounded value lin_bin scales by 16, and both
// scalings are exact, so the sub-bins of bin lin are exactly its members.
RTP_DEVICE int sub_bin(float s, float m, int lin) {
  const float t = __fmul_rn(__fsub_rn(m, s), kLinBinsPerNat * (float)kBins);
  const int d = (int)t - lin * kBins;
  return d < 0 ? 0 : (d > kBins - 1 ? kBins - 1 : d);
}

RTP_DEVICE uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive prefix sum over the block's threads in thread order; `wsum` holds
// one word per warp.  Ends with a barrier, so `wsum` may be reused at once.
RTP_DEVICE uint64_t block_scan_u64(uint64_t v, uint64_t* wsum, uint64_t& excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint64_t off = 0;
  for (int w = 0; w < warp; ++w) off += wsum[w];
  __syncthreads();
  incl += off;
  excl = incl - v;
  return incl;
}

// Candidate path for a cut inside pass-0 bin `lin` (not the tail bin), `need`
// = the mass still to take inside that bin.  Each CTA lists the members of bin
// lin (and counts its keys in higher bins), histograms them into 256 sub-bins
// 1/4096 nat wide (mass and count), and every CTA finds the same cut sub-bin
// from the cluster-wide sums.  If it holds at most kCandCap keys, they go to
// rank 0, which orders them by (score desc, position asc), walks their weights
// to the cut and writes (tau, tiepos, count) into every CTA.  Returns the same
// value in every CTA of the cluster; false (a CTA's list overflowed, or the cut
// sub-bin is too full) leaves the key-window refinement to find the cut.
RTP_DEVICE bool collect_cut(SelSmem& S, cg::cluster_group& cluster, const float* scores, int nloc, int c0,
                            float m, float two_pow_frac, int lin, uint64_t need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  float* list_s = reinterpret_cast<float*>(&S.whlo[0][0]);
  int32_t* list_i = reinterpret_cast<int32_t*>(&S.whhi[0][0]);
  static_assert(sizeof(S.whlo) >= kListCap * sizeof(float), "list fits in the per-warp histograms");

  // members of bin lin -> local list (warp-aggregated appends)
  uint32_t nab = 0;
  for (int base = 0; base < nloc; base += kSelThreads) {
    const int i = base + tid;
    const bool valid = i < nloc;
    const float sc = valid ? scores[i] : 0.f;
    const int d = valid ? lin_bin(sc, m) : kBins;
    nab += d < lin;
    const bool mem = d == lin;
    const uint32_t bal = __ballot_sync(0xffffffffu, mem);
    if (bal) {
      uint32_t b0 = 0;
      if (lane == 0) b0 = atomicAdd(&S.nlist, (uint32_t)__popc(bal));
      b0 = __shfl_sync(0xffffffffu, b0, 0);
      if (mem) {
        const uint32_t slot = b0 + (uint32_t)__popc(bal & ((1u << lane) - 1u));
        if (slot < (uint32_t)kListCap) {
          list_s[slot] = sc;
          list_i[slot] = i;
        }
      }
    }
  }
  nab = warp_sum_u32(nab);
  if (lane == 0) atomicAdd(&S.nabove, nab);
  __syncthreads();
  const int nl = min((int)S.nlist, kListCap);
  for (int j = tid; j < nl; j += kSelThreads) {
    const float sc = list_s[j];
    const int sb = sub_bin(sc, m, lin);
    add_u64_pair(&S.l1lo[sb], &S.l1hi[sb], sel_weight(sc, m, two_pow_frac));
    atomicAdd(&S.l1cnt[sb], 1u);
  }
  __syncthreads();
  S.h1[tid] = pair_value(S.l1lo[tid], S.l1hi[tid]);
  if (tid == 0) S.novf = S.nlist > (uint32_t)kListCap ? 1u : 0u;
  cluster.sync();  // every CTA's sub-bin histogram is complete

  // cluster-wide sub-bin masses and counts, identical in every CTA
  uint64_t a = 0, c = 0;
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r)
    if (r < C) {
      a += cluster.map_shared_rank(S.h1, r)[tid];
      c += cluster.map_shared_rank(S.l1cnt, r)[tid];
    }
  if (warp == 0) {
    uint32_t na = 0, ov = 0;
    if (lane < C) {
      na = *cluster.map_shared_rank(&S.nabove, lane);
      ov = *cluster.map_shared_rank(&S.novf, lane);
    }
    na = warp_sum_u32(na);
    ov = warp_sum_u32(ov);
    if (lane == 0) {
      S.tot_above = na;
      S.tot_ovf = ov;
      S.cut_bin = -1;
    }
  }
  uint64_t em, ec;
  const uint64_t im = block_scan_u64(a, S.wsum, em);  // sub-bin 0 holds the highest scores
  block_scan_u64(c, S.wsum, ec);
  if (em < need && need <= im) {
    S.cut_bin = tid;
    S.cut_above = em;
    S.cut_cnt_above = (uint32_t)ec;
    S.cut_cnt = (uint32_t)c;
  }
  __syncthreads();
  const int sb = S.cut_bin;
  if (S.tot_ovf != 0 || sb < 0 || S.cut_cnt > (uint32_t)kCandCap) return false;

  // the cut sub-bin's keys -> rank 0
  {
    uint32_t* nc = cluster.map_shared_rank(&S.ncand, 0);
    float* cs = cluster.map_shared_rank(S.cand_s, 0);
    int32_t* cp = cluster.map_shared_rank(S.cand_p, 0);
    for (int j = tid; j < nl; j += kSelThreads) {
      const float sc = list_s[j];
      if (sub_bin(sc, m, lin) == sb) {
        const uint32_t slot = atomicAdd(nc, 1u);
        cs[slot] = sc;
        cp[slot] = c0 + list_i[j];
      }
    }
  }
  cluster.sync();  // rank 0 holds all candidates

  if (rank == 0) {
    const int n = (int)S.ncand;  // == S.cut_cnt <= kCandCap
    if (tid < n) {
      const uint32_t kt = score_key(S.cand_s[tid]);
      const int pt = S.cand_p[tid];
      int rk = 0;
      for (int j = 0; j < n; ++j) {
        const uint32_t kj = score_key(S.cand_s[j]);
        rk += (kj > kt || (kj == kt && S.cand_p[j] < pt)) ? 1 : 0;
      }
      S.sort_s[rk] = S.cand_s[tid];
      S.sort_p[rk] = pt;
    }
    if (tid == 0) S.bc_t = n - 1;
    __syncthreads();
    const uint64_t w = tid < n ? sel_weight(S.sort_s[tid], m, two_pow_frac) : 0;
    uint64_t ew;
    const uint64_t iw = block_scan_u64(w, S.wsum, ew);
    const uint64_t need1 = need - S.cut_above;  // >= 1, <= the sub-bin's mass
    if (tid < n && ew < need1 && need1 <= iw) S.bc_t = tid;
    __syncthreads();
    if (tid < C) {
      const int t = S.bc_t;
      *cluster.map_shared_rank(&S.bc_tau, tid) = S.sort_s[t];
      *cluster.map_shared_rank(&S.bc_tiepos, tid) = S.sort_p[t];
      *cluster.map_shared_rank(&S.bc_count, tid) = S.tot_above + S.cut_cnt_above + (uint32_t)t + 1u;
    }
  }
  cluster.sync();  // every CTA holds the cut; no distributed access after this
  return true;
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
  S.l1lo[tid] = 0;
  S.l1hi[tid] = 0;
  S.l1cnt[tid] = 0;
  if (tid == 0) {
    S.nlist = 0;
    S.nabove = 0;
    S.ncand = 0;
  }

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

  // ---- pass 0: 256 linear bins of (max - s), 1/16 nat wide ---------------------
  // (then either the candidate path below or key-window refinement passes)
  uint64_t target = 0, mass_above = 0;
  int lin = -1;               // cut bin of pass 0
  uint32_t kbase = 0;         // key window [kbase, kend) of the refinement passes
  uint64_t kend = 0;
  int shift = 0;
  bool fast = false;
  for (int pass = 0;; ++pass) {
    uint32_t* wlo = S.whlo[warp];
    uint32_t* whi = S.whhi[warp];
    for (int i = lane; i < kBins; i += 32) {
      wlo[i] = 0;
      whi[i] = 0;
    }
    __syncwarp();
    if (pass == 0) {
      for (int base = 0; base < nloc; base += 4 * kSelThreads) {
        float sc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = base + u * kSelThreads + tid;
          sc[u] = i < nloc ? scores[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = base + u * kSelThreads + tid;
          if (i < nloc) {
            const int d = lin_bin(sc[u], m);
            add_u64_pair(&wlo[d], &whi[d], sel_weight(sc[u], m, two_pow_frac));
          }
        }
      }
    } else {
      for (int i = tid; i < nloc; i += kSelThreads) {
        const float sc = scores[i];
        if (lin_bin(sc, m) == lin) {
          const uint32_t k = score_key(sc);
          if (k >= kbase && (uint64_t)k < kend) {
            const int d = (int)((uint64_t)(k - kbase) >> shift);
            add_u64_pair(&wlo[d], &whi[d], sel_weight(sc, m, two_pow_frac));
          }
        }
      }
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
    uint64_t excl;
    const uint64_t incl = block_scan_u64(mine, S.wsum, excl);
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
      if (lin < kBins - 1) {
        fast = collect_cut(S, cluster, scores, nloc, c0, m, two_pow_frac, lin, target - mass_above);
        if (fast) break;
      }
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

  if (fast) {
    // ---- candidate path: (tau, tiepos) came from rank 0; one mask pass -------
    const float tau = S.bc_tau;
    const uint32_t tau_key = score_key(tau);
    const int tpos = S.bc_tiepos;
    for (int base = 0; base < n_chunk; base += 4 * kSelThreads) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * kSelThreads + tid;
        const bool valid = i < nloc;
        const uint32_t k = valid ? score_key(scores[i]) : 0u;
        const bool sel = valid && (k > tau_key || (k == tau_key && c0 + i <= tpos));
        const uint32_t word = __ballot_sync(0xffffffffu, sel);
        const int wpos = base + u * kSelThreads + warp * 32;
        const int w = (c0 + wpos) >> 5;
        if (lane == 0 && mrow && wpos < n_chunk && w < n_words_total) mrow[w] = word;
      }
    }
    if (rank == 0 && tid == 0) {
      tau_bits[qrow] = __float_as_uint(tau);
      tiepos[qrow] = tpos;
      count[qrow] = (int)S.bc_count;
    }
    return;
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
