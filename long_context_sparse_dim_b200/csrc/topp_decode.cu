// a2 + a3 (decode): indexer scores of every cached key and the dynamic top-p cut
// (or, through the same passes with every key weighing 1, a fixed top-k cut).
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
// shared memory.  The cut is found without sorting all keys:
//   pass 0   a 4096-bin histogram of the weights, bins linear in (max - s),
//            1/256 nat wide (the last bin holds the tail).  Summing 16 fine
//            bins gives 256 coarse bins (1/16 nat); every CTA reads all CTAs'
//            coarse bins through distributed shared memory and finds the same
//            coarse cut bin, then the fine cut bin from the 16 fine bins
//            under it;
//   scan     one pass over the scores writes the mask words (keys above the
//            fine cut bin) and sends the keys inside it -- the candidates --
//            to cluster rank 0, with the count of keys above it;
//   rank 0   splits the candidates into 256 sub-bins (1/65536 nat), orders
//            the keys of the cut sub-bin by (score desc, position asc), walks
//            their weights to the cut and sets the candidates' mask bits.
// If the cut lies in the tail bin or the fine cut bin holds more than 512
// keys (long caches, heavy ties), narrowing continues in key space instead (at
// once, without the scan, when the fine bin's mass already proves it too full):
// 256 bins over the order-preserving uint32 image of the fp32 score (8-bit
// digits of the offset inside the fine cut bin, or the coarse tail bin) until
// the bracket is one score value tau;
// ties at tau are resolved by position with a prefix count over the cluster.
// Every mass is a 64-bit fixed-point integer sum, so the result does not depend
// on thread order.  No spin waits: all synchronisation is the hardware cluster
// barrier.
// Caches longer than 16 CTAs x 32768 keys (up to 4x that) give each CTA more
// keys than its shared memory holds: the first 32768 scores stay on chip and
// the rest go to the caller's workspace (written once, read back from L2 by the
// thread that wrote them in every later pass).
#include <cooperative_groups.h>

#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace rtp {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 256;                  // coarse bins, key-space digits, rank 0's sub-bins
constexpr int kFinePerBin = 16;
constexpr int kFineBins = kBins * kFinePerBin;
constexpr int kMaxCluster = 16;
constexpr int kMaxKeysPerCta = 32768;       // scores of one CTA held in shared memory (128 KB)
constexpr int kMaxStream = 4;               // keys per CTA at most kMaxStream x the resident ones
constexpr float kCoarsePerNat = 16.f;       // coarse bin width 1/16 nat
constexpr float kFinePerNat = 256.f;        // fine bin width 1/256 nat
constexpr float kSubPerNat = 65536.f;       // rank 0's sub-bin width 1/65536 nat
constexpr int kCandCap = 512;               // candidates rank 0 resolves
static_assert(kSelThreads == kBins, "one thread per histogram bin");
static_assert(kCandCap <= 4 * kSelThreads, "at most four candidates per thread in the walk");

struct SelSmem {
  union {
    struct {                                  // pass 0, CTA-wide (64-bit masses as lo/hi words)
      uint32_t lo[kFineBins];
      uint32_t hi[kFineBins];
    } f;
    struct {                                  // key-space passes, one histogram per warp
      uint32_t lo[kSelWarps][kBins];
      uint32_t hi[kSelWarps][kBins];
    } w;
    struct {                                  // rank 0, once every candidate has arrived
      uint32_t lo[kBins], hi[kBins], cnt[kBins];
      float s[kCandCap];                      // keys of the cut sub-bin, arrival order
      int32_t p[kCandCap];
      float ss[kCandCap];                     // the same keys in (score desc, position asc) order
      int32_t sp[kCandCap];
    } r;
  } u;
  uint64_t hist[2][kBins];           // this CTA's coarse / key-space histogram, double-buffered
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
  int fine_cut;                      // fine bin holding the cut
  uint64_t fine_above;               // mass of the fine bins above it
  uint64_t fine_mass;                // mass of the fine cut bin
  // rank 0: filled by every CTA between the fine cut and the candidate barrier
  uint32_t ncand;                    // candidates sent (may exceed kCandCap)
  uint32_t nabove;                   // keys above the fine cut bin
  float cand_s[kCandCap];
  int32_t cand_p[kCandCap];
  // rank 0 scratch
  int sub_cut;
  uint64_t sub_above;
  uint32_t sub_cnt_above, nsort;
  int t_cut;
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

// Fixed-point top-p weight round(2^((s - m) log2 e) * 2^frac), or 1 for the
// fixed top-k cut (`unit`): the same passes then count keys instead of weighing
// them.  Every use of a weight in the cut goes through this one function.
RTP_DEVICE uint64_t sel_weight(float s, float m, float two_pow_frac, bool unit) {
  if (unit) return 1ull;
  const float e = ex2f_fast(__fmul_rn(__fsub_rn(s, m), 1.4426950408889634f));
  return __float2ull_rn(__fmul_rn(e, two_pow_frac));
}

// Bins of u = m - s (u rounded once, by __fsub_rn).  The three scalings by
// powers of two are exact, so floor(u * 256) >> 4 == floor(u * 16) and
// floor(u * 65536) >> 8 == floor(u * 256): the bins nest exactly.
RTP_DEVICE int coarse_bin(float s, float m) {  // tail folded into bin 255
  const float t = __fmul_rn(__fsub_rn(m, s), kCoarsePerNat);
  return t >= (float)(kBins - 1) ? kBins - 1 : (int)t;
}
RTP_DEVICE int fine_bin(float s, float m) {  // tail folded into bin 4095 (coarse 255)
  const float t = __fmul_rn(__fsub_rn(m, s), kFinePerNat);
  return t >= (float)(kFineBins - 1) ? kFineBins - 1 : (int)t;
}
RTP_DEVICE int sub_bin(float s, float m, int fine) {  // fine < 4080: u < 15.94, t < 2^20
  const float t = __fmul_rn(__fsub_rn(m, s), kSubPerNat);
  const int d = (int)t - fine * kBins;
  return d < 0 ? 0 : (d > kBins - 1 ? kBins - 1 : d);
}

RTP_DEVICE uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive prefix sum over the block's threads in thread order; `wsum` holds
// one word per warp.  Ends with a barrier, so `wsum` may be reused at once.
RTP_DEVICE uint64_t block_scan_u64(uint64_t v, uint64_t* wsum, uint64_t& excl, uint64_t* total = nullptr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  uint64_t off = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    const uint64_t x = wsum[w];
    off += w < warp ? x : 0;
    all += x;
  }
  __syncthreads();
  if (total) *total = all;
  incl += off;
  excl = incl - v;
  return incl;
}

// Split cluster barrier: arrive (release) after this CTA's last access to
// another CTA's shared memory; wait (acquire) before touching shared memory
// that others may still read.
RTP_DEVICE void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory"); }
RTP_DEVICE void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory"); }

// Cluster-wide histogram of `hb` (256 bins) and the bin holding the cut:
// with `first`, Z = total mass and target = ceil(p Z) are set first (for the
// top-k cut, Z is the number of keys and the target min(k, Z)).  Bins are
// taken in descending score order (`ascending_bins`: bin 0 holds the highest
// scores).  Returns the cut bin; mass_above grows by the mass before it.
RTP_DEVICE int cluster_cut(SelSmem& S, cg::cluster_group& cluster, const uint64_t* hb, bool first,
                           bool ascending_bins, float p, int topk, uint64_t& target, uint64_t& mass_above) {
  const int tid = threadIdx.x;
  const int C = (int)cluster.num_blocks();
  cluster.sync();  // every CTA's histogram of this pass is complete
  uint64_t a = 0;
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r)
    if (r < C) a += cluster.map_shared_rank(hb, r)[tid];
  // position r of the descending score order holds bin r (ascending bins) or bin 255 - r
  uint64_t mine = a;
  if (!ascending_bins) {
    S.red[tid] = a;
    __syncthreads();
    mine = S.red[kBins - 1 - tid];
  }
  uint64_t excl, Z;
  const uint64_t incl = block_scan_u64(mine, S.wsum, excl, &Z);
  if (first) {  // Z = total mass; target = ceil(p Z), or min(k, Z) keys
    if (topk > 0) {
      target = (uint64_t)topk < Z ? (uint64_t)topk : Z;
    } else {
      const double t = ceil((double)p * (double)Z);
      const uint64_t tt = t >= (double)Z ? Z : (uint64_t)t;
      target = tt < 1 ? 1 : tt;
    }
  }
  const uint64_t need = target - mass_above;  // >= 1
  if (excl < need && need <= incl) {  // exactly one position holds the cut
    S.cut_bin = ascending_bins ? tid : (kBins - 1 - tid);
    S.cut_above = excl;
  }
  __syncthreads();
  // (S.cut_bin and S.cut_above are written again only after the next cluster barrier)
  mass_above += S.cut_above;
  return S.cut_bin;
}

// Rank 0, once all n (<= kCandCap) keys of fine bin `fb` are in cand_s/cand_p:
// split them into 256 sub-bins (mass and count), order the keys of the cut
// sub-bin by (score desc, position asc), walk their weights to the cut, write
// the result and set the selected candidates' mask bits (the other CTAs wrote
// the words of the keys above bin fb before the candidate barrier).  `need` is
// the mass still to take inside bin fb: >= 1 and <= the bin's mass, which the
// candidates' weights add up to exactly.
RTP_DEVICE void resolve_candidates(SelSmem& S, int n, int fb, float m, float two_pow_frac, bool unit, uint64_t need,
                                   uint32_t* mrow, int qrow, uint32_t* tau_bits, int32_t* tiepos,
                                   int32_t* count) {
  const int tid = threadIdx.x;
  S.u.r.lo[tid] = 0;
  S.u.r.hi[tid] = 0;
  S.u.r.cnt[tid] = 0;
  if (tid == 0) {
    S.nsort = 0;
    S.sub_cut = 0;
    S.sub_above = 0;
    S.sub_cnt_above = 0;
    S.t_cut = -1;
  }
  __syncthreads();
  for (int j = tid; j < n; j += kSelThreads) {
    const float sc = S.cand_s[j];
    const int d = sub_bin(sc, m, fb);
    add_u64_pair(&S.u.r.lo[d], &S.u.r.hi[d], sel_weight(sc, m, two_pow_frac, unit));
    atomicAdd(&S.u.r.cnt[d], 1u);
  }
  __syncthreads();
  uint64_t em, ec;
  const uint64_t im = block_scan_u64(pair_value(S.u.r.lo[tid], S.u.r.hi[tid]), S.wsum, em);  // sub-bin 0 = highest
  block_scan_u64((uint64_t)S.u.r.cnt[tid], S.wsum, ec);
  if (em < need && need <= im) {
    S.sub_cut = tid;
    S.sub_above = em;
    S.sub_cnt_above = (uint32_t)ec;
  }
  __syncthreads();
  const int sb = S.sub_cut;
  const uint64_t need2 = need - S.sub_above;
  for (int j = tid; j < n; j += kSelThreads) {
    const float sc = S.cand_s[j];
    if (sub_bin(sc, m, fb) == sb) {
      const uint32_t k = atomicAdd(&S.nsort, 1u);
      S.u.r.s[k] = sc;
      S.u.r.p[k] = S.cand_p[j];
    }
  }
  __syncthreads();
  const int ns = (int)S.nsort;
  for (int j = tid; j < ns; j += kSelThreads) {
    const uint32_t kt = score_key(S.u.r.s[j]);
    const int pt = S.u.r.p[j];
    int rk = 0;
    for (int i = 0; i < ns; ++i) {
      const uint32_t ki = score_key(S.u.r.s[i]);
      rk += (ki > kt || (ki == kt && S.u.r.p[i] < pt)) ? 1 : 0;
    }
    S.u.r.ss[rk] = S.u.r.s[j];
    S.u.r.sp[rk] = pt;
  }
  __syncthreads();
  // walk the ordered keys; thread t holds positions 4t .. 4t+3
  uint64_t wv[4], tot = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int idx = 4 * tid + k;
    wv[k] = idx < ns ? sel_weight(S.u.r.ss[idx], m, two_pow_frac, unit) : 0;
    tot += wv[k];
  }
  uint64_t run;
  block_scan_u64(tot, S.wsum, run);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int idx = 4 * tid + k;
    if (idx < ns && run < need2 && need2 <= run + wv[k]) S.t_cut = idx;
    run += wv[k];
  }
  __syncthreads();
  int t = S.t_cut;
  if (t < 0) t = ns > 0 ? ns - 1 : 0;  // not reached: the sub-bin's mass covers need2
  const float tau = S.u.r.ss[t];
  const int tp = S.u.r.sp[t];
  const uint32_t tk = score_key(tau);
  if (mrow) {
    for (int j = tid; j < n; j += kSelThreads) {
      const uint32_t k = score_key(S.cand_s[j]);
      const int pos = S.cand_p[j];
      if (k > tk || (k == tk && pos <= tp)) atomicOr(&mrow[pos >> 5], 1u << (pos & 31));
    }
  }
  if (tid == 0) {
    tau_bits[qrow] = __float_as_uint(tau);
    tiepos[qrow] = tp;
    count[qrow] = (int)(S.nabove + S.sub_cnt_above + (uint32_t)t + 1u);
  }
}

// At most 96 registers a thread, so that two of these CTAs leave room on an SM
// for a CTA of the window attention that runs concurrently.
template <typename T>
__global__ void __maxnreg__(96)
topp_query_kernel(View4 qv, View4 kv, const int32_t* __restrict__ lens, int Hq, int G, int N,
                   int n_chunk, float p, int topk, float two_pow_frac, uint32_t* __restrict__ tau_bits,
                   int32_t* __restrict__ tiepos, int32_t* __restrict__ count,
                   uint32_t* __restrict__ mask, int64_t mask_words, float* __restrict__ spill) {
  pdl_wait();
  pdl_release();
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qrow = blockIdx.x / C;
  const int b = qrow / Hq, h = qrow % Hq, kvh = h / G;
  const bool unit = topk > 0;  // fixed top-k: every key weighs 1

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
  if (n_b == 0 || (!unit && p >= 1.f) || (unit && topk >= n_b)) {
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

  for (int i = tid; i < kFineBins; i += kSelThreads) {
    S.u.f.lo[i] = 0;
    S.u.f.hi[i] = 0;
  }
  if (tid == 0) {
    S.ncand = 0;
    S.nabove = 0;
    S.fine_cut = 0;
    S.fine_above = 0;
  }

  // ---- scores of this CTA's keys (four independent row loads in flight per thread)
  float qf[kIdxDim];
  load_idx_row<T>(static_cast<const T*>(qv.data) + b * qv.sb + h * qv.sh, qf);
  const T* kb = static_cast<const T*>(kv.data) + b * kv.sb + kvh * kv.sh;
  float lmax = -INFINITY;
  const int n_res = min(n_chunk, kMaxKeysPerCta);  // keys whose scores stay in shared memory
  // this CTA's scores past the resident ones; every pass maps key i to thread i % kSelThreads, so
  // each thread reads back only what it wrote
  float* const gsc = spill ? spill + ((int64_t)qrow * C + rank) * (int64_t)(n_chunk - n_res) : nullptr;
  auto score_of = [&](int i) -> float { return i < n_res ? scores[i] : gsc[i - n_res]; };
  constexpr int U = sizeof(T) == 2 ? 4 : 2;
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
        if (i < n_res)
          scores[i] = sc;
        else
          gsc[i - n_res] = sc;
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

  // ---- pass 0: fine histogram of the weights (CTA-wide), then coarse bins ----
  for (int base = 0; base < nloc; base += 4 * kSelThreads) {
    float sc[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kSelThreads + tid;
      sc[u] = i < nloc ? score_of(i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * kSelThreads + tid;
      if (i < nloc) {
        const int f = fine_bin(sc[u], m);
        add_u64_pair(&S.u.f.lo[f], &S.u.f.hi[f], sel_weight(sc[u], m, two_pow_frac, unit));
      }
    }
  }
  __syncthreads();
  {
    // coarse bin tid = fine bins 16 tid .. 16 tid + 15 (rotated start: no bank conflicts)
    uint64_t a = 0;
#pragma unroll
    for (int j = 0; j < kFinePerBin; ++j) {
      const int f = tid * kFinePerBin + ((j + tid) & (kFinePerBin - 1));
      a += pair_value(S.u.f.lo[f], S.u.f.hi[f]);
    }
    S.hist[0][tid] = a;
  }
  uint64_t target = 0, mass_above = 0;
  const int lin = cluster_cut(S, cluster, S.hist[0], true, true, p, topk, target, mass_above);
  int fine = -1;  // the fine cut bin, when the key-space narrowing below starts from it

  if (lin < kBins - 1) {
    // ---- the fine bin of the cut, from the 16 fine bins under coarse bin lin --
    if (warp == 0) {
      uint64_t a = 0;
      if (lane < kFinePerBin) {
        const int f = lin * kFinePerBin + lane;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
          if (r < C) a += pair_value(cluster.map_shared_rank(S.u.f.lo, r)[f], cluster.map_shared_rank(S.u.f.hi, r)[f]);
      }
      uint64_t incl = a;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const uint64_t need = target - mass_above;
      if (lane < kFinePerBin && incl - a < need && need <= incl) {
        S.fine_cut = lin * kFinePerBin + lane;
        S.fine_above = mass_above + (incl - a);
        S.fine_mass = a;
      }
    }
    __syncthreads();
    const int fb = S.fine_cut;
    // A fine bin whose mass exceeds kCandCap times the largest weight a key of it can have (at its
    // upper end, u = fb / 256) certainly holds more candidates than rank 0 takes: skip the candidate
    // scan and narrow in key space at once (the same decision on every CTA of the cluster).
    {
      const double w_max = unit ? 1.0
                                : (double)__float2ull_rn(__fmul_rn(
                                      ex2f_fast(__fmul_rn(-(float)fb / kFinePerNat, 1.4426950408889634f)),
                                      two_pow_frac)) * (1.0 + 9.5367431640625e-07);
      if ((double)S.fine_mass > (double)kCandCap * w_max) {
        fine = fb;
        mass_above = S.fine_above;
        cluster.sync();  // every CTA has read the others' fine bins before the passes below reuse them
        goto key_space;
      }
    }

    // ---- one scan: mask words of the keys above the fine cut bin; its keys
    //      (the candidates) and the count of keys above it go to rank 0 ------
    {
      uint32_t* r_ncand = cluster.map_shared_rank(&S.ncand, 0);
      float* r_cs = cluster.map_shared_rank(S.cand_s, 0);
      int32_t* r_cp = cluster.map_shared_rank(S.cand_p, 0);
      uint32_t nab = 0;
      for (int base = 0; base < n_chunk; base += 4 * kSelThreads) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = base + u * kSelThreads + tid;
          const bool valid = i < nloc;
          const float sc = valid ? score_of(i) : 0.f;
          const int f = valid ? fine_bin(sc, m) : kFineBins;
          const uint32_t word = __ballot_sync(0xffffffffu, f < fb);
          const int wpos = base + u * kSelThreads + warp * 32;
          const int w = (c0 + wpos) >> 5;
          if (lane == 0 && wpos < n_chunk && w < n_words_total) {
            if (mrow) mrow[w] = word;
            nab += (uint32_t)__popc(word);
          }
          const bool cand = f == fb;
          const uint32_t cb = __ballot_sync(0xffffffffu, cand);
          if (cb) {
            uint32_t s0 = 0;
            if (lane == 0) s0 = atomicAdd(r_ncand, (uint32_t)__popc(cb));
            s0 = __shfl_sync(0xffffffffu, s0, 0);
            if (cand) {
              const uint32_t slot = s0 + (uint32_t)__popc(cb & ((1u << lane) - 1u));
              if (slot < (uint32_t)kCandCap) {
                r_cs[slot] = sc;
                r_cp[slot] = c0 + i;
              }
            }
          }
        }
      }
      if (lane == 0 && nab) atomicAdd(cluster.map_shared_rank(&S.nabove, 0), nab);
    }
    cluster.sync();  // every candidate and count is at rank 0
    const uint32_t ntot = *cluster.map_shared_rank(&S.ncand, 0);
    cluster_arrive();  // this CTA's last distributed access
    if (ntot <= (uint32_t)kCandCap) {
      if (rank == 0) resolve_candidates(S, (int)ntot, fb, m, two_pow_frac, unit, target - S.fine_above, mrow, qrow,
                                        tau_bits, tiepos, count);
      // rank 0 keeps its shared memory until every CTA has read the candidate total
      if (rank == 0) cluster_wait();
      return;
    }
    cluster_wait();  // more candidates than rank 0 takes: narrow in key space below
    fine = fb;       // inside the fine cut bin, 16 times narrower than the coarse one
    mass_above = S.fine_above;
  }

key_space:
  // ---- key-space narrowing inside the fine cut bin (or coarse bin lin for the tail) ----
  // key window holding every score of that bin (with a margin)
  uint32_t kbase;
  uint64_t kend;
  int shift = 0;
  {
    const float per_nat = fine >= 0 ? kFinePerNat : kCoarsePerNat;
    const int bin = fine >= 0 ? fine : lin;
    const float hi_s = m - (float)bin / per_nat;
    const float lo_s = m - (float)(bin + 1) / per_nat;
    const float mg = 1e-5f * (fabsf(m) + (float)(bin + 1) / per_nat) + 1e-30f;
    const uint32_t khi = score_key(__fadd_rn(hi_s + mg, 0.0f));
    const uint32_t klo = fine < 0 && lin == kBins - 1 ? 0u : score_key(__fadd_rn(lo_s - mg, 0.0f));
    kbase = klo;
    kend = (uint64_t)khi + 1;
    const uint64_t range = kend - klo;
    while (((range - 1) >> shift) >= (uint64_t)kBins) ++shift;
  }
  for (int pass = 1;; ++pass) {
    uint32_t* wlo = S.u.w.lo[warp];
    uint32_t* whi = S.u.w.hi[warp];
    for (int i = lane; i < kBins; i += 32) {
      wlo[i] = 0;
      whi[i] = 0;
    }
    __syncwarp();
    for (int i = tid; i < nloc; i += kSelThreads) {
      const float sc = score_of(i);
      if (fine >= 0 ? fine_bin(sc, m) == fine : coarse_bin(sc, m) == lin) {
        const uint32_t k = score_key(sc);
        if (k >= kbase && (uint64_t)k < kend) {
          const int d = (int)((uint64_t)(k - kbase) >> shift);
          add_u64_pair(&wlo[d], &whi[d], sel_weight(sc, m, two_pow_frac, unit));
        }
      }
    }
    __syncthreads();
    uint64_t* hb = S.hist[pass & 1];
    {
      uint64_t a = 0;
#pragma unroll
      for (int w = 0; w < kSelWarps; ++w) a += pair_value(S.u.w.lo[w][tid], S.u.w.hi[w][tid]);
      hb[tid] = a;
    }
    // digit bins: bin 255 holds the highest keys
    const int cb = cluster_cut(S, cluster, hb, false, false, p, topk, target, mass_above);
    kbase += (uint32_t)cb << shift;
    const uint64_t e = (uint64_t)kbase + (uint64_t(1) << shift);
    kend = e < kend ? e : kend;
    if (shift == 0) break;            // the bracket is one score value
    shift = shift >= 8 ? shift - 8 : 0;
  }

  // ---- counts at tau: keys above and equal, per CTA, then over the cluster ----
  const uint32_t tau_key = kbase;
  const float tau = key_score(tau_key);
  uint32_t ngt = 0, neq = 0;
  for (int i = tid; i < nloc; i += kSelThreads) {
    const uint32_t k = score_key(score_of(i));
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
  const uint64_t w_tau = sel_weight(tau, m, two_pow_frac, unit);
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
    const uint32_t k = valid ? score_key(score_of(i)) : 0u;
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

bool topp_decode_supported(int64_t N) { return N <= (int64_t)kMaxKeysPerCta * kMaxCluster * kMaxStream; }

// CTAs per query (a power of two <= kMaxCluster) and keys per CTA (a multiple of 32).
static void topp_layout(int64_t Q, int64_t N, int sms, int* C_out, int64_t* n_chunk_out) {
  int C = 1;
  while (C < 8 && Q * C < sms) C <<= 1;
  while ((N + C - 1) / C > kMaxKeysPerCta && C < kMaxCluster) C <<= 1;
  int64_t n_chunk = (N + C - 1) / C;
  n_chunk = (n_chunk + 31) / 32 * 32;
  if (n_chunk == 0) n_chunk = 32;
  *C_out = C;
  *n_chunk_out = n_chunk;
}

size_t topp_decode_workspace_bytes(int64_t B, int64_t Hq, int64_t N) {
  // the layout depends on the SM count only while every CTA's keys fit on chip; past that
  // the cluster has kMaxCluster CTAs whatever the SM count
  int C = 0;
  int64_t n_chunk = 0;
  topp_layout(B * Hq, N, 1, &C, &n_chunk);
  const int64_t per = n_chunk > kMaxKeysPerCta ? (n_chunk - kMaxKeysPerCta) * C : 0;
  return (size_t)(B * Hq * per) * sizeof(float);
}

static int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <typename K, typename... Args>
static cudaError_t launch_cluster(K kern, int grid, int C, size_t smem, cudaStream_t stream, Args... args) {
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
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
  int64_t n_chunk = 0;
  topp_layout(Q, a.N, sms, &C, &n_chunk);
  if (n_chunk > (int64_t)kMaxKeysPerCta * kMaxStream) return cudaErrorInvalidValue;
  if (n_chunk > kMaxKeysPerCta && !a.spill) return cudaErrorInvalidValue;
  const size_t smem = sizeof(SelSmem) + (size_t)(n_chunk < kMaxKeysPerCta ? n_chunk : kMaxKeysPerCta) * sizeof(float);
  if (a.bf16)
    return launch_cluster(topp_query_kernel<__nv_bfloat16>, (int)(Q * C), C, smem, stream, a.q_idx, a.k_idx, a.lens,
                          (int)a.Hq, G, (int)a.N, (int)n_chunk, a.p, (int)a.topk, two_pow_frac, a.tau_bits, a.tiepos,
                          a.count, a.mask, a.mask_words, a.spill);
  return launch_cluster(topp_query_kernel<float>, (int)(Q * C), C, smem, stream, a.q_idx, a.k_idx, a.lens, (int)a.Hq,
                        G, (int)a.N, (int)n_chunk, a.p, (int)a.topk, two_pow_frac, a.tau_bits, a.tiepos, a.count,
                        a.mask, a.mask_words, a.spill);
}

}  // namespace rtp
