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
// shared memory.  The cut is found without sorting by a three-digit radix
// search on the order-preserving uint32 image of the fp32 scores (11 + 11 + 10
// bits, most significant first).  Each digit pass builds a weighted histogram
// (64-bit fixed-point mass + count) per CTA; the cluster reduces it through
// distributed shared memory, each CTA summing one slice of the bins, and the
// CTA holding the cut bin broadcasts it.  After the last digit the cut bin is
// one score value tau; ties at tau are resolved by position with a prefix
// count over the cluster.  Finally every CTA writes its bits of the selection
// mask.  There are no global-memory atomics and no spin waits: all
// synchronisation is the hardware cluster barrier.
#include <cooperative_groups.h>

#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace rtp {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;            // 11-bit digits; the last pass uses 1024 bins
constexpr int kMaxCluster = 16;
constexpr int kMaxKeysPerCta = 32768;  // scores of one CTA held in shared memory (128 KB)

struct SelDecision {
  uint64_t mass_above;  // mass of this pass's bins above the cut bin
  uint64_t bin_mass;
  uint32_t bin;         // cut bin (digit value)
  uint32_t bin_cnt;
  uint32_t cnt_above;
  uint32_t pad;
};

struct SelSmem {
  uint64_t hist_mass[kBins];
  uint32_t hist_cnt[kBins];
  uint64_t red_mass[kBins];
  uint32_t red_cnt[kBins];
  uint64_t slice_mass[kMaxCluster];
  uint32_t slice_cnt[kMaxCluster];
  uint32_t tcount[kMaxCluster];
  SelDecision dec;
  float cmax_self;
  float wmax[kSelWarps];
  uint64_t wmass[kSelWarps];
  uint32_t wcnt[kSelWarps];
  uint32_t wtot[kSelWarps];
};

RTP_DEVICE int ceil_log2(int64_t n) {
  int r = 0;
  while ((int64_t(1) << r) < n) ++r;
  return r;
}

template <typename T>
__global__ void __launch_bounds__(kSelThreads)
topp_decode_kernel(View4 qv, View4 kv, const int32_t* __restrict__ lens, int Hq, int G, int N,
                   int n_chunk, float p, float two_pow_frac, uint32_t* __restrict__ tau_bits,
                   int32_t* __restrict__ tiepos, int32_t* __restrict__ count,
                   uint32_t* __restrict__ mask, int64_t mask_words) {
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

  // ---- scores of this CTA's keys -------------------------------------------
  float qf[kIdxDim];
  load_idx_row<T>(static_cast<const T*>(qv.data) + b * qv.sb + h * qv.sh, qf);
  const T* kb = static_cast<const T*>(kv.data) + b * kv.sb + kvh * kv.sh;
  float lmax = -INFINITY;
  for (int i = tid; i < nloc; i += kSelThreads) {
    float kf[kIdxDim];
    load_idx_row<T>(kb + (int64_t)(c0 + i) * kv.sn, kf);
    const float s = indexer_dot16(qf, kf);
    scores[i] = s;
    lmax = fmaxf(lmax, s);
  }
  lmax = warp_max(lmax);
  if (lane == 0) S.wmax[warp] = lmax;
  __syncthreads();
  if (tid == 0) {
    float m = S.wmax[0];
    for (int w = 1; w < kSelWarps; ++w) m = fmaxf(m, S.wmax[w]);
    S.cmax_self = m;
  }
  cluster.sync();
  float m = -INFINITY;
  for (int r = 0; r < C; ++r) m = fmaxf(m, *cluster.map_shared_rank(&S.cmax_self, r));

  // ---- three radix passes ----------------------------------------------------
  uint64_t target = 0, mass_above = 0;
  uint32_t cnt_above = 0, prefix = 0, tau_cnt = 0;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const int pshift = pass == 1 ? 21 : 10;  // bits of the prefix fixed by earlier passes
    for (int i = tid; i < nb; i += kSelThreads) {
      S.hist_mass[i] = 0;
      S.hist_cnt[i] = 0;
    }
    __syncthreads();
    for (int i = tid; i < nloc; i += kSelThreads) {
      const float s = scores[i];
      const uint32_t k = score_key(s);
      if (pass == 0 || (k >> pshift) == prefix) {
        const uint32_t d = (k >> shift) & (uint32_t)(nb - 1);
        atomicAdd(reinterpret_cast<unsigned long long*>(&S.hist_mass[d]),
                  (unsigned long long)fixed_weight(s, m, two_pow_frac));
        atomicAdd(&S.hist_cnt[d], 1u);
      }
    }
    cluster.sync();  // (A) every CTA's histogram is complete

    // Reduce the bins this CTA owns across the cluster.
    const int sl = nb / C;
    const int lo = rank * sl;
    uint64_t tm = 0;
    uint32_t tc = 0;
    for (int i = tid; i < sl; i += kSelThreads) {
      uint64_t am = 0;
      uint32_t ac = 0;
      for (int r = 0; r < C; ++r) {
        am += cluster.map_shared_rank(S.hist_mass, r)[lo + i];
        ac += cluster.map_shared_rank(S.hist_cnt, r)[lo + i];
      }
      S.red_mass[i] = am;
      S.red_cnt[i] = ac;
      tm += am;
      tc += ac;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      tm += __shfl_xor_sync(0xffffffffu, tm, o);
      tc += __shfl_xor_sync(0xffffffffu, tc, o);
    }
    if (lane == 0) {
      S.wmass[warp] = tm;
      S.wcnt[warp] = tc;
    }
    __syncthreads();
    if (tid < C) {
      uint64_t sm = 0;
      uint32_t sc = 0;
      for (int w = 0; w < kSelWarps; ++w) {
        sm += S.wmass[w];
        sc += S.wcnt[w];
      }
      cluster.map_shared_rank(S.slice_mass, tid)[rank] = sm;
      cluster.map_shared_rank(S.slice_cnt, tid)[rank] = sc;
    }
    cluster.sync();  // (B) all slice totals are known everywhere

    if (pass == 0) {
      uint64_t Z = 0;
      for (int r = 0; r < C; ++r) Z += S.slice_mass[r];
      double t = ceil((double)p * (double)Z);
      uint64_t tt = t >= (double)Z ? Z : (uint64_t)t;
      target = tt < 1 ? 1 : tt;
    }
    const uint64_t need = target - mass_above;  // >= 1
    // The cut slice: walking slices from the highest scores down.
    uint64_t cum = 0;
    uint32_t cumc = 0;
    int cut_r = 0;
    for (int r = C - 1; r >= 0; --r) {
      if (cum + S.slice_mass[r] >= need) {
        cut_r = r;
        break;
      }
      cum += S.slice_mass[r];
      cumc += S.slice_cnt[r];
    }
    if (rank == cut_r && warp == 0) {
      // lane l covers local bins [hi_l - per, hi_l), lane 0 the highest
      const int per = (sl + 31) / 32;
      const int hi_l = sl - lane * per;
      const int lo_l = max(hi_l - per, 0);
      uint64_t lm = 0;
      uint32_t lc = 0;
      for (int i = lo_l; i < hi_l; ++i) {
        lm += S.red_mass[i];
        lc += S.red_cnt[i];
      }
      uint64_t incl = lm;
      uint32_t inclc = lc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t vm = __shfl_up_sync(0xffffffffu, incl, o);
        const uint32_t vc = __shfl_up_sync(0xffffffffu, inclc, o);
        if (lane >= o) {
          incl += vm;
          inclc += vc;
        }
      }
      const uint64_t excl = incl - lm;
      const uint32_t exclc = inclc - lc;
      if (hi_l > lo_l && cum + excl < need && need <= cum + incl) {
        uint64_t ma = cum + excl;
        uint32_t ca = cumc + exclc;
        int bin = lo_l;
        for (int i = hi_l - 1; i >= lo_l; --i) {
          if (ma + S.red_mass[i] >= need) {
            bin = i;
            break;
          }
          ma += S.red_mass[i];
          ca += S.red_cnt[i];
        }
        SelDecision d;
        d.mass_above = ma;
        d.bin_mass = S.red_mass[bin];
        d.bin = (uint32_t)(lo + bin);
        d.bin_cnt = S.red_cnt[bin];
        d.cnt_above = ca;
        d.pad = 0;
        for (int r = 0; r < C; ++r) *cluster.map_shared_rank(&S.dec, r) = d;
      }
    }
    cluster.sync();  // (C) the decision is everywhere
    const SelDecision d = S.dec;
    mass_above += d.mass_above;
    cnt_above += d.cnt_above;
    prefix = pass == 2 ? ((prefix << 10) | d.bin) : ((prefix << 11) | d.bin);
    tau_cnt = d.bin_cnt;
  }

  // ---- ties at tau, by position ---------------------------------------------
  const uint32_t tau_key = prefix;
  const float tau = key_score(tau_key);
  const uint64_t w_tau = fixed_weight(tau, m, two_pow_frac);
  const uint64_t rem = target - mass_above;
  uint64_t n_tau64 = w_tau ? (rem + w_tau - 1) / w_tau : (uint64_t)tau_cnt;
  if (n_tau64 < 1) n_tau64 = 1;
  if (n_tau64 > tau_cnt) n_tau64 = tau_cnt;
  const int n_tau = (int)n_tau64;
  const uint32_t my_tau = S.hist_cnt[tau_key & 1023u];  // this CTA's keys equal to tau
  if (tid < C) cluster.map_shared_rank(S.tcount, tid)[rank] = my_tau;
  cluster.sync();  // (D) last distributed access
  int before = 0;
  for (int r = 0; r < rank; ++r) before += (int)S.tcount[r];
  const int want = n_tau - before;  // how many of this CTA's tau keys are taken

  // ---- mask bits and the tie position ---------------------------------------
  int running = 0;
  for (int base = 0; base < n_chunk; base += kSelThreads) {
    const int i = base + tid;
    const bool valid = i < nloc;
    const uint32_t k = valid ? score_key(scores[i]) : 0u;
    const bool gt = valid && k > tau_key;
    const bool eq = valid && k == tau_key;
    const uint32_t beq = __ballot_sync(0xffffffffu, eq);
    const int wpre = __popc(beq & ((1u << lane) - 1u));
    if (lane == 0) S.wtot[warp] = __popc(beq);
    __syncthreads();
    int woff = 0, rtot = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      const int t = (int)S.wtot[w];
      woff += w < warp ? t : 0;
      rtot += t;
    }
    __syncthreads();
    const int r_eq = running + woff + wpre;
    const bool sel = gt || (eq && r_eq < want);
    if (eq && r_eq == want - 1) tiepos[qrow] = c0 + i;
    const uint32_t word = __ballot_sync(0xffffffffu, sel);
    const int wpos = base + warp * 32;
    const int w = (c0 + wpos) >> 5;
    if (lane == 0 && mrow && wpos < n_chunk && w < n_words_total) mrow[w] = word;
    running += rtot;
  }
  if (rank == 0 && tid == 0) {
    tau_bits[qrow] = __float_as_uint(tau);
    count[qrow] = (int)(cnt_above + (uint32_t)n_tau);
  }
}

bool topp_decode_supported(int64_t N) { return N <= (int64_t)kMaxKeysPerCta * kMaxCluster; }

cudaError_t launch_topp_decode(const LaunchToppDecode& a, cudaStream_t stream) {
  const int64_t Q = a.B * a.Hq;
  if (Q == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // cluster size: enough CTAs to cover the GPU twice, and few enough keys per CTA
  int C = 1;
  while (C < 8 && Q * C < 2 * sms) C <<= 1;
  while ((a.N + C - 1) / C > kMaxKeysPerCta && C < kMaxCluster) C <<= 1;
  int64_t n_chunk = (a.N + C - 1) / C;
  n_chunk = (n_chunk + 31) / 32 * 32;
  if (n_chunk == 0) n_chunk = 32;
  if (n_chunk > kMaxKeysPerCta) return cudaErrorInvalidValue;
  const size_t smem = sizeof(SelSmem) + (size_t)n_chunk * sizeof(float);
  int lg = 0;
  while ((int64_t(1) << lg) < a.N) ++lg;
  const float two_pow_frac = ldexpf(1.f, 63 - lg);
  const int G = (int)(a.Hq / a.Hk);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(Q * C));
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  cudaError_t e;
  if (a.bf16) {
    auto kern = topp_decode_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (C > 8) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    e = cudaLaunchKernelEx(&cfg, kern, a.q_idx, a.k_idx, a.lens, (int)a.Hq, G, (int)a.N, (int)n_chunk, a.p,
                           two_pow_frac, a.tau_bits, a.tiepos, a.count, a.mask, a.mask_words);
  } else {
    auto kern = topp_decode_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (C > 8) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    e = cudaLaunchKernelEx(&cfg, kern, a.q_idx, a.k_idx, a.lens, (int)a.Hq, G, (int)a.N, (int)n_chunk, a.p,
                           two_pow_frac, a.tau_bits, a.tiepos, a.count, a.mask, a.mask_words);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rtp
