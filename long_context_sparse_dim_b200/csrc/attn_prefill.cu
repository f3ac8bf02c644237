// a4 / a5 (prefill): causal attention of T query tokens per sequence over
//   - their selected keys (retrieval heads: threshold form tau, tiepos from
//     rtp_topp_select), or
//   - the last W keys up to their own position (local heads).
//
// "Full Attention Strikes Back ... (RTPurbo)", TL;DR (sparse attention over the
// tokens the indexer picks); "RTPurbo: Turning Dense LLMs into Sparse Attention
// Models ...", "Three Key Insights" 1 (local heads keep a window) and 3.
//
// Design (B200): a CTA takes one query head and 128 query tokens; K/V tiles of
// 64 keys stream through a two-stage cp.async ring (256-byte rows, XOR
// swizzle).  Eight warps each own 16 query rows and run the flash-attention
// recurrence on mma.sync (S = Q K^T, online softmax, P as a bf16 hi + lo pair,
// O += P V).  For the sparse form, key j is admitted for token i iff
// s_ij > tau_i or (s_ij == tau_i and j <= tiepos_i): the indexer tile s is
// recomputed with exactly the instruction the selection used (tcgen05.mma
// kind::f16, M=128, N=64, K=16, projected tiles fed by TMA with the 32-byte
// swizzle), so the predicate sees bit-identical scores.  A ninth warp issues
// those TMA loads and MMAs; warps 0-3 read the accumulators from TMEM (one
// token per lane) and publish a 128 x 64 admission bitmap per tile in shared
// memory; warps skip tiles where none of their rows admits a key.
#include <math.h>

#include "launch.h"
#include "tc05.cuh"

namespace rtp {

namespace {

constexpr int kApRows = 128;
constexpr int kApKeys = 64;
constexpr int kApMathWarps = 8;
constexpr int kApRowBytes = kHeadDim * 2;                 // 256 B
constexpr int kApTileBytes = kApKeys * kApRowBytes;       // 16 KB per K or V tile
constexpr int kApIdxTileBytes = kApKeys * kIdxDim * 2;    // 2 KB
constexpr float kLog2eF = 1.4426950408889634f;
// The MMA accumulators are folded into a round-to-nearest fp32 sum every
// kApFlush tiles: tensor-core accumulation does not round to nearest, so one
// accumulator carried over a million keys would drift by ~1e-3 relative.
constexpr int kApFlush = 16;

struct ApSmem {
  alignas(1024) uint8_t qidx[kApRows * kIdxDim * 2];      // 4 KB (sparse form)
  alignas(1024) uint8_t kidx[2][kApIdxTileBytes];          // 2 x 2 KB (sparse form)
  alignas(128) uint8_t q[kApRows * kApRowBytes];          // 32 KB
  alignas(128) uint8_t kv[2][2][kApTileBytes];            // [stage][K,V] 64 KB
  uint32_t bits[2][kApRows][2];                           // admission bitmaps, double-buffered
  float otot[kApMathWarps][64][32];                       // round-to-nearest running output sums
  uint64_t qidx_full;
  uint64_t kidx_full[2];
  uint64_t kidx_empty[2];
  uint64_t t_full[2];
  uint64_t t_empty[2];
  uint32_t tmem_base;
};

struct ApArgs {
  View4 q, k, v;
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

RTP_DEVICE uint32_t ap_swz(int r, int c) { return (uint32_t)(r * kApRowBytes + ((c ^ (r & 7)) << 4)); }

RTP_DEVICE void cp16(uint32_t dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(pred ? 16 : 0));
}
RTP_DEVICE void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
RTP_DEVICE void cp_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }
RTP_DEVICE void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
RTP_DEVICE void ldsm4t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
RTP_DEVICE void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
RTP_DEVICE float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
RTP_DEVICE void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory"); }

}  // namespace

template <bool SPARSE>
__global__ void __launch_bounds__(kApMathWarps * 32 + (SPARSE ? 32 : 0))
attn_prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, ApArgs A) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  ApSmem& S = *reinterpret_cast<ApSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int t0 = blockIdx.x * kApRows;
  const int bh = blockIdx.y;
  const int b = bh / A.Hq, h = bh % A.Hq, kvh = h / A.G;
  int n_b = A.N;
  if (A.lens) n_b = min(max(A.lens[b], 0), A.N);
  const int qbase = n_b - A.T;
  const int t_last = min(t0 + kApRows, A.T) - 1;
  const int kmax = min(qbase + t_last, n_b - 1);  // last key any row of the block sees
  int klo = 0;
  if (!SPARSE) klo = max(0, qbase + t0 - A.W + 1);
  const int tile0 = klo / kApKeys;
  const int ntiles = kmax >= klo ? (kmax / kApKeys) - tile0 + 1 : 0;
  bool alive = true;

  if (SPARSE) {
    if (tid == 0) {
      mbar_init(&S.qidx_full, 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&S.kidx_full[i], 1);
        mbar_init(&S.kidx_empty[i], 1);
        mbar_init(&S.t_full[i], 1);
        mbar_init(&S.t_empty[i], 128);
      }
      mbar_fence_init();
    }
    if (warp == 0) tmem_alloc(&S.tmem_base, 2 * kApKeys);
    tc_fence_before();
  }
  __syncthreads();
  if (SPARSE) tc_fence_after();
  const uint32_t tmem = SPARSE ? S.tmem_base : 0u;

  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(A.k.data) + b * A.k.sb + kvh * A.k.sh;
  const __nv_bfloat16* vbase = static_cast<const __nv_bfloat16*>(A.v.data) + b * A.v.sb + kvh * A.v.sh;

  if (SPARSE && warp == kApMathWarps) {
    // ---------------- indexer: TMA + tcgen05.mma (one elected lane) ----------------
    if (lane == 0 && ntiles > 0) {
      mbar_expect_tx(&S.qidx_full, kApRows * kIdxDim * 2);
      tma_load_4d(S.qidx, &qmap, &S.qidx_full, 0, t0, h, b);
      int loads = 0, mma_issued = 0;
      for (int i = 0; i < ntiles && i < 2; ++i) {
        mbar_expect_tx(&S.kidx_full[i], kApIdxTileBytes);
        tma_load_4d(S.kidx[i], &kmap, &S.kidx_full[i], 0, (tile0 + i) * kApKeys, kvh, b);
        loads = i + 1;
      }
      mbar_wait(&S.qidx_full, 0, alive, A.err, A.budget);
      const uint64_t adesc = umma_desc_k_sw32(S.qidx);
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kApRows, kApKeys);
      for (int i = 0; i < ntiles; ++i) {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (!mbar_wait(&S.kidx_full[st], ph, alive, A.err, A.budget)) break;
        if (!mbar_wait(&S.t_empty[st], ph ^ 1, alive, A.err, A.budget)) break;
        tc_fence_after();
        umma_f16(tmem + st * kApKeys, adesc, umma_desc_k_sw32(S.kidx[st]), idesc, 0);
        umma_commit(&S.kidx_empty[st]);
        umma_commit(&S.t_full[st]);
        mma_issued = i + 1;
        if (i + 2 < ntiles) {  // refill this stage once the MMA has read it
          if (!mbar_wait(&S.kidx_empty[st], ph, alive, A.err, A.budget)) break;
          mbar_expect_tx(&S.kidx_full[st], kApIdxTileBytes);
          tma_load_4d(S.kidx[st], &kmap, &S.kidx_full[st], 0, (tile0 + i + 2) * kApKeys, kvh, b);
          loads = i + 3;
        }
      }
      // wind down: the last MMA and every TMA load issued land before TMEM is freed
      if (ntiles > 0) {
        mbar_drain(&S.qidx_full, 0, A.err);
        for (int i = loads > 2 ? loads - 2 : 0; i < loads; ++i)
          mbar_drain(&S.kidx_full[i & 1], (i >> 1) & 1, A.err);
        if (mma_issued > 0)
          mbar_drain(&S.t_full[(mma_issued - 1) & 1], ((mma_issued - 1) >> 1) & 1, A.err);
      }
    }
  } else {
    // ---------------- math warps 0-7 ----------------
    const uint32_t qs = smem_addr(S.q);
    // Q tile: 128 rows x 16 chunks
    for (int i = tid; i < kApRows * 16; i += kApMathWarps * 32) {
      const int r = i >> 4, ch = i & 15;
      const int t = t0 + r;
      const bool ok = t < A.T;
      const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(A.q.data) + b * A.q.sb + h * A.q.sh +
                                 (int64_t)(ok ? t : t0) * A.q.sn + ch * 8;
      cp16(qs + ap_swz(r, ch), src, ok);
    }
    auto load_kv = [&](int i, int st) {
      const int key0 = (tile0 + i) * kApKeys;
      const uint32_t ks = smem_addr(S.kv[st][0]), vs = smem_addr(S.kv[st][1]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = tid + u * kApMathWarps * 32;  // 0..1023
        const int r = idx >> 4, ch = idx & 15;
        const int key = key0 + r;
        const bool ok = key >= klo && key <= kmax;
        const int kk = ok ? key : klo;
        cp16(ks + ap_swz(r, ch), kbase + (int64_t)kk * A.k.sn + ch * 8, ok);
        cp16(vs + ap_swz(r, ch), vbase + (int64_t)kk * A.v.sn + ch * 8, ok);
      }
    };
    if (ntiles > 0) load_kv(0, 0);
    cp_commit();

    // per-row thresholds for the indexer epilogue (warps 0-3: row = tid)
    float tau = 0.f;
    int tpos = -1, prow = -1;
    if (SPARSE && warp < 4) {
      const int t = t0 + tid;
      prow = t < A.T ? qbase + t : -1;
      if (t < A.T && prow >= 0) {
        const int64_t qrow = (int64_t)bh * A.T + t;
        tau = __uint_as_float(A.tau_bits[qrow]);
        tpos = A.tiepos[qrow];
      }
    }
    // this warp's two rows per thread
    const int ra = warp * 16 + g, rb = ra + 8;
    const int pa = (t0 + ra < A.T) ? qbase + t0 + ra : -1;
    const int pb = (t0 + rb < A.T) ? qbase + t0 + rb : -1;

    cp_wait_all();
    named_sync(1, kApMathWarps * 32);
    uint32_t qf[8][4];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      ldsm4(qs + ap_swz(r, 2 * kk + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
    float* ot = &S.otot[warp][0][0];  // this thread's 64 sums at ot[e * 32 + lane]
#pragma unroll
    for (int e = 0; e < 64; ++e) ot[e * 32 + lane] = 0.f;
    float ca = 1.f, cb = 1.f;  // rescale factors applied to o since the last fold
    auto fold = [&]() {
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float& acc = ot[(nt * 4 + e) * 32 + lane];
          acc = __fmaf_rn(acc, e < 2 ? ca : cb, o[nt][e]);
          o[nt][e] = 0.f;
        }
      ca = cb = 1.f;
    };

    for (int i = 0; i < ntiles; ++i) {
      const int st = i & 1;
      const int key0 = (tile0 + i) * kApKeys;
      if (i + 1 < ntiles) load_kv(i + 1, st ^ 1);
      cp_commit();
      if (SPARSE && warp < 4) {
        // admission bitmap of row `tid` for this tile
        uint32_t w0 = 0u, w1 = 0u;
        if (mbar_wait(&S.t_full[st], (i >> 1) & 1, alive, A.err, A.budget)) {
          tc_fence_after();
          uint32_t v0[32], v1[32];
          const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + st * kApKeys;
          tmem_ld32(taddr, v0);
          tmem_ld32(taddr + 32, v1);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&S.t_empty[st]);
          const int nv = prow - key0 + 1;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float s0 = __fadd_rn(__fmul_rn(__uint_as_float(v0[j]), 0.25f), 0.0f);
            const float s1 = __fadd_rn(__fmul_rn(__uint_as_float(v1[j]), 0.25f), 0.0f);
            const bool a0 = j < nv && (s0 > tau || (s0 == tau && key0 + j <= tpos));
            const bool a1 = j + 32 < nv && (s1 > tau || (s1 == tau && key0 + 32 + j <= tpos));
            w0 |= (uint32_t)a0 << j;
            w1 |= (uint32_t)a1 << j;
          }
        }
        S.bits[st][tid][0] = w0;
        S.bits[st][tid][1] = w1;
      }
      // K/V tile i (committed one group earlier) and the bitmap are ready
      asm volatile("cp.async.wait_group 1;\n" ::);
      named_sync(1, kApMathWarps * 32);

      // admission of this thread's rows: bits over the tile's 64 keys
      uint64_t adm_a, adm_b;
      if (SPARSE) {
        adm_a = ((uint64_t)S.bits[st][ra][1] << 32) | S.bits[st][ra][0];
        adm_b = ((uint64_t)S.bits[st][rb][1] << 32) | S.bits[st][rb][0];
      } else {
        auto band = [&](int p) -> uint64_t {
          if (p < 0) return 0ull;
          const int lo = max(p - A.W + 1, 0) - key0, hi = p - key0;  // admitted tile columns [lo, hi]
          if (hi < 0 || lo > 63) return 0ull;
          const int l = max(lo, 0), r = min(hi, 63);
          const uint64_t upto = r >= 63 ? ~0ull : ((1ull << (r + 1)) - 1ull);
          return upto & ~((1ull << l) - 1ull);
        };
        adm_a = band(pa);
        adm_b = band(pb);
      }
      if (__any_sync(0xffffffffu, (adm_a | adm_b) != 0ull)) {
        const uint32_t ks = smem_addr(S.kv[st][0]), vs = smem_addr(S.kv[st][1]);
        float sacc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            const int key = 16 * np + (lane & 7) + ((lane >> 4) << 3);
            uint32_t b0, b1, b2, b3;
            ldsm4(ks + ap_swz(key, 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
            mma16816(sacc[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
            mma16816(sacc[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
          }
        }
        // masked, scaled logits and the tile maxima of rows a (g) and b (g + 8)
        float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const int j0 = 8 * nt + 2 * c;
          sacc[nt][0] = ((adm_a >> j0) & 1ull) ? sacc[nt][0] * A.scale_log2 : -INFINITY;
          sacc[nt][1] = ((adm_a >> (j0 + 1)) & 1ull) ? sacc[nt][1] * A.scale_log2 : -INFINITY;
          sacc[nt][2] = ((adm_b >> j0) & 1ull) ? sacc[nt][2] * A.scale_log2 : -INFINITY;
          sacc[nt][3] = ((adm_b >> (j0 + 1)) & 1ull) ? sacc[nt][3] * A.scale_log2 : -INFINITY;
          mxa = fmaxf(mxa, fmaxf(sacc[nt][0], sacc[nt][1]));
          mxb = fmaxf(mxb, fmaxf(sacc[nt][2], sacc[nt][3]));
        }
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        const float mna = fmaxf(ma, mxa), mnb = fmaxf(mb, mxb);
        const float ala = mna == -INFINITY ? 1.f : ex2a(ma - mna);
        const float alb = mnb == -INFINITY ? 1.f : ex2a(mb - mnb);
        ma = mna;
        mb = mnb;
        la *= ala;
        lb *= alb;
        ca *= ala;
        cb *= alb;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[nt][0] *= ala;
          o[nt][1] *= ala;
          o[nt][2] *= alb;
          o[nt][3] *= alb;
        }
        // P in A-fragment form (hi and lo bf16 parts), k-step j covers keys 16j..16j+15
        uint32_t ph[4][4], pl[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const float p0 = sacc[nt][0] == -INFINITY ? 0.f : ex2a(sacc[nt][0] - mna);
          const float p1 = sacc[nt][1] == -INFINITY ? 0.f : ex2a(sacc[nt][1] - mna);
          const float p2 = sacc[nt][2] == -INFINITY ? 0.f : ex2a(sacc[nt][2] - mnb);
          const float p3 = sacc[nt][3] == -INFINITY ? 0.f : ex2a(sacc[nt][3] - mnb);
          la += p0 + p1;
          lb += p2 + p3;
          const uint32_t hab = pack_bf16x2(p0, p1), hcd = pack_bf16x2(p2, p3);
          const uint32_t lab = pack_bf16x2(p0 - bf16_lo(hab), p1 - bf16_hi(hab));
          const uint32_t lcd = pack_bf16x2(p2 - bf16_lo(hcd), p3 - bf16_hi(hcd));
          const int j = nt >> 1, hi8 = nt & 1;
          ph[j][hi8 * 2 + 0] = hab;  // a0 / a2: row g
          ph[j][hi8 * 2 + 1] = hcd;  // a1 / a3: row g + 8
          pl[j][hi8 * 2 + 0] = lab;
          pl[j][hi8 * 2 + 1] = lcd;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
          for (int np = 0; np < 8; ++np) {
            const int key = 16 * j + (lane & 7) + ((lane >> 3) & 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm4t(vs + ap_swz(key, 2 * np + (lane >> 4)), b0, b1, b2, b3);
            mma16816(o[2 * np], ph[j][0], ph[j][1], ph[j][2], ph[j][3], b0, b1);
            mma16816(o[2 * np], pl[j][0], pl[j][1], pl[j][2], pl[j][3], b0, b1);
            mma16816(o[2 * np + 1], ph[j][0], ph[j][1], ph[j][2], ph[j][3], b2, b3);
            mma16816(o[2 * np + 1], pl[j][0], pl[j][1], pl[j][2], pl[j][3], b2, b3);
          }
        }
      }
      if ((i % kApFlush) == kApFlush - 1) fold();
      named_sync(1, kApMathWarps * 32);  // the stage is free for the prefetch two tiles ahead
    }
    cp_wait_all();
    fold();
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = ot[(nt * 4 + e) * 32 + lane];
    // ---- normalise and store ----
    la += __shfl_xor_sync(0xffffffffu, la, 1);
    la += __shfl_xor_sync(0xffffffffu, la, 2);
    lb += __shfl_xor_sync(0xffffffffu, lb, 1);
    lb += __shfl_xor_sync(0xffffffffu, lb, 2);
    const float ia = la > 0.f ? 1.f / la : 0.f, ib = lb > 0.f ? 1.f / lb : 0.f;
    const int ta = t0 + ra, tb = t0 + rb;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = 8 * nt + 2 * c;
      if (A.o_bf16) {
        __nv_bfloat16* oa = static_cast<__nv_bfloat16*>(A.o.data) + b * A.o.sb + h * A.o.sh;
        if (ta < A.T)
          *reinterpret_cast<uint32_t*>(oa + (int64_t)ta * A.o.sn + d) = pack_bf16x2(o[nt][0] * ia, o[nt][1] * ia);
        if (tb < A.T)
          *reinterpret_cast<uint32_t*>(oa + (int64_t)tb * A.o.sn + d) = pack_bf16x2(o[nt][2] * ib, o[nt][3] * ib);
      } else {
        float* of = static_cast<float*>(A.o.data) + b * A.o.sb + h * A.o.sh;
        if (ta < A.T) *reinterpret_cast<float2*>(of + (int64_t)ta * A.o.sn + d) = make_float2(o[nt][0] * ia, o[nt][1] * ia);
        if (tb < A.T) *reinterpret_cast<float2*>(of + (int64_t)tb * A.o.sn + d) = make_float2(o[nt][2] * ib, o[nt][3] * ib);
      }
    }
  }
  if (SPARSE) {
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_free(tmem, 2 * kApKeys);
  }
}

// ---- host ---------------------------------------------------------------------
cudaError_t launch_attn_prefill(const LaunchAttnPrefill& a, cudaStream_t stream) {
  if (a.B * a.Hq * a.T == 0) return cudaSuccess;
  ApArgs A;
  A.q = a.q;
  A.k = a.k;
  A.v = a.v;
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
  const size_t smem = sizeof(ApSmem) + 1024;
  const dim3 grid((unsigned)((a.T + kApRows - 1) / kApRows), (unsigned)(a.B * a.Hq));
  if (a.W > 0) {
    CUtensorMap dummy{};
    cudaFuncSetAttribute(attn_prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_prefill_kernel<false><<<grid, kApMathWarps * 32, smem, stream>>>(dummy, dummy, A);
  } else {
    CUtensorMap qmap, kmap;
    if (!make_idx_map(&qmap, a.q_idx, a.B, a.Hq, a.T, kApRows)) return cudaErrorInvalidValue;
    if (!make_idx_map(&kmap, a.k_idx, a.B, a.Hk, a.N, kApKeys)) return cudaErrorInvalidValue;
    cudaFuncSetAttribute(attn_prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_prefill_kernel<true><<<grid, kApMathWarps * 32 + 32, smem, stream>>>(qmap, kmap, A);
  }
  return cudaGetLastError();
}

}  // namespace rtp
