// C ABI of librtp.so: argument validation on the host, then dispatch to the
// kernels.  Nothing is launched and nothing is written when a check fails.
#include <math.h>
#include <stdint.h>

#include "launch.h"
#include "rtp.h"

namespace {

thread_local int32_t g_last_cuda_error = 0;

rtp_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return RTP_OK;
  g_last_cuda_error = (int32_t)e;
  return RTP_ERR_CUDA;
}

int64_t elt_size(int32_t dt) { return dt == RTP_F32 ? 4 : 2; }

bool dtype_ok(int32_t dt) { return dt == RTP_F32 || dt == RTP_BF16; }

// A 4-D tensor with the given last dimension, contiguous last dim, 16-byte
// aligned base and (for dims longer than 1) 16-byte aligned strides.  An empty
// tensor (a zero dimension) may have a NULL base: nothing is read or written.
rtp_status check4(const rtp_tensor* t, int64_t last) {
  if (!t) return RTP_ERR_INVALID_ARG;
  if (t->ndim != 4) return RTP_ERR_SHAPE;
  if (!dtype_ok(t->dtype)) return RTP_ERR_DTYPE;
  for (int i = 0; i < 4; ++i)
    if (t->shape[i] < 0 || t->stride[i] < 0) return RTP_ERR_SHAPE;
  const bool empty = t->shape[0] == 0 || t->shape[1] == 0 || t->shape[2] == 0;
  if (!t->data && !empty) return RTP_ERR_INVALID_ARG;
  if (t->shape[3] != last) return RTP_ERR_SHAPE;
  if (t->shape[0] > INT32_MAX || t->shape[1] > INT32_MAX || t->shape[2] > INT32_MAX) return RTP_ERR_SHAPE;
  if (t->stride[3] != 1) return RTP_ERR_ALIGNMENT;
  if (((uintptr_t)t->data) % 16) return RTP_ERR_ALIGNMENT;  // (NULL passes: an empty tensor)
  const int64_t es = elt_size(t->dtype);
  for (int i = 0; i < 3; ++i)
    if (t->shape[i] > 1 && (t->stride[i] * es) % 16) return RTP_ERR_ALIGNMENT;
  return RTP_OK;
}

// An f32 tensor of `nd` dims with a contiguous last dim (log-sum-exp rows).
rtp_status check_f32_rows(const rtp_tensor* t, int32_t nd) {
  if (!t || !t->data) return RTP_ERR_INVALID_ARG;
  if (t->ndim != nd) return RTP_ERR_SHAPE;
  if (t->dtype != RTP_F32) return RTP_ERR_DTYPE;
  for (int i = 0; i < nd; ++i)
    if (t->shape[i] < 0 || t->stride[i] < 0) return RTP_ERR_SHAPE;
  if (t->shape[nd - 1] > 1 && t->stride[nd - 1] != 1) return RTP_ERR_ALIGNMENT;
  if (((uintptr_t)t->data) % 4) return RTP_ERR_ALIGNMENT;
  return RTP_OK;
}

rtp::View4 view(const rtp_tensor* t) { return rtp::View4{t->data, t->stride[0], t->stride[1], t->stride[2]}; }
rtp::MutView4 mview(const rtp_tensor* t) {
  return rtp::MutView4{t->data, t->stride[0], t->stride[1], t->stride[2]};
}

bool same_bhn(const rtp_tensor* a, const rtp_tensor* b) {
  return a->shape[0] == b->shape[0] && a->shape[1] == b->shape[1] && a->shape[2] == b->shape[2];
}

rtp_status check_workspace(void* ws, size_t bytes, size_t need) {
  if (need == 0) return RTP_OK;
  if (!ws) return RTP_ERR_WORKSPACE;
  if (((uintptr_t)ws) % 256) return RTP_ERR_ALIGNMENT;
  if (bytes < need) return RTP_ERR_WORKSPACE;
  return RTP_OK;
}

// K and V of one layer: same shape/dtype, last dim 128.
rtp_status check_kv(const rtp_tensor* k, const rtp_tensor* v) {
  rtp_status s;
  if ((s = check4(k, 128)) != RTP_OK) return s;
  if ((s = check4(v, 128)) != RTP_OK) return s;
  if (!same_bhn(k, v)) return RTP_ERR_SHAPE;
  if (k->dtype != v->dtype) return RTP_ERR_DTYPE;
  return RTP_OK;
}

}  // namespace

namespace rtp {
void set_last_cuda_error(int32_t e) { g_last_cuda_error = e; }
}  // namespace rtp

extern "C" {

const char* rtp_status_string(rtp_status s) {
  switch (s) {
    case RTP_OK: return "ok";
    case RTP_ERR_INVALID_ARG: return "invalid argument";
    case RTP_ERR_SHAPE: return "bad shape";
    case RTP_ERR_DTYPE: return "unsupported dtype";
    case RTP_ERR_ALIGNMENT: return "misaligned pointer or stride";
    case RTP_ERR_WORKSPACE: return "workspace missing or too small";
    case RTP_ERR_CUDA: return "CUDA error";
    case RTP_ERR_UNSUPPORTED: return "unsupported configuration";
    default: return "unknown status";
  }
}

int32_t rtp_last_cuda_error(void) { return g_last_cuda_error; }

int32_t rtp_version(void) { return 100; }

// ---- a1 ------------------------------------------------------------------------
rtp_status rtp_index_project(const rtp_tensor* x, const rtp_tensor* P, const rtp_tensor* x_idx,
                             rtp_stream_t stream) {
  rtp_status s;
  if ((s = check4(x, 128)) != RTP_OK) return s;
  if ((s = check4(x_idx, 16)) != RTP_OK) return s;
  if (!P || !P->data) return RTP_ERR_INVALID_ARG;
  if (P->dtype != RTP_F32) return RTP_ERR_DTYPE;
  if (P->ndim != 3 || P->shape[1] != 16 || P->shape[2] != 128 || P->shape[0] < 1) return RTP_ERR_SHAPE;
  if (P->stride[2] != 1 || P->stride[1] != 128 || P->stride[0] != 16 * 128) return RTP_ERR_ALIGNMENT;
  if (((uintptr_t)P->data) % 16) return RTP_ERR_ALIGNMENT;
  if (!same_bhn(x, x_idx)) return RTP_ERR_SHAPE;
  if (x->shape[1] % P->shape[0]) return RTP_ERR_SHAPE;
  rtp::LaunchIndexProject a;
  a.x = view(x);
  a.P = static_cast<const float*>(P->data);
  a.out = mview(x_idx);
  a.B = x->shape[0];
  a.H = x->shape[1];
  a.HP = P->shape[0];
  a.N = x->shape[2];
  a.in_bf16 = x->dtype == RTP_BF16;
  a.out_bf16 = x_idx->dtype == RTP_BF16;
  return cuda_status(rtp::launch_index_project(a, (cudaStream_t)stream));
}

// ---- a2 + a3 ---------------------------------------------------------------------
size_t rtp_topp_select_workspace_size(int64_t B, int64_t Hq, int64_t T, int64_t Hk, int64_t N) {
  (void)Hk;
  if (B < 0 || Hq < 0 || N < 0) return 0;
  // decode: on chip up to 16 x 32768 keys, past that the scores each CTA cannot keep;
  // prefill: the cut lives on chip
  return T <= 1 ? rtp::topp_decode_workspace_bytes(B, Hq, N) : 0;
}

rtp_status rtp_topp_select(const rtp_tensor* q_idx, const rtp_tensor* k_idx, const int32_t* lens, float p,
                           const rtp_selection* out, void* workspace, size_t workspace_bytes,
                           rtp_stream_t stream) {
  rtp_status s;
  if ((s = check4(q_idx, 16)) != RTP_OK) return s;
  if ((s = check4(k_idx, 16)) != RTP_OK) return s;
  if (q_idx->dtype != k_idx->dtype) return RTP_ERR_DTYPE;
  if (q_idx->shape[0] != k_idx->shape[0]) return RTP_ERR_SHAPE;
  if (k_idx->shape[1] < 1 || q_idx->shape[1] % k_idx->shape[1]) return RTP_ERR_SHAPE;
  if (!(p > 0.f) || isnan(p)) return RTP_ERR_INVALID_ARG;
  if (!out || !out->tau_bits || !out->tiepos || !out->count) return RTP_ERR_INVALID_ARG;
  const int64_t N = k_idx->shape[2];
  if (out->mask && out->mask_words < (N + 31) / 32) return RTP_ERR_SHAPE;
  const int64_t T = q_idx->shape[2];
  if ((s = check_workspace(workspace, workspace_bytes,
                           rtp_topp_select_workspace_size(q_idx->shape[0], q_idx->shape[1], T,
                                                          k_idx->shape[1], N))) != RTP_OK)
    return s;
  if (T != 1) {
    if (q_idx->dtype != RTP_BF16) return RTP_ERR_DTYPE;  // the tensor-core score tiles take bf16
    if (q_idx->shape[1] / k_idx->shape[1] > rtp::kPrefillMaxGroup) return RTP_ERR_UNSUPPORTED;
    rtp::LaunchToppPrefill a;
    a.q_idx = view(q_idx);
    a.k_idx = view(k_idx);
    a.lens = lens;
    a.B = q_idx->shape[0];
    a.Hq = q_idx->shape[1];
    a.Hk = k_idx->shape[1];
    a.T = T;
    a.N = N;
    a.p = p;
    a.tau_bits = out->tau_bits;
    a.tiepos = out->tiepos;
    a.count = out->count;
    a.mask = out->mask;
    a.mask_words = out->mask_words;
    cudaError_t e = rtp::device_error_word(&a.err);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(rtp::launch_topp_prefill(a, (cudaStream_t)stream));
  }
  if (!rtp::topp_decode_supported(N)) return RTP_ERR_UNSUPPORTED;
  rtp::LaunchToppDecode a;
  a.q_idx = view(q_idx);
  a.k_idx = view(k_idx);
  a.lens = lens;
  a.B = q_idx->shape[0];
  a.Hq = q_idx->shape[1];
  a.Hk = k_idx->shape[1];
  a.N = N;
  a.p = p;
  a.topk = 0;
  a.bf16 = q_idx->dtype == RTP_BF16;
  a.tau_bits = out->tau_bits;
  a.tiepos = out->tiepos;
  a.count = out->count;
  a.mask = out->mask;
  a.mask_words = out->mask_words;
  a.spill = static_cast<float*>(workspace);
  return cuda_status(rtp::launch_topp_decode(a, (cudaStream_t)stream));
}

rtp_status rtp_topk_select(const rtp_tensor* q_idx, const rtp_tensor* k_idx, const int32_t* lens, int32_t k,
                           const rtp_selection* out, void* workspace, size_t workspace_bytes,
                           rtp_stream_t stream) {
  rtp_status s;
  if ((s = check4(q_idx, 16)) != RTP_OK) return s;
  if ((s = check4(k_idx, 16)) != RTP_OK) return s;
  if (q_idx->dtype != k_idx->dtype) return RTP_ERR_DTYPE;
  if (q_idx->shape[0] != k_idx->shape[0]) return RTP_ERR_SHAPE;
  if (k_idx->shape[1] < 1 || q_idx->shape[1] % k_idx->shape[1]) return RTP_ERR_SHAPE;
  if (k < 1) return RTP_ERR_INVALID_ARG;
  if (!out || !out->tau_bits || !out->tiepos || !out->count) return RTP_ERR_INVALID_ARG;
  const int64_t N = k_idx->shape[2];
  if (out->mask && out->mask_words < (N + 31) / 32) return RTP_ERR_SHAPE;
  if (q_idx->shape[2] != 1) return RTP_ERR_UNSUPPORTED;  // decode form only
  if ((s = check_workspace(workspace, workspace_bytes,
                           rtp_topp_select_workspace_size(q_idx->shape[0], q_idx->shape[1], 1, k_idx->shape[1],
                                                          N))) != RTP_OK)
    return s;
  if (!rtp::topp_decode_supported(N)) return RTP_ERR_UNSUPPORTED;
  rtp::LaunchToppDecode a;
  a.q_idx = view(q_idx);
  a.k_idx = view(k_idx);
  a.lens = lens;
  a.B = q_idx->shape[0];
  a.Hq = q_idx->shape[1];
  a.Hk = k_idx->shape[1];
  a.N = N;
  a.p = 1.f;
  a.topk = k;
  a.bf16 = q_idx->dtype == RTP_BF16;
  a.tau_bits = out->tau_bits;
  a.tiepos = out->tiepos;
  a.count = out->count;
  a.mask = out->mask;
  a.mask_words = out->mask_words;
  a.spill = static_cast<float*>(workspace);
  return cuda_status(rtp::launch_topp_decode(a, (cudaStream_t)stream));
}

// ---- cache maintenance ---------------------------------------------------------------
rtp_status rtp_kv_append(const rtp_tensor* k_new, const rtp_tensor* v_new, const int32_t* pos, int32_t R,
                         const rtp_tensor* P, const rtp_tensor* k_cache, const rtp_tensor* v_cache,
                         const rtp_tensor* k_idx, const rtp_tensor* k_ring, const rtp_tensor* v_ring,
                         int32_t* lens_out, int32_t* ring_lens, rtp_stream_t stream) {
  rtp_status s;
  if ((s = check_kv(k_new, v_new)) != RTP_OK) return s;
  if (!pos) return RTP_ERR_INVALID_ARG;
  if ((void*)lens_out == (const void*)pos || (void*)ring_lens == (const void*)pos) return RTP_ERR_INVALID_ARG;
  if (lens_out && lens_out == ring_lens) return RTP_ERR_INVALID_ARG;
  const int64_t B = k_new->shape[0], H = k_new->shape[1], T = k_new->shape[2];
  if (R < 0 || R > H) return RTP_ERR_INVALID_ARG;
  if (R == H && ring_lens) return RTP_ERR_INVALID_ARG;  // no local heads, no ring
  if (B > INT32_MAX || H > INT32_MAX || T > INT32_MAX) return RTP_ERR_SHAPE;
  int64_t N = 0, W = 1;
  if (R > 0) {
    if ((s = check_kv(k_cache, v_cache)) != RTP_OK) return s;
    if ((s = check4(k_idx, 16)) != RTP_OK) return s;
    if (!P || !P->data) return RTP_ERR_INVALID_ARG;
    if (P->dtype != RTP_F32) return RTP_ERR_DTYPE;
    if (P->ndim != 3 || P->shape[0] != R || P->shape[1] != 16 || P->shape[2] != 128) return RTP_ERR_SHAPE;
    if (P->stride[2] != 1 || P->stride[1] != 128 || P->stride[0] != 16 * 128) return RTP_ERR_ALIGNMENT;
    if (((uintptr_t)P->data) % 16) return RTP_ERR_ALIGNMENT;
    if (k_cache->shape[0] != B || k_cache->shape[1] != R) return RTP_ERR_SHAPE;
    if (k_idx->shape[0] != B || k_idx->shape[1] != R || k_idx->shape[2] != k_cache->shape[2]) return RTP_ERR_SHAPE;
    if (k_cache->dtype != k_new->dtype || k_idx->dtype != k_new->dtype) return RTP_ERR_DTYPE;
    N = k_cache->shape[2];
  }
  if (R < H) {
    if ((s = check_kv(k_ring, v_ring)) != RTP_OK) return s;
    if (k_ring->shape[0] != B || k_ring->shape[1] != H - R || k_ring->shape[2] < 1) return RTP_ERR_SHAPE;
    if (k_ring->dtype != k_new->dtype) return RTP_ERR_DTYPE;
    if (k_ring->shape[2] > INT32_MAX) return RTP_ERR_SHAPE;
    W = k_ring->shape[2];
  }
  rtp::KvAppendArgs a;
  a.k_new = view(k_new);
  a.v_new = view(v_new);
  a.pos = pos;
  a.P = R > 0 ? static_cast<const float*>(P->data) : nullptr;
  a.k_cache = R > 0 ? mview(k_cache) : rtp::MutView4{nullptr, 0, 0, 0};
  a.v_cache = R > 0 ? mview(v_cache) : rtp::MutView4{nullptr, 0, 0, 0};
  a.k_idx = R > 0 ? mview(k_idx) : rtp::MutView4{nullptr, 0, 0, 0};
  a.k_ring = R < H ? mview(k_ring) : rtp::MutView4{nullptr, 0, 0, 0};
  a.v_ring = R < H ? mview(v_ring) : rtp::MutView4{nullptr, 0, 0, 0};
  a.lens_out = lens_out;
  a.ring_lens = ring_lens;
  a.B = (int)B;
  a.H = (int)H;
  a.T = (int)T;
  a.R = R;
  a.N = (int)N;
  a.W = (int)W;
  return cuda_status(rtp::launch_kv_append(a, k_new->dtype == RTP_BF16, (cudaStream_t)stream));
}

// ---- a4 decode -------------------------------------------------------------------
size_t rtp_sparse_attn_decode_workspace_size(int64_t B, int64_t Hq, int64_t Hk, int64_t N) {
  return rtp::attn_decode_workspace_bytes(B, Hq, Hk, N, 0);
}

static rtp_status check_decode_common(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                      const rtp_tensor* o, float scale) {
  rtp_status s;
  if ((s = check4(q, 128)) != RTP_OK) return s;
  if ((s = check_kv(k, v)) != RTP_OK) return s;
  if ((s = check4(o, 128)) != RTP_OK) return s;
  if (q->dtype != k->dtype) return RTP_ERR_DTYPE;
  if (q->shape[0] != k->shape[0] || o->shape[0] != q->shape[0] || o->shape[1] != q->shape[1] ||
      o->shape[2] != q->shape[2])
    return RTP_ERR_SHAPE;
  if (k->shape[1] < 1 || q->shape[1] % k->shape[1]) return RTP_ERR_SHAPE;
  if (q->shape[1] / k->shape[1] > 8) return RTP_ERR_SHAPE;
  if (!isfinite(scale)) return RTP_ERR_INVALID_ARG;
  return RTP_OK;
}

}  // extern "C"

namespace rtp {
rtp_status check_sparse_attn_decode(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                    const int32_t* lens, const rtp_selection* sel, float scale,
                                    const rtp_tensor* o, LaunchAttnDecode* a, bool key_range) {
  rtp_status s;
  if ((s = check_decode_common(q, k, v, o, scale)) != RTP_OK) return s;
  if (q->shape[2] != 1) return RTP_ERR_SHAPE;
  if (!sel || !sel->mask) return RTP_ERR_INVALID_ARG;
  const int64_t N = k->shape[2];
  // a key range's rows past the selection's keys count as not selected (the kernel clamps)
  if (!key_range && sel->mask_words < (N + 31) / 32) return RTP_ERR_SHAPE;
  if (!attn_decode_supported(q->shape[0], k->shape[1], N, 0)) return RTP_ERR_UNSUPPORTED;
  a->q = view(q);
  a->k = view(k);
  a->v = view(v);
  a->lens = lens;
  a->mask = sel->mask;
  a->mask_words = sel->mask_words;
  a->B = q->shape[0];
  a->Hq = q->shape[1];
  a->Hk = k->shape[1];
  a->N = N;
  a->W = 0;
  a->scale = scale;
  a->bf16 = q->dtype == RTP_BF16;
  a->o = mview(o);
  a->o_bf16 = o->dtype == RTP_BF16;
  a->ws = nullptr;
  return RTP_OK;
}
}  // namespace rtp

extern "C" {

rtp_status rtp_sparse_attn_decode(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                  const int32_t* lens, const rtp_selection* sel, float scale,
                                  const rtp_tensor* o, void* workspace, size_t workspace_bytes,
                                  rtp_stream_t stream) {
  rtp::LaunchAttnDecode a;
  rtp_status s;
  if ((s = rtp::check_sparse_attn_decode(q, k, v, lens, sel, scale, o, &a, false)) != RTP_OK) return s;
  const size_t need = rtp_sparse_attn_decode_workspace_size(a.B, a.Hq, a.Hk, a.N);
  if ((s = check_workspace(workspace, workspace_bytes, need)) != RTP_OK) return s;
  a.ws = workspace;
  return cuda_status(rtp::launch_attn_decode(a, (cudaStream_t)stream));
}

rtp_status rtp_sparse_attn_decode_range(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                        const int32_t* lens, const rtp_selection* sel, int64_t key_lo,
                                        float scale, const rtp_tensor* o, const rtp_tensor* lse,
                                        void* workspace, size_t workspace_bytes, rtp_stream_t stream) {
  rtp::LaunchAttnDecode a;
  rtp_status s;
  if (key_lo < 0 || key_lo % 64) return RTP_ERR_INVALID_ARG;
  if ((s = check_f32_rows(lse, 2)) != RTP_OK) return s;
  if ((s = rtp::check_sparse_attn_decode(q, k, v, lens, sel, scale, o, &a, true)) != RTP_OK) return s;
  if (lse->shape[0] != a.B || lse->shape[1] != a.Hq) return RTP_ERR_SHAPE;
  if (key_lo + a.N > INT32_MAX) return RTP_ERR_SHAPE;
  const size_t need = rtp_sparse_attn_decode_workspace_size(a.B, a.Hq, a.Hk, a.N);
  if ((s = check_workspace(workspace, workspace_bytes, need)) != RTP_OK) return s;
  a.ws = workspace;
  a.key_lo = key_lo;
  a.lse = static_cast<float*>(lse->data);
  a.lse_sb = lse->stride[0];
  return cuda_status(rtp::launch_attn_decode(a, (cudaStream_t)stream));
}

rtp_status rtp_attn_combine(const rtp_tensor* o_parts, const rtp_tensor* lse_parts, const rtp_tensor* o,
                            rtp_stream_t stream) {
  rtp_status s;
  if ((s = check4(o_parts, 128)) != RTP_OK) return s;
  if ((s = check4(o, 128)) != RTP_OK) return s;
  if ((s = check_f32_rows(lse_parts, 3)) != RTP_OK) return s;
  if (o_parts->dtype != RTP_F32) return RTP_ERR_DTYPE;
  if (o_parts->shape[0] < 1 || o_parts->shape[0] > INT32_MAX || o_parts->shape[1] != o->shape[0] ||
      o_parts->shape[2] != o->shape[1] || o->shape[2] != 1)
    return RTP_ERR_SHAPE;
  for (int i = 0; i < 3; ++i)
    if (lse_parts->shape[i] != o_parts->shape[i]) return RTP_ERR_SHAPE;
  rtp::AttnCombineArgs a;
  a.o_parts = static_cast<const float*>(o_parts->data);
  a.ps = o_parts->stride[0];
  a.pb = o_parts->stride[1];
  a.ph = o_parts->stride[2];
  a.lse = static_cast<const float*>(lse_parts->data);
  a.ls = lse_parts->stride[0];
  a.lb = lse_parts->stride[1];
  a.S = (int)o_parts->shape[0];
  a.B = (int)o->shape[0];
  a.Hq = (int)o->shape[1];
  a.o = mview(o);
  a.o_bf16 = o->dtype == RTP_BF16;
  return cuda_status(rtp::launch_attn_combine(a, (cudaStream_t)stream));
}

// ---- a4 prefill --------------------------------------------------------------------
size_t rtp_sparse_attn_prefill_workspace_size(int64_t B, int64_t Hq, int64_t T, int64_t Hk, int64_t N) {
  (void)B; (void)Hq; (void)T; (void)Hk; (void)N;
  return 0;
}

rtp_status rtp_sparse_attn_prefill(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                   const rtp_tensor* q_idx, const rtp_tensor* k_idx, const int32_t* lens,
                                   const rtp_selection* sel, float scale, const rtp_tensor* o,
                                   void* workspace, size_t workspace_bytes, rtp_stream_t stream) {
  (void)workspace; (void)workspace_bytes;
  rtp_status s;
  if ((s = check_decode_common(q, k, v, o, scale)) != RTP_OK) return s;
  if ((s = check4(q_idx, 16)) != RTP_OK) return s;
  if ((s = check4(k_idx, 16)) != RTP_OK) return s;
  if (!sel || !sel->tau_bits || !sel->tiepos) return RTP_ERR_INVALID_ARG;
  if (q->dtype != RTP_BF16 || q_idx->dtype != RTP_BF16 || k_idx->dtype != RTP_BF16) return RTP_ERR_DTYPE;
  if (!same_bhn(q, q_idx) || !same_bhn(k, k_idx)) return RTP_ERR_SHAPE;
  if (q->shape[2] > k->shape[2]) return RTP_ERR_SHAPE;
  if (q->shape[1] / k->shape[1] > rtp::kPrefillMaxGroup) return RTP_ERR_UNSUPPORTED;
  rtp::LaunchAttnPrefill a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.q_idx = view(q_idx);
  a.k_idx = view(k_idx);
  a.lens = lens;
  a.tau_bits = sel->tau_bits;
  a.tiepos = sel->tiepos;
  a.B = q->shape[0];
  a.Hq = q->shape[1];
  a.Hk = k->shape[1];
  a.T = q->shape[2];
  a.N = k->shape[2];
  a.W = 0;
  a.scale = scale;
  a.o = mview(o);
  a.o_bf16 = o->dtype == RTP_BF16;
  cudaError_t e = rtp::device_error_word(&a.err);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(rtp::launch_attn_prefill(a, (cudaStream_t)stream));
}

// ---- a5 ----------------------------------------------------------------------------
size_t rtp_window_attn_workspace_size(int64_t B, int64_t Hq, int64_t T, int64_t Hk, int64_t N, int32_t W) {
  if (T <= 1) return rtp::attn_decode_workspace_bytes(B, Hq, Hk, N, W < 1 ? 1 : W);
  return 0;
}

rtp_status rtp_window_attn(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v, const int32_t* lens,
                           int32_t W, float scale, const rtp_tensor* o, void* workspace,
                           size_t workspace_bytes, rtp_stream_t stream) {
  rtp_status s;
  if ((s = check_decode_common(q, k, v, o, scale)) != RTP_OK) return s;
  if (W < 1) return RTP_ERR_INVALID_ARG;
  const int64_t T = q->shape[2];
  const int64_t N = k->shape[2];
  const size_t need = rtp_window_attn_workspace_size(q->shape[0], q->shape[1], T, k->shape[1], N, W);
  if ((s = check_workspace(workspace, workspace_bytes, need)) != RTP_OK) return s;
  if (T != 1) {
    if (q->dtype != RTP_BF16) return RTP_ERR_DTYPE;  // the prefill kernels take bf16
    if (T > N) return RTP_ERR_SHAPE;
    if (q->shape[1] / k->shape[1] > rtp::kPrefillMaxGroup) return RTP_ERR_UNSUPPORTED;
    rtp::LaunchAttnPrefill a;
    a.q = view(q);
    a.k = view(k);
    a.v = view(v);
    a.q_idx = rtp::View4{nullptr, 0, 0, 0};
    a.k_idx = rtp::View4{nullptr, 0, 0, 0};
    a.lens = lens;
    a.tau_bits = nullptr;
    a.tiepos = nullptr;
    a.B = q->shape[0];
    a.Hq = q->shape[1];
    a.Hk = k->shape[1];
    a.T = T;
    a.N = N;
    a.W = W;
    a.scale = scale;
    a.o = mview(o);
    a.o_bf16 = o->dtype == RTP_BF16;
    cudaError_t e = rtp::device_error_word(&a.err);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(rtp::launch_attn_prefill(a, (cudaStream_t)stream));
  }
  rtp::LaunchAttnDecode a;
  a.q = view(q);
  a.k = view(k);
  a.v = view(v);
  a.lens = lens;
  a.mask = nullptr;
  a.mask_words = 0;
  a.B = q->shape[0];
  a.Hq = q->shape[1];
  a.Hk = k->shape[1];
  a.N = N;
  a.W = W;
  a.scale = scale;
  a.bf16 = q->dtype == RTP_BF16;
  a.o = mview(o);
  a.o_bf16 = o->dtype == RTP_BF16;
  a.ws = workspace;
  return cuda_status(rtp::launch_attn_decode(a, (cudaStream_t)stream));
}

}  // extern "C"
