// api.cu -- the C ABI of include/deltakv.h: plan, validation, dispatch.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>

#include "internal.h"

using namespace dkv;

namespace dkv {
Profiler* profiler_create();
void profiler_destroy(Profiler* p);
int profiler_collect(Profiler* p, deltakv_kernel_time* out, int n_max);
}  // namespace dkv

deltakv_plan_s::~deltakv_plan_s() {
  if (p.prof) profiler_destroy(p.prof);
}

namespace {

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

deltakv_status validate_config(const deltakv_config* c) {
  if (!c) return DELTAKV_ERR_INVALID_ARG;
  if (c->layers < 1 || c->batch < 1 || c->kv_heads < 1 || c->q_heads < 1 || c->max_T < 1 ||
      c->stride_s < 1 || c->k < 1 || c->d_c < 1 || c->hidden < 1 || c->d_h < 1)
    return DELTAKV_ERR_INVALID_ARG;
  if (c->q_heads % c->kv_heads != 0) return DELTAKV_ERR_INVALID_ARG;
  if (c->dtype != DELTAKV_BF16 && c->dtype != DELTAKV_F32 && c->dtype != DELTAKV_BF16_CODE4)
    return DELTAKV_ERR_INVALID_ARG;
  if (c->act != DELTAKV_ACT_GELU_ERF && c->act != DELTAKV_ACT_GELU_TANH &&
      c->act != DELTAKV_ACT_NONE)
    return DELTAKV_ERR_INVALID_ARG;
  if (c->q_heads / c->kv_heads > kMaxG) return DELTAKV_ERR_UNSUPPORTED;
  if (c->d_h != 64 && c->d_h != 128) return DELTAKV_ERR_UNSUPPORTED;
  if (c->k > kMaxK) return DELTAKV_ERR_UNSUPPORTED;
  if (c->hidden > kMaxHidden || c->hidden % 32 != 0) return DELTAKV_ERR_UNSUPPORTED;
  bool identity = c->d_c == c->hidden && c->hidden == 2 * c->d_h;
  if (!(c->d_c == 16 || c->d_c == 32 || c->d_c == 64 || identity)) return DELTAKV_ERR_UNSUPPORTED;
  if (identity && c->d_c * c->hidden > 128 * 128) return DELTAKV_ERR_UNSUPPORTED;
  if (c->max_T > (1 << 26)) return DELTAKV_ERR_UNSUPPORTED;
  if (c->dtype == DELTAKV_BF16_CODE4 &&
      (identity || (c->hidden != 128 && c->hidden != 256) || c->act == DELTAKV_ACT_NONE))
    return DELTAKV_ERR_UNSUPPORTED;
  return DELTAKV_OK;
}

void build_plan(const deltakv_config& c, Plan& p) {
  p.cfg = c;
  p.G = c.q_heads / c.kv_heads;
  p.D = 2 * c.d_h;
  p.bf16 = c.dtype != DELTAKV_F32;
  p.code4 = c.dtype == DELTAKV_BF16_CODE4;
  p.esize = p.bf16 ? 2 : 4;
  p.KC = c.k + kExtraCand <= 8 ? 8 : 12;
  const int64_t BH = (int64_t)c.batch * c.kv_heads;
  const int64_t n_ref_max = n_ref_of(c.max_T, c.stride_s);
  const int64_t n_code_max = n_code_of(c.max_T, c.stride_s);
  p.n_ref_cap = std::max<int64_t>(128, ceil_div64(n_ref_max, 128) * 128);
  p.n_code_cap = std::max<int64_t>(128, ceil_div64(n_code_max, 128) * 128);
  // cache planes
  size_t off = 0;
  p.off_refk = off;
  off = align256(off + (size_t)(BH * p.n_ref_cap * c.d_h) * p.esize);
  p.off_refv = off;
  off = align256(off + (size_t)(BH * p.n_ref_cap * c.d_h) * p.esize);
  p.off_code = off;
  off = align256(off + (p.code4 ? (size_t)(BH * p.n_code_cap * c.d_c) / 2
                                : (size_t)(BH * p.n_code_cap * c.d_c) * p.esize));
  p.off_idx = off;
  off = align256(off + (size_t)(BH * p.n_code_cap * c.k) * 4);
  p.off_cscale = 0;
  if (p.code4) {
    p.off_cscale = off;
    off = align256(off + (size_t)(BH * p.n_code_cap) * 2);
  }
  p.cache_bytes = off;
  // workspace: error word, then the compress region and the decode region
  // side by side (a call uses one of them).
  size_t w = kErrBytes;
  p.ws_hnorm = w;
  w = align256(w + (size_t)(BH * p.n_ref_cap) * 4);
  p.ws_hsplit = w;  // 0.5 |x_j|^2 as three bf16 terms in a 16-element row (bf16 caches)
  w = align256(w + (size_t)(BH * p.n_ref_cap) * 32);
  p.ws_cand = w;  // candidate plane; the append path's per-slice lists reuse it (at least 4 KB a head)
  w = align256(w + std::max<size_t>((size_t)(BH * p.n_code_cap * p.KC) * 4, (size_t)BH * 4096));
  const size_t compress_end = w;
  w = kErrBytes;
  // partial slots of one (sequence, kv-head): the CTAs its chunks span; with
  // sequences of different lengths one sequence's kv-heads may hold nearly
  // all chunks, so the bound is taken per kv-head count
  p.nslot_cap = (int)std::max<int64_t>(kMaxSplit, ceil_div64(kNumSMs, c.kv_heads) + 2);
  const int64_t n_refblk_cap = ceil_div64(p.n_ref_cap, 64);
  p.n_chunk_cap = (int)ceil_div64(p.n_ref_cap, kCombineSlots);
  p.ws_S = w;
  w = align256(w + (size_t)(BH * p.n_ref_cap * p.G) * 4);
  p.ws_Smax = w;
  w = align256(w + (size_t)(BH * n_refblk_cap * p.G) * 4);
  p.ws_a = w;
  w = align256(w + (size_t)(BH * p.G * c.hidden) * 4);
  p.ws_cterm = w;
  w = align256(w + (size_t)(BH * p.G) * 4);
  p.ws_mref = w;
  w = align256(w + (size_t)(BH * p.G) * 4);
  p.ws_wtab = w;
  w = align256(w + (size_t)(BH * p.n_ref_cap * p.G) * 4);
  p.ws_part = w;
  w = align256(w + (size_t)(BH * p.nslot_cap * p.G * 2) * 4);
  p.ws_U = w;
  w = align256(w + (size_t)(BH * p.nslot_cap * p.G * c.hidden) * 4);
  p.ws_ochunk = w;
  w = align256(w + (size_t)(BH * p.n_chunk_cap * p.G * (c.d_h + 1)) * 4);
  p.ws_cho = w;  // then the checked lengths [batch]
  w = align256(w + (size_t)(BH + 1 + c.batch) * 4);
  p.ws_decode_end = w;
  p.ws_sparse = w;  // sparse decode: (m, l, output) of every share
  w = align256(w + (size_t)(BH * kSparseSplits * p.G * (c.d_h + 2)) * 4);
  p.ws_mult = w;
  w = align256(w + (size_t)(BH * p.n_ref_cap) * 4);
  p.ws_rowlist = w;  // room for every selected token of a (sequence, kv-head)
  w = align256(w + (size_t)(BH * (p.n_code_cap + p.n_ref_cap)) * 4);
  p.ws_ncode = w;
  w = align256(w + (size_t)BH * 4);
  p.ws_bytes = std::max(compress_end, w);
}

deltakv_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DELTAKV_OK : DELTAKV_ERR_CUDA; }

}  // namespace

extern "C" {

int32_t deltakv_version(void) { return 10000; }

const char* deltakv_status_string(deltakv_status s) {
  switch (s) {
    case DELTAKV_OK: return "ok";
    case DELTAKV_ERR_INVALID_ARG: return "invalid argument";
    case DELTAKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case DELTAKV_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case DELTAKV_ERR_WORKSPACE: return "workspace too small";
    case DELTAKV_ERR_CUDA: return "CUDA runtime error";
    case DELTAKV_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case DELTAKV_ERR_DEVICE_BOUNDS: return "device index or range check failed";
  }
  return "unknown status";
}

deltakv_status deltakv_plan(const deltakv_config* cfg, deltakv_plan_t* plan_out,
                            size_t* cache_bytes_per_layer, size_t* workspace_bytes) {
  if (!plan_out) return DELTAKV_ERR_INVALID_ARG;
  *plan_out = nullptr;
  deltakv_status st = validate_config(cfg);
  if (st != DELTAKV_OK) return st;
  deltakv_plan_s* pl = new (std::nothrow) deltakv_plan_s();
  if (!pl) return DELTAKV_ERR_INVALID_ARG;
  build_plan(*cfg, pl->p);
  if (cache_bytes_per_layer) *cache_bytes_per_layer = pl->p.cache_bytes;
  if (workspace_bytes) *workspace_bytes = pl->p.ws_bytes;
  *plan_out = pl;
  return DELTAKV_OK;
}

deltakv_status deltakv_plan_destroy(deltakv_plan_t plan) {
  delete plan;
  return DELTAKV_OK;
}

deltakv_status deltakv_get_cache_layout(deltakv_plan_t plan, deltakv_cache_layout* out) {
  if (!plan || !out) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  out->ref_k_offset = p.off_refk;
  out->ref_v_offset = p.off_refv;
  out->code_offset = p.off_code;
  out->idx_offset = p.off_idx;
  out->total_bytes = p.cache_bytes;
  out->n_ref_cap = p.n_ref_cap;
  out->n_code_cap = p.n_code_cap;
  out->code_scale_offset = p.off_cscale;
  return DELTAKV_OK;
}

deltakv_status deltakv_compress(deltakv_plan_t plan, int32_t T, const void* K, const void* V,
                                const int64_t kv_strides[3], const void* W1, const float* b1,
                                const void* W2, const float* b2, void* cache, void* workspace,
                                size_t workspace_bytes, deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_compress");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (T < 0 || T > p.cfg.max_T) return DELTAKV_ERR_INVALID_ARG;
  if (T == 0) return DELTAKV_OK;
  if (!K || !V || !kv_strides || !W1 || !W2 || !cache || !workspace) return DELTAKV_ERR_INVALID_ARG;
  if (workspace_bytes < p.ws_bytes) return DELTAKV_ERR_WORKSPACE;
  for (int i = 0; i < 3; ++i)
    if (kv_strides[i] < 0 || (kv_strides[i] * p.esize) % 16 != 0) return DELTAKV_ERR_ALIGNMENT;
  if (kv_strides[2] < p.cfg.d_h) return DELTAKV_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(W1) || !aligned16(W2) || !aligned16(cache) ||
      !aligned16(workspace) || !aligned16(b1) || !aligned16(b2))
    return DELTAKV_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  KVView kv{K, V, kv_strides[0], kv_strides[1], kv_strides[2]};
  cudaError_t e = launch_refpack(p, T, kv, cache, workspace, st);
  if (e == cudaSuccess) {
    // tensor-core search for bf16; CUDA cores for float32 caches and for K/V
    // layouts a TMA descriptor cannot describe (reported before any launch)
    cudaError_t t = cudaErrorNotSupported;
    if (candidates_tc_supported(p)) t = launch_candidates_tc(p, T, kv, cache, workspace, st);
    e = t == cudaErrorNotSupported ? launch_candidates_simt(p, T, kv, cache, workspace, st) : t;
  }
  if (e == cudaSuccess)
    e = encode_tc_supported(p) ? launch_encode_tc(p, T, kv, W1, b1, W2, b2, cache, workspace, st)
                               : launch_encode(p, T, kv, W1, b1, W2, b2, cache, workspace, st);
  return from_cuda(e);
}

deltakv_status deltakv_append(deltakv_plan_t plan, int32_t T0, int32_t T1, const void* K, const void* V,
                              const int64_t kv_strides[3], const void* W1, const float* b1, const void* W2,
                              const float* b2, void* cache, void* workspace, size_t workspace_bytes,
                              deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_append");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (T0 < 0 || T1 < T0 || T1 > p.cfg.max_T) return DELTAKV_ERR_INVALID_ARG;
  if (T1 == T0) return DELTAKV_OK;
  if (!K || !V || !kv_strides || !W1 || !W2 || !cache || !workspace) return DELTAKV_ERR_INVALID_ARG;
  if (workspace_bytes < p.ws_bytes) return DELTAKV_ERR_WORKSPACE;
  for (int i = 0; i < 3; ++i)
    if (kv_strides[i] < 0 || (kv_strides[i] * p.esize) % 16 != 0) return DELTAKV_ERR_ALIGNMENT;
  if (kv_strides[2] < p.cfg.d_h) return DELTAKV_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(W1) || !aligned16(W2) || !aligned16(cache) ||
      !aligned16(workspace) || !aligned16(b1) || !aligned16(b2))
    return DELTAKV_ERR_ALIGNMENT;
  KVView kv{K, V, kv_strides[0], kv_strides[1], kv_strides[2]};
  return from_cuda(launch_append(p, T0, T1, kv, W1, b1, W2, b2, cache, workspace, (cudaStream_t)stream));
}

deltakv_status deltakv_decode_attention(deltakv_plan_t plan, int32_t T, const void* q,
                                        const int64_t q_strides[2], const void* cache,
                                        const void* W3, const float* b3, const void* W4,
                                        const float* b4, float* out,
                                        const int64_t out_strides[2], void* workspace,
                                        size_t workspace_bytes, deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_decode_attention");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (T < 1 || T > p.cfg.max_T) return DELTAKV_ERR_INVALID_ARG;
  if (!q || !q_strides || !cache || !W3 || !W4 || !out || !out_strides || !workspace)
    return DELTAKV_ERR_INVALID_ARG;
  if (workspace_bytes < p.ws_bytes) return DELTAKV_ERR_WORKSPACE;
  if (q_strides[0] < 0 || q_strides[1] < 0 || out_strides[0] < 0 || out_strides[1] < 0)
    return DELTAKV_ERR_INVALID_ARG;
  if ((q_strides[0] * p.esize) % 16 || (q_strides[1] * p.esize) % 16 || (out_strides[0] * 4) % 16 ||
      (out_strides[1] * 4) % 16)
    return DELTAKV_ERR_ALIGNMENT;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(W3) || !aligned16(W4) || !aligned16(out) ||
      !aligned16(workspace) || !aligned16(b3) || !aligned16(b4))
    return DELTAKV_ERR_ALIGNMENT;
  const SeqLens sl{nullptr, T, T};
  return from_cuda(launch_decode(p, contiguous_view(p, cache), sl, q, q_strides[0], q_strides[1], W3, b3, W4, b4,
                                 out, out_strides[0], out_strides[1], workspace, (cudaStream_t)stream));
}

deltakv_status deltakv_page_pool_layout(deltakv_plan_t plan, int32_t n_pages, deltakv_page_layout* out) {
  if (!plan || !out || n_pages < 1) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  const PoolLayout L = pool_layout(p, n_pages);
  out->refs_per_page = (int32_t)L.rp;
  out->codes_per_page = (int32_t)L.cp;
  out->tokens_per_page = (int32_t)(L.rp * p.cfg.stride_s);
  out->n_pages = n_pages;
  out->ref_k_offset = L.off_refk;
  out->ref_v_offset = L.off_refv;
  out->code_offset = L.off_code;
  out->idx_offset = L.off_idx;
  out->code_scale_offset = L.off_cscale;
  out->pool_bytes = L.bytes;
  return DELTAKV_OK;
}

deltakv_status deltakv_pages_from_cache(deltakv_plan_t plan, int32_t T, const void* cache,
                                        const int32_t* page_table, int32_t max_pages, void* pool, int32_t n_pages,
                                        void* workspace, size_t workspace_bytes, deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_pages_from_cache");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (T < 1 || T > p.cfg.max_T || n_pages < 1 || !cache || !page_table || !pool || !workspace)
    return DELTAKV_ERR_INVALID_ARG;
  const int64_t tpp = (int64_t)kPageRefs * p.cfg.stride_s;
  if (max_pages < ceil_div64(T, tpp)) return DELTAKV_ERR_INVALID_ARG;
  if (workspace_bytes < p.ws_bytes) return DELTAKV_ERR_WORKSPACE;
  if (!aligned16(cache) || !aligned16(pool) || !aligned16(workspace) || ((uintptr_t)page_table & 3))
    return DELTAKV_ERR_ALIGNMENT;
  const PoolLayout L = pool_layout(p, n_pages);
  return from_cuda(launch_pages_from_cache(p, T, cache, L, pool, n_pages, page_table, max_pages, workspace,
                                           (cudaStream_t)stream));
}

deltakv_status deltakv_decode_attention_paged(deltakv_plan_t plan, const int32_t* seq_lens, int32_t max_len,
                                              const void* q, const int64_t q_strides[2], const void* pool,
                                              int32_t n_pages, const int32_t* page_table, int32_t max_pages,
                                              const void* W3, const float* b3, const void* W4, const float* b4,
                                              float* out, const int64_t out_strides[2], void* workspace,
                                              size_t workspace_bytes, deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_decode_attention_paged");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (max_len < 1 || max_len > p.cfg.max_T || n_pages < 1) return DELTAKV_ERR_INVALID_ARG;
  if (!seq_lens || !q || !q_strides || !pool || !page_table || !W3 || !W4 || !out || !out_strides || !workspace)
    return DELTAKV_ERR_INVALID_ARG;
  const int64_t tpp = (int64_t)kPageRefs * p.cfg.stride_s;
  if (max_pages < ceil_div64(max_len, tpp)) return DELTAKV_ERR_INVALID_ARG;
  if (workspace_bytes < p.ws_bytes) return DELTAKV_ERR_WORKSPACE;
  if (q_strides[0] < 0 || q_strides[1] < 0 || out_strides[0] < 0 || out_strides[1] < 0)
    return DELTAKV_ERR_INVALID_ARG;
  if ((q_strides[0] * p.esize) % 16 || (q_strides[1] * p.esize) % 16 || (out_strides[0] * 4) % 16 ||
      (out_strides[1] * 4) % 16)
    return DELTAKV_ERR_ALIGNMENT;
  if (!aligned16(q) || !aligned16(pool) || !aligned16(W3) || !aligned16(W4) || !aligned16(out) ||
      !aligned16(workspace) || !aligned16(b3) || !aligned16(b4) || ((uintptr_t)seq_lens & 3) ||
      ((uintptr_t)page_table & 3))
    return DELTAKV_ERR_ALIGNMENT;
  const PoolLayout L = pool_layout(p, n_pages);
  const CacheView cv = pool_view(p, L, pool, n_pages, page_table, max_pages, workspace);
  const SeqLens sl{seq_lens, max_len, max_len};
  return from_cuda(launch_decode(p, cv, sl, q, q_strides[0], q_strides[1], W3, b3, W4, b4, out, out_strides[0],
                                 out_strides[1], workspace, (cudaStream_t)stream));
}

deltakv_status deltakv_decode_attention_sparse(deltakv_plan_t plan, int32_t T, const void* q,
                                               const int64_t q_strides[2], const void* cache, const void* W3,
                                               const float* b3, const void* W4, const float* b4,
                                               const int32_t* tokens, int32_t n_sel, float* out,
                                               const int64_t out_strides[2], void* workspace,
                                               size_t workspace_bytes, deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_decode_attention_sparse");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (T < 1 || T > p.cfg.max_T || n_sel < 1) return DELTAKV_ERR_INVALID_ARG;
  if (!q || !q_strides || !cache || !W3 || !W4 || !tokens || !out || !out_strides || !workspace)
    return DELTAKV_ERR_INVALID_ARG;
  if (workspace_bytes < p.ws_bytes) return DELTAKV_ERR_WORKSPACE;
  if (q_strides[0] < 0 || q_strides[1] < 0 || out_strides[0] < 0 || out_strides[1] < 0)
    return DELTAKV_ERR_INVALID_ARG;
  if ((q_strides[0] * p.esize) % 16 || (q_strides[1] * p.esize) % 16 || (out_strides[0] * 4) % 16 ||
      (out_strides[1] * 4) % 16)
    return DELTAKV_ERR_ALIGNMENT;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(W3) || !aligned16(W4) || !aligned16(out) ||
      !aligned16(workspace) || !aligned16(b3) || !aligned16(b4) || !aligned16(tokens))
    return DELTAKV_ERR_ALIGNMENT;
  // the tensor-core token loop over the gathered rows where the plan and the
  // selection fit it, else the CUDA-core sparse kernels
  cudaError_t e = launch_decode_sparse_tc(p, T, q, q_strides[0], q_strides[1], cache, W3, b3, W4, b4, tokens, n_sel,
                                          out, out_strides[0], out_strides[1], workspace, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported)
    e = launch_decode_sparse(p, T, q, q_strides[0], q_strides[1], cache, W3, b3, W4, b4, tokens, n_sel, out,
                             out_strides[0], out_strides[1], workspace, (cudaStream_t)stream);
  return from_cuda(e);
}

deltakv_status deltakv_reconstruct(deltakv_plan_t plan, int32_t T, const void* cache,
                                   const void* W3, const float* b3, const void* W4,
                                   const float* b4, float* K_out, float* V_out, void* workspace,
                                   size_t workspace_bytes, deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_reconstruct");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (T < 0 || T > p.cfg.max_T) return DELTAKV_ERR_INVALID_ARG;
  if (T == 0) return DELTAKV_OK;
  if (!cache || !W3 || !W4 || !K_out || !V_out || !workspace) return DELTAKV_ERR_INVALID_ARG;
  if (workspace_bytes < p.ws_bytes) return DELTAKV_ERR_WORKSPACE;
  if (!aligned16(cache) || !aligned16(W3) || !aligned16(W4) || !aligned16(K_out) ||
      !aligned16(V_out) || !aligned16(workspace) || !aligned16(b3) || !aligned16(b4))
    return DELTAKV_ERR_ALIGNMENT;
  return from_cuda(launch_reconstruct(p, T, cache, W3, b3, W4, b4, K_out, V_out, workspace,
                                      (cudaStream_t)stream));
}

deltakv_status deltakv_set_profiling(deltakv_plan_t plan, int32_t enable) {
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  if (enable && !plan->p.prof) plan->p.prof = profiler_create();
  if (!enable && plan->p.prof) {
    profiler_destroy(plan->p.prof);
    plan->p.prof = nullptr;
  }
  return DELTAKV_OK;
}

deltakv_status deltakv_profile_collect(deltakv_plan_t plan, deltakv_kernel_time* out,
                                       int32_t n_max, int32_t* n_out) {
  if (!plan || !out || n_max < 0 || !n_out) return DELTAKV_ERR_INVALID_ARG;
  *n_out = 0;
  if (!plan->p.prof) return DELTAKV_OK;
  int n = profiler_collect(plan->p.prof, out, n_max);
  if (n < 0) return DELTAKV_ERR_CUDA;
  *n_out = n;
  return DELTAKV_OK;
}

deltakv_status deltakv_device_status(deltakv_plan_t plan, void* workspace,
                                     deltakv_stream_t stream) {
  if (!plan || !workspace) return DELTAKV_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t word[2] = {0, 0};
  if (cudaStreamSynchronize(st) != cudaSuccess) return DELTAKV_ERR_CUDA;
  if (cudaMemcpy(word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DELTAKV_ERR_CUDA;
  if (word[0] != 0) {
    if (cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return DELTAKV_ERR_CUDA;
    if (word[0] == DELTAKV_ERR_DEVICE_TIMEOUT || word[0] == DELTAKV_ERR_DEVICE_BOUNDS)
      return (deltakv_status)word[0];
    return DELTAKV_ERR_DEVICE_BOUNDS;
  }
  return DELTAKV_OK;
}

}  // extern "C"
