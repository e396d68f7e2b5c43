// internal.h -- plan layout and kernel launchers shared by the library's
// translation units.  Not part of the public ABI (that is include/deltakv.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "deltakv.h"

#include <nvtx3/nvToolsExt.h>

namespace dkv {

// An NVTX range over one C-ABI call, named after the call: a tool that
// records NVTX ranges (nsys, ncu --nvtx) files the call's kernels under that
// name.  With no tool attached a push or pop costs a test of a null pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kMaxK = 8;          // references per token
constexpr int kExtraCand = 4;     // extra candidates the distance kernel keeps
constexpr int kMaxCand = kMaxK + kExtraCand;
constexpr int kMaxG = 8;          // query heads per kv-head
constexpr int kMaxHidden = 256;
constexpr int kMaxSplit = 32;     // decode splits per (sequence, kv-head)
constexpr int kSparseSplits = 64;   // shares of one (sequence, kv-head)'s selection in sparse decode
constexpr int kCombineSlots = 256;// reference slots per combine block
constexpr int kNumSMs = 148;      // B200; used only to size launch grids

// Error word at the start of the workspace: [0] first error code, [1] detail.
constexpr size_t kErrBytes = 256;

// Kernels the library launches (profiling ids).
enum KernelId {
  KID_REFPACK = 0, KID_CAND_SIMT, KID_CAND_TC, KID_ENCODE_SIMT, KID_ENCODE_TC, KID_RECONSTRUCT, KID_DEC_REF,
  KID_DEC_PREP, KID_DEC_STREAM_SIMT, KID_DEC_STREAM_TC, KID_DEC_COMBINE, KID_DEC_FINAL,
  KID_APPEND_REFS, KID_APPEND_ROWS, KID_SPARSE_ATTEND, KID_SPARSE_MERGE, KID_SPARSE_SELECT, KID_COUNT
};
const char* kernel_name(int id);

struct Profiler;  // CUDA-event timing of each launch, off unless enabled

struct Plan {
  Profiler* prof = nullptr;
  deltakv_config cfg;
  int G;                 // q_heads / kv_heads
  int D;                 // 2 d_h
  int esize;             // bytes per element of K, V, refs and weights
  bool bf16;             // element type bf16 (BF16 or BF16_CODE4)
  bool code4;            // codes stored as 4-bit pairs with a bf16 scale per row
  int KC;                // candidates per token kept by the distance kernel
  int64_t n_ref_cap;     // reference rows per (b, head)
  int64_t n_code_cap;    // code rows per (b, head)
  // cache layout (bytes from base)
  size_t off_refk, off_refv, off_code, off_idx, off_cscale, cache_bytes;
  // compress workspace
  size_t ws_hnorm, ws_hsplit, ws_cand;
  // decode workspace
  int nslot_cap;         // decode partial slots per (b, head)
  int n_chunk_cap;       // combine blocks per (b, head)
  size_t ws_S, ws_Smax, ws_mref, ws_a, ws_cterm, ws_wtab, ws_part, ws_U, ws_ochunk, ws_sparse;
  size_t ws_cho;         // sequences of different lengths: int32 chunk offsets [batch * kv_heads + 1], then the
                         // checked lengths [batch]
  size_t ws_decode_end;  // error word + the dense decode's regions (S .. cho)
  // sparse decode on the tensor-core token loop: reference multiplicities
  // [BH][n_ref_cap], listed compressed rows [BH][n_code_cap + n_ref_cap],
  // row counts [BH]
  size_t ws_mult, ws_rowlist, ws_ncode;
  size_t ws_bytes;
};

// Brackets one kernel launch with CUDA events on its stream when the plan's
// profiler is on; does nothing otherwise.
struct ProfScope {
  ProfScope(const Plan& p, cudaStream_t st, int kid);
  ~ProfScope();
  Profiler* prof;
  cudaStream_t st;
  int kid;
  int slot;
};

__host__ __device__ inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Number of references and of compressed rows for a cache of T tokens.
__host__ __device__ inline int64_t n_ref_of(int64_t T, int s) { return T <= 0 ? 0 : ceil_div64(T, s); }
__host__ __device__ inline int64_t n_code_of(int64_t T, int s) { return T - n_ref_of(T, s); }

struct KVView {
  const void* K;
  const void* V;
  int64_t sb, sh, st;    // element strides: batch, head, token
};

// Where a decode reads the compressed cache.  Each plane (reference K and V
// rows, code rows, slot rows, 4-bit scales) is an array of pages; page p
// holds rp reference rows and cp code rows of one (sequence, kv-head).  The
// contiguous cache of a plan is the case of one page per (sequence,
// kv-head): rp = n_ref_cap, cp = n_code_cap, page of (bh, 0) = bh.  A page
// pool instead maps logical page l of (sequence, kv-head) bh to
// ptab[bh * max_pages + l].
struct CacheView {
  const char* base;
  size_t off_refk, off_refv, off_code, off_idx, off_cscale;
  int64_t rp, cp;        // reference rows and code rows per page
  int64_t n_pages;       // pages in each plane
  const int32_t* ptab;   // device [batch * kv_heads][max_pages], or null
  int max_pages;
  uint32_t* err;         // the workspace error word: a page index outside [0, n_pages) is reported there
#ifdef __CUDACC__
  __device__ int64_t page(int64_t bh, int64_t l) const {
    if (!ptab) return bh;
    const int64_t pg = ptab[bh * max_pages + l];
    if (pg < 0 || pg >= n_pages) {  // read page 0 instead (in bounds) and report
      if (atomicCAS(err, 0u, (uint32_t)DELTAKV_ERR_DEVICE_BOUNDS) == 0u) err[1] = (uint32_t)pg;
      return 0;
    }
    return pg;
  }
  // physical row of reference slot j / compressed row r of (sequence, kv-head)
  // bh; a pool page holds 128 reference rows (rp == 128) and fewer than 2^31
  // rows of any plane
  __device__ int64_t ref_row(int64_t bh, int64_t j) const {
    if (!ptab) return bh * rp + j;
    return page(bh, j >> 7) * 128 + (j & 127);
  }
  __device__ int64_t code_row(int64_t bh, int64_t r) const {
    if (!ptab) return bh * cp + r;
    const uint32_t l = (uint32_t)r / (uint32_t)cp;
    return page(bh, l) * cp + (r - (int64_t)l * cp);
  }
#endif
};

// Token counts of one decode: sequence b holds Tb[b] tokens (a device array)
// or, when Tb is null, T_all; T_max bounds them all.
struct SeqLens {
  const int32_t* Tb;
  int T_all, T_max;
  __device__ int T(int b) const { return Tb ? Tb[b] : T_all; }
};

// The contiguous cache of a plan as a CacheView.
CacheView contiguous_view(const Plan& p, const void* cache);

// Page pools: 128 blocks of s tokens per page.
constexpr int kPageRefs = 128;
struct PoolLayout {
  int64_t rp, cp;  // reference rows and code rows per page
  size_t off_refk, off_refv, off_code, off_idx, off_cscale, bytes;
};
PoolLayout pool_layout(const Plan& p, int64_t n_pages);
CacheView pool_view(const Plan& p, const PoolLayout& L, const void* pool, int64_t n_pages, const int32_t* ptab,
                    int max_pages, void* ws);
// Copy the contiguous cache of every (sequence, kv-head) (T tokens) into its pages.
cudaError_t launch_pages_from_cache(const Plan& p, int T, const void* cache, const PoolLayout& L, void* pool,
                                    int64_t n_pages, const int32_t* ptab, int max_pages, void* ws, cudaStream_t st);

// ---- compress ----
cudaError_t launch_refpack(const Plan& p, int T, const KVView& kv, void* cache, void* ws,
                           cudaStream_t st);
cudaError_t launch_candidates_simt(const Plan& p, int T, const KVView& kv, const void* cache,
                                   void* ws, cudaStream_t st);
bool candidates_tc_supported(const Plan& p);
cudaError_t launch_candidates_tc(const Plan& p, int T, const KVView& kv, const void* cache,
                                 void* ws, cudaStream_t st);
cudaError_t launch_decode_sparse(const Plan& p, int T, const void* q, int64_t qsb, int64_t qsh, const void* cache,
                                 const void* W3, const float* b3, const void* W4, const float* b4,
                                 const int32_t* tokens, int n_sel, float* out, int64_t osb, int64_t osh, void* ws,
                                 cudaStream_t st);
cudaError_t launch_append(const Plan& p, int T0, int T1, const KVView& kv, const void* W1, const float* b1,
                          const void* W2, const float* b2, void* cache, void* ws, cudaStream_t st);
cudaError_t launch_encode(const Plan& p, int T, const KVView& kv, const void* W1, const float* b1,
                          const void* W2, const float* b2, void* cache, void* ws,
                          cudaStream_t st);
bool encode_tc_supported(const Plan& p);
cudaError_t launch_encode_tc(const Plan& p, int T, const KVView& kv, const void* W1, const float* b1,
                             const void* W2, const float* b2, void* cache, void* ws,
                             cudaStream_t st);
// ---- reconstruct (tests / debugging) ----
cudaError_t launch_reconstruct(const Plan& p, int T, const void* cache, const void* W3,
                               const float* b3, const void* W4, const float* b4, float* Kout,
                               float* Vout, void* ws, cudaStream_t st);
// ---- decode ----
bool decode_tc_supported(const Plan& p);
int decode_tc_grid(const Plan& p, int64_t N);
// The token loop on the tensor cores; cho: chunk offsets per (sequence,
// kv-head) when the lengths differ (else null); the grid used goes to *grid.
// rowlist / ncode / rl_cap: gathered rows (sparse decode), else null.
cudaError_t launch_decode_tc(const Plan& p, const CacheView& cv, const SeqLens& sl, const int32_t* cho,
                             const void* W3, const float* b3, void* ws, cudaStream_t st, int* grid,
                             const int32_t* rowlist = nullptr, const int32_t* ncode = nullptr, int64_t rl_cap = 0);
// Sparse decode through the tensor-core token loop: the selected tokens'
// compressed rows gathered chunk by chunk, the selected references counted
// in the reference combine.  cudaErrorNotSupported when the plan or the
// selection size does not fit it (the CUDA-core sparse kernels then run).
cudaError_t launch_decode_sparse_tc(const Plan& p, int T, const void* q, int64_t qsb, int64_t qsh, const void* cache,
                                    const void* W3, const float* b3, const void* W4, const float* b4,
                                    const int32_t* tokens, int n_sel, float* out, int64_t osb, int64_t osh, void* ws,
                                    cudaStream_t st);
cudaError_t launch_decode(const Plan& p, const CacheView& cv, const SeqLens& sl, const void* q, int64_t qsb,
                          int64_t qsh, const void* W3, const float* b3, const void* W4, const float* b4, float* out,
                          int64_t osb, int64_t osh, void* ws, cudaStream_t st);

}  // namespace dkv

// The opaque plan handle of the C ABI.
struct deltakv_plan_s {
  dkv::Plan p;
  ~deltakv_plan_s();
};
