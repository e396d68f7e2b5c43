// internal.h -- plan layout and kernel launchers shared by the library's
// translation units.  Not part of the public ABI (that is include/deltakv.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "deltakv.h"

namespace dkv {

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
  KID_APPEND_REFS, KID_APPEND_ROWS, KID_SPARSE_ATTEND, KID_SPARSE_MERGE, KID_COUNT
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
  size_t ws_decode_end;  // error word + the dense decode's regions (S .. ochunk)
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

inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Number of references and of compressed rows for a cache of T tokens.
inline int64_t n_ref_of(int64_t T, int s) { return T <= 0 ? 0 : ceil_div64(T, s); }
inline int64_t n_code_of(int64_t T, int s) { return T - n_ref_of(T, s); }

struct KVView {
  const void* K;
  const void* V;
  int64_t sb, sh, st;    // element strides: batch, head, token
};

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
cudaError_t launch_decode_tc(const Plan& p, int T, const void* cache, const void* W3, const float* b3,
                             void* ws, cudaStream_t st);
cudaError_t launch_decode(const Plan& p, int T, const void* q, int64_t qsb, int64_t qsh,
                          const void* cache, const void* W3, const float* b3, const void* W4,
                          const float* b4, float* out, int64_t osb, int64_t osh, void* ws,
                          cudaStream_t st);

}  // namespace dkv

// The opaque plan handle of the C ABI.
struct deltakv_plan_s {
  dkv::Plan p;
  ~deltakv_plan_s();
};
