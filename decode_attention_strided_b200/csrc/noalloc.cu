// noalloc.cu -- decode attention for callers that cannot allocate device
// memory.
//
// Some callers can't call cudaMalloc (or any allocator) at the point where
// they run decode: code inside a fixed memory budget that was carved up at
// start-up, plugins hosted by an engine that owns every device allocation, or
// paths where an allocation could block or fail mid-step.  For them,
// deltakv_decode_attention_noalloc runs the same decode kernels as
// deltakv_decode_attention, but its scratch lives in the file-scope array
// below instead of a caller-supplied workspace.
//
// The array is kNoAllocScratchBytes (16 MiB) and, once this module is loaded
// on a GPU, that GPU holds it until the process exits.  Only the decode's own
// part of a plan's workspace has to fit, not the compress region: the error
// word, the reference-logit and slot-weight tables (8 G / s bytes per token
// of capacity and kv-head), the per-split partials (about 33 KB per kv-head
// at G = 4, hidden 256) and the combine partials.  One 128k-token sequence
// with 8 kv-heads and 4 query heads per kv-head needs about 3.6 MiB; batch 8
// at 128k needs about 25 MiB and is refused.  Plans whose decode part is
// larger than the array are rejected with DELTAKV_ERR_WORKSPACE.
// Every call shares the
// one array: calls that overlap on the GPU (on different streams, or from
// different host threads without ordering) race on it.
#include <mutex>

#include "internal.h"

namespace dkv {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with cudaGetSymbolAddress.
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }
}  // namespace

}  // namespace dkv

using namespace dkv;

extern "C" deltakv_status deltakv_decode_attention_noalloc(
    deltakv_plan_t plan, int32_t T, const void* q, const int64_t q_strides[2], const void* cache,
    const void* W3, const float* b3, const void* W4, const float* b4, float* out,
    const int64_t out_strides[2], deltakv_stream_t stream) {
  NvtxRange nvtx("deltakv_decode_attention_noalloc");
  if (!plan) return DELTAKV_ERR_INVALID_ARG;
  const Plan& p = plan->p;
  if (T < 1 || T > p.cfg.max_T) return DELTAKV_ERR_INVALID_ARG;
  if (!q || !q_strides || !cache || !W3 || !W4 || !out || !out_strides) return DELTAKV_ERR_INVALID_ARG;
  if (p.ws_decode_end > kNoAllocScratchBytes) return DELTAKV_ERR_WORKSPACE;
  if (q_strides[0] < 0 || q_strides[1] < 0 || out_strides[0] < 0 || out_strides[1] < 0)
    return DELTAKV_ERR_INVALID_ARG;
  if ((q_strides[0] * p.esize) % 16 || (q_strides[1] * p.esize) % 16 || (out_strides[0] * 4) % 16 ||
      (out_strides[1] * 4) % 16)
    return DELTAKV_ERR_ALIGNMENT;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(W3) || !aligned16(W4) || !aligned16(out) ||
      !aligned16(b3) || !aligned16(b4))
    return DELTAKV_ERR_ALIGNMENT;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DELTAKV_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  // The array keeps the previous call's contents; only the error word must
  // start at zero (every other region is written before it is read).
  if (cudaMemsetAsync(scratch, 0, kErrBytes, st) != cudaSuccess) return DELTAKV_ERR_CUDA;
  const SeqLens sl{nullptr, T, T};
  cudaError_t e = launch_decode(p, contiguous_view(p, cache), sl, q, q_strides[0], q_strides[1], W3, b3, W4, b4,
                                out, out_strides[0], out_strides[1], scratch, st);
  return e == cudaSuccess ? DELTAKV_OK : DELTAKV_ERR_CUDA;
}
