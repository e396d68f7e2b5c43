// decode.cu -- split-K decode attention over the compressed cache, with every
// non-reference token rebuilt on demand ("Ricostruzione" of the DeltaKV
// summary; on-demand reconstruction inside attention, section 4).
//
// For query head g of kv-head h, with c = log2(e) / sqrt(d_h):
//   reference slot j :  l_j = c q.K_ref_j                       = S_j
//   other token t    :  l_t = c q.(KV_R + W4_K u_t + b4_K)
//                           = (1/k_eff) sum_i S_{idx_ti} + a.u_t + c q.b4_K
//   with u_t = act(W3 code_t + b3) and a = c W4_K^T q.
// The output  sum_t 2^(l_t - M) V_hat_t / sum_t 2^(l_t - M)  splits as
//   sum_j w_j V_ref_j + W4_V (sum_t p_t u_t) + b4_V sum_t p_t,
//   w_j = 2^(S_j - M) + sum_{t : j in idx_t} p_t / k_eff_t,
// so K_hat and V_hat are never formed: K_R enters through the gathered S
// values, V_R through the per-slot weight table w, and W4 through one GEMV
// per kv-head before (a) and after (W4_V U) the token loop.  This is the same
// arithmetic as rebuilding every token, reassociated.
//
// Kernels, in stream order:
//   decode_ref      S_j for every slot (reads K_ref), per-block maxima
//   decode_prep     a = c W4_K^T q and c q.b4_K per query head
//   decode_stream   per split of the compressed rows: u_t, logits, online
//                   softmax partials (m, l, U = sum p u) and the split's w table
//   decode_combine  per 256-slot chunk: sum_j w_j V_ref_j (reads V_ref)
//   decode_final    merge everything, add W4_V U and b4_V, normalise
#include <cfloat>

#include "common.cuh"
#include "sm100.cuh"

namespace dkv {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kRefBlockSlots = 64;

// Eight consecutive elements as floats (16-byte aligned for bf16, 32 for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
// the same from shared memory (16-byte aligned)
__device__ __forceinline__ void load8s(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 r = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8s(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ------------------------------------------------------------ decode_ref
// One thread per reference row (64 rows per CTA): the row's d_h elements
// with 16-byte loads, every head's dot product at once against the scaled
// queries in shared memory (stored element-major, so one 16-byte shared load
// gives four heads), S and the cleared slot weights written as one vector
// per row.  Each thread's row comes into shared memory by a bulk copy of
// its own, issued before the queries are staged; rows sit 16 bytes apart
// beyond their length, so the threads' 16-byte reads at one offset fall on
// different banks.
template <typename T>
__global__ void __launch_bounds__(kRefBlockSlots)
    decode_ref_kernel(SeqLens sl, int s_, int64_t n_ref_cap, int d_h, int H, int G, float c,
                      const T* __restrict__ q, int64_t qsb, int64_t qsh, CacheView cv,
                      float* __restrict__ S, float* __restrict__ Smax, int n_refblk_cap,
                      float* __restrict__ wtab, uint32_t* __restrict__ err) {
  extern __shared__ __align__(16) unsigned char krow[];  // kRefBlockSlots rows of d_h T + 16 bytes
  __shared__ __align__(16) float qt[128][kMaxG];  // [element][head]
  __shared__ float wmax[kRefBlockSlots / 32][kMaxG];
  __shared__ __align__(8) uint64_t kbar;
  const int b = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t bh = (int64_t)b * H + h;
  const int64_t n_ref = n_ref_of(sl.T(b), s_);
  const T* refk = reinterpret_cast<const T*>(cv.base + cv.off_refk);
  const int64_t j = (int64_t)blockIdx.x * kRefBlockSlots + tid;
  const uint32_t row_bytes = (uint32_t)(d_h * sizeof(T)), row_pitch = row_bytes + 16;
  if (tid == 0) {
    const int64_t jb = (int64_t)blockIdx.x * kRefBlockSlots;
    const int64_t nv = n_ref - jb < 0 ? 0 : (n_ref - jb < kRefBlockSlots ? n_ref - jb : kRefBlockSlots);
    sm100::mbar_init(&kbar, 1);
    sm100::fence_mbar_init();
    sm100::mbar_arrive_expect_tx(&kbar, (uint32_t)nv * row_bytes);
  }
  __syncthreads();
  if (j < n_ref) sm100::bulk_load(krow + tid * row_pitch, refk + cv.ref_row(bh, j) * d_h, row_bytes, &kbar);
  for (int i = tid; i < kMaxG * d_h; i += blockDim.x) {
    const int g = i % kMaxG, e = i / kMaxG;
    qt[e][g] = g < G ? c * to_f(q[b * qsb + (int64_t)(h * G + g) * qsh + e]) : 0.f;
  }
  // the rows have landed (bounded wait; every thread leaves together if it
  // ran out)
  if (!__syncthreads_and(sm100::mbar_wait_drain(&kbar, 0))) {
    if (tid == 0) latch_error(err, DELTAKV_ERR_DEVICE_TIMEOUT, 32);
    return;
  }
  float acc[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) acc[g] = 0.f;
  if (j < n_ref) {
    const T* kr = reinterpret_cast<const T*>(krow + tid * row_pitch);
#pragma unroll 4
    for (int e0 = 0; e0 < d_h; e0 += 8) {
      float v[8];
      load8s(kr + e0, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 qa = *reinterpret_cast<const float4*>(&qt[e0 + i][0]);
        acc[0] = fmaf(qa.x, v[i], acc[0]);
        acc[1] = fmaf(qa.y, v[i], acc[1]);
        acc[2] = fmaf(qa.z, v[i], acc[2]);
        acc[3] = fmaf(qa.w, v[i], acc[3]);
        if (G > 4) {
          const float4 qb = *reinterpret_cast<const float4*>(&qt[e0 + i][4]);
          acc[4] = fmaf(qb.x, v[i], acc[4]);
          acc[5] = fmaf(qb.y, v[i], acc[5]);
          acc[6] = fmaf(qb.z, v[i], acc[6]);
          acc[7] = fmaf(qb.w, v[i], acc[7]);
        }
      }
    }
    float* so = S + (bh * n_ref_cap + j) * G;
    float* wo = wtab + (bh * n_ref_cap + j) * G;
    if (G == 4) {
      *reinterpret_cast<float4*>(so) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(wo) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
#pragma unroll
      for (int g = 0; g < kMaxG; ++g)
        if (g < G) {
          so[g] = acc[g];
          wo[g] = 0.f;
        }
    }
  }
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    float m = j < n_ref ? acc[g] : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[warp][g] = m;
  }
  __syncthreads();
  if (tid < G) {
    float m = -INFINITY;
    for (int w = 0; w < kRefBlockSlots / 32; ++w) m = fmaxf(m, wmax[w][tid]);
    Smax[(bh * n_refblk_cap + blockIdx.x) * G + tid] = m;
  }
}

// ----------------------------------------------------------- decode_prep
template <typename T>
__global__ void __launch_bounds__(256)
    decode_prep_kernel(int d_h, int H, int G, int hidden, float c, const T* __restrict__ q,
                       int64_t qsb, int64_t qsh, const T* __restrict__ W4,
                       const float* __restrict__ b4, float* __restrict__ a,
                       float* __restrict__ cterm, const float* __restrict__ Smax, int n_refblk,
                       int n_refblk_cap, float* __restrict__ mref) {
  __shared__ float qs[kMaxG][128];
  __shared__ float wm[8][kMaxG];
  const int b = blockIdx.z, h = blockIdx.y;
  const int64_t bh = (int64_t)b * H + h;
  {
    // m_ref = max_j S_j of this (sequence, kv-head), from the per-block maxima
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float m[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) m[g] = -INFINITY;
    for (int r = threadIdx.x; r < n_refblk; r += blockDim.x)
#pragma unroll
      for (int g = 0; g < kMaxG; ++g)
        if (g < G) m[g] = fmaxf(m[g], Smax[(bh * n_refblk_cap + r) * G + g]);
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      const float wmax = warp_max(m[g]);
      if (lane == 0 && g < G) wm[warp][g] = wmax;
    }
    __syncthreads();
    if (threadIdx.x < G) {
      float r = wm[0][threadIdx.x];
      for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, wm[w][threadIdx.x]);
      mref[bh * G + threadIdx.x] = r;
    }
  }
  for (int i = threadIdx.x; i < G * d_h; i += blockDim.x) {
    int g = i / d_h, e = i - g * d_h;
    qs[g][e] = c * to_f(q[b * qsb + (int64_t)(h * G + g) * qsh + e]);
  }
  __syncthreads();
  for (int n = threadIdx.x; n < hidden; n += blockDim.x) {
    float acc[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) acc[g] = 0.f;
    for (int e = 0; e < d_h; ++e) {
      float w = to_f(W4[(int64_t)e * hidden + n]);
#pragma unroll
      for (int g = 0; g < kMaxG; ++g)
        if (g < G) acc[g] = fmaf(w, qs[g][e], acc[g]);
    }
    for (int g = 0; g < G; ++g) a[(bh * G + g) * hidden + n] = acc[g];
  }
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int g = 0; g < G; ++g) {
      float acc = 0.f;
      if (b4)
        for (int e = lane; e < d_h; e += 32) acc = fmaf(b4[e], qs[g][e], acc);
      acc = warp_sum(acc);
      if (lane == 0) cterm[bh * G + g] = acc;
    }
  }
}

// --------------------------------------------------------- decode_stream
// One block per (split, kv-head, sequence), 8 warps, one compressed token per
// warp at a time.  The split's slot-weight table lives in shared memory when
// it fits (`wt_in_smem`), else in the split's own region of the workspace.
// Weights added to it are relative to m_ref = max_j S_j, fixed for the call;
// U and l use a per-warp running maximum.
template <typename T>
__global__ void __launch_bounds__(256)
    decode_stream_kernel(SeqLens sl, int s, int d_h, int H, int G, int k, int d_c, int hidden,
                         int act, int ns, int64_t n_ref_cap, int n_refblk, int n_refblk_cap, CacheView cv,
                         const T* __restrict__ W3,
                         const float* __restrict__ b3, const float* __restrict__ a,
                         const float* __restrict__ cterm, const float* __restrict__ S,
                         const float* __restrict__ Smax, float* __restrict__ wtab_g,
                         float* __restrict__ part, float* __restrict__ Upart, int wt_in_smem,
                         int nslot_cap, uint32_t* __restrict__ err) {
  extern __shared__ float smem[];
  float* W3s = smem;                         // [d_c][hidden]
  float* As = W3s + d_c * hidden;            // [G][hidden]
  float* Ured = As + G * hidden;             // [G][hidden]
  float* misc = Ured + G * hidden;           // m_ref[G], m_cta[G], l[G], cterm[G]
  float* cw = misc + 4 * kMaxG;              // [8 warps][d_c] code rows
  float* wt = cw + 8 * d_c;                  // [n_ref][G] when in smem
  const int b = blockIdx.z, h = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int64_t bh = (int64_t)b * H + h;
  const int64_t n_ref = n_ref_of(sl.T(b), s);
  const int64_t n_code = sl.T(b) - n_ref;
  const int64_t c0 = n_code * split / ns, c1 = n_code * (split + 1) / ns;
  const T* code = reinterpret_cast<const T*>(cv.base + cv.off_code);
  // the scale plane exists with 4-bit codes only (its offset is 0 otherwise)
  const __nv_bfloat16* cscale =
      cv.off_cscale ? reinterpret_cast<const __nv_bfloat16*>(cv.base + cv.off_cscale) : nullptr;
  const int32_t* idx = reinterpret_cast<const int32_t*>(cv.base + cv.off_idx);
  // the kv-head's slot-weight table (zeroed by decode_ref), relative to
  // m_ref; with room in shared memory the block sums into a private copy first
  float* wtab = wt_in_smem ? wt : wtab_g + bh * n_ref_cap * G;

  for (int i = tid; i < d_c * hidden; i += blockDim.x) {
    int n = i / d_c, e = i - n * d_c;
    W3s[e * hidden + n] = to_f(W3[i]);
  }
  for (int i = tid; i < G * hidden; i += blockDim.x) {
    As[i] = a[bh * G * hidden + i];
    Ured[i] = 0.f;
  }
  if (wt_in_smem)
    for (int64_t i = tid; i < n_ref * G; i += blockDim.x) wtab[i] = 0.f;
  if (tid < G) {
    float m = -INFINITY;
    for (int r = 0; r < n_refblk; ++r) m = fmaxf(m, Smax[(bh * n_refblk_cap + r) * G + tid]);
    misc[tid] = m;                        // m_ref
    misc[kMaxG + tid] = -INFINITY;        // block max (after the loop)
    misc[2 * kMaxG + tid] = 0.f;          // block l
    misc[3 * kMaxG + tid] = cterm[bh * G + tid];
  }
  __syncthreads();
  if (!wt_in_smem) __threadfence_block();

  const int per_lane = hidden / 32;  // hidden is a multiple of 32 here
  float mw[kMaxG], lw[kMaxG], Uw[kMaxG][8];
  float mref[kMaxG], ct[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    mw[g] = -INFINITY;
    lw[g] = 0.f;
    mref[g] = g < G ? misc[g] : 0.f;
    ct[g] = g < G ? misc[3 * kMaxG + g] : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) Uw[g][i] = 0.f;
  }
  const float* Sb = S + bh * n_ref_cap * G;

  for (int64_t row = c0 + warp; row < c1; row += 8) {
    // the code row, staged in this warp's slice of shared memory
    float* cr = cw + warp * d_c;
    const int64_t prow = cv.code_row(bh, row);  // plane row of the code and of its slots
    for (int e = lane; e < d_c; e += 32) cr[e] = code_at(code, cscale, prow, d_c, e);
    __syncwarp();
    float u[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      u[m] = 0.f;
      if (m < per_lane) {
        int n = lane + 32 * m;
        float acc = b3 ? b3[n] : 0.f;
        for (int e = 0; e < d_c; ++e) acc = fmaf(W3s[e * hidden + n], cr[e], acc);
        u[m] = act_eval(act, acc);
      }
    }
    __syncwarp();
    // reference part of the logits
    int j = lane < k ? idx[prow * k + lane] : -1;
    if (j >= n_ref) { latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j); j = -1; }
    const unsigned valid = __ballot_sync(0xffffffffu, j >= 0);
    const int k_eff = __popc(valid);
    const float inv_k = 1.0f / (float)max(k_eff, 1);
    float lg[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      if (g < G) {
        float part_ = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          if (m < per_lane) part_ = fmaf(As[g * hidden + lane + 32 * m], u[m], part_);
        float sr = j >= 0 ? Sb[(int64_t)j * G + g] : 0.f;
        lg[g] = warp_sum(part_) + warp_sum(sr) * inv_k + ct[g];
      }
    }
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      if (g < G) {
        if (lg[g] > mw[g]) {
          float sc = exp2f(mw[g] - lg[g]);
          lw[g] *= sc;
#pragma unroll
          for (int m = 0; m < 8; ++m) Uw[g][m] *= sc;
          mw[g] = lg[g];
        }
        float p = exp2f(lg[g] - mw[g]);
        lw[g] += p;
#pragma unroll
        for (int m = 0; m < 8; ++m) Uw[g][m] = fmaf(p, u[m], Uw[g][m]);
        float dl = lg[g] - mref[g];
        if (dl > 100.f) latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, 0xFFFFFFFFu);
        float pr = exp2f(fminf(dl, 100.f)) * inv_k;
        if (j >= 0) atomicAdd(&wtab[(int64_t)j * G + g], pr);
      }
    }
  }
  // merge the warps: block max, then rescale and sum l and U
  __shared__ float mws[8][kMaxG];
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) mws[warp][g] = mw[g];
  __syncthreads();
  float mb[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    mb[g] = -INFINITY;
    for (int w = 0; w < 8; ++w) mb[g] = fmaxf(mb[g], mws[w][g]);
  }
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    if (g < G) {
      float sc = mw[g] == -INFINITY ? 0.f : exp2f(mw[g] - mb[g]);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        if (m < per_lane) atomicAdd(&Ured[g * hidden + lane + 32 * m], Uw[g][m] * sc);
      if (lane == 0) atomicAdd(&misc[2 * kMaxG + g], lw[g] * sc);
    }
  }
  __syncthreads();
  const int64_t pb = bh * nslot_cap + split;
  if (tid < G) {
    part[(pb * G + tid) * 2 + 0] = mb[tid];
    part[(pb * G + tid) * 2 + 1] = misc[2 * kMaxG + tid];
  }
  for (int i = tid; i < G * hidden; i += blockDim.x) Upart[pb * G * hidden + i] = Ured[i];
  if (wt_in_smem) {
    float* dst = wtab_g + bh * n_ref_cap * G;
    for (int64_t i = tid; i < n_ref * G; i += blockDim.x)
      if (wt[i] != 0.f) atomicAdd(dst + i, wt[i]);
  }
}

// Partial (m, l, U) slots per kv-head: a fixed count for the CUDA-core
// stream kernel, the CTAs of the even chunk split for the tensor-core one.
struct SlotInfo {
  int tc, ns, grid, nslot_cap, BH;
  int n_ch;            // chunks per (sequence, kv-head) when every sequence has the same length
  const int32_t* cho;  // else the chunk offsets [BH + 1] (decode_sched_kernel)
};

__device__ __forceinline__ int64_t chunk_off(const SlotInfo& si, int64_t bh) {
  return si.cho ? (int64_t)si.cho[bh] : bh * si.n_ch;
}

__device__ __forceinline__ int slots_of(const SlotInfo& si, int64_t bh) {
  if (!si.tc) return si.ns;
  const int64_t x0 = chunk_off(si, bh), x1 = chunk_off(si, bh + 1), N = chunk_off(si, si.BH);
  if (x1 == x0) return 0;
  const int64_t g = N < si.grid ? N : si.grid;  // the CTAs that got chunks (as in the token loop)
  const int64_t first = (x0 * g) / N;
  const int64_t last = ((x1 - 1) * g) / N;
  return (int)(last - first + 1);
}


// -------------------------------------------------------- decode_combine
// M_g = max(m_ref, split maxima).  For 256 slots: weights
// w_j = 2^(S_j - M) + 2^(m_ref - M) sum_splits wtab, then sum_j w_j V_ref_j.
// GP: heads per kv-head as laid out in registers (4 or 8, at least G).
//
// The CTA's V rows (at most 256 x d_h elements, two runs of up to 128
// consecutive rows: a pool page holds 128) come into shared memory by bulk
// copies issued first, so the copy overlaps the weight computation; the sum
// then reads them from shared memory: thread (slot group, 4 consecutive
// elements), every row segment used for all heads of the group.
template <typename T, int GP>
__global__ void __launch_bounds__(256)
    decode_combine_kernel(SeqLens sl, int s, int d_h, int H, int G, SlotInfo si, int64_t n_ref_cap,
                          int n_chunk_cap, CacheView cv, const float* __restrict__ S,
                          const float* __restrict__ mref, const float* __restrict__ wtab_g,
                          const float* __restrict__ part, float* __restrict__ ochunk,
                          const int32_t* __restrict__ mult, uint32_t* __restrict__ err) {
  // kCombineSlots x d_h elements of T; once every thread has read its rows,
  // the partial sums [slot group][head][element] (8 kMaxG 128 floats, at
  // most the rows' size)
  extern __shared__ __align__(128) unsigned char vsm[];
  float* red = reinterpret_cast<float*>(vsm);
  __shared__ __align__(16) float wts[kCombineSlots][GP];
  __shared__ float Mg[kMaxG], mrefg[kMaxG], lw[8][kMaxG];
  __shared__ __align__(8) uint64_t vbar;
  const int b = blockIdx.z, h = blockIdx.y, ch = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t bh = (int64_t)b * H + h;
  const int64_t n_ref = n_ref_of(sl.T(b), s);
  const int64_t j0 = (int64_t)ch * kCombineSlots;
  if (j0 >= n_ref) return;  // past this sequence's references (its final reads n_chunk of its own)
  const int nrows = (int)(n_ref - j0 < kCombineSlots ? n_ref - j0 : kCombineSlots);
  const T* refv = reinterpret_cast<const T*>(cv.base + cv.off_refv);
  if (tid == 0) {
    const uint32_t row_bytes = (uint32_t)(d_h * sizeof(T));
    sm100::mbar_init(&vbar, 1);
    sm100::fence_mbar_init();
    sm100::mbar_arrive_expect_tx(&vbar, (uint32_t)nrows * row_bytes);
    for (int r0 = 0; r0 < nrows; r0 += 128) {
      const int nr = nrows - r0 < 128 ? nrows - r0 : 128;
      sm100::bulk_load(vsm + (size_t)r0 * row_bytes, refv + cv.ref_row(bh, j0 + r0) * d_h, (uint32_t)nr * row_bytes,
                       &vbar);
    }
  }
  if (tid < G) {
    const float m = mref[bh * G + tid];
    mrefg[tid] = m;
    float M = m;
    const int ns = slots_of(si, bh);
    for (int sp = 0; sp < ns; ++sp) M = fmaxf(M, part[((bh * si.nslot_cap + sp) * G + tid) * 2]);
    Mg[tid] = M;
  }
  __syncthreads();
  float lsum[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) lsum[g] = 0.f;
  for (int jj = tid; jj < kCombineSlots; jj += blockDim.x) {
    const int64_t j = j0 + jj;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float w = 0.f;
      if (g < G && j < n_ref) {
        // a reference's own term counts once per selection of it (sparse
        // decode), once otherwise
        float own = exp2f(S[(bh * n_ref_cap + j) * G + g] - Mg[g]);
        if (mult) own *= (float)mult[bh * n_ref_cap + j];
        w = own + wtab_g[(bh * n_ref_cap + j) * G + g] * exp2f(mrefg[g] - Mg[g]);
        lsum[g] += own;
      }
      wts[jj][g] = w;
    }
  }
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    const float ls = warp_sum(lsum[g]);
    if (lane == 0 && g < G) lw[warp][g] = ls;
  }
  // the V rows have landed (bounded wait; every thread leaves together if
  // it ran out)
  if (!__syncthreads_and(sm100::mbar_wait_drain(&vbar, 0))) {
    if (tid == 0) latch_error(err, DELTAKV_ERR_DEVICE_TIMEOUT, 31);
    return;
  }
  // sum_j w_j V_ref_j: thread = (slot group, elements 4 e4 .. 4 e4 + 3)
  const int e4n = d_h / 4, e4 = tid % e4n, grp = tid / e4n, ngrp = blockDim.x / e4n;
  const int spg = kCombineSlots / ngrp;  // slots per group
  float acc[GP][4];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[g][i] = 0.f;
  const int q_end = nrows - grp * spg < spg ? nrows - grp * spg : spg;  // rows past nrows were not copied
#pragma unroll 4
  for (int q = 0; q < q_end; ++q) {
    const int jj = grp * spg + q;
    float v[4];
    const T* row = reinterpret_cast<const T*>(vsm) + (size_t)jj * d_h + e4 * 4;
    if constexpr (sizeof(T) == 2) {
      const uint2 r = *reinterpret_cast<const uint2*>(row);
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
      v[0] = f0.x;
      v[1] = f0.y;
      v[2] = f1.x;
      v[3] = f1.y;
    } else {
      const float4 r = *reinterpret_cast<const float4*>(row);
      v[0] = r.x;
      v[1] = r.y;
      v[2] = r.z;
      v[3] = r.w;
    }
    float w[GP];
#pragma unroll
    for (int g4 = 0; g4 < GP; g4 += 4) {
      const float4 w4 = *reinterpret_cast<const float4*>(&wts[jj][g4]);
      w[g4] = w4.x;
      w[g4 + 1] = w4.y;
      w[g4 + 2] = w4.z;
      w[g4 + 3] = w4.w;
    }
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[g][i] = fmaf(w[g], v[i], acc[g][i]);
  }
  __syncthreads();  // every row read: the rows' space takes the partial sums
#pragma unroll
  for (int g = 0; g < GP; ++g)
    if (g < G)
      *reinterpret_cast<float4*>(&red[(grp * kMaxG + g) * d_h + e4 * 4]) =
          make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  __syncthreads();
  for (int o = tid; o < G * d_h; o += blockDim.x) {
    const int g = o / d_h, e = o - g * d_h;
    float sum = 0.f;
    for (int w = 0; w < ngrp; ++w) sum += red[(w * kMaxG + g) * d_h + e];
    ochunk[((bh * n_chunk_cap + ch) * G + g) * (d_h + 1) + e] = sum;
  }
  if (tid < G) {
    float l = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) l += lw[w][tid];
    ochunk[((bh * n_chunk_cap + ch) * G + tid) * (d_h + 1) + d_h] = l;
  }
}

// ---------------------------------------------------------- decode_final
// kFinalSplit CTAs per (sequence, kv-head), each for d_h / kFinalSplit of
// the output elements (the merge of the splits' maxima, sums and U is
// repeated by each: it is small).
constexpr int kFinalSplit = 4;
template <typename T>
__global__ void __launch_bounds__(256)
    decode_final_kernel(SeqLens sl, int s, int d_h, int H, int G, int hidden, SlotInfo si,
                        int n_chunk_cap, const T* __restrict__ W4, const float* __restrict__ b4,
                        const float* __restrict__ mref, const float* __restrict__ part,
                        const float* __restrict__ Upart, const float* __restrict__ ochunk,
                        float* __restrict__ out, int64_t osb, int64_t osh) {
  __shared__ __align__(16) float Ut[kMaxG][kMaxHidden];
  __shared__ float Mg[kMaxG], Lnr[kMaxG], Lall[kMaxG];
  __shared__ float Oc[kMaxG][128 / kFinalSplit];
  const int b = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
  const int64_t bh = (int64_t)b * H + h;
  const int nout = d_h / kFinalSplit, e_base = blockIdx.x * nout;  // this CTA's output elements
  const int ns = slots_of(si, bh);
  const int64_t pb0 = bh * si.nslot_cap;
  const int n_chunk = (int)((n_ref_of(sl.T(b), s) + kCombineSlots - 1) / kCombineSlots);
  {
    // warp g: the maximum, the token-loop denominator and the reference
    // denominator of head g (the chunks' sums split over the lanes)
    const int warp = tid >> 5, lane = tid & 31;
    for (int g = warp; g < G; g += (int)(blockDim.x >> 5)) {
      float M = mref[bh * G + g];
#pragma unroll 4
      for (int sp = 0; sp < ns; ++sp) M = fmaxf(M, part[((pb0 + sp) * G + g) * 2]);
      float lnr = 0.f;
      for (int sp = lane; sp < ns; sp += 32) {
        float m = part[((pb0 + sp) * G + g) * 2];
        float l = part[((pb0 + sp) * G + g) * 2 + 1];
        if (m != -INFINITY) lnr += l * exp2f(m - M);
      }
      float lr = 0.f;
      for (int c = lane; c < n_chunk; c += 32) lr += ochunk[((bh * n_chunk_cap + c) * G + g) * (d_h + 1) + d_h];
      lnr = warp_sum(lnr);
      lr = warp_sum(lr);
      if (lane == 0) {
        Mg[g] = M;
        Lnr[g] = lnr;
        Lall[g] = lnr + lr;
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < G * hidden; i += blockDim.x) {
    int g = i / hidden, n = i - g * hidden;
    float acc = 0.f;
#pragma unroll 4
    for (int sp = 0; sp < ns; ++sp) {
      float m = part[((pb0 + sp) * G + g) * 2];
      if (m != -INFINITY) acc += Upart[((pb0 + sp) * G + g) * hidden + n] * exp2f(m - Mg[g]);
    }
    Ut[g][n] = acc;
  }
  __syncthreads();
  // the reference chunks' sums for this CTA's elements: threads over
  // (head, element), chunk loads independent of one another
  for (int o = tid; o < G * nout; o += blockDim.x) {
    const int g = o / nout, el = o - g * nout;
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < n_chunk; ++c) acc += ochunk[((bh * n_chunk_cap + c) * G + g) * (d_h + 1) + e_base + el];
    Oc[g][el] = acc;
  }
  __syncthreads();
  // W4_V . U: a warp per output element, its lanes over the hidden units
  // (8 consecutive weights per 16-byte load; hidden <= 256, so one load a
  // lane), every head of the group at once; the weight rows of all of a
  // warp's elements are loaded before any is used
  const int warp = tid >> 5, lane = tid & 31, nw = (int)(blockDim.x >> 5);
  constexpr int kRows = 128 / kFinalSplit / 8;  // elements per warp at d_h = 128, 8 warps
  float w[kRows][8];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int el = warp + r * nw;
    if (el < nout && lane * 8 < hidden) {
      load8(W4 + (int64_t)(d_h + e_base + el) * hidden + lane * 8, w[r]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) w[r][i] = 0.f;
    }
  }
  const int n0 = lane * 8 < hidden ? lane * 8 : 0;  // lanes past hidden hold zero weights
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int el = warp + r * nw;
    if (el >= nout) break;
    float y[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      y[g] = 0.f;
      if (g < G) {
        const float4 u0 = *reinterpret_cast<const float4*>(&Ut[g][n0]);
        const float4 u1 = *reinterpret_cast<const float4*>(&Ut[g][n0 + 4]);
        y[g] = fmaf(w[r][0], u0.x, fmaf(w[r][1], u0.y, fmaf(w[r][2], u0.z, fmaf(w[r][3], u0.w, y[g]))));
        y[g] = fmaf(w[r][4], u1.x, fmaf(w[r][5], u1.y, fmaf(w[r][6], u1.z, fmaf(w[r][7], u1.w, y[g]))));
      }
    }
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      if (g < G) {
        const float yg = warp_sum(y[g]);
        if (lane == g) {
          const int e = e_base + el;
          const float acc = Oc[g][el] + yg + (b4 ? b4[d_h + e] * Lnr[g] : 0.f);
          out[b * osb + (int64_t)(h * G + g) * osh + e] = acc / Lall[g];
        }
      }
    }
  }
}

// ---------------------------------------------------------- decode_sched
// Sequences of different lengths: their lengths checked against [1, T_max]
// (an out-of-range length is reported and read as 1) into `lens`, which the
// other kernels read, and the chunk offsets of the tensor-core token loop:
// cho[bh] = sum over earlier (sequence, kv-head) pairs of their 128-row
// chunk counts, cho[BH] the total.  One block.
__global__ void __launch_bounds__(1024)
    decode_sched_kernel(const int32_t* __restrict__ Tin, int B, int H, int s, int T_max,
                        int32_t* __restrict__ lens, int32_t* __restrict__ cho, uint32_t* __restrict__ err) {
  __shared__ int32_t part[1024];
  __shared__ int32_t Ts[1024];
  const int BH = B * H, tid = threadIdx.x;
  for (int b = tid; b < B; b += blockDim.x) {
    int32_t t = Tin[b];
    if (t < 1 || t > T_max) {
      if (atomicCAS(err, 0u, (uint32_t)DELTAKV_ERR_DEVICE_BOUNDS) == 0u) err[1] = (uint32_t)t;
      t = 1;
    }
    lens[b] = t;
    if (b < 1024) Ts[b] = t;
  }
  __syncthreads();
  const int32_t* Tb = B <= 1024 ? Ts : lens;
  const int per = (BH + blockDim.x - 1) / blockDim.x;  // (sequence, kv-head) pairs per thread
  int32_t sum = 0;
  for (int i = 0; i < per; ++i) {
    const int bh = tid * per + i;
    if (bh < BH) sum += (int32_t)((n_code_of(Tb[bh / H], s) + 127) / 128);
  }
  part[tid] = sum;
  __syncthreads();
  if (tid == 0) {
    int32_t run = 0;
    for (int t = 0; t < (int)blockDim.x; ++t) {
      const int32_t v = part[t];
      part[t] = run;
      run += v;
    }
    cho[BH] = run;
  }
  __syncthreads();
  int32_t run = part[tid];
  for (int i = 0; i < per; ++i) {
    const int bh = tid * per + i;
    if (bh < BH) {
      cho[bh] = run;
      run += (int32_t)((n_code_of(Tb[bh / H], s) + 127) / 128);
    }
  }
}

// ------------------------------------------------------------- launcher
// ------------------------------------------------- sparse selection
// One block per (sequence, kv-head): the selected reference tokens are
// counted per slot (a token selected twice counts twice), the selected other
// tokens' compressed rows listed for the token loop in the order of the
// selection (positions from a ballot prefix per 256 tokens, so the list, and
// with it the token loop's summation order, is the same on every run), and
// their number kept; an index outside [0, T) is reported and skipped.  A
// thread's tokens of eight such groups are loaded before any is used.
__global__ void __launch_bounds__(256)
    sparse_select_kernel(int T, int s, int64_t n_ref_cap, int64_t rl_cap, int n_sel,
                         const int32_t* __restrict__ tokens, int32_t* __restrict__ mult,
                         int32_t* __restrict__ rowlist, int32_t* __restrict__ ncode, uint32_t* __restrict__ err) {
  constexpr int kGroups = 8;
  __shared__ int wsum[8];
  const int64_t bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n_ref = n_ref_of(T, s);
  int32_t* m = mult + bh * n_ref_cap;
  for (int64_t j = tid; j < n_ref; j += blockDim.x) m[j] = 0;
  __syncthreads();
  int base = 0;
  for (int c0 = 0; c0 < n_sel; c0 += kGroups * 256) {
    int tv[kGroups];
#pragma unroll
    for (int u = 0; u < kGroups; ++u) {
      const int i = c0 + u * 256 + tid;
      tv[u] = i < n_sel ? tokens[bh * n_sel + i] : 0;
    }
#pragma unroll
    for (int u = 0; u < kGroups; ++u) {
      if (c0 + u * 256 >= n_sel) break;  // the same for every thread
      const int t = tv[u];
      bool code = false;
      if (c0 + u * 256 + tid < n_sel) {
        if (t < 0 || t >= T) latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)t);
        else if (t % s == 0) atomicAdd(&m[t / s], 1);
        else code = true;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, code);
      if (lane == 0) wsum[warp] = __popc(bal);
      __syncthreads();
      int off = base, total = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const int c = wsum[w];
        off += w < warp ? c : 0;
        total += c;
      }
      if (code) rowlist[bh * rl_cap + off + __popc(bal & ((1u << lane) - 1u))] = t - t / s - 1;
      base += total;
      __syncthreads();  // wsum is reused by the next group
    }
  }
  if (tid == 0) ncode[bh] = base;
}

// Chunk offsets of the token loop over the listed rows: cho[bh] = sum over
// earlier (sequence, kv-head) pairs of their 128-row chunk counts.  One block
// of 1024 threads, each over a contiguous run of pairs; the runs' sums are
// scanned with warp shuffles.
__global__ void __launch_bounds__(1024)
    sparse_cho_kernel(int BH, const int32_t* __restrict__ ncode, int32_t* __restrict__ cho) {
  __shared__ int32_t wtot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (BH + blockDim.x - 1) / blockDim.x;
  int32_t sum = 0;
  for (int i = 0; i < per; ++i) {
    const int bh = tid * per + i;
    if (bh < BH) sum += (ncode[bh] + 127) / 128;
  }
  // inclusive scan within the warp, then across the warps' totals
  int32_t x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += v;
  }
  if (lane == 31) wtot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = (int)(blockDim.x >> 5);
    int32_t w = lane < nw ? wtot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    wtot[lane] = w;  // inclusive totals of warps 0 .. lane
  }
  __syncthreads();
  int32_t run = x - sum + (warp > 0 ? wtot[warp - 1] : 0);
  if (tid == (int)blockDim.x - 1) cho[BH] = run + sum;
  for (int i = 0; i < per; ++i) {
    const int bh = tid * per + i;
    if (bh < BH) {
      cho[bh] = run;
      run += (ncode[bh] + 127) / 128;
    }
  }
}

// The stabilising maximum of a sparse decode, per (sequence, kv-head, head):
// the largest logit estimate over the selection -- S_j of each selected
// reference, the mean of S over the slots of each selected other token (its
// logit less the a . u and constant terms, which the token loop's lazy
// rescaling absorbs).  The dense decode's maximum over every reference can
// lie far above all selected logits, and their softmax weights would then
// underflow in the token loop's fp16 P tile.  One block per (sequence,
// kv-head); 0 when nothing valid is selected.
__global__ void __launch_bounds__(256)
    sparse_mref_kernel(int T, int s, int G, int k, int64_t n_ref_cap, int64_t n_code_cap, int64_t rl_cap,
                       const float* __restrict__ S, const int32_t* __restrict__ mult,
                       const int32_t* __restrict__ rowlist, const int32_t* __restrict__ ncode,
                       const int32_t* __restrict__ idx, float* __restrict__ mref) {
  __shared__ float red[8][kMaxG];
  const int64_t bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n_ref = n_ref_of(T, s);
  const float* Sb = S + bh * n_ref_cap * G;
  float m[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) m[g] = -INFINITY;
  // eight slots' counts, then their S rows, in flight at a time
  for (int64_t j0 = tid; j0 < n_ref; j0 += 8 * (int64_t)blockDim.x) {
    int mv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      mv[u] = j < n_ref ? mult[bh * n_ref_cap + j] : 0;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t j = j0 + (int64_t)u * blockDim.x;
      if (mv[u] > 0)
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < G) m[g] = fmaxf(m[g], Sb[j * G + g]);
    }
  }
  // four listed rows at a time: their rows of the list, then their slots,
  // then the slots' S rows
  const int nc = ncode[bh];
  for (int i0 = tid; i0 < nc; i0 += 4 * (int)blockDim.x) {
    int64_t r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * (int)blockDim.x;
      r[u] = i < nc ? rowlist[bh * rl_cap + i] : -1;
    }
    int js[4][kMaxK];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int q = 0; q < kMaxK; ++q) js[u][q] = (r[u] >= 0 && q < k) ? idx[(bh * n_code_cap + r[u]) * k + q] : -1;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float sum[kMaxG];
#pragma unroll
      for (int g = 0; g < kMaxG; ++g) sum[g] = 0.f;
      int ke = 0;
#pragma unroll
      for (int q = 0; q < kMaxK; ++q) {
        const int j = js[u][q];
        if (j < 0 || j >= n_ref) continue;
        ++ke;
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < G) sum[g] += Sb[(int64_t)j * G + g];
      }
      if (ke > 0)
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < G) m[g] = fmaxf(m[g], sum[g] / (float)ke);
    }
  }
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    float v = m[g];
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[warp][g] = v;
  }
  __syncthreads();
  if (tid < G) {
    float v = -INFINITY;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v = fmaxf(v, red[w][tid]);
    mref[bh * G + tid] = v == -INFINITY ? 0.f : v;
  }
}

// Selected tokens of a sparse decode on the tensor-core token loop.
struct SparseSel {
  const int32_t* tokens;
  int n_sel;
};

template <typename E>
static cudaError_t decode_launch(const Plan& p, const CacheView& cv, const SeqLens& sl_in, const void* q, int64_t qsb,
                                 int64_t qsh, const void* W3, const float* b3, const void* W4, const float* b4,
                                 float* out, int64_t osb, int64_t osh, void* ws, cudaStream_t st,
                                 const SparseSel* sel = nullptr) {
  const auto& c = p.cfg;
  const int H = c.kv_heads, B = c.batch, G = p.G;
  const int64_t n_ref = n_ref_of(sl_in.T_max, c.stride_s);  // the longest sequence's; shorter ones stop early
  const float cs = kLog2e / sqrtf((float)c.d_h);
  char* w = (char*)ws;
  float* S = (float*)(w + p.ws_S);
  float* Smax = (float*)(w + p.ws_Smax);
  float* a = (float*)(w + p.ws_a);
  float* cterm = (float*)(w + p.ws_cterm);
  float* mref = (float*)(w + p.ws_mref);
  float* wtab = (float*)(w + p.ws_wtab);
  float* part = (float*)(w + p.ws_part);
  float* Upart = (float*)(w + p.ws_U);
  float* ochunk = (float*)(w + p.ws_ochunk);
  int32_t* cho = (int32_t*)(w + p.ws_cho);
  int32_t* lens = cho + (int64_t)B * H + 1;
  SeqLens sl = sl_in;
  int32_t* mult = nullptr;
  int32_t* rowlist = nullptr;
  int32_t* ncode = nullptr;
  if (sel) {
    // the selection: reference multiplicities, the listed compressed rows and
    // the token loop's chunk offsets over them
    mult = (int32_t*)(w + p.ws_mult);
    rowlist = (int32_t*)(w + p.ws_rowlist);
    ncode = (int32_t*)(w + p.ws_ncode);
    {
      ProfScope ps(p, st, KID_SPARSE_SELECT);
      sparse_select_kernel<<<B * H, 256, 0, st>>>(sl.T_all, c.stride_s, p.n_ref_cap, p.n_code_cap + p.n_ref_cap,
                                                  sel->n_sel, sel->tokens, mult, rowlist, ncode, (uint32_t*)ws);
      sparse_cho_kernel<<<1, 1024, 0, st>>>(B * H, ncode, cho);
    }
    cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return e0;
  }
  if (sl.Tb) {
    // checked lengths and chunk offsets first: every later kernel reads them
    decode_sched_kernel<<<1, 1024, 0, st>>>(sl_in.Tb, B, H, c.stride_s, sl.T_max, lens, cho, (uint32_t*)ws);
    cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return e0;
    sl.Tb = lens;
  }
  const int n_refblk = (int)ceil_div64(n_ref, kRefBlockSlots);
  const int n_refblk_cap = (int)ceil_div64(p.n_ref_cap, kRefBlockSlots);
  const int n_chunk = (int)ceil_div64(n_ref, kCombineSlots);

  {
    ProfScope ps(p, st, KID_DEC_REF);
    const size_t kbytes = (size_t)kRefBlockSlots * (c.d_h * sizeof(E) + 16);
    decode_ref_kernel<E><<<dim3(n_refblk, H, B), kRefBlockSlots, kbytes, st>>>(
        sl, c.stride_s, p.n_ref_cap, c.d_h, H, G, cs, (const E*)q, qsb, qsh, cv, S, Smax, n_refblk_cap, wtab,
        (uint32_t*)ws);
  }
  {
    ProfScope ps(p, st, KID_DEC_PREP);
    decode_prep_kernel<E><<<dim3(1, H, B), 256, 0, st>>>(c.d_h, H, G, c.hidden, cs, (const E*)q, qsb,
                                                         qsh, (const E*)W4, b4, a, cterm, Smax, n_refblk,
                                                         n_refblk_cap, mref);
  }
  if (sel) {
    ProfScope ps(p, st, KID_SPARSE_SELECT);
    sparse_mref_kernel<<<B * H, 256, 0, st>>>(sl.T_all, c.stride_s, G, c.k, p.n_ref_cap, p.n_code_cap,
                                              p.n_code_cap + p.n_ref_cap, S, mult, rowlist, ncode,
                                              (const int32_t*)(cv.base + cv.off_idx), mref);
    cudaError_t e1 = cudaGetLastError();
    if (e1 != cudaSuccess) return e1;
  }
  SlotInfo si{};
  si.nslot_cap = p.nslot_cap;
  si.BH = B * H;
  cudaError_t e = cudaErrorNotSupported;
  if (decode_tc_supported(p)) {
    const int32_t* chop = (sl.Tb || sel) ? cho : nullptr;
    int grid = 0;
    e = launch_decode_tc(p, cv, sl, chop, W3, b3, ws, st, &grid, rowlist, ncode, p.n_code_cap + p.n_ref_cap);
    if (e == cudaSuccess) {
      si.tc = 1;
      si.n_ch = (int)ceil_div64(n_code_of(sl.T_all, c.stride_s), 128);
      si.cho = chop;
      si.grid = grid;
    }
  }
  if (e == cudaErrorNotSupported && sel) return e;  // the caller takes the CUDA-core sparse kernels
  if (e == cudaErrorNotSupported) {
    // splits: enough blocks for about two waves, never more rows than splits
    const int64_t n_code = n_code_of(sl.T_max, c.stride_s);
    int ns = (int)ceil_div64(2 * kNumSMs, (int64_t)B * H);
    ns = (int)std::min<int64_t>(std::min<int64_t>(ns, p.nslot_cap), std::max<int64_t>(1, n_code / 64));
    size_t base = sizeof(float) * (size_t)(c.d_c * c.hidden + 2 * G * c.hidden + 4 * kMaxG + 8 * c.d_c);
    size_t wt_bytes = sizeof(float) * (size_t)(n_ref * G);
    int wt_in_smem = base + wt_bytes <= 200 * 1024;
    size_t smem = base + (wt_in_smem ? wt_bytes : 0);
    auto ks = decode_stream_kernel<E>;
    e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps(p, st, KID_DEC_STREAM_SIMT);
    ks<<<dim3(ns, H, B), 256, smem, st>>>(sl, c.stride_s, c.d_h, H, G, c.k, c.d_c, c.hidden, (int)c.act, ns,
                                          p.n_ref_cap, n_refblk, n_refblk_cap, cv, (const E*)W3, b3, a, cterm,
                                          S, Smax, wtab, part, Upart, wt_in_smem, p.nslot_cap, (uint32_t*)ws);
    e = cudaGetLastError();
    si.tc = 0;
    si.ns = ns;
  }
  if (e != cudaSuccess) return e;
  {
    ProfScope ps(p, st, KID_DEC_COMBINE);
    const size_t vbytes = (size_t)kCombineSlots * c.d_h * sizeof(E);
    auto kc = G <= 4 ? decode_combine_kernel<E, 4> : decode_combine_kernel<E, 8>;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)vbytes);
    if (e != cudaSuccess) return e;
    kc<<<dim3(n_chunk, H, B), 256, vbytes, st>>>(sl, c.stride_s, c.d_h, H, G, si, p.n_ref_cap, p.n_chunk_cap, cv,
                                                 S, mref, wtab, part, ochunk, mult, (uint32_t*)ws);
  }
  {
    ProfScope ps(p, st, KID_DEC_FINAL);
    decode_final_kernel<E><<<dim3(kFinalSplit, H, B), 256, 0, st>>>(
        sl, c.stride_s, c.d_h, H, G, c.hidden, si, p.n_chunk_cap, (const E*)W4, b4, mref, part, Upart, ochunk,
        out, osb, osh);
  }
  return cudaGetLastError();
}

CacheView contiguous_view(const Plan& p, const void* cache) {
  CacheView v{};
  v.base = (const char*)cache;
  v.off_refk = p.off_refk;
  v.off_refv = p.off_refv;
  v.off_code = p.off_code;
  v.off_idx = p.off_idx;
  v.off_cscale = p.off_cscale;
  v.rp = p.n_ref_cap;
  v.cp = p.n_code_cap;
  v.n_pages = (int64_t)p.cfg.batch * p.cfg.kv_heads;
  v.ptab = nullptr;
  v.max_pages = 1;
  v.err = nullptr;
  return v;
}

cudaError_t launch_decode_sparse_tc(const Plan& p, int T, const void* q, int64_t qsb, int64_t qsh, const void* cache,
                                    const void* W3, const float* b3, const void* W4, const float* b4,
                                    const int32_t* tokens, int n_sel, float* out, int64_t osb, int64_t osh, void* ws,
                                    cudaStream_t st) {
  // the row list holds up to n_code_cap + n_ref_cap entries per (sequence, kv-head)
  if (!decode_tc_supported(p) || p.code4 || (int64_t)n_sel > p.n_code_cap + p.n_ref_cap) return cudaErrorNotSupported;
  const SparseSel sel{tokens, n_sel};
  const CacheView cv = contiguous_view(p, cache);
  const SeqLens sl{nullptr, T, T};
  if (p.bf16)
    return decode_launch<__nv_bfloat16>(p, cv, sl, q, qsb, qsh, W3, b3, W4, b4, out, osb, osh, ws, st, &sel);
  return decode_launch<float>(p, cv, sl, q, qsb, qsh, W3, b3, W4, b4, out, osb, osh, ws, st, &sel);
}

cudaError_t launch_decode(const Plan& p, const CacheView& cv, const SeqLens& sl, const void* q, int64_t qsb,
                          int64_t qsh, const void* W3, const float* b3, const void* W4, const float* b4, float* out,
                          int64_t osb, int64_t osh, void* ws, cudaStream_t st) {
  if (p.bf16)
    return decode_launch<__nv_bfloat16>(p, cv, sl, q, qsb, qsh, W3, b3, W4, b4, out, osb, osh, ws, st);
  return decode_launch<float>(p, cv, sl, q, qsb, qsh, W3, b3, W4, b4, out, osb, osh, ws, st);
}

}  // namespace dkv
