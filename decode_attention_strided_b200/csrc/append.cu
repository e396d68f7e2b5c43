// append.cu -- streaming compression: the tokens [T0, T1) of a layer whose
// packed cache already holds the compressed tokens [0, T0).
//
// DeltaKV summary, section 3, "Processo di Compressione" steps 1-4, applied
// to tokens as they arrive during decoding ("durante l'inferenza" in the same
// section): a new token t with t mod s == 0 becomes a reference (its K, V rows
// are copied into the reference planes); every other new token searches all
// earlier references (slots j with j s < t, including references appended by
// the same call), keeps the k nearest by squared L2 over [K ; V] (ties to the
// lower slot), subtracts their mean and compresses the residual with the MLP.
// The slots are the exact top-k of float32 distances, so they match the oracle
// under the same near-tie rule as compression in one call; where two
// references lie within float32 rounding of the same distance the two paths
// may keep different ones.  Everything else is what one call over [0, T1)
// writes.
//
// Few tokens arrive per call, so the kernels are plain CUDA-core code with
// exact fp32 distances (no candidate search and re-rank): each new token's
// references are split over several CTAs (a scan kernel), whose lists one
// CTA per (token, kv-head) merges before the MLP (a finish kernel).
#include <cfloat>
#include <climits>

#include "common.cuh"
#include "sm100.cuh"

namespace dkv {

using namespace sm100;

namespace {
constexpr int kScanThreads = 256;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kFinishThreads = 512;
constexpr int kFinishWarps = kFinishThreads / 32;
constexpr int kAppendKMax = 8;    // references per token (k <= 8)
constexpr int kAppendRows = 8;    // reference rows in flight per warp
constexpr int kAppendSplitMax = 64;  // scan CTAs per (token, sequence x kv-head)

// NV consecutive elements of E held as raw 32-bit words (NV * sizeof(E) is
// 8, 16 or 32 bytes, aligned to that size or to 16), converted on use.
template <typename E, int NV>
struct Frag {
  static constexpr int kBytes = NV * (int)sizeof(E);
  static constexpr int kWords = kBytes / 4;
  uint32_t w[kWords];
  // global load cached in L2 only: the append kernels start before the
  // grid ahead of them on the stream has finished (programmatic launch), so
  // they read nothing through the read-only path, which assumes data that
  // no grid changes during the kernel's lifetime
  __device__ __forceinline__ void ldcg(const E* p) {
    if constexpr (kBytes % 16 == 0) {
#pragma unroll
      for (int c = 0; c < kBytes / 16; ++c) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p) + c);
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
      }
    } else {
      const uint2 v = __ldcg(reinterpret_cast<const uint2*>(p));
      w[0] = v.x;
      w[1] = v.y;
    }
  }
  // load through a generic pointer (shared or global memory)
  __device__ __forceinline__ void ld(const E* p) {
    if constexpr (kBytes % 16 == 0) {
#pragma unroll
      for (int c = 0; c < kBytes / 16; ++c) {
        const uint4 v = reinterpret_cast<const uint4*>(p)[c];
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
      }
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      w[0] = v.x;
      w[1] = v.y;
    }
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < kWords; ++i) w[i] = 0u;
  }
  // element i as float (bf16: element 2c in the low half of word c)
  __device__ __forceinline__ float operator[](int i) const {
    if constexpr (sizeof(E) == 2)
      return __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
    else
      return __uint_as_float(w[i]);
  }
};

// Sums of eight per-lane partials p[0..7] over the warp, one sum per lane:
// lane l ends with the total of row (l >> 2) & 7.  Three exchange steps
// each hand half of the remaining rows to the partner lane (4 + 2 + 1
// shuffles), two plain steps finish the sums: 9 shuffles for 8 rows.
__device__ __forceinline__ float warp_sum8(const float (&p)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float q4[4], q2[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b4 ? p[i + 4] : p[i], send = b4 ? p[i] : p[i + 4];
    q4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b3 ? q4[i + 2] : q4[i], send = b3 ? q4[i] : q4[i + 2];
    q2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float q = (b2 ? q2[1] : q2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? q2[0] : q2[1], 4);
  q += __shfl_xor_sync(0xffffffffu, q, 2);
  q += __shfl_xor_sync(0xffffffffu, q, 1);
  return q;
}

// The k-th smallest entry of an ascending list (k in [1, KC]; no entry is
// NaN): the largest of its first k, which needs no dynamic register index.
template <int KC>
__device__ __forceinline__ float kth_entry(const float (&bd)[KC], int k) {
  float v = bd[0];
#pragma unroll
  for (int i = 1; i < KC; ++i) v = i < k ? fmaxf(v, bd[i]) : v;
  return v;
}

// Rank of entry i among the n entries (d, j) in shared memory, ordered by
// distance with ties to the lower slot.  Slots are distinct, so the ranks
// are 0 .. n - 1, each once.
__device__ __forceinline__ int list_rank(const float* cd, const int* cj, int n, int i) {
  const float d = cd[i];
  const int j = cj[i];
  int r = 0;
#pragma unroll 8
  for (int e = 0; e < n; ++e) r += cd[e] < d || (cd[e] == d && cj[e] < j);
  return r;
}

// The k nearest of several ascending k-lists held in shared memory (list w:
// entries [w * stride, w * stride + k) of cd, cj; an empty entry has slot
// INT_MAX), by the whole block.  No entry above the smallest k-th distance
// of a full list can rank below k (that list alone holds k entries at or
// below it), so only entries at or below it are ranked: usually little more
// than k of them.  Writes the m = min(k, valid entries) nearest, in order,
// to od, oj and returns m.  Distances are non-negative (sums of squares), so
// their bit patterns order like their values.
template <int N>  // at most N entries
struct SelectScratch {
  float sd[N];
  int sj[N];
  unsigned tau;
  int n;
};
template <int N>
__device__ __forceinline__ int select_k(const float* cd, const int* cj, int n, int stride, int k,
                                        SelectScratch<N>& x, float* od, int* oj) {
  const int tid = threadIdx.x, nt = blockDim.x;
  if (tid == 0) {
    x.tau = __float_as_uint(FLT_MAX);
    x.n = 0;
  }
  __syncthreads();
  for (int i0 = 0; i0 < n; i0 += nt) {
    // the warp's smallest k-th distance first, then one atomic per warp
    const int i = i0 + tid;
    unsigned v = (i < n && i % stride == k - 1 && cj[i] != INT_MAX) ? __float_as_uint(cd[i]) : 0xffffffffu;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((tid & 31) == 0 && v != 0xffffffffu) atomicMin(&x.tau, v);
  }
  __syncthreads();
  const float tau = __uint_as_float(x.tau);
  for (int i = tid; i < n; i += nt)
    if (i % stride < k && cj[i] != INT_MAX && cd[i] <= tau) {
      const int q = atomicAdd(&x.n, 1);
      x.sd[q] = cd[i];
      x.sj[q] = cj[i];
    }
  __syncthreads();
  const int m = x.n;
  for (int i = tid; i < m; i += nt) {
    const int r = list_rank(x.sd, x.sj, m, i);
    if (r < k) {
      od[r] = x.sd[i];
      oj[r] = x.sj[i];
    }
  }
  __syncthreads();
  return m < k ? m : k;
}
}  // namespace

// New reference rows j in [j0, j1): copy K and V of token j s into the
// reference planes.
template <typename E>
__global__ void append_refs_kernel(int s, int d_h, int H, int64_t j0, int64_t n_ref_cap, const E* __restrict__ K,
                                   const E* __restrict__ V, int64_t sb, int64_t sh, int64_t st,
                                   E* __restrict__ refk, E* __restrict__ refv) {
  const int b = blockIdx.z, h = blockIdx.y;
  const int64_t j = j0 + blockIdx.x, t = j * s, bh = (int64_t)b * H + h;
  const E* kr = K + b * sb + h * sh + t * st;
  const E* vr = V + b * sb + h * sh + t * st;
  for (int e = threadIdx.x; e < d_h; e += blockDim.x) {
    refk[(bh * n_ref_cap + j) * d_h + e] = kr[e];
    refv[(bh * n_ref_cap + j) * d_h + e] = vr[e];
  }
}

struct AppendParams {
  int s, d_h, H, k, d_c, hidden, act;
  __nv_bfloat16* cscale;  // per-row scales of 4-bit codes, else null
  int64_t row0;  // first code row of the call
  int64_t n_ref_cap, n_code_cap;
  int64_t sb, sh, st;
  uint32_t* err;
};

// Reference scan: one (new non-reference token, slice of its references,
// sequence x kv-head) per CTA.  The token's code row is row0 + blockIdx.y;
// the slice is references [blockIdx.x * per, (blockIdx.x + 1) * per) of the
// slots j with j s < t.  Lane l of a warp holds elements [NV l, NV l + NV)
// of [K ; V] (D = 32 NV); the warps take groups of kAppendRows rows in turn,
// with every row of a group in flight, and keep a k-list each, held alike by
// all lanes: a group's distances that beat the list's k-th entry (usually
// none once the list has filled) are inserted one at a time in slot order.
// The warps' lists meet by rank in shared memory; the slice's k nearest
// (distance, slot) go to the scratch list of (token, slice).
template <typename E, int NV>
__global__ void __launch_bounds__(kScanThreads, 2)
    append_scan_kernel(const AppendParams P, int per, const E* __restrict__ K, const E* __restrict__ V,
                       const E* __restrict__ refk, const E* __restrict__ refv, float* __restrict__ lists) {
  __shared__ float cd[kScanWarps * kAppendKMax];
  __shared__ int cj[kScanWarps * kAppendKMax];
  __shared__ SelectScratch<kScanWarps * kAppendKMax> sx;
  __shared__ float od[kAppendKMax];
  __shared__ int oj[kAppendKMax];
  // K, V and the reference planes may have been written by the kernel
  // before this one on the stream; the finish kernel may start staging its
  // weights as soon as every scan CTA is running
  grid_dep_wait();
  grid_dep_launch();
  const int bh = blockIdx.z, b = bh / P.H, h = bh % P.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d_h = P.d_h, k = P.k;
  const int64_t row = P.row0 + blockIdx.y;
  const int64_t t = token_of_code_row(row, P.s);
  const int e0 = lane * NV;  // this lane's elements (D = 32 NV)
  const bool inK = e0 < d_h;
  float x[NV];
  {
    Frag<E, NV> f;
    f.ldcg((inK ? K + e0 : V + (e0 - d_h)) + b * P.sb + h * P.sh + t * P.st);
#pragma unroll
    for (int i = 0; i < NV; ++i) x[i] = f[i];
  }
  const int64_t ns = (t + P.s - 1) / P.s;  // slots j with j s < t
  const int64_t jlo = (int64_t)blockIdx.x * per, jhi = jlo + per < ns ? jlo + per : ns;
  const E* rs = (inK ? refk + e0 : refv + (e0 - d_h)) + (int64_t)bh * P.n_ref_cap * d_h;
  float bd[kAppendKMax];
  int bi[kAppendKMax];
#pragma unroll
  for (int i = 0; i < kAppendKMax; ++i) {
    bd[i] = FLT_MAX;
    bi[i] = INT_MAX;
  }
  float thr = FLT_MAX;  // the list's k-th distance
  const int mine = (lane >> 2) & 7;  // the row whose distance this lane ends with
  // rows of this warp's next group, in flight while the current one is used
  constexpr int64_t kStep = (int64_t)kScanWarps * kAppendRows;
  Frag<E, NV> nxt[kAppendRows];
  auto fetch = [&](int64_t g0) {
#pragma unroll
    for (int u = 0; u < kAppendRows; ++u) {
      if (g0 + u < jhi) nxt[u].ldcg(rs + (g0 + u) * d_h);
      else nxt[u].zero();
    }
  };
  fetch(jlo + (int64_t)warp * kAppendRows);
  for (int64_t j0 = jlo + (int64_t)warp * kAppendRows; j0 < jhi; j0 += kStep) {
    Frag<E, NV> v[kAppendRows];
#pragma unroll
    for (int u = 0; u < kAppendRows; ++u) v[u] = nxt[u];
    if (j0 + kStep < jhi) fetch(j0 + kStep);
    float part[kAppendRows];
#pragma unroll
    for (int u = 0; u < kAppendRows; ++u) {
      float a = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const float df = x[i] - v[u][i];
        a = fmaf(df, df, a);
      }
      part[u] = a;
    }
    const float d = warp_sum8(part, lane);
    unsigned m = __ballot_sync(0xffffffffu, (lane & 3) == 0 && j0 + mine < jhi && d < thr);
    while (m) {
      const int src = __ffs(m) - 1;
      const float dd = __shfl_sync(0xffffffffu, d, src);
      topk_insert_inorder<kAppendKMax>(bd, bi, dd, (int)(j0 + (src >> 2)));
      thr = kth_entry<kAppendKMax>(bd, k);
      m &= m - 1;
      m &= __ballot_sync(0xffffffffu, d < thr);
    }
  }
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < kAppendKMax; ++i) {
      cd[warp * kAppendKMax + i] = bd[i];
      cj[warp * kAppendKMax + i] = i < k ? bi[i] : INT_MAX;
    }
  __syncthreads();
  const int m = select_k(cd, cj, kScanWarps * kAppendKMax, kAppendKMax, k, sx, od, oj);
  float* o = lists + (((int64_t)bh * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * (2 * kAppendKMax);
  if (tid < k) {
    o[tid] = tid < m ? od[tid] : FLT_MAX;
    o[kAppendKMax + tid] = __int_as_float(tid < m ? oj[tid] : INT_MAX);
  }
}

// Shared memory of the finish kernel beyond its static arrays: W1 then W2
// when they are bf16 (at most 160 KB for d_h <= 128, hidden <= 256 and
// d_c <= 64), staged by bulk copies; float32 weights are read from global
// memory after an L2 prefetch.
template <typename E>
static size_t finish_weight_bytes(int d_h, int hidden, int d_c) {
  return ((size_t)hidden * 2 * d_h + (size_t)d_c * hidden) * sizeof(E);
}

// Finish one new non-reference token of one (sequence, kv-head): merge the
// slices' lists into the k nearest, r = x_t - their mean, the compressor
// MLP, and the code and slot rows.  Launched behind the scan kernel with
// programmatic stream serialisation: everything before grid_dep_wait() (the
// weights' copy into shared memory, the token's own row) overlaps the scan.
template <typename E, int NV>
__global__ void __launch_bounds__(kFinishThreads, 1)
    append_finish_kernel(const AppendParams P, int nsplit, const E* __restrict__ K, const E* __restrict__ V,
                         const E* __restrict__ W1, const float* __restrict__ b1, const E* __restrict__ W2,
                         const float* __restrict__ b2, const E* __restrict__ refk, const E* __restrict__ refv,
                         const float* __restrict__ lists, E* __restrict__ code, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char wsm[];
  __shared__ float xs[2 * 128], r[2 * 128], cbuf[64];
  __shared__ __align__(16) float hbuf[kMaxHidden];
  __shared__ float md[kAppendKMax][2 * 128];
  __shared__ float cd[kAppendSplitMax * kAppendKMax];
  __shared__ int cj[kAppendSplitMax * kAppendKMax];
  __shared__ SelectScratch<kAppendSplitMax * kAppendKMax> sx;
  __shared__ float seld[kAppendKMax];
  __shared__ int sel[kAppendKMax];
  __shared__ __align__(8) uint64_t wbar;
  const int bh = blockIdx.z, b = bh / P.H, h = bh % P.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d_h = P.d_h, D = 2 * d_h, k = P.k;
  const int64_t row = P.row0 + blockIdx.y;
  const int64_t t = token_of_code_row(row, P.s);
  const uint32_t w1_bytes = (uint32_t)(P.hidden * D * sizeof(E)), w2_bytes = (uint32_t)(P.d_c * P.hidden * sizeof(E));
  constexpr bool kSmemW = sizeof(E) == 2;
  const E* w1 = W1;
  const E* w2 = W2;
  if constexpr (kSmemW) {
    if (tid == 0) {
      mbar_init(&wbar, 1);
      fence_mbar_init();
      mbar_arrive_expect_tx(&wbar, w1_bytes + w2_bytes);
      constexpr uint32_t kPiece = 32 * 1024;
      for (uint32_t o = 0; o < w1_bytes; o += kPiece)
        bulk_load(wsm + o, reinterpret_cast<const unsigned char*>(W1) + o, min(kPiece, w1_bytes - o), &wbar);
      bulk_load(wsm + w1_bytes, W2, w2_bytes, &wbar);
    }
    w1 = reinterpret_cast<const E*>(wsm);
    w2 = reinterpret_cast<const E*>(wsm + w1_bytes);
  } else {
    for (uint32_t o = tid * 128u; o < w1_bytes; o += kFinishThreads * 128u)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const unsigned char*>(W1) + o));
    for (uint32_t o = tid * 128u; o < w2_bytes; o += kFinishThreads * 128u)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const unsigned char*>(W2) + o));
  }
  for (int e = tid; e < D; e += kFinishThreads)
    xs[e] = to_f(e < d_h ? K[b * P.sb + h * P.sh + t * P.st + e] : V[b * P.sb + h * P.sh + t * P.st + (e - d_h)]);
  grid_dep_launch();
  grid_dep_wait();  // the scan's lists are complete and visible
  // merge: the first k entries of every slice's list, ranked together
  const int n = nsplit * k;
  const float* l = lists + ((int64_t)bh * gridDim.y + blockIdx.y) * nsplit * (2 * kAppendKMax);
  for (int i = tid; i < n; i += kFinishThreads) {
    const int sp = i / k, q = i - sp * k;
    cd[i] = __ldcg(l + sp * 2 * kAppendKMax + q);
    cj[i] = __float_as_int(__ldcg(l + sp * 2 * kAppendKMax + kAppendKMax + q));
  }
  __syncthreads();
  const int k_eff = select_k(cd, cj, n, k, k, sx, seld, sel);
  // r = x_t - mean of the chosen references: warp q loads reference sel[q]
  if (warp < k_eff) {
    const int e0 = lane * NV;
    const bool inK = e0 < d_h;
    const E* rs = (inK ? refk + e0 : refv + (e0 - d_h)) + (int64_t)bh * P.n_ref_cap * d_h;
    Frag<E, NV> f;
    f.ldcg(rs + (int64_t)sel[warp] * d_h);
#pragma unroll
    for (int i = 0; i < NV; ++i) md[warp][e0 + i] = f[i];
  }
  __syncthreads();
  {
    const float inv = 1.0f / (float)(k_eff > 0 ? k_eff : 1);
    for (int e = tid; e < D; e += kFinishThreads) {
      float m = 0.f;
      for (int q = 0; q < k_eff; ++q) m += md[q][e];
      r[e] = xs[e] - m * inv;
    }
  }
  __syncthreads();
  if constexpr (kSmemW) {
    // every thread sees the copies land (bounded), then all leave together
    // if any wait ran out
    if (!__syncthreads_and(mbar_wait_drain(&wbar, 0))) {
      if (tid == 0) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 30);
      return;
    }
  }
  // hidden = act(W1 r + b1): a warp takes 8 weight rows at a time, lane l
  // multiplying elements [NV l, NV l + NV) of each (hidden is a multiple of
  // 32, so of 8)
  {
    float rr[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) rr[i] = r[lane * NV + i];
    for (int u0 = warp * kAppendRows; u0 < P.hidden; u0 += kFinishWarps * kAppendRows) {
      Frag<E, NV> wv[kAppendRows];
#pragma unroll
      for (int u = 0; u < kAppendRows; ++u) wv[u].ld(w1 + (int64_t)(u0 + u) * D + lane * NV);
      float part[kAppendRows];
#pragma unroll
      for (int u = 0; u < kAppendRows; ++u) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) a = fmaf(wv[u][i], rr[i], a);
        part[u] = a;
      }
      const float s = warp_sum8(part, lane);
      if ((lane & 3) == 0) {
        const int u = u0 + ((lane >> 2) & 7);
        hbuf[u] = act_eval(P.act, s + (b1 ? b1[u] : 0.f));
      }
    }
  }
  __syncthreads();
  // code = W2 hidden + b2: a warp takes 8 outputs (d_c <= 64: one pass),
  // lane l over elements 4 l, 4 l + 128, ... of each row
  for (int o0 = warp * kAppendRows; o0 < P.d_c; o0 += kFinishWarps * kAppendRows) {
    float part[kAppendRows];
#pragma unroll
    for (int u = 0; u < kAppendRows; ++u) part[u] = 0.f;
    for (int c = lane * 4; c < P.hidden; c += 128) {
      const float4 hv = *reinterpret_cast<const float4*>(&hbuf[c]);
#pragma unroll
      for (int u = 0; u < kAppendRows; ++u) {
        if (o0 + u < P.d_c) {
          Frag<E, 4> wv;
          wv.ld(w2 + (int64_t)(o0 + u) * P.hidden + c);
          part[u] = fmaf(wv[0], hv.x, fmaf(wv[1], hv.y, fmaf(wv[2], hv.z, fmaf(wv[3], hv.w, part[u]))));
        }
      }
    }
    const float acc = warp_sum8(part, lane);
    const int o = o0 + ((lane >> 2) & 7);
    if ((lane & 3) == 0 && o < P.d_c) {
      const float cv = acc + (b2 ? b2[o] : 0.f);
      if (P.cscale) cbuf[o] = cv;
      else code[((int64_t)bh * P.n_code_cap + row) * P.d_c + o] = from_f<E>(cv);
    }
  }
  if (P.cscale) {
    // 4-bit codes: the whole row's scale first, then the packed nibbles
    __syncthreads();
    if (tid == 0) {
      float amax = 0.f;
      for (int o = 0; o < P.d_c; ++o) amax = fmaxf(amax, fabsf(cbuf[o]));
      const __nv_bfloat16 sb = __float2bfloat16_rn(amax / 7.0f);
      const float sc = __bfloat162float(sb);
      uint8_t* c8 = reinterpret_cast<uint8_t*>(code) + ((int64_t)bh * P.n_code_cap + row) * (P.d_c / 2);
      for (int o = 0; o < P.d_c; o += 2) {
        int q0 = 0, q1 = 0;
        if (sc > 0.f) {
          q0 = (int)fminf(fmaxf(rintf(__fdiv_rn(cbuf[o], sc)), -7.f), 7.f);
          q1 = (int)fminf(fmaxf(rintf(__fdiv_rn(cbuf[o + 1], sc)), -7.f), 7.f);
        }
        c8[o / 2] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
      }
      P.cscale[(int64_t)bh * P.n_code_cap + row] = sb;
    }
  }
  if (tid < k) idx[((int64_t)bh * P.n_code_cap + row) * k + tid] = tid < k_eff ? sel[tid] : -1;
}

// Launch with programmatic stream serialisation: the grid may start while
// the previous kernel on the stream is still running, and waits for it in
// grid_dep_wait().
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename E, int NV>
static cudaError_t launch_rows(const AppendParams& P, int per, int nsplit, dim3 gs, dim3 gf, const KVView& kv,
                               const void* W1, const float* b1, const void* W2, const float* b2, const E* refk,
                               const E* refv, float* lists, E* code, int32_t* idx, cudaStream_t st) {
  cudaError_t e = launch_pdl(append_scan_kernel<E, NV>, gs, dim3(kScanThreads), 0, st, P, per, (const E*)kv.K,
                             (const E*)kv.V, refk, refv, lists);
  if (e != cudaSuccess) return e;
  const size_t wb = sizeof(E) == 2 ? finish_weight_bytes<E>(P.d_h, P.hidden, P.d_c) : 0;
  if (wb) {
    e = cudaFuncSetAttribute(append_finish_kernel<E, NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wb);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(append_finish_kernel<E, NV>, gf, dim3(kFinishThreads), wb, st, P, nsplit, (const E*)kv.K,
                    (const E*)kv.V, (const E*)W1, b1, (const E*)W2, b2, refk, refv, (const float*)lists, code, idx);
}

template <typename E>
static cudaError_t append_launch(const Plan& p, int T0, int T1, const KVView& kv, const void* W1, const float* b1,
                                 const void* W2, const float* b2, void* cache, void* ws, cudaStream_t st) {
  const auto& c = p.cfg;
  char* cb = (char*)cache;
  E* refk = (E*)(cb + p.off_refk);
  E* refv = (E*)(cb + p.off_refv);
  const int64_t j0 = n_ref_of(T0, c.stride_s), j1 = n_ref_of(T1, c.stride_s);
  if (j1 > j0) {
    ProfScope ps(p, st, KID_APPEND_REFS);
    append_refs_kernel<E><<<dim3((unsigned)(j1 - j0), c.kv_heads, c.batch), 128, 0, st>>>(
        c.stride_s, c.d_h, c.kv_heads, j0, p.n_ref_cap, (const E*)kv.K, (const E*)kv.V, kv.sb, kv.sh, kv.st, refk,
        refv);
  }
  const int64_t r0 = n_code_of(T0, c.stride_s), r1 = n_code_of(T1, c.stride_s);
  if (r1 > r0) {
    AppendParams P;
    P.s = c.stride_s;
    P.d_h = c.d_h;
    P.H = c.kv_heads;
    P.k = c.k;
    P.d_c = c.d_c;
    P.hidden = c.hidden;
    P.act = (int)c.act;
    P.row0 = r0;
    P.n_ref_cap = p.n_ref_cap;
    P.n_code_cap = p.n_code_cap;
    P.cscale = p.code4 ? (__nv_bfloat16*)(cb + p.off_cscale) : nullptr;
    P.sb = kv.sb;
    P.sh = kv.sh;
    P.st = kv.st;
    P.err = (uint32_t*)ws;
    // split each token's references over enough CTAs for two per SM; the
    // slices' lists live in the compress region's candidate plane, so long
    // appends go in chunks of rows that fit it
    const int64_t rows = r1 - r0, BH = (int64_t)c.batch * c.kv_heads;
    const int64_t ns_max = n_ref_of(T1, c.stride_s);
    const int64_t list_bytes = 2 * kAppendKMax * 4;
    const int64_t scratch = std::max<int64_t>((int64_t)BH * p.n_code_cap * p.KC * 4, BH * 4096);
    float* lists = (float*)((char*)ws + p.ws_cand);
    E* code = (E*)(cb + p.off_code);
    int32_t* idx = (int32_t*)(cb + p.off_idx);
    ProfScope ps(p, st, KID_APPEND_ROWS);
    for (int64_t c0 = 0; c0 < rows;) {
      const int64_t left = rows - c0;
      int64_t nsplit = (2 * kNumSMs + left * BH - 1) / (left * BH);
      nsplit = std::min<int64_t>(std::min<int64_t>(nsplit, kAppendSplitMax),
                                 std::max<int64_t>(1, ns_max / (kScanWarps * kAppendRows)));
      nsplit = std::max<int64_t>(std::min<int64_t>(nsplit, scratch / (BH * list_bytes)), 1);
      const int64_t n = std::min<int64_t>(left, std::max<int64_t>(1, scratch / (BH * nsplit * list_bytes)));
      P.row0 = r0 + c0;
      const int per = (int)((ns_max + nsplit - 1) / nsplit);
      const dim3 gs((unsigned)nsplit, (unsigned)n, (unsigned)BH), gf(1, (unsigned)n, (unsigned)BH);
      const cudaError_t e =
          c.d_h == 128
              ? launch_rows<E, 8>(P, per, (int)nsplit, gs, gf, kv, W1, b1, W2, b2, refk, refv, lists, code, idx, st)
              : launch_rows<E, 4>(P, per, (int)nsplit, gs, gf, kv, W1, b1, W2, b2, refk, refv, lists, code, idx, st);
      if (e != cudaSuccess) return e;
      c0 += n;
    }
  }
  return cudaGetLastError();
}

cudaError_t launch_append(const Plan& p, int T0, int T1, const KVView& kv, const void* W1, const float* b1,
                          const void* W2, const float* b2, void* cache, void* ws, cudaStream_t st) {
  if (p.bf16)
    return append_launch<__nv_bfloat16>(p, T0, T1, kv, W1, b1, W2, b2, cache, ws, st);
  return append_launch<float>(p, T0, T1, kv, W1, b1, W2, b2, cache, ws, st);
}

}  // namespace dkv
