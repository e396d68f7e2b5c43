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

namespace dkv {

namespace {
constexpr int kAppendThreads = 512;
constexpr int kAppendWarps = kAppendThreads / 32;
constexpr int kAppendKMax = 8;   // references per token (k <= 8)
constexpr int kAppendRows = 8;   // reference rows in flight per warp

// N consecutive elements as floats (N = 4 or 8; 8- to 32-byte aligned).
template <int N>
__device__ __forceinline__ void loadv(const __nv_bfloat16* p, float (&v)[N]) {
#pragma unroll
  for (int c = 0; c < N; c += 4) {
    const uint2 r = __ldg(reinterpret_cast<const uint2*>(p + c));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
    const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
    v[c] = f0.x;
    v[c + 1] = f0.y;
    v[c + 2] = f1.x;
    v[c + 3] = f1.y;
  }
}
template <int N>
__device__ __forceinline__ void loadv(const float* p, float (&v)[N]) {
#pragma unroll
  for (int c = 0; c < N; c += 4) {
    const float4 r = __ldg(reinterpret_cast<const float4*>(p + c));
    v[c] = r.x;
    v[c + 1] = r.y;
    v[c + 2] = r.z;
    v[c + 3] = r.w;
  }
}
}  // namespace

// Insert (d, j) into a list sorted by (distance, slot), branch-free: every
// position is computed from the old list directly.  No-op when (d, j) does
// not precede the last entry.
template <int KC>
__device__ __forceinline__ void topk_insert_any(float (&bd)[KC], int (&bi)[KC], float d, int j) {
  bool lt[KC];
#pragma unroll
  for (int i = 0; i < KC; ++i) lt[i] = d < bd[i] || (d == bd[i] && j < bi[i]);
#pragma unroll
  for (int i = KC - 1; i > 0; --i) {
    bd[i] = lt[i - 1] ? bd[i - 1] : (lt[i] ? d : bd[i]);
    bi[i] = lt[i - 1] ? bi[i - 1] : (lt[i] ? j : bi[i]);
  }
  bd[0] = lt[0] ? d : bd[0];
  bi[0] = lt[0] ? j : bi[0];
}

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
// with every row of a group in flight.  Writes the slice's k nearest
// (distance, slot) to the scratch list of (token, slice).
template <typename E, int NV>
__global__ void __launch_bounds__(kAppendThreads)
    append_scan_kernel(const AppendParams P, int per, const E* __restrict__ K, const E* __restrict__ V,
                       const E* __restrict__ refk, const E* __restrict__ refv, float* __restrict__ lists) {
  __shared__ float wd[kAppendWarps][kAppendKMax];
  __shared__ int wj[kAppendWarps][kAppendKMax];
  const int bh = blockIdx.z, b = bh / P.H, h = bh % P.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d_h = P.d_h;
  const int64_t row = P.row0 + blockIdx.y;
  const int64_t t = token_of_code_row(row, P.s);
  const int e0 = lane * NV;  // this lane's elements (D = 32 NV)
  const bool inK = e0 < d_h;
  float x[NV];
  loadv<NV>((inK ? K + e0 : V + (e0 - d_h)) + b * P.sb + h * P.sh + t * P.st, x);
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
  for (int64_t j0 = jlo + (int64_t)warp * kAppendRows; j0 < jhi; j0 += (int64_t)kAppendWarps * kAppendRows) {
    float v[kAppendRows][NV];
#pragma unroll
    for (int u = 0; u < kAppendRows; ++u)
      if (j0 + u < jhi) loadv<NV>(rs + (j0 + u) * d_h, v[u]);
#pragma unroll
    for (int u = 0; u < kAppendRows; ++u) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const float df = x[i] - v[u][i];
        part = fmaf(df, df, part);
      }
      const float d = warp_sum(part);
      if (lane == 0 && j0 + u < jhi) topk_insert_inorder<kAppendKMax>(bd, bi, d, (int)(j0 + u));
    }
  }
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < kAppendKMax; ++i) {
      wd[warp][i] = bd[i];
      wj[warp][i] = bi[i];
    }
  __syncthreads();
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kAppendKMax; ++i) {
      bd[i] = FLT_MAX;
      bi[i] = INT_MAX;
    }
    for (int w = 0; w < kAppendWarps; ++w)
      for (int i = 0; i < kAppendKMax; ++i)
        if (wj[w][i] != INT_MAX) topk_insert<kAppendKMax>(bd, bi, wd[w][i], wj[w][i]);
    float* o = lists + (((int64_t)bh * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * (2 * kAppendKMax);
    for (int i = 0; i < kAppendKMax; ++i) {
      o[i] = bd[i];
      o[kAppendKMax + i] = __int_as_float(bi[i]);
    }
  }
}

// Finish one new non-reference token of one (sequence, kv-head): merge the
// slices' lists into the k nearest, r = x_t - their mean, the compressor
// MLP, and the code and slot rows.
template <typename E, int NV>
__global__ void __launch_bounds__(kAppendThreads)
    append_finish_kernel(const AppendParams P, int nsplit, const E* __restrict__ K, const E* __restrict__ V,
                         const E* __restrict__ W1, const float* __restrict__ b1, const E* __restrict__ W2,
                         const float* __restrict__ b2, const E* __restrict__ refk, const E* __restrict__ refv,
                         const float* __restrict__ lists, E* __restrict__ code, int32_t* __restrict__ idx) {
  __shared__ float r[2 * 128], hbuf[kMaxHidden], cbuf[64];
  __shared__ int sel[kAppendKMax], sel_n;
  const int bh = blockIdx.z, b = bh / P.H, h = bh % P.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d_h = P.d_h, D = 2 * d_h;
  const int64_t row = P.row0 + blockIdx.y;
  const int64_t t = token_of_code_row(row, P.s);
  if (warp == 0) {
    // merge the slices' lists: lane l folds slices l, l + 32, ..., then the
    // lanes' lists meet in a shuffle tree
    float bd[kAppendKMax];
    int bi[kAppendKMax];
#pragma unroll
    for (int i = 0; i < kAppendKMax; ++i) {
      bd[i] = FLT_MAX;
      bi[i] = INT_MAX;
    }
    const float* l = lists + ((int64_t)bh * gridDim.y + blockIdx.y) * nsplit * (2 * kAppendKMax);
    for (int sp = lane; sp < nsplit; sp += 32)
#pragma unroll
      for (int i = 0; i < kAppendKMax; ++i) {
        const int j = __float_as_int(l[sp * 2 * kAppendKMax + kAppendKMax + i]);
        topk_insert_any<kAppendKMax>(bd, bi, l[sp * 2 * kAppendKMax + i], j);
      }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      float od[kAppendKMax];
      int oj[kAppendKMax];
#pragma unroll
      for (int i = 0; i < kAppendKMax; ++i) {
        od[i] = __shfl_xor_sync(0xffffffffu, bd[i], o);
        oj[i] = __shfl_xor_sync(0xffffffffu, bi[i], o);
      }
#pragma unroll
      for (int i = 0; i < kAppendKMax; ++i)
        topk_insert_any<kAppendKMax>(bd, bi, od[i], oj[i]);
    }
    if (lane == 0) {
      int n = 0;
      for (int i = 0; i < P.k; ++i)
        if (bi[i] != INT_MAX) sel[n++] = bi[i];
      sel_n = n;
    }
  }
  __syncthreads();
  const int k_eff = sel_n;
  // r = x_t - mean of the chosen references (warp 0: lane l, elements NV l..)
  if (warp == 0) {
    const int e0 = lane * NV;
    const bool inK = e0 < d_h;
    float x[NV], m[NV];
    loadv<NV>((inK ? K + e0 : V + (e0 - d_h)) + b * P.sb + h * P.sh + t * P.st, x);
    const E* rs = (inK ? refk + e0 : refv + (e0 - d_h)) + (int64_t)bh * P.n_ref_cap * d_h;
#pragma unroll
    for (int i = 0; i < NV; ++i) m[i] = 0.f;
    for (int q = 0; q < k_eff; ++q) {
      float v[NV];
      loadv<NV>(rs + (int64_t)sel[q] * d_h, v);
#pragma unroll
      for (int i = 0; i < NV; ++i) m[i] += v[i];
    }
    const float inv = 1.0f / (float)(k_eff > 0 ? k_eff : 1);
#pragma unroll
    for (int i = 0; i < NV; ++i) r[e0 + i] = x[i] - m[i] * inv;
  }
  __syncthreads();
  // code = W2 act(W1 r + b1) + b2: a warp per weight row at a time, lane l
  // multiplying elements [NV l, NV l + NV) of the row (D = 32 NV; hidden is
  // a multiple of 32, so a W2 row is hidden / 32 elements a lane)
  {
    float rr[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) rr[i] = r[lane * NV + i];
    for (int u = warp; u < P.hidden; u += kAppendWarps) {
      float wv[NV];
      loadv<NV>(W1 + (int64_t)u * D + lane * NV, wv);
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < NV; ++i) acc = fmaf(wv[i], rr[i], acc);
      acc = warp_sum(acc);
      if (lane == 0) hbuf[u] = act_eval(P.act, acc + (b1 ? b1[u] : 0.f));
    }
  }
  __syncthreads();
  for (int o = warp; o < P.d_c; o += kAppendWarps) {
    float acc = 0.f;
    const E* w = W2 + (int64_t)o * P.hidden;
    for (int u = lane * 4; u < P.hidden; u += 128) {
      float wv[4];
      loadv<4>(w + u, wv);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc = fmaf(wv[i], hbuf[u + i], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
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
  if (tid < P.k) idx[((int64_t)bh * P.n_code_cap + row) * P.k + tid] = tid < k_eff ? sel[tid] : -1;
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
    // split each token's references over enough CTAs to fill the GPU; the
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
      nsplit = std::min<int64_t>(std::min<int64_t>(nsplit, 64),
                                 std::max<int64_t>(1, ns_max / (kAppendWarps * kAppendRows)));
      nsplit = std::max<int64_t>(std::min<int64_t>(nsplit, scratch / (BH * list_bytes)), 1);
      const int64_t n = std::min<int64_t>(left, std::max<int64_t>(1, scratch / (BH * nsplit * list_bytes)));
      P.row0 = r0 + c0;
      const int per = (int)((ns_max + nsplit - 1) / nsplit);
      const dim3 gs((unsigned)nsplit, (unsigned)n, (unsigned)BH), gf(1, (unsigned)n, (unsigned)BH);
      if (c.d_h == 128) {
        append_scan_kernel<E, 8><<<gs, kAppendThreads, 0, st>>>(P, per, (const E*)kv.K, (const E*)kv.V, refk, refv,
                                                                lists);
        append_finish_kernel<E, 8><<<gf, kAppendThreads, 0, st>>>(P, (int)nsplit, (const E*)kv.K, (const E*)kv.V,
                                                                  (const E*)W1, b1, (const E*)W2, b2, refk, refv,
                                                                  lists, code, idx);
      } else {
        append_scan_kernel<E, 4><<<gs, kAppendThreads, 0, st>>>(P, per, (const E*)kv.K, (const E*)kv.V, refk, refv,
                                                                lists);
        append_finish_kernel<E, 4><<<gf, kAppendThreads, 0, st>>>(P, (int)nsplit, (const E*)kv.K, (const E*)kv.V,
                                                                  (const E*)W1, b1, (const E*)W2, b2, refk, refv,
                                                                  lists, code, idx);
      }
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
