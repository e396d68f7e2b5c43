// compress_simt.cu -- reference packing, the CUDA-core nearest-reference
// search, the fused gather-mean-residual + compressor MLP (encode) and the
// debug reconstruction.
//
// Method: DeltaKV (gist.science summary, section 3 "Metodologia"):
//   "Struttura della Compressione"  references every s-th token, kept whole;
//   "Processo di Compressione" 1    k most similar earlier references by L2;
//   step 2                          their mean KV_R;
//   step 3                          residual x_t - KV_R;
//   step 4                          light MLP compressor to d_c;
//   "Ricostruzione"                 KV_R + decompressed residual.
#include <cfloat>
#include <climits>

#include "common.cuh"

namespace dkv {

// ---------------------------------------------------------------- refpack
// Copy reference rows (token j*s) into the cache's ref planes and store half
// their squared norm, 0.5 * |x_j|^2, for the tensor-core distance kernel.
// One warp per reference row.
template <typename T>
__global__ void refpack_kernel(int s, int d_h, int H, int64_t n_ref, int64_t n_ref_cap,
                               const T* __restrict__ K, const T* __restrict__ V, int64_t sb,
                               int64_t sh, int64_t st, T* __restrict__ refk,
                               T* __restrict__ refv, float* __restrict__ hnorm,
                               __nv_bfloat16* __restrict__ hsplit) {
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t j = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (j >= n_ref) return;
  const int64_t t = j * s;
  const T* kr = K + b * sb + h * sh + t * st;
  const T* vr = V + b * sb + h * sh + t * st;
  const int64_t bh = (int64_t)b * H + h;
  T* ok = refk + (bh * n_ref_cap + j) * d_h;
  T* ov = refv + (bh * n_ref_cap + j) * d_h;
  float acc = 0.f;
  for (int e = lane; e < d_h; e += 32) {
    T a = kr[e], c = vr[e];
    ok[e] = a;
    ov[e] = c;
    float fa = to_f(a), fc = to_f(c);
    acc = fmaf(fa, fa, acc);
    acc = fmaf(fc, fc, acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) hnorm[bh * n_ref_cap + j] = 0.5f * acc;
  if (hsplit != nullptr && lane < 2) {
    // h = 0.5 |x_j|^2 = hi + mid + lo in bf16 (24 significant bits), then
    // zeros: the K = 16 row that the distance kernel's last MMA adds
    const float hv = 0.5f * acc;
    const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
    const float r1 = hv - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    __align__(16) __nv_bfloat16 row[8];
    for (int i = 0; i < 8; ++i) row[i] = __float2bfloat16_rn(0.f);
    if (lane == 0) {
      row[0] = hi;
      row[1] = mid;
      row[2] = lo;
    }
    reinterpret_cast<uint4*>(hsplit + (bh * n_ref_cap + j) * 16)[lane] = *reinterpret_cast<const uint4*>(row);
  }
}

cudaError_t launch_refpack(const Plan& p, int T, const KVView& kv, void* cache, void* ws,
                           cudaStream_t st) {
  const auto& c = p.cfg;
  int64_t n_ref = n_ref_of(T, c.stride_s);
  if (n_ref == 0) return cudaSuccess;
  dim3 grid((unsigned)ceil_div64(n_ref, 8), c.kv_heads, c.batch);
  char* cb = (char*)cache;
  float* hn = (float*)((char*)ws + p.ws_hnorm);
  ProfScope ps(p, st, KID_REFPACK);
  if (p.bf16) {
    using T_ = __nv_bfloat16;
    refpack_kernel<T_><<<grid, 256, 0, st>>>(c.stride_s, c.d_h, c.kv_heads, n_ref, p.n_ref_cap,
                                             (const T_*)kv.K, (const T_*)kv.V, kv.sb, kv.sh,
                                             kv.st, (T_*)(cb + p.off_refk),
                                             (T_*)(cb + p.off_refv), hn,
                                             (__nv_bfloat16*)((char*)ws + p.ws_hsplit));
  } else {
    refpack_kernel<float><<<grid, 256, 0, st>>>(c.stride_s, c.d_h, c.kv_heads, n_ref,
                                                 p.n_ref_cap, (const float*)kv.K,
                                                 (const float*)kv.V, kv.sb, kv.sh, kv.st,
                                                 (float*)(cb + p.off_refk),
                                                 (float*)(cb + p.off_refv), hn, nullptr);
  }
  return cudaGetLastError();
}

// --------------------------------------------------- candidate search (SIMT)
// For each token of a 64-token tile, the KC nearest earlier references by
// squared L2 distance over [K ; V], computed directly as sum (x - r)^2 in
// fp32 on CUDA cores.  References are staged 32 at a time in shared memory;
// each thread owns one token and keeps its KC best in registers.  Used for
// float32 caches (whose tolerance leaves no room for tensor-core rounding)
// and for shapes the tensor-core kernel does not cover.
constexpr int kCandTile = 64;
constexpr int kCandRefChunk = 32;

template <typename T, int KC>
__global__ void __launch_bounds__(kCandTile)
    cand_simt_kernel(int T_, int s, int d_h, int H, int64_t n_ref_cap, int64_t n_code_cap,
                     const T* __restrict__ K, const T* __restrict__ V, int64_t sb, int64_t sh,
                     int64_t st, const T* __restrict__ refk, const T* __restrict__ refv,
                     int32_t* __restrict__ cand) {
  extern __shared__ float smem[];
  const int D = 2 * d_h;
  float* xs = smem;                          // [kCandTile][D + 1]
  float* rs = xs + kCandTile * (D + 1);      // [kCandRefChunk][D]
  const int b = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
  const int64_t bh = (int64_t)b * H + h;
  const int64_t t0 = (int64_t)blockIdx.x * kCandTile;
  const T* Kb = K + b * sb + h * sh;
  const T* Vb = V + b * sb + h * sh;
  for (int i = tid; i < kCandTile * D; i += blockDim.x) {
    int r = i / D, e = i - r * D;
    int64_t t = t0 + r;
    float v = 0.f;
    if (t < T_) v = e < d_h ? to_f(Kb[t * st + e]) : to_f(Vb[t * st + e - d_h]);
    xs[r * (D + 1) + e] = v;
  }
  const int64_t t = t0 + tid;
  const int n_cand = t < T_ ? (int)((t + s - 1) / s) : 0;  // slots j with j*s < t
  const int64_t t_last = min(t0 + kCandTile, (int64_t)T_) - 1;
  const int nc_tile = (int)((t_last + s - 1) / s);
  float bd[KC];
  int bi[KC];
#pragma unroll
  for (int i = 0; i < KC; ++i) { bd[i] = FLT_MAX; bi[i] = INT_MAX; }
  for (int j0 = 0; j0 < nc_tile; j0 += kCandRefChunk) {
    __syncthreads();
    for (int i = tid; i < kCandRefChunk * D; i += blockDim.x) {
      int r = i / D, e = i - r * D;
      int64_t j = j0 + r;
      float v = 0.f;
      if (j < nc_tile)
        v = e < d_h ? to_f(refk[(bh * n_ref_cap + j) * d_h + e])
                    : to_f(refv[(bh * n_ref_cap + j) * d_h + e - d_h]);
      rs[r * D + e] = v;
    }
    __syncthreads();
    float acc[kCandRefChunk];
#pragma unroll
    for (int r = 0; r < kCandRefChunk; ++r) acc[r] = 0.f;
    const float* xrow = xs + tid * (D + 1);
    for (int e = 0; e < D; ++e) {
      float xv = xrow[e];
#pragma unroll
      for (int r = 0; r < kCandRefChunk; ++r) {
        float df = xv - rs[r * D + e];
        acc[r] = fmaf(df, df, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kCandRefChunk; ++r)
      if (j0 + r < n_cand) topk_insert<KC>(bd, bi, acc[r], j0 + r);
  }
  if (t < T_ && (t % s) != 0) {
    int32_t* o = cand + (bh * n_code_cap + code_row_of(t, s)) * KC;
#pragma unroll
    for (int i = 0; i < KC; ++i) o[i] = bi[i] == INT_MAX ? -1 : bi[i];
  }
}

template <typename E, int KC>
static cudaError_t cand_simt_launch(const Plan& p, int T, const KVView& kv, const void* cache,
                                    void* ws, cudaStream_t st) {
  const auto& c = p.cfg;
  const int D = p.D;
  size_t smem = sizeof(float) * (size_t)(kCandTile * (D + 1) + kCandRefChunk * D);
  auto kern = cand_simt_kernel<E, KC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const char* cb = (const char*)cache;
  dim3 grid((unsigned)ceil_div64(T, kCandTile), c.kv_heads, c.batch);
  ProfScope ps(p, st, KID_CAND_SIMT);
  kern<<<grid, kCandTile, smem, st>>>(T, c.stride_s, c.d_h, c.kv_heads, p.n_ref_cap,
                                      p.n_code_cap, (const E*)kv.K, (const E*)kv.V, kv.sb, kv.sh,
                                      kv.st, (const E*)(cb + p.off_refk),
                                      (const E*)(cb + p.off_refv),
                                      (int32_t*)((char*)ws + p.ws_cand));
  return cudaGetLastError();
}

cudaError_t launch_candidates_simt(const Plan& p, int T, const KVView& kv, const void* cache,
                                   void* ws, cudaStream_t st) {
  if (n_code_of(T, p.cfg.stride_s) == 0) return cudaSuccess;
  if (p.bf16)
    return p.KC == 8 ? cand_simt_launch<__nv_bfloat16, 8>(p, T, kv, cache, ws, st)
                     : cand_simt_launch<__nv_bfloat16, 12>(p, T, kv, cache, ws, st);
  return p.KC == 8 ? cand_simt_launch<float, 8>(p, T, kv, cache, ws, st)
                   : cand_simt_launch<float, 12>(p, T, kv, cache, ws, st);
}

// -------------------------------------------------------------- encode
// For a tile of 32 compressed rows of one (b, head):
//  1. (one warp per token) exact fp32 distances sum (x_t - r_j)^2 to the KC
//     candidates, the k smallest by (distance, slot), their mean KV_R and the
//     residual x_t - KV_R; the slots go to the idx plane;
//  2. h = act(W1 r + b1) for the 32 residuals;
//  3. code = W2 h + b2, rounded to the cache type, to the code plane.
constexpr int kEncTile = 32;

template <typename T, int KC>
__global__ void __launch_bounds__(256)
    encode_simt_kernel(int T_, int s, int d_h, int H, int k, int d_c, int hidden, int act,
                       int64_t n_ref_cap, int64_t n_code_cap, const T* __restrict__ K,
                       const T* __restrict__ V, int64_t sb, int64_t sh, int64_t st,
                       const T* __restrict__ W1, const float* __restrict__ b1,
                       const T* __restrict__ W2, const float* __restrict__ b2,
                       const T* __restrict__ refk, const T* __restrict__ refv,
                       T* __restrict__ code, int32_t* __restrict__ idx_out,
                       const int32_t* __restrict__ cand, uint32_t* __restrict__ err) {
  extern __shared__ float smem[];
  const int D = 2 * d_h;
  float* R = smem;                              // [kEncTile][D]
  float* Hs = R + kEncTile * D;                 // [kEncTile][hidden + 1]
  float* Wc = Hs + kEncTile * (hidden + 1);     // [16][hidden]   W1 chunk, transposed
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int64_t bh = (int64_t)b * H + h;
  const int64_t n_code = T_ - (T_ + s - 1) / s;
  const int64_t row0 = (int64_t)blockIdx.x * kEncTile;
  const T* Kb = K + b * sb + h * sh;
  const T* Vb = V + b * sb + h * sh;
  const T* rk = refk + bh * n_ref_cap * d_h;
  const T* rv = refv + bh * n_ref_cap * d_h;
  const int per_lane = D / 32;  // 4 or 8

  // ---- 1. selection, mean, residual (warp per token)
  for (int r = warp; r < kEncTile; r += 8) {
    const int64_t row = row0 + r;
    float* Rr = R + r * D;
    if (row >= n_code) {
      for (int e = lane; e < D; e += 32) Rr[e] = 0.f;
      continue;
    }
    const int64_t t = token_of_code_row(row, s);
    float xv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < per_lane) {
        int e = lane + 32 * i;
        xv[i] = e < d_h ? to_f(Kb[t * st + e]) : to_f(Vb[t * st + e - d_h]);
      }
    const int32_t* cr = cand + (bh * n_code_cap + row) * KC;
    float cd[KC];
    int cj[KC];
#pragma unroll
    for (int i = 0; i < KC; ++i) {
      int j = cr[i];
      if (j >= 0 && (int64_t)j * s >= t) {  // not an earlier reference: drop it
        latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j);
        j = -1;
      }
      cj[i] = j;
      float part = 0.f;
      if (j >= 0) {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < per_lane) {
            int e = lane + 32 * q;
            float rvv = e < d_h ? to_f(rk[(int64_t)j * d_h + e]) : to_f(rv[(int64_t)j * d_h + e - d_h]);
            float df = xv[q] - rvv;
            part = fmaf(df, df, part);
          }
      }
      part = warp_sum(part);
      cd[i] = j >= 0 ? part : FLT_MAX;
      if (j < 0) cj[i] = INT_MAX;
    }
    // k smallest of the KC candidates by (distance, slot), ascending
    int sel[kMaxK];
    int k_eff = 0;
#pragma unroll
    for (int q = 0; q < kMaxK; ++q) {
      sel[q] = -1;
      if (q < k) {
        int best = -1;
        float bdv = FLT_MAX;
        int bj = INT_MAX;
#pragma unroll
        for (int i = 0; i < KC; ++i) {
          bool better = cj[i] != INT_MAX && (cd[i] < bdv || (cd[i] == bdv && cj[i] < bj));
          if (better) { best = i; bdv = cd[i]; bj = cj[i]; }
        }
        if (best >= 0) {
          sel[q] = bj;
          ++k_eff;
#pragma unroll
          for (int i = 0; i < KC; ++i)
            if (i == best) cj[i] = INT_MAX;
        }
      }
    }
    if (lane < k) {
      int v = -1;
#pragma unroll
      for (int q = 0; q < kMaxK; ++q)
        if (q == lane) v = sel[q];
      idx_out[(bh * n_code_cap + row) * k + lane] = v;
    }
    const float inv = 1.0f / (float)max(k_eff, 1);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < per_lane) {
        int e = lane + 32 * q;
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxK; ++i)
          if (i < k && sel[i] >= 0)
            m += e < d_h ? to_f(rk[(int64_t)sel[i] * d_h + e]) : to_f(rv[(int64_t)sel[i] * d_h + e - d_h]);
        Rr[e] = xv[q] - m * inv;
      }
  }
  __syncthreads();

  // ---- 2. Hs = act(R W1^T + b1); thread tid owns hidden unit n = tid
  {
    float acc[kEncTile];
#pragma unroll
    for (int r = 0; r < kEncTile; ++r) acc[r] = 0.f;
    for (int e0 = 0; e0 < D; e0 += 16) {
      for (int i = tid; i < 16 * hidden; i += blockDim.x) {
        int n = i / 16, e = i - n * 16;
        Wc[e * hidden + n] = to_f(W1[(int64_t)n * D + e0 + e]);
      }
      __syncthreads();
      if (tid < hidden) {
#pragma unroll 4
        for (int e = 0; e < 16; ++e) {
          float w = Wc[e * hidden + tid];
#pragma unroll
          for (int r = 0; r < kEncTile; ++r) acc[r] = fmaf(R[r * D + e0 + e], w, acc[r]);
        }
      }
      __syncthreads();
    }
    if (tid < hidden) {
      float bias = b1 ? b1[tid] : 0.f;
#pragma unroll
      for (int r = 0; r < kEncTile; ++r) Hs[r * (hidden + 1) + tid] = act_eval(act, acc[r] + bias);
    }
  }
  __syncthreads();

  // ---- 3. code = Hs W2^T + b2
  for (int i = tid; i < kEncTile * d_c; i += blockDim.x) {
    int r = i / d_c, o = i - r * d_c;
    int64_t row = row0 + r;
    if (row >= n_code) continue;
    const T* w2 = W2 + (int64_t)o * hidden;
    const float* hr = Hs + r * (hidden + 1);
    float acc = b2 ? b2[o] : 0.f;
    for (int n = 0; n < hidden; ++n) acc = fmaf(hr[n], to_f(w2[n]), acc);
    code[(bh * n_code_cap + row) * d_c + o] = from_f<T>(acc);
  }
}

template <typename E, int KC>
static cudaError_t encode_launch(const Plan& p, int T, const KVView& kv, const void* W1,
                                 const float* b1, const void* W2, const float* b2, void* cache,
                                 void* ws, cudaStream_t st) {
  const auto& c = p.cfg;
  const int D = p.D;
  size_t smem = sizeof(float) * (size_t)(kEncTile * D + kEncTile * (c.hidden + 1) + 16 * c.hidden);
  auto kern = encode_simt_kernel<E, KC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  char* cb = (char*)cache;
  int64_t n_code = n_code_of(T, c.stride_s);
  dim3 grid((unsigned)ceil_div64(n_code, kEncTile), c.kv_heads, c.batch);
  ProfScope ps(p, st, KID_ENCODE_SIMT);
  kern<<<grid, 256, smem, st>>>(T, c.stride_s, c.d_h, c.kv_heads, c.k, c.d_c, c.hidden, (int)c.act,
                                p.n_ref_cap, p.n_code_cap, (const E*)kv.K, (const E*)kv.V, kv.sb,
                                kv.sh, kv.st, (const E*)W1, b1, (const E*)W2, b2,
                                (const E*)(cb + p.off_refk), (const E*)(cb + p.off_refv),
                                (E*)(cb + p.off_code), (int32_t*)(cb + p.off_idx),
                                (const int32_t*)((char*)ws + p.ws_cand), (uint32_t*)ws);
  return cudaGetLastError();
}

cudaError_t launch_encode(const Plan& p, int T, const KVView& kv, const void* W1, const float* b1,
                          const void* W2, const float* b2, void* cache, void* ws,
                          cudaStream_t st) {
  if (n_code_of(T, p.cfg.stride_s) == 0) return cudaSuccess;
  if (p.code4) return cudaErrorNotSupported;  // 4-bit codes are written by the tensor-core encoder
  if (p.bf16)
    return p.KC == 8 ? encode_launch<__nv_bfloat16, 8>(p, T, kv, W1, b1, W2, b2, cache, ws, st)
                     : encode_launch<__nv_bfloat16, 12>(p, T, kv, W1, b1, W2, b2, cache, ws, st);
  return p.KC == 8 ? encode_launch<float, 8>(p, T, kv, W1, b1, W2, b2, cache, ws, st)
                   : encode_launch<float, 12>(p, T, kv, W1, b1, W2, b2, cache, ws, st);
}

// --------------------------------------------------------- reconstruct
// Dense float32 K_hat, V_hat for every token ("Ricostruzione"): reference
// rows as stored, other tokens KV_R + W4 act(W3 code + b3) + b4.  One block
// per 32 tokens; warp-per-token for the mean, thread-per-unit for the MLPs.
template <typename T>
__global__ void __launch_bounds__(256)
    reconstruct_kernel(int T_, int s, int d_h, int H, int k, int d_c, int hidden, int act,
                       int64_t n_ref_cap, int64_t n_code_cap, const T* __restrict__ refk,
                       const T* __restrict__ refv, const T* __restrict__ code,
                       const __nv_bfloat16* __restrict__ cscale,
                       const int32_t* __restrict__ idx, const T* __restrict__ W3,
                       const float* __restrict__ b3, const T* __restrict__ W4,
                       const float* __restrict__ b4, float* __restrict__ Kout,
                       float* __restrict__ Vout, uint32_t* __restrict__ err) {
  extern __shared__ float smem[];
  const int D = 2 * d_h;
  float* Cs = smem;                       // [32][d_c]
  float* Us = Cs + 32 * d_c;              // [32][hidden + 1]
  const int b = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
  const int64_t bh = (int64_t)b * H + h;
  const int64_t t0 = (int64_t)blockIdx.x * 32;
  const int64_t n_ref = (T_ + s - 1) / s;
  const T* rk = refk + bh * n_ref_cap * d_h;
  const T* rv = refv + bh * n_ref_cap * d_h;
  for (int i = tid; i < 32 * d_c; i += blockDim.x) {
    int r = i / d_c, o = i - r * d_c;
    int64_t t = t0 + r;
    float v = 0.f;
    if (t < T_ && t % s != 0) v = code_at(code, cscale, bh * n_code_cap + code_row_of(t, s), d_c, o);
    Cs[i] = v;
  }
  __syncthreads();
  for (int i = tid; i < 32 * hidden; i += blockDim.x) {
    int r = i / hidden, n = i - r * hidden;
    const T* w3 = W3 + (int64_t)n * d_c;
    float acc = b3 ? b3[n] : 0.f;
    for (int e = 0; e < d_c; ++e) acc = fmaf(to_f(w3[e]), Cs[r * d_c + e], acc);
    Us[r * (hidden + 1) + n] = act_eval(act, acc);
  }
  __syncthreads();
  for (int i = tid; i < 32 * D; i += blockDim.x) {
    int r = i / D, e = i - r * D;
    int64_t t = t0 + r;
    if (t >= T_) continue;
    float v;
    if (t % s == 0) {
      int64_t j = t / s;
      v = e < d_h ? to_f(rk[j * d_h + e]) : to_f(rv[j * d_h + e - d_h]);
    } else {
      const int32_t* ir = idx + (bh * n_code_cap + code_row_of(t, s)) * k;
      float m = 0.f;
      int k_eff = 0;
      for (int i2 = 0; i2 < k; ++i2) {
        int j = ir[i2];
        if (j < 0) continue;
        if (j >= n_ref) { latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j); continue; }
        m += e < d_h ? to_f(rk[(int64_t)j * d_h + e]) : to_f(rv[(int64_t)j * d_h + e - d_h]);
        ++k_eff;
      }
      const T* w4 = W4 + (int64_t)e * hidden;
      float y = b4 ? b4[e] : 0.f;
      for (int n = 0; n < hidden; ++n) y = fmaf(to_f(w4[n]), Us[r * (hidden + 1) + n], y);
      v = m / (float)max(k_eff, 1) + y;
    }
    float* out = e < d_h ? Kout : Vout;
    out[(bh * T_ + t) * d_h + (e < d_h ? e : e - d_h)] = v;
  }
}

cudaError_t launch_reconstruct(const Plan& p, int T, const void* cache, const void* W3,
                               const float* b3, const void* W4, const float* b4, float* Kout,
                               float* Vout, void* ws, cudaStream_t st) {
  const auto& c = p.cfg;
  if (T == 0) return cudaSuccess;
  size_t smem = sizeof(float) * (size_t)(32 * c.d_c + 32 * (c.hidden + 1));
  dim3 grid((unsigned)ceil_div64(T, 32), c.kv_heads, c.batch);
  const char* cb = (const char*)cache;
  ProfScope ps(p, st, KID_RECONSTRUCT);
  if (p.bf16) {
    using T_ = __nv_bfloat16;
    auto kern = reconstruct_kernel<T_>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 256, smem, st>>>(T, c.stride_s, c.d_h, c.kv_heads, c.k, c.d_c, c.hidden,
                                  (int)c.act, p.n_ref_cap, p.n_code_cap,
                                  (const T_*)(cb + p.off_refk), (const T_*)(cb + p.off_refv),
                                  (const T_*)(cb + p.off_code),
                                  p.code4 ? (const __nv_bfloat16*)(cb + p.off_cscale) : nullptr,
                                  (const int32_t*)(cb + p.off_idx),
                                  (const T_*)W3, b3, (const T_*)W4, b4, Kout, Vout, (uint32_t*)ws);
  } else {
    auto kern = reconstruct_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, 256, smem, st>>>(T, c.stride_s, c.d_h, c.kv_heads, c.k, c.d_c, c.hidden,
                                  (int)c.act, p.n_ref_cap, p.n_code_cap,
                                  (const float*)(cb + p.off_refk), (const float*)(cb + p.off_refv),
                                  (const float*)(cb + p.off_code), nullptr,
                                  (const int32_t*)(cb + p.off_idx), (const float*)W3, b3,
                                  (const float*)W4, b4, Kout, Vout, (uint32_t*)ws);
  }
  return cudaGetLastError();
}

}  // namespace dkv
