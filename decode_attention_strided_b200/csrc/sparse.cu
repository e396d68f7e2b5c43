// sparse.cu -- decode attention over a caller-selected subset of the cached
// tokens, reconstructing only those tokens.
//
// DeltaKV summary, section 3 "Ricostruzione" with section 4 ("OmniKV"
// integration): a sparse-attention selector names the tokens that matter for
// the current query; only they are rebuilt (reference rows as stored, every
// other token as the mean of its references plus the decompressor MLP of its
// code) and attended.  For query head hq of kv-head h:
//   out = sum_{t in sel(b, h)} softmax_t(q . K_hat_t / sqrt(d_h)) V_hat_t.
// The selection is an input (the selector itself is not part of this path).
//
// Kernels: each CTA takes a contiguous share of one (sequence, kv-head)'s
// selection, rebuilds 32 tokens at a time into shared memory (the same
// arithmetic as deltakv_reconstruct, in fp32) and folds them into a running
// softmax for the group's query heads; a second kernel merges the shares.
#include <cfloat>

#include "common.cuh"

namespace dkv {

namespace {
constexpr int kSpTok = 32;  // tokens rebuilt per round
}

struct SparseParams {
  int T, s, d_h, H, G, k, d_c, hidden, act, n_sel, per, nsplit;
  int64_t n_ref_cap, n_code_cap, qsb, qsh;
  float scale;  // 1 / sqrt(d_h)
};

template <typename E>
__global__ void __launch_bounds__(256)
    sparse_attend_kernel(const SparseParams P, const E* __restrict__ q, const int32_t* __restrict__ tokens,
                         const E* __restrict__ refk, const E* __restrict__ refv, const E* __restrict__ code,
                         const int32_t* __restrict__ idx, const E* __restrict__ W3, const float* __restrict__ b3,
                         const E* __restrict__ W4, const float* __restrict__ b4, float* __restrict__ part,
                         uint32_t* __restrict__ err) {
  extern __shared__ float smem[];
  const int d_h = P.d_h, D = 2 * d_h, G = P.G, hidden = P.hidden, d_c = P.d_c;
  float* X = smem;                          // [kSpTok][D] rebuilt tokens
  float* Cs = X + kSpTok * D;               // [kSpTok][d_c]
  float* Us = Cs + kSpTok * d_c;            // [kSpTok][hidden + 1]
  float* qs = Us + kSpTok * (hidden + 1);   // [G][d_h], scaled
  float* lg = qs + kMaxG * d_h;             // [G][kSpTok]
  float* mrun = lg + kMaxG * kSpTok;        // [G]
  float* lrun = mrun + kMaxG;               // [G]
  float* alpha = lrun + kMaxG;              // [G]
  int* tok = (int*)(alpha + kMaxG);         // [kSpTok], -1 = empty
  const int b = blockIdx.z, h = blockIdx.y, sp = blockIdx.x, tid = threadIdx.x;
  const int64_t bh = (int64_t)b * P.H + h;
  const int64_t n_ref = (P.T + P.s - 1) / P.s;
  const E* rk = refk + bh * P.n_ref_cap * d_h;
  const E* rv = refv + bh * P.n_ref_cap * d_h;
  for (int i = tid; i < G * d_h; i += blockDim.x) {
    const int g = i / d_h, e = i - g * d_h;
    qs[g * d_h + e] = P.scale * to_f(q[b * P.qsb + (int64_t)(h * G + g) * P.qsh + e]);
  }
  if (tid < G) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.f;
  }
  // this thread's output elements: (g, e) = o / d_h, o % d_h for
  // o = tid + 256 w, w < 4 (G d_h <= 1024)
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int i_lo = sp * P.per, i_hi = min(P.n_sel, i_lo + P.per);
  for (int i0 = i_lo; i0 < i_hi; i0 += kSpTok) {
    __syncthreads();
    if (tid < kSpTok) {
      int t = -1;
      if (i0 + tid < i_hi) {
        t = tokens[bh * P.n_sel + i0 + tid];
        if (t < 0 || t >= P.T) {
          latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)t);
          t = -1;
        }
      }
      tok[tid] = t;
    }
    __syncthreads();
    // rebuild: codes, u = act(W3 c + b3), x = KV_R + W4 u + b4
    for (int i = tid; i < kSpTok * d_c; i += blockDim.x) {
      const int r = i / d_c, o = i - r * d_c, t = tok[r];
      float v = 0.f;
      if (t >= 0 && t % P.s != 0) v = to_f(code[(bh * P.n_code_cap + code_row_of(t, P.s)) * d_c + o]);
      Cs[i] = v;
    }
    __syncthreads();
    for (int i = tid; i < kSpTok * hidden; i += blockDim.x) {
      const int r = i / hidden, n = i - r * hidden;
      const E* w3 = W3 + (int64_t)n * d_c;
      float a = b3 ? b3[n] : 0.f;
      for (int e = 0; e < d_c; ++e) a = fmaf(to_f(w3[e]), Cs[r * d_c + e], a);
      Us[r * (hidden + 1) + n] = act_eval(P.act, a);
    }
    __syncthreads();
    for (int i = tid; i < kSpTok * D; i += blockDim.x) {
      const int r = i / D, e = i - r * D, t = tok[r];
      float v = 0.f;
      if (t >= 0) {
        if (t % P.s == 0) {
          const int64_t j = t / P.s;
          v = e < d_h ? to_f(rk[j * d_h + e]) : to_f(rv[j * d_h + e - d_h]);
        } else {
          const int32_t* ir = idx + (bh * P.n_code_cap + code_row_of(t, P.s)) * P.k;
          float m = 0.f;
          int k_eff = 0;
          for (int i2 = 0; i2 < P.k; ++i2) {
            const int j = ir[i2];
            if (j < 0) continue;
            if (j >= n_ref) {
              latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j);
              continue;
            }
            m += e < d_h ? to_f(rk[(int64_t)j * d_h + e]) : to_f(rv[(int64_t)j * d_h + e - d_h]);
            ++k_eff;
          }
          const E* w4 = W4 + (int64_t)e * hidden;
          float y = b4 ? b4[e] : 0.f;
          for (int n = 0; n < hidden; ++n) y = fmaf(to_f(w4[n]), Us[r * (hidden + 1) + n], y);
          v = m / (float)max(k_eff, 1) + y;
        }
      }
      X[r * D + e] = v;
    }
    __syncthreads();
    // logits of the round
    for (int i = tid; i < G * kSpTok; i += blockDim.x) {
      const int g = i / kSpTok, r = i - g * kSpTok;
      float a = -INFINITY;
      if (tok[r] >= 0) {
        a = 0.f;
        for (int e = 0; e < d_h; ++e) a = fmaf(qs[g * d_h + e], X[r * D + e], a);
      }
      lg[g * kSpTok + r] = a;
    }
    __syncthreads();
    if (tid < G) {
      float m = mrun[tid];
      for (int r = 0; r < kSpTok; ++r) m = fmaxf(m, lg[tid * kSpTok + r]);
      const float al = m == -INFINITY ? 1.f : expf(mrun[tid] - m);
      float l = lrun[tid] * al;
      for (int r = 0; r < kSpTok; ++r) {
        const float p = lg[tid * kSpTok + r] == -INFINITY ? 0.f : expf(lg[tid * kSpTok + r] - m);
        lg[tid * kSpTok + r] = p;
        l += p;
      }
      alpha[tid] = al;
      mrun[tid] = m;
      lrun[tid] = l;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int o = tid + w * (int)blockDim.x;
      if (o < G * d_h) {
        const int g = o / d_h, e = o - g * d_h;
        float a = acc[w] * alpha[g];
        for (int r = 0; r < kSpTok; ++r) a = fmaf(lg[g * kSpTok + r], X[r * D + d_h + e], a);
        acc[w] = a;
      }
    }
  }
  __syncthreads();
  // partial of this share: m, l per head, then the unnormalised output
  float* pp = part + (bh * P.nsplit + sp) * G * (d_h + 2);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int o = tid + w * (int)blockDim.x;
    if (o < G * d_h) {
      const int g = o / d_h, e = o - g * d_h;
      pp[g * (d_h + 2) + 2 + e] = acc[w];
    }
  }
  if (tid < G) {
    pp[tid * (d_h + 2)] = mrun[tid];
    pp[tid * (d_h + 2) + 1] = lrun[tid];
  }
}

// Merge the shares of every (sequence, query head).
__global__ void sparse_merge_kernel(const SparseParams P, const float* __restrict__ part, float* __restrict__ out,
                                    int64_t osb, int64_t osh) {
  const int b = blockIdx.z, h = blockIdx.y, g = blockIdx.x;
  const int64_t bh = (int64_t)b * P.H + h;
  const int d_h = P.d_h;
  float M = -INFINITY;
  for (int sp = 0; sp < P.nsplit; ++sp) M = fmaxf(M, part[((bh * P.nsplit + sp) * P.G + g) * (d_h + 2)]);
  float L = 0.f;
  for (int sp = 0; sp < P.nsplit; ++sp) {
    const float* pp = part + ((bh * P.nsplit + sp) * P.G + g) * (d_h + 2);
    if (pp[0] != -INFINITY) L += pp[1] * expf(pp[0] - M);
  }
  for (int e = threadIdx.x; e < d_h; e += blockDim.x) {
    float o = 0.f;
    for (int sp = 0; sp < P.nsplit; ++sp) {
      const float* pp = part + ((bh * P.nsplit + sp) * P.G + g) * (d_h + 2);
      if (pp[0] != -INFINITY) o += pp[2 + e] * expf(pp[0] - M);
    }
    out[b * osb + (int64_t)(h * P.G + g) * osh + e] = L > 0.f ? o / L : 0.f;
  }
}

size_t sparse_smem_bytes(const Plan& p) {
  const auto& c = p.cfg;
  return sizeof(float) * ((size_t)kSpTok * 2 * c.d_h + (size_t)kSpTok * c.d_c + (size_t)kSpTok * (c.hidden + 1) +
                          (size_t)kMaxG * c.d_h + (size_t)kMaxG * kSpTok + 3 * kMaxG) +
         sizeof(int) * kSpTok;
}

template <typename E>
static cudaError_t sparse_launch(const Plan& p, int T, const void* q, int64_t qsb, int64_t qsh, const void* cache,
                                 const void* W3, const float* b3, const void* W4, const float* b4,
                                 const int32_t* tokens, int n_sel, float* out, int64_t osb, int64_t osh, void* ws,
                                 cudaStream_t st) {
  const auto& c = p.cfg;
  const char* cb = (const char*)cache;
  SparseParams P;
  P.T = T;
  P.s = c.stride_s;
  P.d_h = c.d_h;
  P.H = c.kv_heads;
  P.G = p.G;
  P.k = c.k;
  P.d_c = c.d_c;
  P.hidden = c.hidden;
  P.act = (int)c.act;
  P.n_sel = n_sel;
  P.n_ref_cap = p.n_ref_cap;
  P.n_code_cap = p.n_code_cap;
  P.qsb = qsb;
  P.qsh = qsh;
  P.scale = 1.0f / sqrtf((float)c.d_h);
  const int64_t BH = (int64_t)c.batch * c.kv_heads;
  // shares of at least one round each, about two CTAs per SM in total
  int nsplit = (int)std::min<int64_t>((n_sel + kSpTok - 1) / kSpTok, std::max<int64_t>(1, 2 * kNumSMs / BH));
  nsplit = std::max(1, std::min(nsplit, kSparseSplits));
  P.nsplit = nsplit;
  P.per = (n_sel + nsplit - 1) / nsplit;
  float* part = (float*)((char*)ws + p.ws_sparse);
  const size_t smem = sparse_smem_bytes(p);
  auto kern = sparse_attend_kernel<E>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  {
    ProfScope ps(p, st, KID_SPARSE_ATTEND);
    kern<<<dim3(nsplit, c.kv_heads, c.batch), 256, smem, st>>>(
        P, (const E*)q, tokens, (const E*)(cb + p.off_refk), (const E*)(cb + p.off_refv),
        (const E*)(cb + p.off_code), (const int32_t*)(cb + p.off_idx), (const E*)W3, b3, (const E*)W4, b4, part,
        (uint32_t*)ws);
  }
  {
    ProfScope ps(p, st, KID_SPARSE_MERGE);
    sparse_merge_kernel<<<dim3(p.G, c.kv_heads, c.batch), 128, 0, st>>>(P, part, out, osb, osh);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_sparse(const Plan& p, int T, const void* q, int64_t qsb, int64_t qsh, const void* cache,
                                 const void* W3, const float* b3, const void* W4, const float* b4,
                                 const int32_t* tokens, int n_sel, float* out, int64_t osb, int64_t osh, void* ws,
                                 cudaStream_t st) {
  if (p.cfg.dtype == DELTAKV_BF16)
    return sparse_launch<__nv_bfloat16>(p, T, q, qsb, qsh, cache, W3, b3, W4, b4, tokens, n_sel, out, osb, osh, ws,
                                        st);
  return sparse_launch<float>(p, T, q, qsb, qsh, cache, W3, b3, W4, b4, tokens, n_sel, out, osb, osh, ws, st);
}

}  // namespace dkv
