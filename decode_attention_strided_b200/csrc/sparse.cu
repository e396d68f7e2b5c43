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
// selection, 16 tokens per pass, and never forms K_hat or V_hat rows.  The
// decompressor's output layer is linear, so for a non-reference token with
// code c, u = act(W3 c + b3) and reference mean (mk, mv):
//   q . k_hat = q . mk + (W4_K^T q) . u + q . b4_K
//   sum_t p_t v_hat_t = sum_t p_t mv_t + W4_V (sum_t p_t u_t) + b4_V sum_t p_t
// (reference tokens: q . K_ref and V_ref alone).  Per token that leaves the
// first layer (d_c x hidden MACs) plus O(G (d_h + hidden)), instead of the
// second layer's 2 d_h x hidden.  W4_K^T q is folded once per CTA and W4_V
// is applied once per CTA to the accumulated sum of p u.  A second kernel
// merges the shares' (max, sum, output) triples.
#include <cfloat>

#include "common.cuh"

namespace dkv {

namespace {
constexpr int kSpR = 16;           // tokens per pass
constexpr int kSpRP = kSpR + 4;    // row stride of the transposed code tile (keeps float4 rows aligned)
constexpr int kSpThreads = 256;
constexpr int kSpWarps = kSpThreads / 32;
static_assert(kSpWarps >= kMaxG, "one warp per query head of a group");
static_assert(kSpR == 2 * kSpWarps, "two tokens per warp in the logit step");
}  // namespace

struct SparseParams {
  int T, s, d_h, H, G, k, d_c, hidden, act, n_sel, per, nsplit;
  int64_t n_ref_cap, n_code_cap, qsb, qsh;
  float scale;  // 1 / sqrt(d_h)
  const __nv_bfloat16* cscale;  // per-row scales of 4-bit codes, else null
};

// Shared-memory carve-up (in floats; every region starts on 16 bytes).
struct SpLayout {
  int w3t, b3, qs, qw, qb, cst, u, mk, mv, zp, st, ints, total;
};

__host__ __device__ inline int sp_take(int& o, int n) {
  const int r = o;
  o += (n + 3) & ~3;
  return r;
}

__host__ __device__ inline SpLayout sp_layout(int d_c, int hidden, int G, int d_h, int k) {
  SpLayout L;
  int o = 0;
  L.w3t = sp_take(o, d_c * (hidden + 1));  // W3 transposed, [d_c][hidden + 1]
  L.b3 = sp_take(o, hidden);
  L.qs = sp_take(o, G * d_h);             // q / sqrt(d_h), [G][d_h]
  L.qw = sp_take(o, G * hidden);          // W4_K^T q, [G][hidden]
  L.qb = sp_take(o, G);                   // q . b4_K
  L.cst = sp_take(o, d_c * kSpRP);        // codes of the pass, [d_c][kSpRP]
  L.u = sp_take(o, kSpR * hidden);        // act(W3 c + b3), [kSpR][hidden]
  L.mk = sp_take(o, kSpR * d_h);          // K part of the reference mean (or the reference row)
  L.mv = sp_take(o, kSpR * d_h);          // V part
  L.zp = sp_take(o, G * kSpR);            // logits, then softmax weights, [G][kSpR]
  L.st = sp_take(o, 4 * kMaxG);           // running max, sum, sum over non-reference tokens, rescale
  L.ints = sp_take(o, 2 * kSpR + kSpR * k);  // token, kind (-1 empty, 0 reference, 1 coded), slots
  L.total = o;
  return L;
}

template <typename E> __device__ __forceinline__ float2 load2(const E* p);
template <> __device__ __forceinline__ float2 load2<float>(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
template <> __device__ __forceinline__ float2 load2<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

// Eight consecutive elements of a reference row, loaded in one go (16 bytes
// of bf16, 32 of float) so that all of a token's slots are in flight together.
template <typename E> struct Row8;
template <> struct Row8<__nv_bfloat16> {
  uint4 v;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { v = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void add_to(float (&a)[8]) const {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[2 * i] += __uint_as_float(w[i] << 16);  // bf16 -> fp32 is exact
      a[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <> struct Row8<float> {
  float4 x, y;
  __device__ __forceinline__ void load(const float* p) {
    x = __ldg(reinterpret_cast<const float4*>(p));
    y = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void add_to(float (&a)[8]) const {
    a[0] += x.x;
    a[1] += x.y;
    a[2] += x.z;
    a[3] += x.w;
    a[4] += y.x;
    a[5] += y.y;
    a[6] += y.z;
    a[7] += y.w;
  }
};

// Sum each of N (a power of two <= 32) values over the warp.  Returns the
// total of value g(lane) = the lane's position among the N groups of 32 / N
// lanes; lanes with (lane % (32 / N)) == 0 hold distinct g.  log2(N) halving
// exchanges plus log2(32 / N) plain ones instead of 5 N shuffles.
template <int N>
__device__ __forceinline__ float warp_sum_scatter(float (&v)[N], int lane, int& g) {
  g = 0;
  int off = 16;
#pragma unroll
  for (int c = N; c > 1; c >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < c / 2; ++i) {
      const float keep = up ? v[i + c / 2] : v[i];
      const float send = up ? v[i] : v[i + c / 2];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
    g += up ? c / 2 : 0;
  }
  float r = v[0];
#pragma unroll
  for (; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
  return r;
}

template <typename E, int GM>
__global__ void __launch_bounds__(kSpThreads, GM <= 4 ? 2 : 1)
    sparse_attend_kernel(const SparseParams P, const E* __restrict__ q, const int32_t* __restrict__ tokens,
                         const E* __restrict__ refk, const E* __restrict__ refv, const E* __restrict__ code,
                         const int32_t* __restrict__ idx, const E* __restrict__ W3, const float* __restrict__ b3,
                         const E* __restrict__ W4, const float* __restrict__ b4, float* __restrict__ part,
                         uint32_t* __restrict__ err) {
  extern __shared__ __align__(16) float smem[];
  const int d_h = P.d_h, G = P.G, hidden = P.hidden, d_c = P.d_c, K = P.k, HP = hidden + 1;
  const SpLayout L = sp_layout(d_c, hidden, G, d_h, K);
  float* W3t = smem + L.w3t;
  float* b3s = smem + L.b3;
  float* qs = smem + L.qs;
  float* qW = smem + L.qw;
  float* qb = smem + L.qb;
  float* CsT = smem + L.cst;
  float* U = smem + L.u;
  float* MK = smem + L.mk;
  float* MV = smem + L.mv;
  float* zp = smem + L.zp;
  float* m_s = smem + L.st;
  float* l_s = m_s + kMaxG;
  float* lb_s = l_s + kMaxG;
  float* al_s = lb_s + kMaxG;
  int* tok = (int*)(smem + L.ints);
  int* kind = tok + kSpR;
  int* slots = kind + kSpR;
  const int b = blockIdx.z, h = blockIdx.y, sp = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t bh = (int64_t)b * P.H + h;
  const int64_t n_ref = (P.T + P.s - 1) / P.s;
  const E* rk = refk + bh * P.n_ref_cap * d_h;
  const E* rv = refv + bh * P.n_ref_cap * d_h;
  const E* cd = code + bh * P.n_code_cap * d_c;
  const int32_t* ix = idx + bh * P.n_code_cap * K;

  // ---- per-CTA constants
  for (int i = tid; i < G * d_h; i += kSpThreads) {
    const int g = i / d_h, e = i - g * d_h;
    qs[i] = P.scale * to_f(q[b * P.qsb + (int64_t)(h * G + g) * P.qsh + e]);
  }
  for (int i = tid; i < d_c * hidden; i += kSpThreads) {
    const int n = i / d_c, e = i - n * d_c;
    W3t[e * HP + n] = to_f(W3[i]);
  }
  for (int n = tid; n < hidden; n += kSpThreads) b3s[n] = b3 ? b3[n] : 0.f;
  if (tid < kMaxG) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
    lb_s[tid] = 0.f;
    al_s[tid] = 1.f;
  }
  __syncthreads();
  for (int n = tid; n < hidden; n += kSpThreads) {
    float a[GM];
#pragma unroll
    for (int g = 0; g < GM; ++g) a[g] = 0.f;
#pragma unroll 4
    for (int e = 0; e < d_h; ++e) {
      const float w = to_f(W4[(int64_t)e * hidden + n]);
#pragma unroll
      for (int g = 0; g < GM; ++g)
        if (g < G) a[g] = fmaf(qs[g * d_h + e], w, a[g]);
    }
#pragma unroll
    for (int g = 0; g < GM; ++g)
      if (g < G) qW[g * hidden + n] = a[g];
  }
  if (warp < G) {
    float a = 0.f;
    if (b4)
      for (int e = lane; e < d_h; e += 32) a = fmaf(qs[warp * d_h + e], b4[e], a);
    a = warp_sum(a);
    if (lane == 0) qb[warp] = a;
  }
  __syncthreads();
  // this lane's slice of the folded query: e = lane + 32 i, n = lane + 32 i
  float qe[GM][4], qn[GM][8];
#pragma unroll
  for (int g = 0; g < GM; ++g) {
#pragma unroll
    for (int i = 0; i < 4; ++i) qe[g][i] = (g < G && lane + 32 * i < d_h) ? qs[g * d_h + lane + 32 * i] : 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) qn[g][i] = (g < G && lane + 32 * i < hidden) ? qW[g * hidden + lane + 32 * i] : 0.f;
  }
  float qbl[GM];
#pragma unroll
  for (int g = 0; g < GM; ++g) qbl[g] = g < G ? qb[g] : 0.f;

  // accumulators of the columns c = tid + 256 j of [U | MV] (hidden + d_h <= 512)
  float acc[2][GM];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int g = 0; g < GM; ++g) acc[j][g] = 0.f;
  const int ncol = hidden + d_h;
  const int i_lo = sp * P.per, i_hi = min(P.n_sel, i_lo + P.per);
  int t_next = -1;
  if (tid < kSpR && i_lo + tid < i_hi) t_next = tokens[bh * P.n_sel + i_lo + tid];

  for (int i0 = i_lo; i0 < i_hi; i0 += kSpR) {
    __syncthreads();  // the previous pass's readers are done
    // tokens of this pass (loaded one pass ahead)
    if (tid < kSpR) {
      int t = t_next, ty = -1;
      if (i0 + tid < i_hi) {
        if (t < 0 || t >= P.T) {
          latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)t);
          t = -1;
        } else {
          ty = (t % P.s == 0) ? 0 : 1;
        }
      } else {
        t = -1;
      }
      tok[tid] = t;
      kind[tid] = ty;
      t_next = (i0 + kSpR + tid < i_hi) ? tokens[bh * P.n_sel + i0 + kSpR + tid] : -1;
    }
    __syncthreads();
    // codes (transposed) and slot lists of the coded tokens: every load of
    // the step is issued before the first store
    {
      float2 cv[4];
      int cr[4], ce[4];
      const int hc = d_c >> 1;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = tid + m * kSpThreads;
        cr[m] = -1;
        cv[m] = make_float2(0.f, 0.f);
        if (i < kSpR * hc) {
          const int r = i / hc;
          cr[m] = r;
          ce[m] = 2 * (i - r * hc);
          if (kind[r] == 1) {
            if (P.cscale) {
              const int64_t crow = bh * P.n_code_cap + code_row_of(tok[r], P.s);
              cv[m] = make_float2(code_at(code, P.cscale, crow, d_c, ce[m]),
                                  code_at(code, P.cscale, crow, d_c, ce[m] + 1));
            } else {
              cv[m] = load2(cd + code_row_of(tok[r], P.s) * d_c + ce[m]);
            }
          }
        }
      }
      int sv = -1;
      if (tid < kSpR * K) {
        const int r = tid / K, j = tid - r * K;
        if (kind[r] == 1) {
          sv = ix[code_row_of(tok[r], P.s) * K + j];
          if (sv >= n_ref) {
            latch_error(err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)sv);
            sv = -1;
          }
        }
        slots[tid] = sv < 0 ? -1 : sv;
      }
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (cr[m] >= 0) {
          CsT[ce[m] * kSpRP + cr[m]] = cv[m].x;
          CsT[(ce[m] + 1) * kSpRP + cr[m]] = cv[m].y;
        }
    }
    __syncthreads();
    // reference part, issued now and consumed after the first decompressor
    // layer: thread (ir, e8) sums elements e8 .. e8 + 7 of the rows of token
    // ir's references (the reference row itself for a reference token)
    const int per_row = d_h >> 3;
    const bool has_item = tid < kSpR * per_row;
    const int ir = has_item ? tid / per_row : 0;
    const int e8 = has_item ? 8 * (tid - ir * per_row) : 0;
    const int ity = has_item ? kind[ir] : -1;
    Row8<E> rka[4], rva[4];
    int js[4];
#pragma unroll
    for (int j2 = 0; j2 < 4; ++j2) {
      int j = -1;
      if (ity == 0 && j2 == 0) j = tok[ir] / P.s;
      if (ity == 1 && j2 < K) j = slots[ir * K + j2];
      js[j2] = j;
      if (j >= 0) {
        rka[j2].load(rk + (int64_t)j * d_h + e8);
        rva[j2].load(rv + (int64_t)j * d_h + e8);
      }
    }
    // first decompressor layer: thread (n0, half) owns columns n0 and n0 + hidden/2
    // for the pass's tokens 8 half .. 8 half + 7
    if (tid < hidden) {
      const int hh = hidden >> 1, n0 = tid % hh, half = tid / hh, n1 = n0 + hh;
      float a0[8], a1[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        a0[r] = b3s[n0];
        a1[r] = b3s[n1];
      }
      const float* cc = CsT + half * 8;
#pragma unroll 4
      for (int e = 0; e < d_c; ++e) {
        const float w0 = W3t[e * HP + n0], w1 = W3t[e * HP + n1];
        const float4 c0 = *reinterpret_cast<const float4*>(cc + e * kSpRP);
        const float4 c1 = *reinterpret_cast<const float4*>(cc + e * kSpRP + 4);
        const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          a0[r] = fmaf(w0, cv[r], a0[r]);
          a1[r] = fmaf(w1, cv[r], a1[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int rr = half * 8 + r;
        const bool on = kind[rr] == 1;
        U[rr * hidden + n0] = on ? act_fast(P.act, a0[r]) : 0.f;
        U[rr * hidden + n1] = on ? act_fast(P.act, a1[r]) : 0.f;
      }
    }
    if (has_item) {
      float mk[8], mv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mk[i] = mv[i] = 0.f;
      int ke = 0;
#pragma unroll
      for (int j2 = 0; j2 < 4; ++j2)
        if (js[j2] >= 0) {
          rka[j2].add_to(mk);
          rva[j2].add_to(mv);
          ++ke;
        }
      if (ity == 1 && K > 4) {  // slots 4 .. 7
#pragma unroll
        for (int j2 = 0; j2 < 4; ++j2) {
          const int j = (4 + j2 < K) ? slots[ir * K + 4 + j2] : -1;
          js[j2] = j;
          if (j >= 0) {
            rka[j2].load(rk + (int64_t)j * d_h + e8);
            rva[j2].load(rv + (int64_t)j * d_h + e8);
          }
        }
#pragma unroll
        for (int j2 = 0; j2 < 4; ++j2)
          if (js[j2] >= 0) {
            rka[j2].add_to(mk);
            rva[j2].add_to(mv);
            ++ke;
          }
      }
      const float kf = (float)max(ke, 1);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        mk[i] /= kf;
        mv[i] /= kf;
      }
      float4* dk = reinterpret_cast<float4*>(MK + ir * d_h + e8);
      float4* dv = reinterpret_cast<float4*>(MV + ir * d_h + e8);
      dk[0] = make_float4(mk[0], mk[1], mk[2], mk[3]);
      dk[1] = make_float4(mk[4], mk[5], mk[6], mk[7]);
      dv[0] = make_float4(mv[0], mv[1], mv[2], mv[3]);
      dv[1] = make_float4(mv[4], mv[5], mv[6], mv[7]);
    }
    __syncthreads();
    // logits: warp w takes tokens w and w + 8
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = warp + rr * kSpWarps, ty = kind[r];
      float pz[GM];
#pragma unroll
      for (int g = 0; g < GM; ++g) pz[g] = 0.f;
      if (ty >= 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (lane + 32 * i < d_h) {
            const float x = MK[r * d_h + lane + 32 * i];
#pragma unroll
            for (int g = 0; g < GM; ++g) pz[g] = fmaf(qe[g][i], x, pz[g]);
          }
        if (ty == 1) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (lane + 32 * i < hidden) {
              const float u = U[r * hidden + lane + 32 * i];
#pragma unroll
              for (int g = 0; g < GM; ++g) pz[g] = fmaf(qn[g][i], u, pz[g]);
            }
        }
      }
      int g;
      const float z = warp_sum_scatter<GM>(pz, lane, g);  // warp-uniform ty: all lanes take part
      if ((lane & (32 / GM - 1)) == 0 && g < G) {
        float qbg = 0.f;
#pragma unroll
        for (int g2 = 0; g2 < GM; ++g2)
          if (g2 == g) qbg = qbl[g2];
        zp[g * kSpR + r] = ty < 0 ? -INFINITY : z + (ty == 1 ? qbg : 0.f);
      }
    }
    __syncthreads();
    // running softmax: warp g, lane r < kSpR
    if (warp < G) {
      const int g = warp;
      const float z = lane < kSpR ? zp[g * kSpR + lane] : -INFINITY;
      const float m0 = m_s[g];
      const float m1 = fmaxf(m0, warp_max(z));
      const float p = (z == -INFINITY) ? 0.f : expf(z - m1);
      const float l = warp_sum(p);
      const float lb = warp_sum((lane < kSpR && kind[lane] == 1) ? p : 0.f);
      if (lane < kSpR) zp[g * kSpR + lane] = p;
      if (lane == 0) {
        const float al = (m1 == -INFINITY) ? 1.f : expf(m0 - m1);
        m_s[g] = m1;
        l_s[g] = l_s[g] * al + l;
        lb_s[g] = lb_s[g] * al + lb;
        al_s[g] = al;
      }
    }
    __syncthreads();
    // accumulate sum_t p_t [u_t | mv_t]
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = tid + j * kSpThreads;
      if (c < ncol) {
        const bool isu = c < hidden;
        const float* y = isu ? U + c : MV + (c - hidden);
        const int ys = isu ? hidden : d_h;
#pragma unroll
        for (int g = 0; g < GM; ++g)
          if (g < G) acc[j][g] *= al_s[g];
#pragma unroll
        for (int r = 0; r < kSpR; r += 4) {
          const float y0 = y[r * ys], y1 = y[(r + 1) * ys], y2 = y[(r + 2) * ys], y3 = y[(r + 3) * ys];
#pragma unroll
          for (int g = 0; g < GM; ++g)
            if (g < G) {
              const float4 p4 = *reinterpret_cast<const float4*>(zp + g * kSpR + r);
              acc[j][g] = fmaf(p4.w, y3, fmaf(p4.z, y2, fmaf(p4.y, y1, fmaf(p4.x, y0, acc[j][g]))));
            }
        }
      }
    }
  }
  __syncthreads();
  // sum p u -> U as [G][hidden]; sum p mv -> MK as [G][d_h]
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int c = tid + j * kSpThreads;
    if (c < ncol) {
#pragma unroll
      for (int g = 0; g < GM; ++g)
        if (g < G) {
          if (c < hidden)
            U[g * hidden + c] = acc[j][g];
          else
            MK[g * d_h + c - hidden] = acc[j][g];
        }
    }
  }
  __syncthreads();
  // unnormalised output of the share: sum p mv + W4_V (sum p u) + b4_V sum_{coded} p
  float* pp = part + (bh * P.nsplit + sp) * G * (d_h + 2);
  for (int e = warp; e < d_h; e += kSpWarps) {
    float a[GM];
#pragma unroll
    for (int g = 0; g < GM; ++g) a[g] = 0.f;
    const E* w4 = W4 + (int64_t)(d_h + e) * hidden;
    for (int n = lane; n < hidden; n += 32) {
      const float w = to_f(w4[n]);
#pragma unroll
      for (int g = 0; g < GM; ++g)
        if (g < G) a[g] = fmaf(w, U[g * hidden + n], a[g]);
    }
    int g;
    const float v = warp_sum_scatter<GM>(a, lane, g);
    if ((lane & (32 / GM - 1)) == 0 && g < G)
      pp[g * (d_h + 2) + 2 + e] = MK[g * d_h + e] + v + (b4 ? b4[d_h + e] * lb_s[g] : 0.f);
  }
  if (tid < G) {
    pp[tid * (d_h + 2)] = m_s[tid];
    pp[tid * (d_h + 2) + 1] = l_s[tid];
  }
}

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
  return sizeof(float) * (size_t)sp_layout(c.d_c, c.hidden, p.G, c.d_h, c.k).total;
}

template <typename E, int GM>
static cudaError_t sparse_attend(const Plan& p, const SparseParams& P, const void* q, const void* cache,
                                 const void* W3, const float* b3, const void* W4, const float* b4,
                                 const int32_t* tokens, float* part, void* ws, cudaStream_t st) {
  const auto& c = p.cfg;
  const char* cb = (const char*)cache;
  const size_t smem = sparse_smem_bytes(p);
  auto kern = sparse_attend_kernel<E, GM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(p, st, KID_SPARSE_ATTEND);
  kern<<<dim3(P.nsplit, c.kv_heads, c.batch), kSpThreads, smem, st>>>(
      P, (const E*)q, tokens, (const E*)(cb + p.off_refk), (const E*)(cb + p.off_refv), (const E*)(cb + p.off_code),
      (const int32_t*)(cb + p.off_idx), (const E*)W3, b3, (const E*)W4, b4, part, (uint32_t*)ws);
  return cudaGetLastError();
}

template <typename E>
static cudaError_t sparse_launch(const Plan& p, int T, const void* q, int64_t qsb, int64_t qsh, const void* cache,
                                 const void* W3, const float* b3, const void* W4, const float* b4,
                                 const int32_t* tokens, int n_sel, float* out, int64_t osb, int64_t osh, void* ws,
                                 cudaStream_t st) {
  const auto& c = p.cfg;
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
  P.cscale = p.code4 ? (const __nv_bfloat16*)((const char*)cache + p.off_cscale) : nullptr;
  const int64_t BH = (int64_t)c.batch * c.kv_heads;
  // shares of at least one pass each, about two CTAs per SM in total
  int nsplit = (int)std::min<int64_t>((n_sel + kSpR - 1) / kSpR, std::max<int64_t>(1, 2 * kNumSMs / BH));
  nsplit = std::max(1, std::min(nsplit, kSparseSplits));
  P.nsplit = nsplit;
  P.per = (n_sel + nsplit - 1) / nsplit;
  float* part = (float*)((char*)ws + p.ws_sparse);
  cudaError_t e = p.G <= 4 ? sparse_attend<E, 4>(p, P, q, cache, W3, b3, W4, b4, tokens, part, ws, st)
                            : sparse_attend<E, 8>(p, P, q, cache, W3, b3, W4, b4, tokens, part, ws, st);
  if (e != cudaSuccess) return e;
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
  if (p.bf16)
    return sparse_launch<__nv_bfloat16>(p, T, q, qsb, qsh, cache, W3, b3, W4, b4, tokens, n_sel, out, osb, osh, ws,
                                        st);
  return sparse_launch<float>(p, T, q, qsb, qsh, cache, W3, b3, W4, b4, tokens, n_sel, out, osb, osh, ws, st);
}

}  // namespace dkv
