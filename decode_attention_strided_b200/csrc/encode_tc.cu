// encode_tc.cu -- exact re-rank + reference mean + residual + compressor MLP
// on the 5th-generation tensor cores, writing the packed cache.
//
// DeltaKV summary, section 3, "Processo di Compressione" steps 1-4 (the
// selection is finished here from the k + 4 candidates the tensor-core search
// kept):
//   1. exact fp32 distances |x_t - r_j|^2 to the candidates; the k smallest
//      by (distance, slot) are the token's references (idx plane);
//   2. KV_R = their mean;  3. r = x_t - KV_R;
//   4. code = W2 act(W1 r + b1) + b2  (code plane, rounded to bf16).
//
// One persistent CTA per SM, 8 warps.  W1 [hidden x D] and W2 [d_c x hidden]
// stay in shared memory as fp16 for the whole launch (bf16 values are exact
// in fp16); per 64-row tile:
//   phase 1  8 lanes per token, 32 tokens in flight: gather the k + 4
//            candidate rows, exact distances, choose k, reload them for the
//            mean, residual r -> R tile (64 tokens x D, K-major)
//   phase 2  tcgen05.mma  D1^T = W1 . R^T  (M = 128 hidden units per half,
//            N = 64 tokens; fp32 in TMEM): TMEM lanes are hidden units
//   phase 3  all 8 warps: thread = hidden unit, act(D1 + b1) over its 64
//            tokens -> H tile stored as hidden rows of 64 tokens, which is
//            the MN-major A operand of
//   phase 4  tcgen05.mma  codes = H . W2^T  (M = 128 with 64 tokens, N = d_c)
//   phase 5  TMEM -> + b2 -> bf16 codes
// Precision: every MMA operand that is not a weight is split into two fp16
// terms, hi = fp16(v) and lo = fp16(v - hi), and multiplied twice, so r and
// act(.) enter with about 22 significant bits.  With a single fp16 (or bf16)
// term the unrounded codes would differ from exact ones by enough to flip
// the final bf16 rounding of a code element often, and each flip moves the
// decoded token.
#include <cfloat>
#include <climits>

#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace dkv {
using namespace sm100;

namespace enc {
constexpr int ROWS = 64;       // compressed rows per tile (the MMA runs M = 128)
constexpr int MMA_M = 128;
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t D2_COL = 256;  // TMEM column of the second accumulator
}  // namespace enc

// tcgen05 kind::f16 instruction descriptor, fp16 A/B, fp32 D, K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of element (row, col) of a K-major operand stored as 128-byte
// swizzled atoms of `rows_per_atom` rows x 64 fp16 columns.
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, int rows_per_atom) {
  const int atom = col >> 6, c = col & 63;
  return (uint32_t)(atom * rows_per_atom * 128 + row * 128 + ((((c >> 3) ^ (row & 7))) << 4) + (c & 7) * 2);
}

// MN-major, 128-byte swizzle descriptor: 64 contiguous M-elements per 128-byte
// row, 8-row K groups `sbo` bytes apart, 64-element M blocks `lbo` apart.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128_enc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// v = hi + lo with hi = fp16(v), lo = fp16(v - hi), for two values at once.
__device__ __forceinline__ void split_half2(float a, float b, __half2& hi, __half2& lo) {
  hi = __floats2half2_rn(a, b);
  const float2 h = __half22float2(hi);
  lo = __floats2half2_rn(a - h.x, b - h.y);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

struct EncParams {
  int T, s, d_h, H, k, d_c, hidden, act, BH;
  int64_t n_code, n_ref, n_ref_cap, n_code_cap;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t sb, sh, st;
  const __nv_bfloat16* W1;
  const float* b1;
  const __nv_bfloat16* W2;
  const float* b2;
  const __nv_bfloat16* refk;
  const __nv_bfloat16* refv;
  __nv_bfloat16* code;
  int32_t* idx;
  const int32_t* cand;
  uint32_t* err;
  int n_tiles, tiles_per_bh;
};

// EPL: elements of [K ; V] per lane with 8 lanes per row (D / 8);
// KC: candidates per token; ACT: activation; HAS_B: biases present.
template <int EPL> struct RowPack;
template <> struct RowPack<32> { static constexpr int V4 = 4; };  // 4 x 16 B
template <> struct RowPack<16> { static constexpr int V4 = 2; };  // 2 x 16 B

template <int EPL>
__device__ __forceinline__ void load_row(const __nv_bfloat16* src, uint4 (&r)[RowPack<EPL>::V4]) {
#pragma unroll
  for (int i = 0; i < RowPack<EPL>::V4; ++i) r[i] = __ldg(reinterpret_cast<const uint4*>(src) + i);
}

template <int EPL>
__device__ __forceinline__ void unpack_row(const uint4 (&r)[RowPack<EPL>::V4], float (&f)[EPL]) {
#pragma unroll
  for (int i = 0; i < RowPack<EPL>::V4; ++i) {
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&r[i]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 v = __bfloat1622float2(p2[q]);
      f[8 * i + 2 * q] = v.x;
      f[8 * i + 2 * q + 1] = v.y;
    }
  }
}

__device__ __forceinline__ float group8_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 4, 8);
  v += __shfl_xor_sync(0xffffffffu, v, 2, 8);
  v += __shfl_xor_sync(0xffffffffu, v, 1, 8);
  return v;
}

template <int ACT>
__device__ __forceinline__ float enc_act(float v) {
  if (ACT == DELTAKV_ACT_GELU_ERF) return gelu_fast(v);
  return act_eval(ACT, v);
}

template <int EPL, int KC, int ACT>
__global__ void __launch_bounds__(enc::THREADS, 1) encode_tc_kernel(const EncParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int D = EPL * 8;
  constexpr int KA = D / 64;                       // 64-column atoms along D
  const int hidden = P.hidden, hid_atoms = (hidden + 63) / 64;
  // shared memory: W1 [hidden rows][D] K-major (A of GEMM1^T), then the
  // R tile (B of GEMM1^T: 64 token rows x D, hi atoms then lo atoms) which
  // the H tile (A of GEMM2, MN-major: hidden rows x 64 tokens, hi then lo)
  // later overwrites, then W2 [d_c rows][hidden] K-major (B of GEMM2)
  unsigned char* sW1 = smem;
  unsigned char* sR = sW1 + (size_t)KA * hidden * 128;
  const size_t r_part = (size_t)KA * enc::ROWS * 128;          // one of hi / lo
  const size_t h_part = (size_t)hidden * 128;                  // one of hi / lo
  const size_t rh_b = r_part > h_part ? 2 * r_part : 2 * h_part;
  unsigned char* sW2 = sR + rh_b;
  uint64_t* mma_bar = (uint64_t*)(sW2 + (((size_t)hid_atoms * P.d_c * 128 + 1023) & ~size_t(1023)));
  uint32_t* tmem_slot = (uint32_t*)(mma_bar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;

  // ---- weights -> fp16 (bf16 values are exact in fp16), swizzled K-major
  for (int i = tid; i < hidden * D / 8; i += blockDim.x) {
    const int n = i / (D / 8), c8 = (i % (D / 8)) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(P.W1 + (int64_t)n * D + c8);
    const __nv_bfloat162* b2v = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint4 out;
    __half2* o2 = reinterpret_cast<__half2*>(&out);
#pragma unroll
    for (int q = 0; q < 4; ++q) o2[q] = __float22half2_rn(__bfloat1622float2(b2v[q]));
    *reinterpret_cast<uint4*>(sW1 + sw128_offset(n, c8, hidden)) = out;
  }
  for (int i = tid; i < P.d_c * hid_atoms * 8; i += blockDim.x) {
    const int o = i / (hid_atoms * 8), c8 = (i % (hid_atoms * 8)) * 8;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (c8 < hidden) {
      const uint4 raw = *reinterpret_cast<const uint4*>(P.W2 + (int64_t)o * hidden + c8);
      const __nv_bfloat162* b2v = reinterpret_cast<const __nv_bfloat162*>(&raw);
      __half2* o2 = reinterpret_cast<__half2*>(&out);
#pragma unroll
      for (int q = 0; q < 4; ++q) o2[q] = __float22half2_rn(__bfloat1622float2(b2v[q]));
    }
    *reinterpret_cast<uint4*>(sW2 + sw128_offset(o, c8, P.d_c)) = out;
  }
  if (tid == 0) {
    mbar_init(mma_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, enc::TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t mma_phase = 0;
  bool ok = true;

  const int grp = lane >> 3, s8 = lane & 7;   // row within the warp's 4, lane within the row
  const int e0 = s8 * EPL;                     // this lane's first element of [K ; V]
  const bool inK = e0 < P.d_h;

  for (int tile = blockIdx.x; tile < P.n_tiles && ok; tile += gridDim.x) {
    const int bh = tile / P.tiles_per_bh;
    const int64_t row0 = (int64_t)(tile % P.tiles_per_bh) * enc::ROWS;
    const int b = bh / P.H, h = bh % P.H;
    const __nv_bfloat16* Kb = P.K + b * P.sb + h * P.sh;
    const __nv_bfloat16* Vb = P.V + b * P.sb + h * P.sh;
    const __nv_bfloat16* rk = P.refk + (int64_t)bh * P.n_ref_cap * P.d_h;
    const __nv_bfloat16* rv = P.refv + (int64_t)bh * P.n_ref_cap * P.d_h;

    // ------------------------------- phase 1: re-rank, mean, residual (8 lanes / row)
    for (int n = warp * 4 + grp; n < enc::ROWS; n += 32) {
      const int64_t row = row0 + n;
      const bool live = row < P.n_code;
      const int64_t t = live ? (row / (P.s - 1)) * P.s + (row % (P.s - 1)) + 1 : 0;
      const int32_t* cr = P.cand + ((int64_t)bh * P.n_code_cap + row) * KC;
      const int myc0 = (live && s8 < KC) ? cr[s8] : -1;
      const int myc1 = (live && s8 + 8 < KC) ? cr[s8 + 8] : -1;
      float xv[EPL];
      {
        uint4 xr[RowPack<EPL>::V4];
        if (live) load_row<EPL>(inK ? Kb + t * P.st + e0 : Vb + t * P.st + (e0 - P.d_h), xr);
        else
#pragma unroll
          for (int i = 0; i < RowPack<EPL>::V4; ++i) xr[i] = make_uint4(0, 0, 0, 0);
        unpack_row<EPL>(xr, xv);
      }
      int cj[KC];
      float cd[KC];
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        int j = c < 8 ? __shfl_sync(0xffffffffu, myc0, c, 8) : __shfl_sync(0xffffffffu, myc1, c - 8, 8);
        if (j >= 0 && (int64_t)j * P.s >= t) {  // not an earlier reference: drop it
          if (s8 == 0) latch_error(P.err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j);
          j = -1;
        }
        cj[c] = j;
      }
      // exact distances, 4 candidate rows in flight at a time
#pragma unroll
      for (int c0 = 0; c0 < KC; c0 += 4) {
        uint4 rr[4][RowPack<EPL>::V4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = cj[c0 + u];
          if (j >= 0) load_row<EPL>(inK ? rk + (int64_t)j * P.d_h + e0 : rv + (int64_t)j * P.d_h + (e0 - P.d_h), rr[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float part = 0.f;
          if (cj[c0 + u] >= 0) {
            float rf[EPL];
            unpack_row<EPL>(rr[u], rf);
#pragma unroll
            for (int q = 0; q < EPL; ++q) {
              const float df = xv[q] - rf[q];
              part = fmaf(df, df, part);
            }
          }
          part = group8_sum(part);
          cd[c0 + u] = cj[c0 + u] >= 0 ? part : FLT_MAX;
        }
      }
      // the k smallest (distance, slot), ascending
      uint32_t chosen = 0;
      int k_eff = 0, my_sel = -1;
      for (int qk = 0; qk < P.k; ++qk) {
        int best = -1;
        float bdv = FLT_MAX;
        int bj = INT_MAX;
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          const bool avail = cj[c] >= 0 && !(chosen & (1u << c));
          if (avail && (cd[c] < bdv || (cd[c] == bdv && cj[c] < bj))) {
            best = c;
            bdv = cd[c];
            bj = cj[c];
          }
        }
        if (best >= 0) {
          chosen |= 1u << best;
          ++k_eff;
        }
        if (s8 == qk) my_sel = best >= 0 ? bj : -1;
      }
      if (live && s8 < P.k) P.idx[((int64_t)bh * P.n_code_cap + row) * P.k + s8] = my_sel;
      // mean of the chosen rows (reloaded: they are in L2), residual
      float m[EPL];
#pragma unroll
      for (int q = 0; q < EPL; ++q) m[q] = 0.f;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        if (chosen & (1u << c)) {
          const int j = cj[c];
          uint4 rr[RowPack<EPL>::V4];
          load_row<EPL>(inK ? rk + (int64_t)j * P.d_h + e0 : rv + (int64_t)j * P.d_h + (e0 - P.d_h), rr);
          float rf[EPL];
          unpack_row<EPL>(rr, rf);
#pragma unroll
          for (int q = 0; q < EPL; ++q) m[q] += rf[q];
        }
      }
      const float inv = 1.0f / (float)max(k_eff, 1);
      // r = hi + lo (fp16) into the R tile: row n, columns e0 .. e0 + EPL
#pragma unroll
      for (int v = 0; v < EPL / 8; ++v) {
        __half2 hi2[4], lo2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = 8 * v + 2 * q;
          const float r0 = live ? xv[i] - m[i] * inv : 0.f;
          const float r1 = live ? xv[i + 1] - m[i + 1] * inv : 0.f;
          split_half2(r0, r1, hi2[q], lo2[q]);
        }
        const uint32_t off = sw128_offset(n, e0 + 8 * v, enc::ROWS);
        *reinterpret_cast<uint4*>(sR + off) = *reinterpret_cast<const uint4*>(hi2);
        *reinterpret_cast<uint4*>(sR + r_part + off) = *reinterpret_cast<const uint4*>(lo2);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ------------------------------ phase 2: D1^T = W1 . R^T (hidden x tokens)
    if (tid == 0) {
      const uint32_t w0 = smem_u32(sW1), r0 = smem_u32(sR);
      const uint32_t idesc = idesc_f16_f32(128, enc::ROWS);
#pragma unroll 1
      for (int hh = 0; hh < hidden / 128; ++hh)
#pragma unroll 1
        for (int part = 0; part < 2; ++part)
#pragma unroll 1
          for (int k16 = 0; k16 < D / 16; ++k16) {
            const int atom = k16 >> 2, off = (k16 & 3) * 32;
            umma_f16(tmem + enc::ROWS * hh,
                     desc_kmajor_sw128(w0 + atom * hidden * 128 + hh * 128 * 128 + off),
                     desc_kmajor_sw128(r0 + part * (uint32_t)r_part + atom * enc::ROWS * 128 + off), idesc,
                     (part | k16) != 0);
          }
      umma_commit(mma_bar);
    }
    if (!mbar_wait(mma_bar, mma_phase, abort_flag)) { ok = false; break; }
    mma_phase ^= 1;
    tc_fence_after();

    // ---------------- phase 3: H = act(D1 + b1), hidden rows x 64 tokens (all 8 warps)
    if (warp < 4 * (hidden / 128)) {
      const int q = warp & 3, hh = warp >> 2;
      const int unit = 128 * hh + 32 * q + lane;
      const float bias = P.b1 ? P.b1[unit] : 0.f;
      float v[64];
      tmem_ld64(tmem + ((uint32_t)(32 * q) << 16) + enc::ROWS * hh, v);
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        __half2 hi2[4], lo2[4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
          split_half2(enc_act<ACT>(v[8 * c8 + 2 * x] + bias), enc_act<ACT>(v[8 * c8 + 2 * x + 1] + bias), hi2[x],
                      lo2[x]);
        // MN-major row `unit` of 64 tokens: 16-byte chunk c8, swizzled by row
        const uint32_t off = (uint32_t)unit * 128 + (((c8 ^ (unit & 7))) << 4);
        *reinterpret_cast<uint4*>(sR + off) = *reinterpret_cast<const uint4*>(hi2);
        *reinterpret_cast<uint4*>(sR + h_part + off) = *reinterpret_cast<const uint4*>(lo2);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // --------------------------- phase 4: codes = H . W2^T (tokens x d_c)
    if (tid == 0) {
      const uint32_t w0 = smem_u32(sW2), h0 = smem_u32(sR);
      const uint32_t idesc = idesc_f16_f32(enc::MMA_M, P.d_c) | (1u << 15);  // A MN-major
#pragma unroll 1
      for (int part = 0; part < 2; ++part)
#pragma unroll 1
        for (int k16 = 0; k16 < hidden / 16; ++k16) {
          // A: 16 hidden rows per step; the second 64-token block (rows of the
          // M = 128 MMA that no token owns) reads the same rows again
          const uint64_t ad = desc_mnmajor_sw128_enc(h0 + part * (uint32_t)h_part + k16 * 16 * 128, 0, 1024);
          const uint64_t bd = desc_kmajor_sw128(w0 + (k16 >> 2) * P.d_c * 128 + (k16 & 3) * 32);
          umma_f16(tmem + enc::D2_COL, ad, bd, idesc, (part | k16) != 0);
        }
      umma_commit(mma_bar);
    }
    if (!mbar_wait(mma_bar, mma_phase, abort_flag)) { ok = false; break; }
    mma_phase ^= 1;
    tc_fence_after();

    // ----------------------------------------- phase 5: codes = D2 + b2
    if (warp < 2) {
      const int n = warp * 32 + lane;
      const int64_t row = row0 + n;
      for (int c0 = 0; c0 < P.d_c; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + enc::D2_COL + c0, v);
        if (row < P.n_code) {
          uint4 o[2];
          __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(o);
#pragma unroll
          for (int x = 0; x < 8; ++x)
            o2[x] = __floats2bfloat162_rn(v[2 * x] + (P.b2 ? P.b2[c0 + 2 * x] : 0.f),
                                          v[2 * x + 1] + (P.b2 ? P.b2[c0 + 2 * x + 1] : 0.f));
          uint4* dst = reinterpret_cast<uint4*>(P.code + ((int64_t)bh * P.n_code_cap + row) * P.d_c + c0);
          dst[0] = o[0];
          dst[1] = o[1];
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (!ok) {
    if (lane == 0) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 10);
    *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, enc::TMEM_COLS);
  }
}

size_t encode_tc_smem(const Plan& p) {
  const int D = p.D, hidden = p.cfg.hidden, d_c = p.cfg.d_c;
  const int hid_atoms = (hidden + 63) / 64;
  const size_t w1 = (size_t)(D / 64) * hidden * 128;
  const size_t rh = std::max(2 * (size_t)(D / 64) * enc::ROWS * 128, 2 * (size_t)hidden * 128);
  const size_t w2 = ((size_t)hid_atoms * d_c * 128 + 1023) & ~size_t(1023);
  return 1024 + w1 + rh + w2 + 64;
}

bool encode_tc_supported(const Plan& p) {
  const auto& c = p.cfg;
  return c.dtype == DELTAKV_BF16 && (c.d_h == 64 || c.d_h == 128) && (c.hidden == 128 || c.hidden == 256) &&
         c.d_c % 16 == 0 && c.d_c <= 256 && encode_tc_smem(p) <= 227 * 1024;
}

namespace {
template <int EPL, int KC, int ACT>
cudaError_t encode_tc_launch3(const EncParams& P, size_t smem, int grid, cudaStream_t st) {
  auto kern = encode_tc_kernel<EPL, KC, ACT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, enc::THREADS, smem, st>>>(P);
  return cudaGetLastError();
}
template <int EPL, int KC>
cudaError_t encode_tc_launch(const EncParams& P, size_t smem, int grid, cudaStream_t st) {
  if (P.act == DELTAKV_ACT_GELU_ERF) return encode_tc_launch3<EPL, KC, DELTAKV_ACT_GELU_ERF>(P, smem, grid, st);
  if (P.act == DELTAKV_ACT_GELU_TANH) return encode_tc_launch3<EPL, KC, DELTAKV_ACT_GELU_TANH>(P, smem, grid, st);
  return encode_tc_launch3<EPL, KC, DELTAKV_ACT_NONE>(P, smem, grid, st);
}
}  // namespace

cudaError_t launch_encode_tc(const Plan& p, int T, const KVView& kv, const void* W1, const float* b1,
                             const void* W2, const float* b2, void* cache, void* ws, cudaStream_t st) {
  const auto& c = p.cfg;
  const int64_t n_code = n_code_of(T, c.stride_s);
  if (n_code == 0) return cudaSuccess;
  char* cb = (char*)cache;
  EncParams P;
  P.T = T;
  P.s = c.stride_s;
  P.d_h = c.d_h;
  P.H = c.kv_heads;
  P.k = c.k;
  P.d_c = c.d_c;
  P.hidden = c.hidden;
  P.act = (int)c.act;
  P.BH = c.batch * c.kv_heads;
  P.n_code = n_code;
  P.n_ref = n_ref_of(T, c.stride_s);
  P.n_ref_cap = p.n_ref_cap;
  P.n_code_cap = p.n_code_cap;
  P.K = (const __nv_bfloat16*)kv.K;
  P.V = (const __nv_bfloat16*)kv.V;
  P.sb = kv.sb;
  P.sh = kv.sh;
  P.st = kv.st;
  P.W1 = (const __nv_bfloat16*)W1;
  P.b1 = b1;
  P.W2 = (const __nv_bfloat16*)W2;
  P.b2 = b2;
  P.refk = (const __nv_bfloat16*)(cb + p.off_refk);
  P.refv = (const __nv_bfloat16*)(cb + p.off_refv);
  P.code = (__nv_bfloat16*)(cb + p.off_code);
  P.idx = (int32_t*)(cb + p.off_idx);
  P.cand = (const int32_t*)((char*)ws + p.ws_cand);
  P.err = (uint32_t*)ws;
  P.tiles_per_bh = (int)ceil_div64(n_code, enc::ROWS);
  P.n_tiles = P.tiles_per_bh * P.BH;
  int dev = 0, sms = kNumSMs;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(P.n_tiles, sms);
  const size_t smem = encode_tc_smem(p);
  ProfScope ps(p, st, KID_ENCODE_TC);
  if (c.d_h == 128)
    return p.KC == 8 ? encode_tc_launch<32, 8>(P, smem, grid, st) : encode_tc_launch<32, 12>(P, smem, grid, st);
  return p.KC == 8 ? encode_tc_launch<16, 8>(P, smem, grid, st) : encode_tc_launch<16, 12>(P, smem, grid, st);
}

}  // namespace dkv
