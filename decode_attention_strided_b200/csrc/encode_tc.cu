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
//   phase 1  warp per token: gather, re-rank, mean, residual r -> A tiles
//   phase 2  tcgen05.mma  D1 = R . W1^T                   (fp32 in TMEM)
//   phase 3  TMEM -> + b1 -> act -> H tiles (alias the A tiles)
//   phase 4  tcgen05.mma  D2 = H . W2^T
//   phase 5  TMEM -> + b2 -> bf16 codes
// Precision: every MMA operand that is not a weight is split into two fp16
// terms, hi = fp16(v) and lo = fp16(v - hi), and multiplied twice, so r and
// act(.) enter with about 22 significant bits.  With a single fp16 (or bf16)
// term the unrounded codes would differ from exact ones by enough to flip
// the final bf16 rounding of a code element often, and each flip moves the
// decoded token.
// The MMA is M = 128; a tile uses only its first 64 rows, the other 64 read
// the neighbouring operand atom (in-bounds shared memory) and their results
// are never read, which halves the A footprint so the weights fit.
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
constexpr int ATOM = ROWS * 128;  // bytes of one 64-row x 64-column fp16 atom
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

// EPL bf16 (or fp16) values in one vector register group.
template <int EPL> struct PackT;
template <> struct PackT<8> { using type = uint4; };
template <> struct PackT<4> { using type = uint2; };
template <int EPL> using Pack = typename PackT<EPL>::type;

template <int EPL>
__device__ __forceinline__ void unpack(const Pack<EPL>& p, float (&f)[EPL]) {
  const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&p);
#pragma unroll
  for (int q = 0; q < EPL / 2; ++q) {
    const float2 v = __bfloat1622float2(p2[q]);
    f[2 * q] = v.x;
    f[2 * q + 1] = v.y;
  }
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

// EPL: bf16 elements of x each lane holds (D / 32); KC: candidates per token.
template <int EPL, int KC>
__global__ void __launch_bounds__(enc::THREADS, 1) encode_tc_kernel(const EncParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int D = EPL * 32;
  const int hid_atoms = (P.hidden + 63) / 64;
  const int rh_atoms = max(D / 64, hid_atoms);
  unsigned char* sW1 = smem;                                        // [D/64][hidden][128 B]
  unsigned char* sRH = sW1 + (D / 64) * P.hidden * 128;             // hi atoms, then lo atoms
  unsigned char* sLo = sRH + rh_atoms * enc::ATOM;                  //   [rh_atoms][64][128 B] each
  unsigned char* sW2 = sLo + rh_atoms * enc::ATOM;                  // [hid_atoms][d_c][128 B]
  uint64_t* mma_bar = (uint64_t*)(sW2 + ((hid_atoms * P.d_c * 128 + 1023) & ~1023));
  uint32_t* tmem_slot = (uint32_t*)(mma_bar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;

  // ---- weights -> fp16, 128-byte swizzled K-major atoms (once per CTA)
  for (int i = tid; i < P.hidden * D / 8; i += blockDim.x) {
    const int n = i / (D / 8), c8 = (i % (D / 8)) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(P.W1 + (int64_t)n * D + c8);
    const __nv_bfloat162* b2v = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint4 out;
    __half2* o2 = reinterpret_cast<__half2*>(&out);
#pragma unroll
    for (int q = 0; q < 4; ++q) o2[q] = __float22half2_rn(__bfloat1622float2(b2v[q]));
    *reinterpret_cast<uint4*>(sW1 + sw128_offset(n, c8, P.hidden)) = out;
  }
  for (int i = tid; i < P.d_c * hid_atoms * 8; i += blockDim.x) {
    const int o = i / (hid_atoms * 8), c8 = (i % (hid_atoms * 8)) * 8;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (c8 < P.hidden) {
      const uint4 raw = *reinterpret_cast<const uint4*>(P.W2 + (int64_t)o * P.hidden + c8);
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

  for (int tile = blockIdx.x; tile < P.n_tiles && ok; tile += gridDim.x) {
    const int bh = tile / P.tiles_per_bh;
    const int64_t row0 = (int64_t)(tile % P.tiles_per_bh) * enc::ROWS;
    const int b = bh / P.H, h = bh % P.H;
    const __nv_bfloat16* Kb = P.K + b * P.sb + h * P.sh;
    const __nv_bfloat16* Vb = P.V + b * P.sb + h * P.sh;
    const __nv_bfloat16* rk = P.refk + (int64_t)bh * P.n_ref_cap * P.d_h;
    const __nv_bfloat16* rv = P.refv + (int64_t)bh * P.n_ref_cap * P.d_h;
    const int e0 = lane * EPL;  // this lane's first element of [K ; V]
    const bool inK = e0 < P.d_h;

    // ------------------------------------------ phase 1: re-rank, mean, residual
    // Two rows per warp at a time; every gather of a row pair is issued before
    // any of them is used, so the L2 round trips overlap.
    for (int n0 = warp * 2; n0 < enc::ROWS; n0 += 16) {
      constexpr int NR = 2;
      Pack<EPL> xr[NR], rr[NR][KC];
      int jj[NR][KC];
      int64_t tt[NR];
      bool live[NR];
#pragma unroll
      for (int u = 0; u < NR; ++u) {
        const int64_t row = row0 + n0 + u;
        live[u] = row < P.n_code;
        tt[u] = live[u] ? (row / (P.s - 1)) * P.s + (row % (P.s - 1)) + 1 : 0;
        const int my_c = (live[u] && lane < KC) ? P.cand[((int64_t)bh * P.n_code_cap + row) * KC + lane] : -1;
        if (live[u]) {
          const __nv_bfloat16* src = inK ? Kb + tt[u] * P.st + e0 : Vb + tt[u] * P.st + (e0 - P.d_h);
          xr[u] = *reinterpret_cast<const Pack<EPL>*>(src);
        }
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          int j = __shfl_sync(0xffffffffu, my_c, c);
          if (j >= 0 && (int64_t)j * P.s >= tt[u]) {  // not an earlier reference: drop it
            if (lane == 0) latch_error(P.err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j);
            j = -1;
          }
          jj[u][c] = j;
        }
      }
#pragma unroll
      for (int u = 0; u < NR; ++u)
#pragma unroll
        for (int c = 0; c < KC; ++c)
          if (jj[u][c] >= 0) {
            const int j = jj[u][c];
            const __nv_bfloat16* src = inK ? rk + (int64_t)j * P.d_h + e0 : rv + (int64_t)j * P.d_h + (e0 - P.d_h);
            rr[u][c] = *reinterpret_cast<const Pack<EPL>*>(src);
          }
#pragma unroll
      for (int u = 0; u < NR; ++u) {
        const int n = n0 + u;
        const int64_t row = row0 + n;
        float rres[EPL];
        if (live[u]) {
          float xv[EPL];
          unpack<EPL>(xr[u], xv);
          float cd[KC];
#pragma unroll
          for (int c = 0; c < KC; ++c) {
            float part = 0.f;
            if (jj[u][c] >= 0) {
              float rf[EPL];
              unpack<EPL>(rr[u][c], rf);
#pragma unroll
              for (int q = 0; q < EPL; ++q) {
                const float df = xv[q] - rf[q];
                part = fmaf(df, df, part);
              }
            }
            part = warp_sum(part);
            cd[c] = jj[u][c] >= 0 ? part : FLT_MAX;
          }
          // the k smallest (distance, slot) of the candidates, ascending
          uint32_t chosen = 0;
          int k_eff = 0, my_sel = -1;
          for (int q = 0; q < P.k; ++q) {
            int best = -1;
            float bdv = FLT_MAX;
            int bj = INT_MAX;
#pragma unroll
            for (int c = 0; c < KC; ++c) {
              const bool avail = jj[u][c] >= 0 && !(chosen & (1u << c));
              if (avail && (cd[c] < bdv || (cd[c] == bdv && jj[u][c] < bj))) {
                best = c;
                bdv = cd[c];
                bj = jj[u][c];
              }
            }
            if (best >= 0) {
              chosen |= 1u << best;
              ++k_eff;
            }
            if (lane == q) my_sel = best >= 0 ? bj : -1;
          }
          if (lane < P.k) P.idx[((int64_t)bh * P.n_code_cap + row) * P.k + lane] = my_sel;
          const float inv = 1.0f / (float)max(k_eff, 1);
          float m[EPL];
#pragma unroll
          for (int q = 0; q < EPL; ++q) m[q] = 0.f;
#pragma unroll
          for (int c = 0; c < KC; ++c)
            if (chosen & (1u << c)) {
              float rf[EPL];
              unpack<EPL>(rr[u][c], rf);
#pragma unroll
              for (int q = 0; q < EPL; ++q) m[q] += rf[q];
            }
#pragma unroll
          for (int q = 0; q < EPL; ++q) rres[q] = xv[q] - m[q] * inv;
        } else {
#pragma unroll
          for (int q = 0; q < EPL; ++q) rres[q] = 0.f;
        }
        // r = hi + lo in fp16, into the swizzled A tiles
        __half2 hi2[EPL / 2], lo2[EPL / 2];
#pragma unroll
        for (int q = 0; q < EPL / 2; ++q) split_half2(rres[2 * q], rres[2 * q + 1], hi2[q], lo2[q]);
        const uint32_t off = sw128_offset(n, e0, enc::ROWS);
        *reinterpret_cast<Pack<EPL>*>(sRH + off) = *reinterpret_cast<const Pack<EPL>*>(hi2);
        *reinterpret_cast<Pack<EPL>*>(sLo + off) = *reinterpret_cast<const Pack<EPL>*>(lo2);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // --------------------------------------------------- phase 2: GEMM1
    if (tid == 0) {
      const uint32_t w0 = smem_u32(sW1);
      const uint32_t idesc = idesc_f16_f32(enc::MMA_M, P.hidden);
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        const uint32_t a0 = smem_u32(part == 0 ? sRH : sLo);
#pragma unroll 1
        for (int k16 = 0; k16 < D / 16; ++k16) {
          const int atom = k16 >> 2, off = (k16 & 3) * 32;
          umma_f16(tmem, desc_kmajor_sw128(a0 + atom * enc::ATOM + off),
                   desc_kmajor_sw128(w0 + atom * P.hidden * 128 + off), idesc, (part | k16) != 0);
        }
      }
      umma_commit(mma_bar);
    }
    if (!mbar_wait(mma_bar, mma_phase, abort_flag)) { ok = false; break; }
    mma_phase ^= 1;
    tc_fence_after();

    // ------------------------------------------- phase 3: act(D1 + b1) -> H
    // rows 0..63 live in TMEM lanes 0..63: warps 0, 1 (columns of the first
    // half) and 4, 5 (second half) read them
    if ((warp & 3) < 2) {
      const int q = warp & 3, half = warp >> 2, n = q * 32 + lane;
      const int cols = P.hidden / 2;
      for (int c0 = half * cols; c0 < (half + 1) * cols; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + c0, v);
        __half2 hi2[8], lo2[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float a = act_fast(P.act, v[2 * x] + (P.b1 ? P.b1[c0 + 2 * x] : 0.f));
          const float bq = act_fast(P.act, v[2 * x + 1] + (P.b1 ? P.b1[c0 + 2 * x + 1] : 0.f));
          split_half2(a, bq, hi2[x], lo2[x]);
        }
        const uint32_t o0 = sw128_offset(n, c0, enc::ROWS), o1 = sw128_offset(n, c0 + 8, enc::ROWS);
        *reinterpret_cast<uint4*>(sRH + o0) = *reinterpret_cast<const uint4*>(&hi2[0]);
        *reinterpret_cast<uint4*>(sRH + o1) = *reinterpret_cast<const uint4*>(&hi2[4]);
        *reinterpret_cast<uint4*>(sLo + o0) = *reinterpret_cast<const uint4*>(&lo2[0]);
        *reinterpret_cast<uint4*>(sLo + o1) = *reinterpret_cast<const uint4*>(&lo2[4]);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // --------------------------------------------------- phase 4: GEMM2
    if (tid == 0) {
      const uint32_t w0 = smem_u32(sW2);
      const uint32_t idesc = idesc_f16_f32(enc::MMA_M, P.d_c);
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        const uint32_t h0 = smem_u32(part == 0 ? sRH : sLo);
#pragma unroll 1
        for (int k16 = 0; k16 < P.hidden / 16; ++k16) {
          const int atom = k16 >> 2, off = (k16 & 3) * 32;
          umma_f16(tmem + enc::D2_COL, desc_kmajor_sw128(h0 + atom * enc::ATOM + off),
                   desc_kmajor_sw128(w0 + atom * P.d_c * 128 + off), idesc, (part | k16) != 0);
        }
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
  const size_t w2 = ((size_t)hid_atoms * d_c * 128 + 1023) & ~size_t(1023);
  const size_t rh = 2 * (size_t)std::max(D / 64, hid_atoms) * enc::ATOM;
  // the M = 128 reads of the last lo atom run 8 KB past it: W2 (and, when W2
  // is shorter than that, the padding below) keeps them inside the block
  const size_t tail = w2 < (size_t)enc::ATOM ? (size_t)enc::ATOM - w2 : 0;
  return 1024 + w1 + rh + w2 + tail + 64;
}

bool encode_tc_supported(const Plan& p) {
  const auto& c = p.cfg;
  return c.dtype == DELTAKV_BF16 && (c.d_h == 64 || c.d_h == 128) && c.hidden % 32 == 0 &&
         c.hidden <= 256 && c.d_c % 16 == 0 && c.d_c <= 256 && encode_tc_smem(p) <= 227 * 1024;
}

namespace {
template <int EPL, int KC>
cudaError_t encode_tc_launch(const EncParams& P, size_t smem, int grid, cudaStream_t st) {
  auto kern = encode_tc_kernel<EPL, KC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, enc::THREADS, smem, st>>>(P);
  return cudaGetLastError();
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
  ProfScope ps(p, st, KID_ENCODE);
  if (c.d_h == 128)
    return p.KC == 8 ? encode_tc_launch<8, 8>(P, smem, grid, st) : encode_tc_launch<8, 12>(P, smem, grid, st);
  return p.KC == 8 ? encode_tc_launch<4, 8>(P, smem, grid, st) : encode_tc_launch<4, 12>(P, smem, grid, st);
}

}  // namespace dkv
