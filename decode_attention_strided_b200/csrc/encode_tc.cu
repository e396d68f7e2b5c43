// encode_tc.cu -- exact re-rank + reference mean + residual + compressor MLP
// on the 5th-generation tensor cores, writing the packed cache.
//
// DeltaKV summary, section 3, "Processo di Compressione" steps 1-4 (the
// selection is finished here from the k + 4 candidates the tensor-core search
// kept):
//   1. exact fp32 distances |x_t - r_j|^2 to the candidates; the k smallest
//      by (distance, slot) are the token's references (idx plane);
//   2. KV_R = their mean;  3. r = x_t - KV_R;
//   4. code = W2 act(W1 r + b1) + b2  (code plane: bf16, or 4-bit values with
//      one bf16 scale per row).
//
// One persistent CTA per SM, 16 warps with fixed roles, per 64-row tile:
//   gather warps (11)  16 lanes per token row, a pair of rows at a time,
//            pairs claimed from a shared counter in tile order; the next
//            pair's x and candidate slots are loaded ahead, and with k + 4 = 8
//            its candidate rows too, at the end of the current pair's work
//            (kept in registers for the mean), else four at a time; exact
//            fp32 distances, each candidate ranked by one lane, the chosen
//            set by ballot; r = x - mean -> R tile (64
//            tokens x D, K-major, hi and lo), double-buffered so the next
//            tile's gather overlaps
//   MMA warp  tcgen05.mma  D1^T = W1 . R^T  (A = W1 held in tensor memory
//            for the whole launch, M = 128 hidden units per half, N = 64
//            tokens); then codes = H . W2^T (A = the H tile through an
//            MN-major descriptor, M = 128 with 64 tokens, N = d_c)
//   activation warps (4)  thread = hidden unit: act(D1 + b1) over the tile's
//            64 tokens -> H tile (hidden rows of 64 tokens, hi and lo), then
//            TMEM -> + b2 -> bf16 codes (or 4-bit codes and their scale)
// W1 and W2 are converted to fp16 once per launch (bf16 values of normal
// range are exact in fp16).
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
constexpr int ROWS = 64;          // compressed rows per tile (GEMM1^T N; GEMM2 runs M = 128)
constexpr int MMA_M = 128;
constexpr int GATHER_WARPS = 11;  // warps 0-10: re-rank, mean, residual
constexpr int MMA_WARP = 11;      // warp 11: TMEM allocation and MMA issue
constexpr int ACT0 = 12;          // warps 12-15: activation and code store; warp w reads TMEM lanes 32 (w % 4)..
constexpr int ACT_WARPS = 4;
constexpr int THREADS = 16 * 32;  // four warps per scheduler: 128 registers a thread
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t W1_COL = 0;    // W1 halves, D/2 packed columns each
constexpr uint32_t D1_COL = 256;  // GEMM1^T accumulators, 64 columns per half
constexpr uint32_t D2_COL = 384;  // GEMM2 accumulator, d_c columns
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

// One code row of 4-bit codes from the GEMM2 accumulator (TMEM lane = row,
// DC fp32 columns from taddr): + b2, quantised by quantize_row4 and stored as
// DC / 2 bytes plus its bf16 scale when `live`.  Warp-collective (every lane
// runs the TMEM loads).
template <int DC>
__device__ __forceinline__ void store_code4_row(uint32_t taddr, const float* b2, uint8_t* dst, __nv_bfloat16* sdst,
                                                bool live) {
  float cv[DC];
#pragma unroll
  for (int c0 = 0; c0 < DC; c0 += 16) {
    float v[16];
    tmem_ld16(taddr + c0, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) cv[c0 + i] = v[i] + (b2 ? b2[c0 + i] : 0.f);
  }
  uint8_t pk[DC / 2];
  const __nv_bfloat16 sb = quantize_row4<DC>(cv, pk);
  if (live) {
    if constexpr (DC == 16) {
      *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(pk);
    } else {
#pragma unroll
      for (int i = 0; i < DC / 32; ++i) reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(pk)[i];
    }
    *sdst = sb;
  }
}

// n / d for 0 <= n < 2^31 by one multiply-high, one add and one shift
// (division by an invariant integer, Granlund and Montgomery 1994, Thm 4.2:
// l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1; the add cannot wrap
// because n < 2^31).
struct FastDiv {
  uint32_t m, l;
  __device__ __forceinline__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> l; }
};
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while (((uint64_t)1 << l) < d) ++l;
  FastDiv f;
  f.m = (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << l) - d)) / d + 1);
  f.l = l;
  return f;
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
  __nv_bfloat16* cscale;  // 4-bit codes: per-row scales (the code plane then holds d_c / 2 bytes a row)
  int32_t* idx;
  const int32_t* cand;
  uint32_t* err;
  int n_tiles, tiles_per_bh;
  FastDiv div_tiles, div_sm1, div_H;  // by tiles_per_bh, s - 1 and H
  float inv_k;                          // 1 / k, rounded as the device rounds 1.0f / k
};

// EPL: elements of [K ; V] per lane with 16 lanes per row (D / 16).
template <int EPL> struct RowPack;
template <> struct RowPack<16> { static constexpr int V4 = 2; };  // 2 x 16 B
template <> struct RowPack<8> { static constexpr int V4 = 1; };   // 1 x 16 B

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

// Sum over the 16 lanes of each row group; the whole warp takes part (a
// constant full mask: both groups run every shuffle together).
__device__ __forceinline__ float group16_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 8, 16);
  v += __shfl_xor_sync(0xffffffffu, v, 4, 16);
  v += __shfl_xor_sync(0xffffffffu, v, 2, 16);
  v += __shfl_xor_sync(0xffffffffu, v, 1, 16);
  return v;
}

// Candidate rows in flight at a time: all of them when there are 8 (they
// stay in registers for the mean), else four (the chosen ones are loaded
// again, from L2, for the mean).
template <int KC> struct CandBatch { static constexpr int N = KC == 8 ? 8 : 4; };

template <int ACT>
__device__ __forceinline__ float enc_act(float v) {
  if (ACT == DELTAKV_ACT_GELU_ERF) return gelu_fast(v);
  return act_eval(ACT, v);
}

// Row n of a 64-row tile: its code row, token and this lane's x slice.
struct GatherRow {
  int64_t row, t;
  int64_t last_ref;        // the latest reference before token t (slot q of row = q (s - 1) + r)
  bool inrow;              // n < ROWS (the last pass of a tile may run past it)
  const __nv_bfloat16* x;  // this lane's slice of x_t (valid when live)
  const int32_t* cand;     // the row's candidate slots
  bool live;
};

template <int KC>
__device__ __forceinline__ GatherRow gather_row(const EncParams& P, int tile, int n, bool inK, int e0) {
  GatherRow g;
  // unsigned 32-bit index arithmetic: tiles, rows and tokens of one
  // (sequence, kv-head) are below 2^31
  const uint32_t bh = P.div_tiles.div((uint32_t)tile);
  const uint32_t row = ((uint32_t)tile - bh * (uint32_t)P.tiles_per_bh) * enc::ROWS + (uint32_t)n;
  g.row = row;
  g.inrow = n < enc::ROWS;
  g.live = g.inrow && g.row < P.n_code;
  // row = q (s - 1) + r with r < s - 1 is token t = q s + r + 1 = row + q + 1;
  // the references before it are slots 0 .. q
  const uint32_t q = P.div_sm1.div(row);
  g.t = g.live ? (int64_t)(row + q + 1u) : 0;
  g.last_ref = q;
  const uint32_t b = P.div_H.div(bh), h = bh - b * (uint32_t)P.H;
  g.x = (inK ? P.K + e0 : P.V + (e0 - P.d_h)) + (int64_t)b * P.sb + (int64_t)h * P.sh + g.t * P.st;
  g.cand = P.cand + ((int64_t)bh * P.n_code_cap + g.row) * KC;
  return g;
}

template <int EPL, int KC>
__device__ __forceinline__ void gather_prefetch(const EncParams& P, const GatherRow& g, int s16,
                                                uint4 (&x)[RowPack<EPL>::V4], int& c) {
  if (g.live) {
    load_row<EPL>(g.x, x);
  } else {
#pragma unroll
    for (int i = 0; i < RowPack<EPL>::V4; ++i) x[i] = make_uint4(0, 0, 0, 0);
  }
  c = (g.live && s16 < KC) ? g.cand[s16] : -1;
}

struct EncBars {
  uint64_t r_full[2], r_empty[2], d1_full, d1_empty, h_full, h_empty, d2_full, d2_empty;
  uint64_t drain;  // the MMA warp's last commit
};

template <int EPL, int KC, int ACT>
__global__ void __launch_bounds__(enc::THREADS, 1) encode_tc_kernel(const EncParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int D = EPL * 16;
  constexpr int KA = D / 64;                       // 64-column atoms along D
  const int hidden = P.hidden, nh = hidden / 128, hid_atoms = hidden / 64;
  // shared memory: two R tiles (B of GEMM1^T: 64 token rows x D, K-major,
  // hi atoms then lo atoms), the H tile (A of GEMM2, MN-major: hidden rows x
  // 64 tokens, hi then lo), W2 [d_c rows][hidden] K-major (B of GEMM2)
  const size_t r_part = (size_t)KA * enc::ROWS * 128;          // one of hi / lo
  const size_t h_part = (size_t)hidden * 128;                  // one of hi / lo
  unsigned char* sR = smem;                                    // [2][hi, lo]
  unsigned char* sH = sR + 4 * r_part;
  unsigned char* sW2 = sH + 2 * h_part;
  EncBars* bars = (EncBars*)(sW2 + (((size_t)hid_atoms * P.d_c * 128 + 1023) & ~size_t(1023)));
  uint32_t* tmem_slot = (uint32_t*)(bars + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  uint32_t* q_claim = tmem_slot + 2;  // the row-pair counter of the gather

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;

  // W2 -> fp16, swizzled K-major (bf16 values of normal range are exact in fp16)
  for (int i = tid; i < P.d_c * hid_atoms * 8; i += blockDim.x) {
    const int o = i / (hid_atoms * 8), c8 = (i % (hid_atoms * 8)) * 8;
    const uint4 raw = *reinterpret_cast<const uint4*>(P.W2 + (int64_t)o * hidden + c8);
    const __nv_bfloat162* b2v = reinterpret_cast<const __nv_bfloat162*>(&raw);
    uint4 out;
    __half2* o2 = reinterpret_cast<__half2*>(&out);
#pragma unroll
    for (int q = 0; q < 4; ++q) o2[q] = __float22half2_rn(__bfloat1622float2(b2v[q]));
    *reinterpret_cast<uint4*>(sW2 + sw128_offset(o, c8, P.d_c)) = out;
  }
  if (tid == 0) {
    mbar_init(&bars->r_full[0], enc::ROWS / 2);  // one arrival per row pair
    mbar_init(&bars->r_full[1], enc::ROWS / 2);
    *q_claim = 0;
    mbar_init(&bars->r_empty[0], 1);
    mbar_init(&bars->r_empty[1], 1);
    mbar_init(&bars->d1_full, 1);
    mbar_init(&bars->d1_empty, enc::ACT_WARPS);
    mbar_init(&bars->h_full, enc::ACT_WARPS);
    mbar_init(&bars->h_empty, 1);
    mbar_init(&bars->d2_full, 1);
    mbar_init(&bars->d2_empty, enc::ACT_WARPS);
    mbar_init(&bars->drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == enc::MMA_WARP) {
    tmem_alloc(tmem_slot, enc::TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // tiles of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int n_local = P.n_tiles > (int)blockIdx.x ? (P.n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp >= enc::ACT0 && warp < enc::ACT0 + enc::ACT_WARPS) {
    // W1 -> tensor memory, fp16: A of GEMM1^T, half hh at columns
    // W1_COL + hh D/2, lane = hidden unit within the half
    const int q = warp & 3;
    for (int hh = 0; hh < nh; ++hh) {
      const __nv_bfloat16* wrow = P.W1 + (int64_t)(hh * 128 + q * 32 + lane) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        uint32_t r[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(wrow + 2 * c0) + v);
          const __nv_bfloat162* b2v = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            __half2 h2 = __float22half2_rn(__bfloat1622float2(b2v[x]));
            r[4 * v + x] = *reinterpret_cast<uint32_t*>(&h2);
          }
        }
        tmem_st32(tmem + ((uint32_t)(q * 32) << 16) + enc::W1_COL + hh * (D / 2) + c0, r);
      }
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- the gather: exact re-rank, mean, residual, one row pair at a time
  // A tile's 64 rows are 32 pairs; a warp takes one pair (16 lanes a row).
  // Pairs are claimed from one counter in shared memory in tile order (claim
  // c is pair c % 32 of this CTA's tile c / 32), so a warp that finishes
  // early takes the next pair instead of idling behind a fixed share of the
  // rows.  Each pair arrives once on its tile's r_full.
  constexpr int PAIRS = enc::ROWS / 2;
  const int grp = lane >> 4, s16 = lane & 15;  // row within the pair, lane within the row
  const int e0 = s16 * EPL;                    // this lane's first element of [K ; V]
  const bool inK = e0 < P.d_h;
  constexpr int NB = CandBatch<KC>::N;
  // The x slice and candidate slot of the next pair are loaded before the
  // current pair's work, so only the candidate rows' latency sits on its path.
  uint4 pf_x[RowPack<EPL>::V4];
  int pf_c = -1;
  auto claim = [&]() -> uint32_t {
    uint32_t c = 0;
    if (lane == 0) c = atomicAdd(q_claim, 1u);
    return __shfl_sync(0xffffffffu, c, 0);
  };
  auto valid = [&](uint32_t c) { return c / PAIRS < (uint32_t)n_local; };
  auto prefetch = [&](uint32_t c) {
    const int tile = blockIdx.x + (int)(c / PAIRS) * gridDim.x;
    gather_prefetch<EPL, KC>(P, gather_row<KC>(P, tile, (int)(c % PAIRS) * 2 + grp, inK, e0), s16, pf_x, pf_c);
  };
  // the next pair's candidate slots (checked) and, with k + 4 = 8, its
  // candidate rows: loaded at the end of the current pair's work
  uint4 nrr[NB][RowPack<EPL>::V4];
  int ncj[KC];
  auto load_cands = [&](uint32_t c) {
    const int tile = blockIdx.x + (int)(c / PAIRS) * gridDim.x;
    const GatherRow g = gather_row<KC>(P, tile, (int)(c % PAIRS) * 2 + grp, inK, e0);
    const int bh = (int)P.div_tiles.div((uint32_t)tile);
    const __nv_bfloat16* rs = (inK ? P.refk + e0 : P.refv + (e0 - P.d_h)) + (int64_t)bh * P.n_ref_cap * P.d_h;
#pragma unroll
    for (int cc = 0; cc < KC; ++cc) {
      int j = __shfl_sync(0xffffffffu, pf_c, cc, 16);
      if (j >= 0 && j > g.last_ref) {  // not an earlier reference: drop it
        if (s16 == 0) latch_error(P.err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j);
        j = -1;
      }
      ncj[cc] = j;
    }
    if constexpr (NB == KC) {
#pragma unroll
      for (int u = 0; u < NB; ++u)
        if (ncj[u] >= 0) load_row<EPL>(rs + (int64_t)ncj[u] * P.d_h, nrr[u]);
    }
  };
  // pair c, whose x slices and slots are in pf_x / pf_c; the loads of pair
  // cn (when valid) are issued before the work
  auto process = [&](uint32_t c, uint32_t cn) -> bool {
    const int it = (int)(c / PAIRS), rb = it & 1;
    const int tile = blockIdx.x + it * gridDim.x;
    // the R buffer is free once GEMM1 of the tile two back is complete
    if (it >= 2 && !mbar_wait(&bars->r_empty[rb], ((it >> 1) - 1) & 1, abort_flag)) return false;
    const int bh = (int)P.div_tiles.div((uint32_t)tile);
    // this lane's slice of reference row j: rs + j d_h
    const __nv_bfloat16* rs = (inK ? P.refk + e0 : P.refv + (e0 - P.d_h)) + (int64_t)bh * P.n_ref_cap * P.d_h;
    unsigned char* sRb = sR + rb * 2 * r_part;
    const int n = (int)(c % PAIRS) * 2 + grp;
    const GatherRow g = gather_row<KC>(P, tile, n, inK, e0);
    float xr[EPL];
    unpack_row<EPL>(pf_x, xr);
    int cj[KC];
    float cd[KC];
#pragma unroll
    for (int u = 0; u < KC; ++u) cj[u] = ncj[u];
    uint4 rr[NB][RowPack<EPL>::V4];
    if constexpr (NB == KC) {
#pragma unroll
      for (int u = 0; u < NB; ++u)
#pragma unroll
        for (int i = 0; i < RowPack<EPL>::V4; ++i) rr[u][i] = nrr[u][i];
    }
    if (valid(cn)) prefetch(cn);
    // exact distances; with NB == KC the rows were loaded at the end of the
    // previous pair and stay in registers for the mean, else NB at a time
#pragma unroll
    for (int c0 = 0; c0 < KC; c0 += NB) {
      if constexpr (NB != KC) {
#pragma unroll
        for (int u = 0; u < NB; ++u) {
          const int j = cj[c0 + u];
          if (j >= 0) load_row<EPL>(rs + (int64_t)j * P.d_h, rr[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < NB; ++u) {
        float part = 0.f;
        if (cj[c0 + u] >= 0) {
          // even and odd elements accumulate in the two lanes of a packed
          // fp32x2 register
          unsigned long long acc = 0ull;
#pragma unroll
          for (int i = 0; i < RowPack<EPL>::V4; ++i) {
            const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&rr[u][i]);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const float2 v = __bfloat1622float2(p2[x]);
              asm("{\n\t.reg .b64 a, b, d;\n\t"
                  "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\t"
                  "sub.rn.f32x2 d, a, b;\n\tfma.rn.f32x2 %0, d, d, %0;\n\t}"
                  : "+l"(acc)
                  : "f"(xr[8 * i + 2 * x]), "f"(xr[8 * i + 2 * x + 1]), "f"(v.x), "f"(v.y));
            }
          }
          float e0, e1;
          asm("mov.b64 {%0, %1}, %2;" : "=f"(e0), "=f"(e1) : "l"(acc));
          part = e0 + e1;
        }
        part = group16_sum(part);
        cd[c0 + u] = cj[c0 + u] >= 0 ? part : FLT_MAX;
      }
    }
    // the k smallest (distance, slot), ascending: lane c of the row ranks
    // candidate c against the others; ranks below k are the references
    float my_d = FLT_MAX;
    int my_j = -1, n_valid = 0;
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      if (s16 == c) {
        my_d = cd[c];
        my_j = cj[c];
      }
      n_valid += cj[c] >= 0 ? 1 : 0;
    }
    int rank = 0;
#pragma unroll
    for (int c = 0; c < KC; ++c)
      rank += (cj[c] >= 0 && (cd[c] < my_d || (cd[c] == my_d && cj[c] < my_j))) ? 1 : 0;
    const bool pick = s16 < KC && my_j >= 0 && rank < P.k;
    const uint32_t chosen = (__ballot_sync(0xffffffffu, pick) >> (16 * grp)) & 0xFFFFu;
    const int k_eff = min(P.k, n_valid);
    if (g.live) {
      int32_t* idx_row = P.idx + ((int64_t)bh * P.n_code_cap + g.row) * P.k;
      if (pick) idx_row[rank] = my_j;
      if (s16 >= k_eff && s16 < P.k) idx_row[s16] = -1;
    }
    // r = x - mean of the chosen rows, formed in place as x - sum_c inv r_c
    // (k_eff < k only for the earliest tokens, which see fewer than k references)
    const float inv = k_eff == P.k ? P.inv_k : 1.0f / (float)max(k_eff, 1);
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      if (chosen & (1u << c)) {
        uint4 rc[RowPack<EPL>::V4];
        if constexpr (NB == KC) {
#pragma unroll
          for (int i = 0; i < RowPack<EPL>::V4; ++i) rc[i] = rr[c][i];
        } else {
          load_row<EPL>(rs + (int64_t)cj[c] * P.d_h, rc);  // reloaded: it is in L2
        }
#pragma unroll
        for (int i = 0; i < RowPack<EPL>::V4; ++i) {
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&rc[i]);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 v = __bfloat1622float2(p2[x]);
            xr[8 * i + 2 * x] = fmaf(-inv, v.x, xr[8 * i + 2 * x]);
            xr[8 * i + 2 * x + 1] = fmaf(-inv, v.y, xr[8 * i + 2 * x + 1]);
          }
        }
      }
    }
    if (valid(cn)) load_cands(cn);
    // r = hi + lo (fp16) into the R tile: row n, columns e0 .. e0 + EPL
#pragma unroll
    for (int v = 0; v < EPL / 8; ++v) {
      __half2 hi2[4], lo2[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = 8 * v + 2 * q;
        split_half2(g.live ? xr[i] : 0.f, g.live ? xr[i + 1] : 0.f, hi2[q], lo2[q]);
      }
      if (g.inrow) {
        const uint32_t off = sw128_offset(n, e0 + 8 * v, enc::ROWS);
        *reinterpret_cast<uint4*>(sRb + off) = *reinterpret_cast<const uint4*>(hi2);
        *reinterpret_cast<uint4*>(sRb + r_part + off) = *reinterpret_cast<const uint4*>(lo2);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->r_full[rb]);
    return true;
  };

  if (warp < enc::GATHER_WARPS) {
    // ------------------------------------ gather warps: pairs until none is left
    bool ok = true;
    uint32_t c = claim();
    if (valid(c)) {
      prefetch(c);
      load_cands(c);
    }
    while (ok && valid(c)) {
      const uint32_t cn = claim();
      ok = process(c, cn);
      c = cn;
    }
    if (!ok) {
      if (lane == 0) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 10);
      *abort_flag = 1;
    }
  } else if (warp == enc::MMA_WARP) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t r_base = smem_u32(sR), h0 = smem_u32(sH), w0 = smem_u32(sW2);
      const uint32_t id1 = idesc_f16_f32(128, enc::ROWS);
      const uint32_t id2 = idesc_f16_f32(enc::MMA_M, P.d_c) | (1u << 15);  // A MN-major
      bool ok = true;
      for (int it = 0; it <= n_local && ok; ++it) {
        if (it < n_local) {
          // GEMM1^T of tile it: D1[hh] = W1[hh] . R^T  (hidden x tokens)
          const int rb = it & 1;
          if (!mbar_wait(&bars->r_full[rb], (it >> 1) & 1, abort_flag)) { ok = false; break; }
          if (it >= 1 && !mbar_wait(&bars->d1_empty, (it - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t rt = r_base + rb * 2 * (uint32_t)r_part;
          for (int hh = 0; hh < nh; ++hh)
#pragma unroll 1
            for (int part = 0; part < 2; ++part)
#pragma unroll
              for (int k16 = 0; k16 < D / 16; ++k16)
                umma_f16_ts(tmem + enc::D1_COL + enc::ROWS * hh, tmem + enc::W1_COL + hh * (D / 2) + k16 * 8,
                            desc_kmajor_sw128(rt + part * (uint32_t)r_part + (k16 >> 2) * enc::ROWS * 128 +
                                              (k16 & 3) * 32),
                            id1, (part | k16) != 0);
          umma_commit(&bars->r_empty[rb]);
          umma_commit(&bars->d1_full);
        }
        if (it >= 1) {
          // GEMM2 of tile it - 1: codes = H . W2^T (tokens x d_c)
          const int pt = it - 1;
          if (!mbar_wait(&bars->h_full, pt & 1, abort_flag)) { ok = false; break; }
          if (pt >= 1 && !mbar_wait(&bars->d2_empty, (pt - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int part = 0; part < 2; ++part)
#pragma unroll 1
            for (int k16 = 0; k16 < hidden / 16; ++k16) {
              // A: 16 hidden rows per step; the second 64-token block (rows of
              // the M = 128 MMA that no token owns) reads the same rows again
              const uint64_t ad = desc_mnmajor_sw128_enc(h0 + part * (uint32_t)h_part + k16 * 16 * 128, 0, 1024);
              const uint64_t bd = desc_kmajor_sw128(w0 + (k16 >> 2) * P.d_c * 128 + (k16 & 3) * 32);
              umma_f16(tmem + enc::D2_COL, ad, bd, id2, (part | k16) != 0);
            }
          umma_commit(&bars->h_empty);
          umma_commit(&bars->d2_full);
        }
      }
      if (!ok) {
        latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 11);
        *abort_flag = 1;
      }
      // every MMA issued has completed before tensor memory is released
      if (!umma_drain(&bars->drain)) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 13);
    }
  } else if (warp >= enc::ACT0 && warp < enc::ACT0 + enc::ACT_WARPS) {
    // ------------------- activation H = act(D1 + b1), then the code store
    const int q = warp & 3;
    bool ok = true;
    for (int it = 0; it < n_local && ok; ++it) {
      const int tile = blockIdx.x + it * gridDim.x;
      if (!mbar_wait(&bars->d1_full, it & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      for (int hh = 0; hh < nh; ++hh) {
        const int unit = 128 * hh + 32 * q + lane;
        const float bias = P.b1 ? P.b1[unit] : 0.f;
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          float v[32];
          tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + enc::D1_COL + enc::ROWS * hh + 32 * cc, v);
          if (hh == nh - 1 && cc == 1) {
            // the accumulator is in registers: GEMM1 of the next tile may start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->d1_empty);
          }
          if (hh == 0 && cc == 0 && it >= 1 && !mbar_wait(&bars->h_empty, (it - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            __half2 hi2[4], lo2[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              if (ACT == DELTAKV_ACT_GELU_ERF) {
                const float2 g2 = gelu_fast2(v[8 * c4 + 2 * x] + bias, v[8 * c4 + 2 * x + 1] + bias);
                split_half2(g2.x, g2.y, hi2[x], lo2[x]);
              } else {
                split_half2(enc_act<ACT>(v[8 * c4 + 2 * x] + bias), enc_act<ACT>(v[8 * c4 + 2 * x + 1] + bias),
                            hi2[x], lo2[x]);
              }
            }
            // MN-major row `unit` of 64 tokens: 16-byte chunk c8, swizzled by row
            const int c8 = 4 * cc + c4;
            const uint32_t off = (uint32_t)unit * 128 + (((c8 ^ (unit & 7))) << 4);
            *reinterpret_cast<uint4*>(sH + off) = *reinterpret_cast<const uint4*>(hi2);
            *reinterpret_cast<uint4*>(sH + h_part + off) = *reinterpret_cast<const uint4*>(lo2);
          }
        }
        if (!ok) break;
      }
      if (!ok) break;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->h_full);
      // this tile's codes wait for GEMM2, which the MMA warp issues after
      // GEMM1 of the next tile: meanwhile take row pairs of the next tile
      // (a pair claimed from the tile after it is worked too: its R buffer
      // is free, GEMM1 of this tile being complete)
      if (!ok) break;
      // codes = D2 + b2 (TMEM lanes 0-63: the first two activation warps)
      if (!mbar_wait(&bars->d2_full, it & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (q < 2 && P.cscale) {
        const int bh = tile / P.tiles_per_bh;
        const int64_t row = (int64_t)(tile % P.tiles_per_bh) * enc::ROWS + q * 32 + lane;
        const int64_t prow = (int64_t)bh * P.n_code_cap + row;
        const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + enc::D2_COL;
        uint8_t* dst = reinterpret_cast<uint8_t*>(P.code) + prow * (P.d_c / 2);
        const bool live = row < P.n_code;
        if (P.d_c == 16) store_code4_row<16>(ta, P.b2, dst, P.cscale + prow, live);
        else if (P.d_c == 32) store_code4_row<32>(ta, P.b2, dst, P.cscale + prow, live);
        else store_code4_row<64>(ta, P.b2, dst, P.cscale + prow, live);
      } else if (q < 2) {
        const int bh = tile / P.tiles_per_bh;
        const int64_t row = (int64_t)(tile % P.tiles_per_bh) * enc::ROWS + q * 32 + lane;
        for (int c0 = 0; c0 < P.d_c; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + enc::D2_COL + c0, v);
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->d2_empty);
    }
    if (!ok) {
      if (lane == 0) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 12);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == enc::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, enc::TMEM_COLS);
  }
}

size_t encode_tc_smem(const Plan& p) {
  const int D = p.D, hidden = p.cfg.hidden, d_c = p.cfg.d_c;
  const size_t r = 4 * (size_t)(D / 64) * enc::ROWS * 128;   // two tiles, hi and lo
  const size_t h = 2 * (size_t)hidden * 128;                 // hi and lo
  const size_t w2 = ((size_t)(hidden / 64) * d_c * 128 + 1023) & ~size_t(1023);
  return 1024 + r + h + w2 + sizeof(EncBars) + 64;
}

bool encode_tc_supported(const Plan& p) {
  const auto& c = p.cfg;
  return p.bf16 && (c.d_h == 64 || c.d_h == 128) && (c.hidden == 128 || c.hidden == 256) &&
         c.d_c % 16 == 0 && c.d_c <= 64 && encode_tc_smem(p) <= 227 * 1024;
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
  P.cscale = p.code4 ? (__nv_bfloat16*)(cb + p.off_cscale) : nullptr;
  P.idx = (int32_t*)(cb + p.off_idx);
  P.cand = (const int32_t*)((char*)ws + p.ws_cand);
  P.err = (uint32_t*)ws;
  P.tiles_per_bh = (int)ceil_div64(n_code, enc::ROWS);
  P.n_tiles = P.tiles_per_bh * P.BH;
  P.div_tiles = make_fastdiv((uint32_t)P.tiles_per_bh);
  P.div_sm1 = make_fastdiv((uint32_t)(P.s - 1));
  P.div_H = make_fastdiv((uint32_t)P.H);
  P.inv_k = 1.0f / (float)c.k;  // IEEE division, correctly rounded on host and device alike
  int dev = 0, sms = kNumSMs;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(P.n_tiles, sms);
  const size_t smem = encode_tc_smem(p);
  ProfScope ps(p, st, KID_ENCODE_TC);
  if (c.d_h == 128)
    return p.KC == 8 ? encode_tc_launch<16, 8>(P, smem, grid, st) : encode_tc_launch<16, 12>(P, smem, grid, st);
  return p.KC == 8 ? encode_tc_launch<8, 8>(P, smem, grid, st) : encode_tc_launch<8, 12>(P, smem, grid, st);
}

}  // namespace dkv
