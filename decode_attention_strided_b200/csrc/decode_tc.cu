// decode_tc.cu -- the token loop of decode attention over the compressed cache
// on the 5th-generation tensor cores (bf16 caches).
//
// DeltaKV summary, section 3 "Ricostruzione" and section 4 (reconstruction
// on demand inside the attention that reads the cache).  For query head g of
// kv-head h and compressed token t (logits in log2 units, c = log2 e/sqrt d_h):
//   u_t  = act(W3 code_t + b3)                       GEMM1 + act, per token
//   l_tg = a_g . u_t + c q_g.b4_K + mean_i S[idx_ti][g]
//          (a_g = c W4_K^T q_g,  S[j][g] = c q_g . K_ref_j)
//   p_tg = 2^(l_tg - m_g)   with m_g the segment's scale (below)
//   U_g += sum_t p_tg u_t         (W4_V U_g is applied once per kv-head later)
//   w[j][g] += p_tg / k_eff for j in idx_t   (V_ref side, per-slot weights)
// so no token's K or V is ever materialised.  Per 128-token chunk:
//   producer warp  TMA: the chunk's codes (zero-filled past the last row)
//                  and slots into a ring of 2-4 stages
//   MMA warp       D1 = codes . W3^T  (M=128, N=hidden, K=d_c; bf16, exact
//                  products) and U += u^T . [P_hi, P_lo rows] (M=128 hidden
//                  units, N=16, K=128 tokens; the u tile read through an
//                  MN-major descriptor; one accumulator per kv-head segment,
//                  resident in tensor memory; p enters as two fp16 terms,
//                  which the N = 16 shape holds at no extra cost), in the
//                  causal order of their inputs: GEMM1(i + 1), then U(i)
//   activation     8 warps, one token row and one hidden half per thread:
//                  u = act(D1 + b3) (exact GELU through gelu_tanhfit2, one
//                  MUFU tanh per value) rounded to an fp16 u tile (two
//                  buffers) for the U MMA, and a_g . u summed in fp32 from
//                  the unrounded u (the logit needs more than fp16 u holds);
//                  D1 is released to the next GEMM1 after its last TMEM load
//   softmax        4 warps: the chunk's slots copied to registers and its
//                  S gathers issued as soon as it lands (which frees the ring
//                  stage for the producer), the two halves' logit parts
//                  added, chunk maximum, fp16 P tile (two buffers), slot-weight
//                  reductions into the global table
// Scale (lazy rescaling): every segment starts at m_g = max_j S[j][g] and
// keeps it while no chunk maximum exceeds m_g by more than 8 (so p <= 2^8
// fits fp16 with room to spare); only then the softmax warps rescale the U
// accumulator in tensor memory (after its MMAs so far have completed) and
// their denominators, and raise m_g.  The common chunk never waits on the
// MMAs of the previous one.
// A persistent grid splits the flattened (kv-head, chunk) list evenly; each
// CTA writes one partial (m, l, U) per kv-head segment it touches.
#include <cfloat>
#include <climits>
#include <cstring>
#include <mutex>
#include <type_traits>

#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace dkv {
using namespace sm100;

namespace dtc {
constexpr int CH = 128;                 // tokens per chunk (MMA M)
#ifndef DTC_ACT
#define DTC_ACT 8
#endif
constexpr int ACT = DTC_ACT;            // activation warps from 2 (ACT / 4 per TMEM lane quarter)
constexpr int PARTS = ACT / 4;          // hidden units split into PARTS column ranges
constexpr int SMX = 4;                  // softmax warps after them (one per lane quarter)
constexpr int ACT0 = 2;
constexpr int THREADS = (ACT0 + ACT + SMX) * 32;
constexpr int MAX_STAGES = 4;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns: D1 [0, hidden), the segment's U accumulator [256, 288)
// (hidden halves of 16 columns: head g's hi term in column g, its lo term in
// column 8 + g)
constexpr uint32_t COL_D1 = 0, COL_U = 256;
constexpr int PRODUCER = 0, MMA = 1;
constexpr float TAU = 8.0f;             // log2 headroom before a rescale
}  // namespace dtc

// Heads per kv-head as the kernel lays them out (a multiple of 4).
__host__ __device__ constexpr int dtc_gp(int G) { return G <= 4 ? 4 : 8; }

// Even split of N chunks over `grid` CTAs: CTA c owns chunks x with
// floor(x grid / N) == c.
__host__ __device__ inline int64_t dtc_begin(int64_t c, int64_t N, int grid) {
  return (c * N + grid - 1) / grid;
}
__host__ __device__ inline int64_t dtc_owner(int64_t x, int64_t N, int grid) { return (x * grid) / N; }

struct DecTcParams {
  int s, d_h, G, k, d_c, hidden, act, H, BH;
  int64_t n_ref_cap;
  CacheView cv;         // where the codes and slots are (contiguous cache or page pool)
  SeqLens sl;           // tokens of every sequence
  int n_ch_all;         // chunks per (sequence, kv-head) when every sequence has T_all tokens
  const int32_t* cho;   // else chunk offsets per (sequence, kv-head), [BH + 1]
  // Gathered rows (sparse decode): the compressed rows of (sequence, kv-head)
  // bh are rowlist[bh * rl_cap + i], i < ncode[bh], not rows 0 .. n_code - 1
  const int32_t* rowlist;
  const int32_t* ncode;
  int64_t rl_cap;
  int grid, nslot_cap, n_refblk, n_refblk_cap;
  int code_swz;        // 32, 64 or 128: bytes per swizzled row of the code tile
  int code_atoms;      // 64-column atoms of the code tile (2 when d_c = 128)
  int nst;             // stages of the input ring (2..MAX_STAGES)
  int code4;           // 4-bit codes: staged packed, expanded to an fp16 code tile
  const uint8_t* code4p;
  const __nv_bfloat16* cscale;
  const int32_t* idx;
  const __nv_bfloat16* W3;
  const float* b3;
  const float* a;
  const float* cterm;
  const float* S;
  const float* Smax;
  const float* mref;  // per (sequence, kv-head, head): max_j S_j
  float* wtab;
  float* part;
  float* Upart;
  uint32_t* err;
};

// K-major smem descriptor for 32-, 64- or 128-byte swizzled rows.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr, int swz) {
  const uint64_t type = swz == 128 ? 2 : (swz == 64 ? 4 : 6);
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)((8 * swz) >> 4) << 32;  // 8-row groups
  d |= (uint64_t)1 << 46;
  d |= type << 61;
  return d;
}

// MN-major, 128-byte swizzle: 64 contiguous M-elements per 128-byte row,
// K rows 128 bytes apart (8-row groups `sbo` apart), M blocks `lbo` apart.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// kind::f16 instruction descriptors.
__host__ __device__ constexpr uint32_t idesc_kind_f16(bool bf16, int M, int N, bool a_mn) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (a_mn ? (1u << 15) : 0u) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of byte `bo` of row `row` in a K-major tile with `swz`-byte rows.
__device__ __forceinline__ uint32_t swz_off(int row, int bo, int swz) {
  const int mask = swz / 16 - 1;
  const int chunk = (bo >> 4) ^ (((row * swz) >> 7) & mask);
  return (uint32_t)(row * swz + (chunk << 4) + (bo & 15));
}


__device__ __forceinline__ void tmem_ld16f(uint32_t taddr, float (&v)[16]) {
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

// 16 consecutive 32-bit columns of this thread's TMEM lane; complete with
// tmem_st_wait.
__device__ __forceinline__ void tmem_st16f(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
      : "memory");
}

// Split 16-column TMEM load: issue now, wait later (the registers are
// in/out operands of the wait, so nothing reads them before it).
__device__ __forceinline__ void tmem_ld_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

// acc += (x0, x1) * (y0, y1), one packed fp32 instruction.
__device__ __forceinline__ void fma2_acc(float2& acc, float x0, float x1, float y0, float y1) {
  asm("{\n\t.reg .b64 x, y, d;\n\t"
      "mov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %5};\n\tmov.b64 d, {%0, %1};\n\t"
      "fma.rn.f32x2 d, x, y, d;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "+f"(acc.x), "+f"(acc.y)
      : "f"(x0), "f"(x1), "f"(y0), "f"(y1));
}

__host__ __device__ inline size_t dtc_align(size_t x) { return (x + 1023) & ~size_t(1023); }

// Offsets of the shared-memory regions (from a 1024-aligned base).
struct DecLayout {
  size_t code, idx, stg, w3, b3, av, zb, u, p, fl, bar, total;
  __host__ __device__ DecLayout(int d_c, int k, int hidden, int nst, bool code4, int gp) {
    const size_t code_b = (size_t)dtc::CH * d_c * 2, idx_b = (size_t)dtc::CH * k * 4;
    const size_t w3_b = (size_t)hidden * d_c * 2, av_b = (size_t)hidden * gp * 4;
    const size_t zb_b = (size_t)dtc::PARTS * dtc::CH * gp * 4;
    const size_t u_b = (size_t)(hidden / 64) * dtc::CH * 128, p_b = 2 * 2 * 16 * 128;
    size_t o = 0;
    code = o; o = dtc_align(o + nst * dtc_align(code_b));
    idx = o;  o = dtc_align(o + nst * dtc_align(idx_b));
    stg = o;  o = dtc_align(o + (code4 ? nst * dtc_align((size_t)dtc::CH * (d_c / 2 + 2)) : 0));
    w3 = o;   o = dtc_align(o + w3_b);
    b3 = o;   o = dtc_align(o + (size_t)hidden * 4);
    av = o;   o = dtc_align(o + 2 * dtc_align(av_b));
    zb = o;   o = dtc_align(o + 2 * zb_b);
    u = o;    o = dtc_align(o + 2 * u_b);
    p = o;    o = dtc_align(o + p_b);
    fl = o;   o += 128 * sizeof(float);  // 112 used (below)
    bar = o;  o += 32 * 8;
    total = o;
  }
};

template <int ACT, bool HAS_B3, int GP>
__global__ void __launch_bounds__(dtc::THREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap mapC, const DecTcParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const DecLayout L(P.d_c, P.k, P.hidden, P.nst, P.code4 != 0, GP);
  const size_t stg_b = dtc_align((size_t)dtc::CH * (P.d_c / 2 + 2));
  const size_t code_b = dtc_align((size_t)dtc::CH * P.d_c * 2), idx_b = dtc_align((size_t)dtc::CH * P.k * 4);
  const size_t av_b = dtc_align((size_t)P.hidden * GP * 4), zb_b = (size_t)dtc::PARTS * dtc::CH * GP * 4;
  const size_t u_b = (size_t)(P.hidden / 64) * dtc::CH * 128;
  const int NST = P.nst;
  auto sCode = [&](int i) { return base + L.code + i * code_b; };
  auto sIdx = [&](int i) { return (int32_t*)(base + L.idx + i * idx_b); };
  auto sStg = [&](int i) { return base + L.stg + i * stg_b; };  // 4-bit codes, then scales
  unsigned char* sW3 = base + L.w3;
  float* sB3 = (float*)(base + L.b3);
  auto sAv = [&](int i) { return (float*)(base + L.av + i * av_b); };  // a_g, [hidden / 2][GP][2]
  auto sZb = [&](int i) { return (float*)(base + L.zb + i * zb_b); };  // logit parts, [part][row][GP]
  auto sU = [&](int i) { return base + L.u + i * u_b; };
  auto sP = [&](int i) { return base + L.p + i * 2 * 16 * 128; };
  float* fl = (float*)(base + L.fl);
  float* m_ref = fl;          // [8]     segment's reference-logit maximum
  float* ctv = fl + 8;        // [8]     segment's constant logit term
  float* lred = fl + 16;      // [4][8]  per-warp denominators at a segment end
  float* mred = fl + 48;      // [2][4][8] per-warp chunk maxima, by chunk parity
  uint64_t* bar = (uint64_t*)(base + L.bar);
  uint64_t* in_full = bar + 0;    // [MAX_STAGES]
  uint64_t* in_empty = bar + 4;   // [MAX_STAGES]
  uint64_t* d1_full = bar + 8;    // GEMM1(i) complete
  uint64_t* d1_free = bar + 9;    // the activation warps have loaded D1(i)
  uint64_t* u_full = bar + 10;    // [2] u tile and logit parts of chunk i written
  uint64_t* u_empty = bar + 12;   // [2] U(i) complete: the u tile is free again
  uint64_t* z_empty = bar + 14;   // [2] the softmax warps have read the logit parts
  uint64_t* p_full = bar + 16;    // [2]
  uint64_t* p_empty = bar + 18;   // [2]
  uint64_t* ua_done = bar + 20;   // [2]  U(j) complete
  uint64_t* ua_free = bar + 22;   // the segment's U accumulator has been read
  uint64_t* drain = bar + 23;     // the MMA warp's last commit
  uint64_t* code_ready = bar + 24;  // [MAX_STAGES] 4-bit codes expanded (producer warp)
  uint32_t* tmem_slot = (uint32_t*)(bar + 28);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int G = P.G, hidden = P.hidden, part_w = hidden / dtc::PARTS;
  // the flattened (sequence, kv-head, chunk) list: chunk x belongs to the
  // last bh with coff(bh) <= x; every role visits its chunks in order and
  // walks bh forward from the previous one
  auto coff = [&](int bh) -> int64_t { return P.cho ? (int64_t)P.cho[bh] : (int64_t)bh * P.n_ch_all; };
  const int64_t N = coff(P.BH);
  // the chunks go to the first min(grid, N) CTAs (every one of them gets at
  // least one, so the CTAs that share a (sequence, kv-head) are consecutive);
  // the rest have nothing to do
  const int gridp = (int)(N < P.grid ? N : P.grid);
  const bool has = (int)blockIdx.x < gridp;
  const int64_t x_begin = has ? dtc_begin(blockIdx.x, N, gridp) : 0;
  const int64_t x_end = has ? dtc_begin(blockIdx.x + 1, N, gridp) : 0;
  const int n_local = (int)(x_end - x_begin);
  int bh_start = 0;
  if (n_local > 0) {
    if (!P.cho) {
      bh_start = (int)(x_begin / P.n_ch_all);
    } else {
      int lo = 0, hi = P.BH - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (coff(mid) <= x_begin) lo = mid; else hi = mid - 1;
      }
      bh_start = lo;
    }
  }
  auto bh_of = [&](int64_t x, int hint) {
    int bh = hint;
    while (bh + 1 < P.BH && coff(bh + 1) <= x) ++bh;
    return bh;
  };
  auto n_code_bh = [&](int bh) -> int64_t {
    return P.ncode ? (int64_t)P.ncode[bh] : n_code_of(P.sl.T(bh / P.H), P.s);
  };

  // ---- one-time set-up: W3 (K-major, swizzled like the code tile; bf16, or
  // fp16 next to 4-bit codes, whose expanded values q * scale fp16 holds
  // exactly), b3, zero P tiles (their padding rows are never written),
  // barriers, TMEM
  {
    const int swz = P.code_swz;
    const int row_elems = swz / 2;
    for (int i = tid; i < hidden * P.d_c / 8; i += blockDim.x) {
      const int n = i / (P.d_c / 8), c8 = (i % (P.d_c / 8)) * 8;
      uint4 v = *reinterpret_cast<const uint4*>(P.W3 + (int64_t)n * P.d_c + c8);
      if (P.code4) {
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&v);
        uint4 hv;
        __half2* h2 = reinterpret_cast<__half2*>(&hv);
#pragma unroll
        for (int x = 0; x < 4; ++x) h2[x] = __float22half2_rn(__bfloat1622float2(b2[x]));
        v = hv;
      }
      const int atom = c8 / row_elems, col = c8 % row_elems;
      *reinterpret_cast<uint4*>(sW3 + (size_t)atom * hidden * swz + swz_off(n, col * 2, swz)) = v;
    }
    for (int i = tid; i < hidden; i += blockDim.x) sB3[i] = HAS_B3 ? P.b3[i] : 0.f;
    for (int i = tid; i < 2 * 2 * 16 * 128 / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sP(0))[i] = 0u;
  }
  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&in_full[i], 1);
      mbar_init(&in_empty[i], 1 + dtc::SMX);  // the GEMM1 commit and the softmax warps
      mbar_init(&code_ready[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&u_full[i], dtc::ACT);
      mbar_init(&u_empty[i], 1);
      mbar_init(&z_empty[i], dtc::SMX);
      mbar_init(&p_full[i], dtc::SMX);
      mbar_init(&p_empty[i], 1);
      mbar_init(&ua_done[i], 1);
    }
    mbar_init(d1_full, 1);
    mbar_init(d1_free, dtc::ACT);
    mbar_init(ua_free, dtc::SMX);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == dtc::MMA) {
    tmem_alloc(tmem_slot, dtc::TMEM_COLS);
    tmem_relinquish();
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == dtc::PRODUCER && P.rowlist) {
    // ------------------------------------------ producer, gathered rows
    // the chunk's rows are entries of the (sequence, kv-head)'s row list: the
    // warp copies each row's codes into the swizzled code tile and its slots
    // into the slot tile with plain loads and stores (rows past the list's
    // end: zero codes, no slots), then marks the stage full
    if (n_local > 0) {
      bool ok = true;
      int bh = bh_start;
      const int swz = P.code_swz, row_elems = swz / 2;
      const char* cbase = P.cv.base + P.cv.off_code;
      for (int it = 0; it < n_local && ok; ++it) {
        const int64_t x = x_begin + it;
        bh = bh_of(x, bh);
        const int64_t row0 = (x - coff(bh)) * dtc::CH;
        const int64_t n_code = n_code_bh(bh);
        const int st = it % NST;
        ok = mbar_wait(&in_empty[st], ((it / NST) & 1) ^ 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        unsigned char* tile = sCode(st);
        int32_t* sidx = sIdx(st);
#pragma unroll 1
        for (int r = lane; r < dtc::CH; r += 32) {
          const bool valid = row0 + r < n_code;
          const int64_t cr = valid ? (int64_t)P.rowlist[(int64_t)bh * P.rl_cap + row0 + r] : 0;
          const int64_t prow = P.cv.code_row(bh, cr);
          const uint4* src = reinterpret_cast<const uint4*>(cbase + prow * P.d_c * 2);
          for (int e = 0; e < P.d_c; e += 8) {  // 16 bytes: 8 bf16 codes
            const uint4 v = valid ? __ldg(src + e / 8) : make_uint4(0u, 0u, 0u, 0u);
            const int atom = e / row_elems, col = e % row_elems;
            *reinterpret_cast<uint4*>(tile + (size_t)atom * dtc::CH * swz + swz_off(r, col * 2, swz)) = v;
          }
          for (int kk = 0; kk < P.k; ++kk) sidx[r * P.k + kk] = valid ? __ldg(P.idx + prow * P.k + kk) : -1;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&in_full[st]);
      }
      if (!ok && lane == 0) {
        latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 20);
        *abort_flag = 1;
      }
    }
  } else if (warp == dtc::PRODUCER && P.code4) {
    // -------------------------------------------- producer, 4-bit codes
    // lane 0 issues chunk it's copies (packed codes and scales into the
    // stage's staging area, slots into its slot area); then the warp expands
    // chunk it - 1's codes into the fp16 code tile (q * scale, rows past the
    // last token zero) and marks it ready for GEMM1
    if (n_local > 0) {
      const uint32_t c4_bytes = (uint32_t)(dtc::CH * P.d_c / 2), s_bytes = (uint32_t)(dtc::CH * 2);
      const uint32_t idx_bytes = (uint32_t)(dtc::CH * P.k * 4);
      const int swz = P.code_swz, hb = P.d_c / 2;
      bool ok = true;
      int issued = 0;
      int pbh = bh_start, ebh = bh_start;  // issuing and expanding cursors
      for (int it = 0; it <= n_local && ok; ++it) {
        if (it < n_local) {
          const int64_t x = x_begin + it;
          pbh = bh_of(x, pbh);
          const int64_t row0 = (x - coff(pbh)) * dtc::CH;
          const int st = it % NST;
          ok = mbar_wait(&in_empty[st], ((it / NST) & 1) ^ 1, abort_flag);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          if (lane == 0) {
            const int64_t prow = P.cv.code_row(pbh, row0);
            mbar_arrive_expect_tx(&in_full[st], c4_bytes + s_bytes + idx_bytes);
            bulk_load(sStg(st), P.code4p + prow * hb, c4_bytes, &in_full[st]);
            bulk_load(sStg(st) + c4_bytes, P.cscale + prow, s_bytes, &in_full[st]);
            bulk_load(sIdx(st), P.idx + prow * P.k, idx_bytes, &in_full[st]);
          }
          issued = it + 1;
        }
        if (it >= 1) {
          const int j = it - 1, sj = j % NST;
          ok = mbar_wait(&in_full[sj], (j / NST) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          ebh = bh_of(x_begin + j, ebh);
          const int64_t row0 = (x_begin + j - coff(ebh)) * dtc::CH;
          const int64_t n_code = n_code_bh(ebh);
          const uint8_t* c8 = sStg(sj);
          const __nv_bfloat16* sc = reinterpret_cast<const __nv_bfloat16*>(sStg(sj) + c4_bytes);
          unsigned char* tile = sCode(sj);
#pragma unroll 1
          for (int r = lane; r < dtc::CH; r += 32) {
            const bool valid = row0 + r < n_code;
            const float scale = valid ? __bfloat162float(sc[r]) : 0.f;
            for (int e8 = 0; e8 < P.d_c; e8 += 8) {
              const uint32_t w = *reinterpret_cast<const uint32_t*>(c8 + r * hb + e8 / 2);  // 8 codes
              uint4 o;
              __half2* h2 = reinterpret_cast<__half2*>(&o);
#pragma unroll
              for (int x = 0; x < 4; ++x) {
                const int byte = (int)((w >> (8 * x)) & 0xFF);
                const float q0 = (float)(((byte & 0xF) ^ 8) - 8), q1 = (float)(((byte >> 4) ^ 8) - 8);
                h2[x] = __floats2half2_rn(q0 * scale, q1 * scale);
              }
              *reinterpret_cast<uint4*>(tile + swz_off(r, e8 * 2, swz)) = o;
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&code_ready[sj]);
        }
      }
      if (!ok && lane == 0) {
        latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 20);
        *abort_flag = 1;
      }
      if (lane == 0) {
        for (int i = 0; i < NST && issued > i; ++i) {
          const int j = issued - 1 - i;
          if (!mbar_wait_drain(&in_full[j % NST], (j / NST) & 1)) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 24);
        }
      }
    }
  } else if (warp == dtc::PRODUCER) {
    // ------------------------------------------------------------ producer
    // the whole warp follows the ring; lane 0 issues the copies
    if (n_local > 0) {
      const uint32_t code_bytes = (uint32_t)(dtc::CH * P.d_c * 2), idx_bytes = (uint32_t)(dtc::CH * P.k * 4);
      bool ok = true;
      int issued = 0;
      int bh = bh_start;
      for (int it = 0; it < n_local && ok; ++it) {
        const int64_t x = x_begin + it;
        bh = bh_of(x, bh);
        const int64_t row0 = (x - coff(bh)) * dtc::CH;
        // a chunk never straddles a page: a page holds a multiple of 128 code rows
        const int64_t prow = P.cv.code_row(bh, row0);
        const int st = it % NST;
        ok = mbar_wait(&in_empty[st], ((it / NST) & 1) ^ 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&in_full[st], code_bytes + idx_bytes);
          for (int a = 0; a < P.code_atoms; ++a)
            tma_load_3d(&mapC, &in_full[st], sCode(st) + (size_t)a * dtc::CH * 128, a * 64, (int)(prow % P.cv.cp),
                        (int)(prow / P.cv.cp));
          bulk_load(sIdx(st), P.idx + prow * P.k, idx_bytes, &in_full[st]);
        }
        __syncwarp();
        issued = it + 1;
      }
      if (!ok && lane == 0) {
        latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 20);
        *abort_flag = 1;
      }
      // the copies of the last chunks issued (one per stage) land before the
      // block can finish, also after an abort
      if (lane == 0) {
        for (int i = 0; i < NST && issued > i; ++i) {
          const int j = issued - 1 - i;
          if (!mbar_wait_drain(&in_full[j % NST], (j / NST) & 1)) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 24);
        }
      }
      __syncwarp();
    }
  } else if (warp == dtc::MMA) {
    // ------------------------------------------------------------- MMA warp
    // The whole warp follows the chunks and waits; lane 0 issues.  Causal
    // order of the events the MMAs wait for:
    //   d1_free(i)  the activation warps have loaded D1(i)  -> GEMM1(i + 1)
    //   p_full(i)   the softmax warps have written P(i)     -> U(i)
    // (p_full(i) follows the activation warps' end of chunk i, which follows
    // their d1_free(i)).  The first U of a segment restarts the accumulator,
    // once the softmax warps have read the previous segment's.
    if (n_local > 0) {
      const uint32_t id_g1 = idesc_kind_f16(!P.code4, dtc::CH, hidden, false);  // fp16 next to 4-bit codes
      const uint32_t id_u = idesc_kind_f16(false, 128, 16, true);
      const int swz = P.code_swz, per_row = swz / 32;  // k16 steps per swizzled row
      // the code tile of a stage is ready: its TMA copy has landed, or with
      // 4-bit codes the producer warp has expanded it
      auto code_wait = [&](int j) {
        return P.code4 ? mbar_wait(&code_ready[j % NST], (j / NST) & 1, abort_flag)
                       : mbar_wait(&in_full[j % NST], (j / NST) & 1, abort_flag);
      };
      auto gemm1 = [&](int j) {
        const int st = j % NST;
        if (lane == 0) {
          const uint32_t c0 = smem_u32(sCode(st)), w0 = smem_u32(sW3);
          for (int k16 = 0; k16 < P.d_c / 16; ++k16) {
            const int atom = k16 / per_row, off = (k16 % per_row) * 32;
            umma_f16(tmem + dtc::COL_D1, desc_kmajor(c0 + atom * dtc::CH * swz + off, swz),
                     desc_kmajor(w0 + atom * hidden * swz + off, swz), id_g1, k16 != 0);
          }
          umma_commit(d1_full);
          umma_commit(&in_empty[st]);
        }
        __syncwarp();
      };
      bool ok = code_wait(0);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        gemm1(0);
      } else {
        ok = false;
      }
      int useg = -1, uprev = -1, ubh = bh_start;
      for (int i = 0; i < n_local && ok; ++i) {
        if (i + 1 < n_local) {
          ok = mbar_wait(d1_free, i & 1, abort_flag) && code_wait(i + 1);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          gemm1(i + 1);
        }
        const int jb = i & 1;
        ubh = bh_of(x_begin + i, ubh);
        const bool first = ubh != uprev;
        ok = mbar_wait(&p_full[jb], (i >> 1) & 1, abort_flag) &&
             (!first || useg < 0 || mbar_wait(ua_free, useg & 1, abort_flag));
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (first) { ++useg; uprev = ubh; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t u0 = smem_u32(sU(jb)), p0 = smem_u32(sP(jb));
          for (int h2 = 0; h2 < hidden / 128; ++h2)
            for (int k16 = 0; k16 < dtc::CH / 16; ++k16) {
              const uint64_t ad = desc_mnmajor_sw128(u0 + (2 * h2) * dtc::CH * 128 + k16 * 16 * 128,
                                                     dtc::CH * 128, 1024);
              const uint64_t bd = desc_kmajor(p0 + (k16 >> 2) * 16 * 128 + (k16 & 3) * 32, 128);
              umma_f16(tmem + dtc::COL_U + 16 * h2, ad, bd, id_u, !(first && k16 == 0));
            }
          umma_commit(&ua_done[jb]);
          umma_commit(&u_empty[jb]);
          umma_commit(&p_empty[jb]);
        }
        __syncwarp();
      }
      if (!ok && lane == 0) {
        latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 21);
        *abort_flag = 1;
      }
      // every MMA lane 0 issued has completed before tensor memory is released
      if (lane == 0 && !umma_drain(drain)) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 25);
      __syncwarp();
    }
  } else if (warp >= dtc::ACT0 && warp < dtc::ACT0 + dtc::ACT) {
    // ------------------------------------------------- activation warps
    // Thread (lane quarter q, lane) owns token row n of the chunk and one
    // range of hidden units: u = act(D1 + b3) on its columns, rounded to fp16
    // into the u tile (the U MMA's operand), and its share of every head's
    // logit term a_g . u, summed in fp32 from the unrounded u, into the logit
    // parts.
    const int aw = warp - dtc::ACT0;        // 0 .. ACT - 1
    const int q = warp & 3, n = q * 32 + lane;
    const int hh = aw >> 2;                 // hidden range
    bool ok = true;
    int prev_bh = -1, seg_count = 0, bh = bh_start;
    int64_t seg_x0 = 0, seg_ncode = 0;  // the segment's first chunk and row count
    const float* av = sAv(0);
    for (int it = 0; it < n_local && ok; ++it) {
      const int64_t x = x_begin + it;
      bh = bh_of(x, bh);
      const int ub = it & 1;
      if (bh != prev_bh) {
        seg_x0 = coff(bh);
        seg_ncode = n_code_bh(bh);
      }
      // rows past the sequence's last compressed token (the chunk's padding)
      // hold whatever the buffer holds: their u is zero
      const bool rvalid = (x - seg_x0) * dtc::CH + n < seg_ncode;
      if (bh != prev_bh) {
        // a_g of this kv-head into the buffer of this segment's parity, as
        // pairs of adjacent hidden units per head (heads >= G zero).  Its
        // last readers, the chunks of two segments back, are behind every
        // activation warp: all of them passed the previous segment's barrier.
        prev_bh = bh;
        float* dst = sAv(seg_count & 1);
        const float* ab = P.a + (int64_t)bh * G * hidden;
        for (int i = tid - dtc::ACT0 * 32; i < GP * hidden; i += dtc::ACT * 32) {
          const int g = i / hidden, c = i % hidden;
          dst[((c >> 1) * GP + g) * 2 + (c & 1)] = g < G ? ab[(int64_t)g * hidden + c] : 0.f;
        }
        named_bar(2, dtc::ACT * 32);
        av = dst;
        ++seg_count;
      }
      ok = mbar_wait(&z_empty[ub], ((it >> 1) & 1) ^ 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      unsigned char* ut = sU(ub);
      const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + dtc::COL_D1 + hh * part_w;
      float2 za[GP];  // per head: partial sums over even and odd hidden units
#pragma unroll
      for (int g = 0; g < GP; ++g) za[g] = make_float2(0.f, 0.f);
      // the u buffer is free once U(it - 2) is complete
      ok = mbar_wait(&u_empty[ub], ((it >> 1) & 1) ^ 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      // 16 columns of D1 at a time, two per pass of a rolled loop (one code
      // copy for every sub-block keeps the loop inside the instruction
      // cache): each sub-block's TMEM load is issued before the previous one
      // is computed (a wait covers every earlier load, so each wait comes
      // right before its sub-block is used)
      uint32_t ra[16], rc[16];
      // masked: the chunk holds rows past the sequence's last compressed
      // token (only the last chunk of a (sequence, kv-head) can); their u is
      // set to zero (the rows hold whatever the buffer holds)
      auto block = [&](const uint32_t (&r)[16], int c0, auto masked) {
#pragma unroll
        for (int v8 = 0; v8 < 2; ++v8) {
          uint4 pk;
          __half2* h2 = reinterpret_cast<__half2*>(&pk);
#pragma unroll
          for (int x2 = 0; x2 < 4; ++x2) {
            const int e = 8 * v8 + 2 * x2;  // column c0 + e
            float z0 = __uint_as_float(r[e]), z1 = __uint_as_float(r[e + 1]);
            if (HAS_B3) {
              const float2 bb = *reinterpret_cast<const float2*>(sB3 + c0 + e);
              z0 += bb.x;
              z1 += bb.y;
            }
            float2 u2;
            if (ACT == DELTAKV_ACT_GELU_ERF) {
              u2 = gelu_tanhfit2(z0, z1);
            } else {
              u2 = make_float2(act_eval(ACT, z0), act_eval(ACT, z1));
            }
            if constexpr (decltype(masked)::value) {
              if (!rvalid) u2 = make_float2(0.f, 0.f);
            }
            h2[x2] = __floats2half2_rn(u2.x, u2.y);
            const float* ap = av + ((c0 + e) >> 1) * GP * 2;
#pragma unroll
            for (int g = 0; g < GP; g += 2) {
              const float4 a4 = *reinterpret_cast<const float4*>(ap + 2 * g);  // heads g, g + 1
              fma2_acc(za[g], u2.x, u2.y, a4.x, a4.y);
              fma2_acc(za[g + 1], u2.x, u2.y, a4.z, a4.w);
            }
          }
          const int col = c0 + 8 * v8;
          *reinterpret_cast<uint4*>(ut + (col >> 6) * dtc::CH * 128 + swz_off(n, (col & 63) * 2, 128)) = pk;
        }
      };
      // D1 of this chunk once its GEMM1 is complete; this range's columns
      // 16 at a time, two per pass of the rolled loop
      ok = mbar_wait(d1_full, it & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      const int nsb = part_w / 16;  // even: part_w is 32, 64 or 128
      auto run = [&](auto masked) {
        tmem_ld_issue(trow, ra);
#pragma unroll 1
        for (int sb = 0; sb < nsb; sb += 2) {
          const int c0 = hh * part_w + 16 * sb;
          const bool last = sb + 2 >= nsb;
          tmem_ld_wait(ra);
          tmem_ld_issue(trow + 16 * (sb + 1), rc);
          if (last) {
            // both last sub-blocks in registers: D1 goes to the next GEMM1
            // two sub-blocks before the end of this chunk's work
            tmem_ld_wait(rc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(d1_free);
          }
          block(ra, c0, masked);
          if (!last) {
            tmem_ld_wait(rc);
            tmem_ld_issue(trow + 16 * (sb + 2), ra);
          }
          block(rc, c0 + 16, masked);
        }
      };
      if ((x - seg_x0 + 1) * dtc::CH <= seg_ncode) {
        run(std::false_type{});
      } else {
        run(std::true_type{});
      }
      if (!ok) break;
      {
        float* zr = sZb(ub) + ((size_t)hh * dtc::CH + n) * GP;
#pragma unroll
        for (int g = 0; g < GP; g += 4)
          *reinterpret_cast<float4*>(zr + g) = make_float4(za[g].x + za[g].y, za[g + 1].x + za[g + 1].y,
                                                           za[g + 2].x + za[g + 2].y, za[g + 3].x + za[g + 3].y);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&u_full[ub]);
    }
    if (!ok) {
      latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 22);
      *abort_flag = 1;
    }
  } else if (warp >= dtc::ACT0 + dtc::ACT && warp < dtc::ACT0 + dtc::ACT + dtc::SMX) {
    // ---------------------------------------------------- softmax warps
    const int sw = warp - (dtc::ACT0 + dtc::ACT);   // 0..3
    const int q = warp & 3, n = q * 32 + lane;      // token row / hidden unit in a half (TMEM lane quarter)
    // per-thread copies of the segment state (identical in every thread,
    // except lt: this thread's own share of the softmax denominator)
    float m_run[GP], lt[GP], wsc[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      m_run[g] = lt[g] = 0.f;
      wsc[g] = 1.f;
    }
    bool ok = true;
    int prev_bh = -1, seg_first = 0, bh = bh_start;
    int64_t n_code = 0, n_ref = 0;
    for (int it = 0; it < n_local && ok; ++it) {
      const int64_t x = x_begin + it;
      bh = bh_of(x, bh);
      const int64_t row0 = (x - coff(bh)) * dtc::CH;
      const int st = it % NST, zb = it & 1;
      if (bh != prev_bh) {
        prev_bh = bh;
        seg_first = it;
        n_code = n_code_bh(bh);
        n_ref = n_ref_of(P.sl.T(bh / P.H), P.s);
        named_bar(3, dtc::SMX * 32);
        if (sw == 0 && lane < G) {
          const int g = lane;
          m_ref[g] = P.mref[(int64_t)bh * G + g];
          ctv[g] = P.cterm[(int64_t)bh * G + g];
        }
        named_bar(3, dtc::SMX * 32);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          m_run[g] = g < G ? m_ref[g] : 0.f;
          lt[g] = 0.f;
          wsc[g] = 1.f;
        }
      }
      // the chunk's slots into registers and the reference logits S[idx]
      // requested; the ring stage is then free for the producer
      const int64_t row = row0 + n;
      const bool valid = row < n_code;
      if (!mbar_wait(&in_full[st], (it / NST) & 1, abort_flag)) { ok = false; break; }
      int js[kMaxK];
      {
        const int32_t* ir = sIdx(st) + n * P.k;
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) js[i] = (i < P.k && valid) ? ir[i] : -1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&in_empty[st]);
      const float* Sb = P.S + (int64_t)bh * P.n_ref_cap * G;
      float4 sv[kMaxK];
      int k_eff = 0;
#pragma unroll
      for (int i = 0; i < kMaxK; ++i) {
        sv[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        const int j = js[i];
        if (j >= 0 && j < n_ref) {
          ++k_eff;
          if (G == 4) sv[i] = __ldg(reinterpret_cast<const float4*>(Sb + (int64_t)j * 4));
        } else if (j >= n_ref) {
          latch_error(P.err, DELTAKV_ERR_DEVICE_BOUNDS, (uint32_t)j);
          js[i] = -1;
        }
      }
      float lg[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) lg[g] = 0.f;
      if (G != 4) {
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
          const int j = js[i];
          if (j < 0) continue;
#pragma unroll
          for (int g = 0; g < GP; ++g)
            if (g < G) lg[g] += Sb[(int64_t)j * G + g];
        }
      }
      // the hidden ranges' parts of a_g . u
      if (!mbar_wait(&u_full[zb], (it >> 1) & 1, abort_flag)) { ok = false; break; }
      float zz[GP];
      {
        const float* z0 = sZb(zb) + (size_t)n * GP;
#pragma unroll
        for (int g = 0; g < GP; g += 4) {
          float4 acc = *reinterpret_cast<const float4*>(z0 + g);
#pragma unroll
          for (int pt = 1; pt < dtc::PARTS; ++pt) {
            const float4 v = *reinterpret_cast<const float4*>(z0 + pt * dtc::CH * GP + g);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
          }
          zz[g] = acc.x; zz[g + 1] = acc.y; zz[g + 2] = acc.z; zz[g + 3] = acc.w;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&z_empty[zb]);
      if (G == 4) {
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
          lg[0] += sv[i].x; lg[1] += sv[i].y; lg[2] += sv[i].z; lg[3] += sv[i].w;
        }
      }
      const float inv_k = 1.0f / (float)max(k_eff, 1);
      // chunk maximum of every head's logits: warp reduction, then across the
      // four warps through a slot pair indexed by chunk parity
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        if (g < G) {
          lg[g] = zz[g] + ctv[g] + lg[g] * inv_k;
          float wm;
          const float mv = valid ? lg[g] : -INFINITY;
          asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(wm) : "f"(mv));
          if (lane == 0) mred[zb * 32 + sw * 8 + g] = wm;
        }
      }
      named_bar(3, dtc::SMX * 32);
      // lazy rescaling: the scale m_run moves only when a chunk maximum
      // exceeds it by more than TAU (the same decision in every thread)
      float mnew[GP];
      bool raise = false;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        mnew[g] = m_run[g];
        if (g < G) {
          float m = -INFINITY;
#pragma unroll
          for (int w = 0; w < dtc::SMX; ++w) m = fmaxf(m, mred[zb * 32 + w * 8 + g]);
          if (m > m_run[g] + dtc::TAU) {
            mnew[g] = m;
            raise = true;
          }
        }
      }
      if (raise) {
        float alpha[GP];
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          alpha[g] = g < G ? exp2f(m_run[g] - mnew[g]) : 1.f;
          lt[g] *= alpha[g];
          m_run[g] = mnew[g];
          wsc[g] = g < G ? exp2f(fminf(m_run[g] - m_ref[g], 100.f)) : 1.f;
        }
        if (it > seg_first) {
          // the accumulator holds the segment's chunks so far: once their
          // MMAs are complete, scale it in place
          const int j = it - 1;
          ok = mbar_wait(&ua_done[j & 1], (j >> 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            if (h2 < hidden / 128) {
              // columns g (hi) and 8 + g (lo) of head g
              float du[16];
              const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + dtc::COL_U + 16 * h2;
              tmem_ld16f(ta, du);
#pragma unroll
              for (int c = 0; c < 16; ++c)
                if ((c & 7) < GP) du[c] *= alpha[c & 7];
              tmem_st16f(ta, du);
            }
          }
          tmem_st_wait();
          tc_fence_before();
        }
      }
      float p[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        p[g] = (g < G && valid) ? exp2f(lg[g] - m_run[g]) : 0.f;
        lt[g] += p[g];
      }
      if (!mbar_wait(&p_empty[zb], ((it >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
      {
        // p = hi + lo: rows g and 8 + g of the P tile (G <= 8)
        unsigned char* pt = sP(zb);
        const int atom = n >> 6, cc = n & 63;
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (g < G) {
            const __half hi = __float2half_rn(p[g]);
            const __half lo = __float2half_rn(p[g] - __half2float(hi));
            *reinterpret_cast<__half*>(pt + atom * 16 * 128 + swz_off(g, cc * 2, 128)) = hi;
            *reinterpret_cast<__half*>(pt + atom * 16 * 128 + swz_off(8 + g, cc * 2, 128)) = lo;
          }
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[zb]);
      // slot weights, relative to the reference maximum, into the kv-head's
      // global table
      if (valid && k_eff > 0) {
        float* wt = P.wtab + (int64_t)bh * P.n_ref_cap * G;
        float sc[GP];
#pragma unroll
        for (int g = 0; g < GP; ++g) sc[g] = g < G ? p[g] * wsc[g] * inv_k : 0.f;
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
          const int j = js[i];
          if (j < 0) continue;
          if (G == 4) {
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(wt + (int64_t)j * 4), "f"(sc[0]),
                         "f"(sc[1]), "f"(sc[2]), "f"(sc[3])
                         : "memory");
          } else {
#pragma unroll
            for (int g = 0; g < GP; ++g)
              if (g < G) atomicAdd(wt + (int64_t)j * G + g, sc[g]);
          }
        }
      }
      const bool seg_end = (it == n_local - 1) || (x + 1 >= coff(bh + 1));
      if (seg_end) {
        // the segment's U once its last MMA is complete, then its denominator
        ok = mbar_wait(&ua_done[it & 1], (it >> 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        const int64_t pb = (int64_t)bh * P.nslot_cap + (int64_t)blockIdx.x - dtc_owner(coff(bh), N, gridp);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          if (h2 < hidden / 128) {
            float du[16];  // columns g (hi) and 8 + g (lo) of head g
            tmem_ld16f(tmem + ((uint32_t)(q * 32) << 16) + dtc::COL_U + 16 * h2, du);
            const int unit = 128 * h2 + n;
#pragma unroll
            for (int g = 0; g < GP; ++g)
              if (g < G) P.Upart[(pb * G + g) * hidden + unit] = du[g] + du[8 + g];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ua_free);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (g < G) {
            const float ls = warp_sum(lt[g]);
            if (lane == 0) lred[sw * 8 + g] = ls;
          }
        }
        named_bar(3, dtc::SMX * 32);
        if (sw == 0 && lane < G) {
          float l = 0.f;
          for (int w = 0; w < dtc::SMX; ++w) l += lred[w * 8 + lane];
          float mr = m_run[0];
#pragma unroll
          for (int g = 1; g < GP; ++g)
            if (lane == g) mr = m_run[g];
          P.part[(pb * G + lane) * 2 + 0] = mr;
          P.part[(pb * G + lane) * 2 + 1] = l;
        }
      }
    }
    if (!ok) {
      latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 23);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == dtc::MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, dtc::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host
namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn_dec() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}
}  // namespace

// Stages of the input ring: as many (up to 4) as shared memory holds.
int decode_tc_stages(const Plan& p) {
  const auto& c = p.cfg;
  for (int nst = dtc::MAX_STAGES; nst >= 2; --nst)
    if (DecLayout(c.d_c, c.k, c.hidden, nst, p.code4, dtc_gp(p.G)).total + 1024 <= 227 * 1024) return nst;
  return 0;
}

bool decode_tc_supported(const Plan& p) {
  const auto& c = p.cfg;
  if (!p.bf16 || !encode_fn_dec()) return false;
  // u = act(W3 c + b3) enters the U MMA as one fp16 term, so each value
  // V-side carries a relative error of up to 2^-12.  With a nonlinear codec
  // that stays inside the attention tolerance; a linear codec (no
  // activation) feeds larger, unsquashed u and takes the fp32 token loop.
  if (c.act == DELTAKV_ACT_NONE) return false;
  if (!(c.hidden == 128 || c.hidden == 256)) return false;
  if (!(c.d_c == 16 || c.d_c == 32 || c.d_c == 64 || c.d_c == 128)) return false;
  if (2 * p.G > 16) return false;
  return decode_tc_stages(p) >= 2 && (!p.code4 || c.d_c <= 64);
}

int decode_tc_grid(const Plan& p, int64_t N) {
  (void)p;
  return (int)std::min<int64_t>(N, kNumSMs);
}

cudaError_t launch_decode_tc(const Plan& p, const CacheView& cv, const SeqLens& sl, const int32_t* cho,
                             const void* W3, const float* b3, void* ws, cudaStream_t st, int* grid_out,
                             const int32_t* rowlist, const int32_t* ncode, int64_t rl_cap) {
  const auto& c = p.cfg;
  const int BH = c.batch * c.kv_heads;
  const int n_ch_all = (int)ceil_div64(n_code_of(sl.T_all, c.stride_s), dtc::CH);
  // with one length for all, the grid covers the chunks; else one CTA per SM
  // (CTAs past the end of the list have nothing to do)
  const int grid = cho ? kNumSMs : decode_tc_grid(p, (int64_t)n_ch_all * BH);
  *grid_out = grid;
  if (grid == 0) return cudaSuccess;
  char* w = (char*)ws;
  DecTcParams P;
  P.s = c.stride_s; P.d_h = c.d_h; P.G = p.G; P.k = c.k; P.d_c = c.d_c; P.hidden = c.hidden;
  P.act = (int)c.act; P.H = c.kv_heads; P.BH = BH;
  P.n_ref_cap = p.n_ref_cap;
  P.cv = cv; P.sl = sl; P.n_ch_all = n_ch_all; P.cho = cho;
  P.rowlist = rowlist; P.ncode = ncode; P.rl_cap = rl_cap;
  P.grid = grid; P.nslot_cap = p.nslot_cap;
  P.n_refblk = (int)ceil_div64(n_ref_of(sl.T_max, c.stride_s), 64);
  P.n_refblk_cap = (int)ceil_div64(p.n_ref_cap, 64);
  P.code_swz = c.d_c >= 64 ? 128 : c.d_c * 2;
  P.code_atoms = c.d_c > 64 ? c.d_c / 64 : 1;
  P.nst = decode_tc_stages(p);
  P.code4 = p.code4 ? 1 : 0;
  P.code4p = (const uint8_t*)(cv.base + cv.off_code);
  P.cscale = p.code4 ? (const __nv_bfloat16*)(cv.base + cv.off_cscale) : nullptr;
  P.idx = (const int32_t*)(cv.base + cv.off_idx);
  P.W3 = (const __nv_bfloat16*)W3; P.b3 = b3;
  P.a = (const float*)(w + p.ws_a); P.cterm = (const float*)(w + p.ws_cterm);
  P.S = (const float*)(w + p.ws_S); P.Smax = (const float*)(w + p.ws_Smax);
  P.mref = (const float*)(w + p.ws_mref);
  P.wtab = (float*)(w + p.ws_wtab); P.part = (float*)(w + p.ws_part); P.Upart = (float*)(w + p.ws_U);
  P.err = (uint32_t*)ws;
  CUtensorMap mapC;
  memset(&mapC, 0, sizeof(mapC));  // unused with 4-bit codes (the producer copies them untiled)
  if (!p.code4) {
    // pages of cp code rows; rows past a sequence's last token are loaded
    // as they are and masked by the activation and softmax warps
    cuuint64_t dims[3] = {(cuuint64_t)c.d_c, (cuuint64_t)cv.cp, (cuuint64_t)cv.n_pages};
    cuuint64_t str[2] = {(cuuint64_t)c.d_c * 2, (cuuint64_t)cv.cp * c.d_c * 2};
    cuuint32_t box[3] = {(cuuint32_t)std::min(c.d_c, 64), (cuuint32_t)dtc::CH, 1};
    cuuint32_t es[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = P.code_swz == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : P.code_swz == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                     : CU_TENSOR_MAP_SWIZZLE_32B;
    if (encode_fn_dec()(&mapC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<char*>(cv.base + cv.off_code), dims,
                        str, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  const int gp = dtc_gp(p.G);
  const size_t smem = DecLayout(c.d_c, c.k, c.hidden, P.nst, p.code4, gp).total + 1024;
  void (*kern)(const CUtensorMap, const DecTcParams) = nullptr;
  const bool hb = b3 != nullptr;
#define DTC_PICK(A)                                                                                      \
  kern = gp == 4 ? (hb ? decode_tc_kernel<A, true, 4> : decode_tc_kernel<A, false, 4>)                   \
                 : (hb ? decode_tc_kernel<A, true, 8> : decode_tc_kernel<A, false, 8>)
  switch ((int)c.act) {
    case DELTAKV_ACT_GELU_ERF:
      DTC_PICK(DELTAKV_ACT_GELU_ERF);
      break;
    case DELTAKV_ACT_GELU_TANH:
      DTC_PICK(DELTAKV_ACT_GELU_TANH);
      break;
    default:
      return cudaErrorNotSupported;  // decode_tc_supported excludes the linear codec
  }
#undef DTC_PICK
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(p, st, KID_DEC_STREAM_TC);
  kern<<<P.grid, dtc::THREADS, smem, st>>>(mapC, P);
  return cudaGetLastError();
}

}  // namespace dkv
