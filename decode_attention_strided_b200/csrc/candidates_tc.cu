// candidates_tc.cu -- nearest strided references on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA), with a fused running top-k.
//
// DeltaKV summary, section 3, "Processo di Compressione" step 1: for every
// non-reference token the k most similar earlier references by L2 distance
// over [K ; V].  Ranking by |x_t - r_j|^2 equals ranking by
//     e(t, j) = |r_j|^2 / 2 - <x_t, r_j>
// (the token's own norm is common to the row), so the hot loop is the causal
// contraction X[T x D] . R[n_ref x D]^T with a per-column bias.  It runs as
// bf16 x bf16 -> fp32 MMAs; the epilogue keeps, per token, the KC = k + 4
// smallest e in registers (ties to the lower slot).  The GEMM form loses
// precision to cancellation when x_t is close to r_j, so the encode kernel
// re-ranks these KC candidates with exact fp32 distances before choosing k.
//
// Work unit: two 128-token tiles of one (sequence, kv-head) -- 256 tokens
// share every reference tile that is staged in shared memory.
// Warp roles (320 threads, one CTA per SM, persistent):
//   warps 0-7  warp w owns token tile w / 4, TMEM lanes 32 (w % 4)..: at the
//              start of a unit it writes its token rows into tensor memory
//              (the A operand), then drains that tile's accumulator into the
//              rows' running top-k lists
//   warp 8     TMA producer: whole reference tiles (128 rows x D) into a
//              3-slot ring
//   warp 9     MMA issuer: M=128, N=128, K=16 tcgen05.mma with A in tensor
//              memory and B in shared memory, fp32 accumulators in TMEM
// TMEM (512 columns): A of token tile 0 and 1 (D/2 columns each, two bf16
// per column), then one 128-column accumulator per token tile.  The MMAs of
// tile 1 run while the epilogue drains tile 0 and the other way round.
// The ranking key e is formed inside the accumulator: A holds -x_t, and one
// more K = 16 MMA per tile adds a ones row times the bf16 split of h_j (three
// terms, 24 significant bits), so the epilogue reads e directly.
// Shape choices: an M = 128 MMA occupies the tensor pipe for at least about
// 58 cycles whatever its N, so N = 128 (64 cycles of math) keeps it math-bound;
// with A in tensor memory each MMA reads only its 4 KB of B from shared
// memory, which leaves shared-memory bandwidth for the TMA writes and the
// epilogue.
#include <cfloat>
#include <climits>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace dkv {
using namespace sm100;

namespace tcc {
constexpr int TM = 128;                     // tokens per tile (MMA M)
constexpr int TPU = 2;                      // token tiles per unit
constexpr int RN = 128;                     // references per tile (MMA N)
constexpr int NSLOT = 3;                    // reference tiles in flight
constexpr int BATOM = RN * 128;             // bytes: 128 reference rows x 128 B
constexpr int HATOM = RN * 32;              // bytes: 128 rows x 16 bf16 (32-byte swizzle)
constexpr int CHUNK = 16;                   // columns per slow-path chunk
constexpr int SPILL = 32 * CHUNK * 4;       // bytes per warp: 32 lanes x CHUNK floats
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (EPI_WARPS + 2) * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t A_COL = 0;               // A of tile i at A_COL + i * 128
constexpr uint32_t D_COL = 256;             // accumulator of tile i at D_COL + i * RN
constexpr int PRODUCER_WARP = EPI_WARPS;
constexpr int MMA_WARP = EPI_WARPS + 1;
__host__ __device__ constexpr int spill_bytes(int) { return EPI_WARPS * SPILL; }
}  // namespace tcc

struct TcParams {
  int T, s, H, BH, n_units, n_pairs, d_h;
  int n_ref;
  int64_t n_ref_cap, n_code_cap;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  int64_t sb, sh, st;
  const float* hnorm;
  int32_t* cand;
  uint32_t* err;
};

struct UnitInfo {
  int p, bh, t0;
  int R[tcc::TPU];
  int Rmax;
};

// Static schedule: units sorted by decreasing cost (later token pairs see more
// references), dealt to the persistent CTAs in a zig-zag.
__device__ __forceinline__ bool unit_of(const TcParams& P, int round, UnitInfo& u) {
  const int G = gridDim.x, c = blockIdx.x;
  const int idx = round * G + ((round & 1) ? (G - 1 - c) : c);
  if (idx >= P.n_units) return false;
  u.p = P.n_pairs - 1 - idx / P.BH;
  u.bh = idx % P.BH;
  u.t0 = u.p * tcc::TM * tcc::TPU;
  u.Rmax = 0;
#pragma unroll
  for (int i = 0; i < tcc::TPU; ++i) {
    const int lo = u.t0 + i * tcc::TM;
    const int hi = min(lo + tcc::TM, P.T) - 1;  // last token of the tile
    int R = 0;
    if (hi >= lo && hi >= 1) {
      const int ns = min((hi + P.s - 1) / P.s, P.n_ref);  // slots seen by the tile's last token
      R = (ns + tcc::RN - 1) / tcc::RN;
    }
    u.R[i] = R;
    u.Rmax = max(u.Rmax, R);
  }
  return true;
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Minimum of 16 consecutive values (eight three-input minima).
__device__ __forceinline__ float min16(const float* v) {
  const float a0 = min3f(v[0], v[1], v[2]), a1 = min3f(v[3], v[4], v[5]), a2 = min3f(v[6], v[7], v[8]);
  const float a3 = min3f(v[9], v[10], v[11]), a4 = min3f(v[12], v[13], v[14]);
  return fminf(min3f(a0, a1, a2), min3f(a3, a4, v[15]));
}

// One 64-column block of one token row's accumulator, which holds
// e = |r_j|^2 / 2 - <x_t, r_j> for slots jb .. jb + 63: fold it into the
// row's running list.
template <int KC>
__device__ __forceinline__ void cand_block(float (&v)[64], int jb, int cnt, int cnt_lo, bool first,
                                           float (&bd)[KC], int (&bi)[KC], float* sp, int sw) {
  if (jb + 64 > cnt_lo) {
#pragma unroll
    for (int x = 0; x < 64; ++x)
      if (jb + x >= cnt) v[x] = FLT_MAX;
  }
  if (first) {
    // the list is empty: every value is taken, without branching
#pragma unroll
    for (int x = 0; x < 64; ++x) topk_insert_inorder<KC>(bd, bi, v[x], jb + x);
    return;
  }
  // fast path: most blocks hold nothing below any lane's k-th best; the
  // per-chunk minima also let the slow path skip chunks without a candidate
  float cm[64 / tcc::CHUNK];
#pragma unroll
  for (int c = 0; c < 64 / tcc::CHUNK; ++c) cm[c] = min16(v + c * tcc::CHUNK);
  if (!__any_sync(0xffffffffu, fminf(min3f(cm[0], cm[1], cm[2]), cm[3]) < bd[KC - 1])) return;
#pragma unroll
  for (int c = 0; c < 64 / tcc::CHUNK; ++c) {
    const float thr = bd[KC - 1];
    if (!__any_sync(0xffffffffu, cm[c] < thr)) continue;
    // bit x = (v_x < thr): the sign of v_x - thr shifted in from the top
    // (one funnel shift per value), in two independent 8-bit chains
    uint32_t ma = 0u, mb = 0u;
#pragma unroll
    for (int x = tcc::CHUNK / 2 - 1; x >= 0; --x) {
      ma = __funnelshift_l(__float_as_uint(v[c * tcc::CHUNK + x] - thr), ma, 1);
      mb = __funnelshift_l(__float_as_uint(v[c * tcc::CHUNK + tcc::CHUNK / 2 + x] - thr), mb, 1);
    }
    uint32_t m = ma | (mb << (tcc::CHUNK / 2));
    if (!__any_sync(0xffffffffu, __popc(m) > 1)) {
      // at most one candidate per lane: it is the chunk's minimum
      if (m) topk_insert_inorder<KC>(bd, bi, cm[c], jb + c * tcc::CHUNK + __ffs(m) - 1);
      continue;
    }
    if (m) {
#pragma unroll
      for (int i4 = 0; i4 < tcc::CHUNK / 4; ++i4)
        reinterpret_cast<float4*>(sp)[i4 ^ sw] =
            make_float4(v[c * tcc::CHUNK + 4 * i4], v[c * tcc::CHUNK + 4 * i4 + 1], v[c * tcc::CHUNK + 4 * i4 + 2],
                        v[c * tcc::CHUNK + 4 * i4 + 3]);
    }
    __syncwarp();
    while (m) {
      const int x = __ffs(m) - 1;
      m &= m - 1;
      const float vx = sp[x ^ (sw << 2)];  // float4 slot (x / 4) ^ sw, element x % 4
      topk_insert_inorder<KC>(bd, bi, vx, jb + c * tcc::CHUNK + x);
    }
    __syncwarp();
  }
}

template <int NKC, int KC>
__global__ void __launch_bounds__(tcc::THREADS, 1)
    cand_tc_kernel(const __grid_constant__ CUtensorMap mapRK, const __grid_constant__ CUtensorMap mapRV,
                   const __grid_constant__ CUtensorMap mapH, const TcParams P) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int D = NKC * 64;
  // one ring slot: NKC reference atoms, then the tile's split half-norm
  // rows (128 x 32 bytes, 32-byte swizzle)
  constexpr int SLOT = NKC * tcc::BATOM + tcc::HATOM;
  unsigned char* sB = smem;                                     // [NSLOT] slots
  unsigned char* sOnes = sB + tcc::NSLOT * SLOT;                // 128 rows of (1, 1, 1, 0, ...)
  float* spill = (float*)(sOnes + tcc::HATOM);                  // [EPI_WARPS][32][CHUNK]
  uint64_t* b_full = (uint64_t*)((unsigned char*)spill + tcc::spill_bytes(KC));  // [NSLOT]
  uint64_t* b_empty = b_full + tcc::NSLOT;                      // [NSLOT]
  uint64_t* a_full = b_empty + tcc::NSLOT;                      // [1]
  uint64_t* d_full = a_full + 1;                                // [TPU]
  uint64_t* d_empty = d_full + tcc::TPU;                        // [TPU]
  uint64_t* drain = d_empty + tcc::TPU;                         // [1] the MMA warp's last commit
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int HALF = NKC / 2;  // atoms per d_h (K part, then V part)

  if (threadIdx.x == 0) {
    for (int i = 0; i < tcc::NSLOT; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    mbar_init(a_full, tcc::EPI_WARPS);
    for (int i = 0; i < tcc::TPU; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], tcc::EPI_WARPS / tcc::TPU);  // the warps of token tile i
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == tcc::PRODUCER_WARP && lane == 0) {
    prefetch_tensormap(&mapRK);
    prefetch_tensormap(&mapRV);
    prefetch_tensormap(&mapH);
  }
  // the ones operand of the norm MMA: row m = (1, 1, 1, 0 x 13), 32-byte
  // swizzle (16-byte chunk c of row m sits at chunk c ^ ((m >> 2) & 1))
  for (int i = threadIdx.x; i < tcc::TM * 2; i += blockDim.x) {
    const int m = i >> 1, c = i & 1;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (c == 0) {
      v.x = 0x3F803F80u;  // bf16 1.0, 1.0
      v.y = 0x00003F80u;  // 1.0, 0
    }
    *reinterpret_cast<uint4*>(sOnes + m * 32 + ((c ^ ((m >> 2) & 1)) << 4)) = v;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == tcc::MMA_WARP) {
    tmem_alloc(tmem_slot, tcc::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == tcc::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t b_it = 0;
      bool ok = true;
      UnitInfo u;
      for (int round = 0; ok && unit_of(P, round, u); ++round) {
        for (int r = 0; r < u.Rmax && ok; ++r, ++b_it) {
          const int sl = b_it % tcc::NSLOT;
          const uint32_t ph = (b_it / tcc::NSLOT) & 1;
          if (!mbar_wait(&b_empty[sl], ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&b_full[sl], SLOT);
          unsigned char* dst = sB + sl * SLOT;
          for (int kc = 0; kc < NKC; ++kc) {
            if (kc < HALF)
              tma_load_3d(&mapRK, &b_full[sl], dst + kc * tcc::BATOM, kc * 64, r * tcc::RN, u.bh);
            else
              tma_load_3d(&mapRV, &b_full[sl], dst + kc * tcc::BATOM, (kc - HALF) * 64, r * tcc::RN, u.bh);
          }
          tma_load_3d(&mapH, &b_full[sl], dst + NKC * tcc::BATOM, 0, r * tcc::RN, u.bh);
        }
      }
      if (!ok) {
        latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 1);
        *abort_flag = 1;
      }
      // every reference load issued (b_it of them, the last NSLOT one per
      // slot) lands before the block can finish, also after an abort
      for (int i = 0; i < tcc::NSLOT && b_it > (uint32_t)i; ++i) {
        const uint32_t it = b_it - 1 - i;
        if (!mbar_wait_drain(&b_full[it % tcc::NSLOT], (it / tcc::NSLOT) & 1))
          latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 4);
      }
    }
  } else if (warp == tcc::MMA_WARP) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(tcc::TM, tcc::RN);
      const uint32_t b_base = smem_u32(sB);
      uint32_t b_it = 0, acc_it = 0, unit_it = 0;
      bool ok = true;
      UnitInfo u;
      for (int round = 0; ok && unit_of(P, round, u); ++round) {
        if (u.Rmax == 0) continue;
        if (!mbar_wait(a_full, unit_it & 1, abort_flag)) { ok = false; break; }
        ++unit_it;
        for (int r = 0; r < u.Rmax && ok; ++r, ++acc_it, ++b_it) {
          const int sl = b_it % tcc::NSLOT;
          if (!mbar_wait(&b_full[sl], (b_it / tcc::NSLOT) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
          for (int i = 0; i < tcc::TPU; ++i) {
            if (acc_it >= 1 && !mbar_wait(&d_empty[i], (acc_it - 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem + tcc::D_COL + i * tcc::RN;
            const uint32_t a = tmem + tcc::A_COL + i * 128;
#pragma unroll
            for (int k16 = 0; k16 < D / 16; ++k16)
              umma_f16_ts(d, a + k16 * 8,
                           desc_kmajor_sw128(b_base + sl * SLOT + (k16 >> 2) * tcc::BATOM + (k16 & 3) * 32), idesc,
                           k16 != 0);
            // + h_j: ones (A, shared memory) times the split half-norm rows
            umma_f16(d, desc_kmajor_sw32(smem_u32(sOnes)), desc_kmajor_sw32(b_base + sl * SLOT + NKC * tcc::BATOM),
                     idesc, 1u);
            umma_commit(&d_full[i]);
          }
          if (!ok) break;
          umma_commit(&b_empty[sl]);
        }
      }
      if (!ok) {
        latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 2);
        *abort_flag = 1;
      }
      // every MMA issued has completed before tensor memory is released
      if (!umma_drain(drain)) latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 5);
    }
  } else {
    // ------------------------------------------------ token rows + epilogue
    const int q = warp & 3, ti = warp >> 2, row = q * 32 + lane;
    float* sp = spill + warp * (32 * tcc::CHUNK) + lane * tcc::CHUNK;  // this lane's CHUNK floats
    const int sw = (lane >> 1) & 3;  // float4 swizzle: 8 lanes of a phase hit 8 distinct bank groups
    uint32_t acc_it = 0;
    bool ok = true;
    UnitInfo u;
    for (int round = 0; ok && unit_of(P, round, u); ++round) {
      if (u.Rmax == 0) continue;
      const int t = u.t0 + ti * tcc::TM + row;
      // A of token tile ti: this thread's token row, [K ; V] as bf16 pairs.
      // Every MMA that read it in the previous unit is complete: this warp
      // consumed that unit's last accumulator of tile ti.
      {
        const int b = u.bh / P.H, h = u.bh % P.H;
        const __nv_bfloat16* kr = P.K + b * P.sb + h * P.sh + (int64_t)t * P.st;
        const __nv_bfloat16* vr = P.V + b * P.sb + h * P.sh + (int64_t)t * P.st;
        const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + tcc::A_COL + ti * 128;
#pragma unroll 1
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          // columns c0 .. c0 + 31 hold elements 2 c0 .. 2 c0 + 63 of [K ; V]
          const int e = 2 * c0;
          const __nv_bfloat16* src = e < P.d_h ? kr + e : vr + (e - P.d_h);
          uint32_t w[32];
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4) {
            const uint4 x = t < P.T ? __ldg(reinterpret_cast<const uint4*>(src) + v4) : make_uint4(0, 0, 0, 0);
            // -x_t: flip the sign bits of both bf16 halves
            w[4 * v4] = x.x ^ 0x80008000u;
            w[4 * v4 + 1] = x.y ^ 0x80008000u;
            w[4 * v4 + 2] = x.z ^ 0x80008000u;
            w[4 * v4 + 3] = x.w ^ 0x80008000u;
          }
          tmem_st32(ta + c0, w);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full);
      }
      const int first = u.t0 + ti * tcc::TM;
      const int cnt = t < P.T ? min((t + P.s - 1) / P.s, P.n_ref) : 0;  // valid slots j < cnt
      const int cnt_lo = min((first + P.s - 1) / P.s, P.n_ref);         // smallest cnt in the tile
      float bd[KC];
      int bi[KC];
#pragma unroll
      for (int x = 0; x < KC; ++x) {
        bd[x] = FLT_MAX;
        bi[x] = INT_MAX;
      }
      for (int r = 0; r < u.Rmax; ++r, ++acc_it) {
        if (!mbar_wait(&d_full[ti], acc_it & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dcol = tmem + ((uint32_t)(q * 32) << 16) + tcc::D_COL + ti * tcc::RN;
#pragma unroll 1
        for (int hf = 0; hf < tcc::RN / 64; ++hf) {
          float v[64];
          tmem_ld64(dcol + hf * 64, v);
          if (hf == tcc::RN / 64 - 1) {
            // the accumulator is in registers: the next MMAs may reuse it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[ti]);
          }
          cand_block<KC>(v, r * tcc::RN + hf * 64, cnt, cnt_lo, r == 0 && hf == 0, bd, bi, sp, sw);
        }
      }
      if (!ok) break;
      if (t < P.T && (t % P.s) != 0) {
        int32_t* o = P.cand + ((int64_t)u.bh * P.n_code_cap + (t - t / P.s - 1)) * KC;
#pragma unroll
        for (int x = 0; x < KC; ++x) o[x] = bi[x] == INT_MAX ? -1 : bi[x];
      }
    }
    if (!ok) {
      latch_error(P.err, DELTAKV_ERR_DEVICE_TIMEOUT, 3);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == tcc::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, tcc::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// bf16 tensor map with a 64 x rows box in the 128-byte swizzle layout.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
              cuuint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t box[5] = {64, box_rows, 1, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The split half-norm plane: box 16 x RN rows, 32-byte swizzle.
bool make_map_h(CUtensorMap* m, const void* base, const cuuint64_t* dims, const cuuint64_t* strides) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t box[3] = {16, tcc::RN, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = kNumSMs;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : kNumSMs;
}

template <int NKC, int KC>
size_t smem_bytes() {
  return 1024 + (size_t)tcc::NSLOT * (NKC * tcc::BATOM + tcc::HATOM) + tcc::HATOM + (size_t)tcc::spill_bytes(KC) + 256;
}

template <int NKC, int KC>
cudaError_t launch_tc(const CUtensorMap& mRK, const CUtensorMap& mRV, const CUtensorMap& mH, const TcParams& P,
                      int grid, cudaStream_t st) {
  auto kern = cand_tc_kernel<NKC, KC>;
  const size_t smem = smem_bytes<NKC, KC>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, tcc::THREADS, smem, st>>>(mRK, mRV, mH, P);
  return cudaGetLastError();
}

}  // namespace

bool candidates_tc_supported(const Plan& p) {
  return p.bf16 && (p.cfg.d_h == 64 || p.cfg.d_h == 128) && encode_fn() != nullptr;
}

cudaError_t launch_candidates_tc(const Plan& p, int T, const KVView& kv, const void* cache, void* ws,
                                 cudaStream_t st) {
  const auto& c = p.cfg;
  const int64_t n_code = n_code_of(T, c.stride_s);
  if (n_code == 0) return cudaSuccess;
  const int n_ref = (int)n_ref_of(T, c.stride_s);
  const int d_h = c.d_h;
  CUtensorMap mRK, mRV, mH;
  {
    const char* cb = (const char*)cache;
    cuuint64_t dims[3] = {(cuuint64_t)d_h, (cuuint64_t)n_ref, (cuuint64_t)c.batch * c.kv_heads};
    cuuint64_t str[2] = {(cuuint64_t)d_h * 2, (cuuint64_t)p.n_ref_cap * d_h * 2};
    if (!make_map(&mRK, cb + p.off_refk, 3, dims, str, tcc::RN) ||
        !make_map(&mRV, cb + p.off_refv, 3, dims, str, tcc::RN))
      return cudaErrorNotSupported;
    // split half-norm rows: 16 bf16 (32 bytes) per reference, 32-byte swizzle
    cuuint64_t hdims[3] = {16, (cuuint64_t)n_ref, (cuuint64_t)c.batch * c.kv_heads};
    cuuint64_t hstr[2] = {32, (cuuint64_t)p.n_ref_cap * 32};
    if (!make_map_h(&mH, (const char*)ws + p.ws_hsplit, hdims, hstr)) return cudaErrorNotSupported;
  }
  TcParams P;
  P.T = T;
  P.s = c.stride_s;
  P.H = c.kv_heads;
  P.BH = c.batch * c.kv_heads;
  P.d_h = d_h;
  P.K = (const __nv_bfloat16*)kv.K;
  P.V = (const __nv_bfloat16*)kv.V;
  P.sb = kv.sb;
  P.sh = kv.sh;
  P.st = kv.st;
  P.n_pairs = (int)ceil_div64(T, tcc::TM * tcc::TPU);
  P.n_units = P.n_pairs * P.BH;
  P.n_ref = n_ref;
  P.n_ref_cap = p.n_ref_cap;
  P.n_code_cap = p.n_code_cap;
  P.hnorm = (const float*)((const char*)ws + p.ws_hnorm);
  P.cand = (int32_t*)((char*)ws + p.ws_cand);
  P.err = (uint32_t*)ws;
  const int grid = std::min(P.n_units, sm_count());
  ProfScope ps(p, st, KID_CAND_TC);
  if (d_h == 128)
    return p.KC == 8 ? launch_tc<4, 8>(mRK, mRV, mH, P, grid, st) : launch_tc<4, 12>(mRK, mRV, mH, P, grid, st);
  return p.KC == 8 ? launch_tc<2, 8>(mRK, mRV, mH, P, grid, st) : launch_tc<2, 12>(mRK, mRV, mH, P, grid, st);
}

}  // namespace dkv
