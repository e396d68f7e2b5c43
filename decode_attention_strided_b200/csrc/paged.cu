// paged.cu -- the compressed cache in pages drawn from a shared pool.
//
// DeltaKV summary, section 4 ("Implementazione: Sparse-vLLM"): the serving
// system keeps the irregular, compressed cache under a memory manager that
// is decoupled from the attention kernels.  Here the cache of one
// (sequence, kv-head) is a list of pages of 128 consecutive blocks of s
// tokens -- 128 reference rows, 128 (s - 1) code rows, their slot rows and,
// with 4-bit codes, their scales -- and a page table maps each logical page
// to a physical page of the pool, so sequences of different lengths share
// one pool and a sequence grows a page at a time.
//
// Pool layout: one plane per kind of row, each an array of pages (page p of
// the code plane holds code rows p cp .. p cp + cp - 1), planes 256-byte
// aligned.  Every page holds a multiple of 128 code rows, so a 128-row chunk
// of the decode's token loop never straddles two pages.
#include <cstring>

#include "common.cuh"

namespace dkv {

PoolLayout pool_layout(const Plan& p, int64_t n_pages) {
  const auto& c = p.cfg;
  PoolLayout L{};
  L.rp = kPageRefs;
  L.cp = (int64_t)kPageRefs * (c.stride_s - 1);
  size_t off = 0;
  L.off_refk = off;
  off = align256(off + (size_t)(n_pages * L.rp * c.d_h) * p.esize);
  L.off_refv = off;
  off = align256(off + (size_t)(n_pages * L.rp * c.d_h) * p.esize);
  L.off_code = off;
  off = align256(off + (p.code4 ? (size_t)(n_pages * L.cp * c.d_c) / 2 : (size_t)(n_pages * L.cp * c.d_c) * p.esize));
  L.off_idx = off;
  off = align256(off + (size_t)(n_pages * L.cp * c.k) * 4);
  L.off_cscale = 0;
  if (p.code4) {
    L.off_cscale = off;
    off = align256(off + (size_t)(n_pages * L.cp) * 2);
  }
  L.bytes = off;
  return L;
}

CacheView pool_view(const Plan& p, const PoolLayout& L, const void* pool, int64_t n_pages, const int32_t* ptab,
                    int max_pages, void* ws) {
  (void)p;
  CacheView v{};
  v.base = (const char*)pool;
  v.off_refk = L.off_refk;
  v.off_refv = L.off_refv;
  v.off_code = L.off_code;
  v.off_idx = L.off_idx;
  v.off_cscale = L.off_cscale;
  v.rp = L.rp;
  v.cp = L.cp;
  v.n_pages = n_pages;
  v.ptab = ptab;
  v.max_pages = max_pages;
  v.err = (uint32_t*)ws;
  return v;
}

namespace {

// One span of consecutive rows of one plane: rows [l rows_pp, min((l + 1)
// rows_pp, n_rows)) of (sequence, kv-head) bh, from its contiguous rows to
// page ptab[bh][l].  The span starts on a multiple of 128 rows in both
// buffers, so both ends of its 16-byte words are aligned; a tail shorter than
// 16 bytes is copied byte by byte.
struct Plane {
  const char* src;    // the plane in the contiguous cache
  char* dst;          // the plane in the pool
  int64_t cap;        // rows per (sequence, kv-head) in the cache
  int64_t rows_pp;    // rows per page
  int64_t n_rows;     // rows in use per (sequence, kv-head)
  int row_bytes;
};

__global__ void __launch_bounds__(256)
    pages_from_cache_kernel(Plane pl0, Plane pl1, Plane pl2, Plane pl3, Plane pl4, int n_planes,
                            const int32_t* __restrict__ ptab, int max_pages, int64_t n_pages,
                            uint32_t* __restrict__ err) {
  const int l = blockIdx.x, bh = blockIdx.y, plane = blockIdx.z;
  if (plane >= n_planes) return;
  const Plane pl = plane == 0 ? pl0 : plane == 1 ? pl1 : plane == 2 ? pl2 : plane == 3 ? pl3 : pl4;
  const int64_t r0 = (int64_t)l * pl.rows_pp;
  if (r0 >= pl.n_rows) return;
  const int64_t r1 = min(r0 + pl.rows_pp, pl.n_rows);
  const int64_t pg = ptab[(int64_t)bh * max_pages + l];
  if (pg < 0 || pg >= n_pages) {
    if (threadIdx.x == 0 && atomicCAS(err, 0u, (uint32_t)DELTAKV_ERR_DEVICE_BOUNDS) == 0u) err[1] = (uint32_t)pg;
    return;
  }
  const char* s = pl.src + ((int64_t)bh * pl.cap + r0) * pl.row_bytes;
  char* d = pl.dst + pg * pl.rows_pp * pl.row_bytes;
  const int64_t bytes = (r1 - r0) * pl.row_bytes;
  const int64_t n16 = bytes / 16;
  for (int64_t i = threadIdx.x; i < n16; i += blockDim.x)
    reinterpret_cast<uint4*>(d)[i] = reinterpret_cast<const uint4*>(s)[i];
  for (int64_t i = n16 * 16 + threadIdx.x; i < bytes; i += blockDim.x) d[i] = s[i];
}

}  // namespace

cudaError_t launch_pages_from_cache(const Plan& p, int T, const void* cache, const PoolLayout& L, void* pool,
                                    int64_t n_pages, const int32_t* ptab, int max_pages, void* ws,
                                    cudaStream_t st) {
  const auto& c = p.cfg;
  const char* cb = (const char*)cache;
  char* pb = (char*)pool;
  const int64_t n_ref = n_ref_of(T, c.stride_s), n_code = n_code_of(T, c.stride_s);
  const int code_bytes = p.code4 ? c.d_c / 2 : c.d_c * p.esize;
  Plane pl[5];
  pl[0] = Plane{cb + p.off_refk, pb + L.off_refk, p.n_ref_cap, L.rp, n_ref, c.d_h * p.esize};
  pl[1] = Plane{cb + p.off_refv, pb + L.off_refv, p.n_ref_cap, L.rp, n_ref, c.d_h * p.esize};
  pl[2] = Plane{cb + p.off_code, pb + L.off_code, p.n_code_cap, L.cp, n_code, code_bytes};
  pl[3] = Plane{cb + p.off_idx, pb + L.off_idx, p.n_code_cap, L.cp, n_code, c.k * 4};
  pl[4] = Plane{cb + p.off_cscale, pb + L.off_cscale, p.n_code_cap, L.cp, n_code, 2};
  const int n_planes = p.code4 ? 5 : 4;
  const int n_lp = (int)ceil_div64(T, (int64_t)kPageRefs * c.stride_s);  // logical pages in use
  if (n_lp == 0) return cudaSuccess;
  pages_from_cache_kernel<<<dim3(n_lp, c.batch * c.kv_heads, n_planes), 256, 0, st>>>(
      pl[0], pl[1], pl[2], pl[3], pl[4], n_planes, ptab, max_pages, n_pages, (uint32_t*)ws);
  return cudaGetLastError();
}

}  // namespace dkv
