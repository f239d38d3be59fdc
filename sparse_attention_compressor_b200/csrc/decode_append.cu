// Decode-time cache append ("Cache layers": the K=V sliding window plus the compressor's buffer /
// pool / count / overlap state, and the indexer's own copy at index_head_dim; "Hybrid attention":
// entries appear once their source window has closed).
//
// One new token per sequence at t = ctx - 1. Its kv row is rotated at pos0 + t and written to the
// paged window cache. For compressed layers the un-rotated row also goes into a ring of the last
// L rows (slot t mod L): that ring is the compressor buffer, and for CSA (L = 2m) its older half is
// the overlap carried from the previous window. When t + 1 is a multiple of m, entry
// w = (t+1)/m - 1 closes: it pools the ring rows of its window [(w+1)m - L, (w+1)m) (clipped at
// 0) with the prefill compressor's pooling (pool_window.cuh) and is written, rotated at
// pos0 + w*m, to the pool pages. CSA does the same for the indexer key row (its own ring and
// gate, no rotation). The token count is ctx itself, so the state needs no counter of its own.
//
// Windows of L >= 64 rows (HCA): one block of 8 warps per sequence; warp 0 writes the new row and
// on a closing window the 8 warps split the window's rows and merge in shared memory. Shorter
// windows take one warp per part: a CSA layer with D = 512 and cI = 128 runs both parts in one
// 64-thread block per sequence (warp 0 the kv row and main pool, warp 1 the indexer's), other
// shapes one launch per part. The pooling reads the new token's row from its input rather than
// back from the ring. Prefill chunks (several tokens per sequence) have their own two kernels
// below.
#include "pool_window.cuh"
#include "sac_kernels.h"

namespace sac {
namespace {

struct AppendPart {
  const int32_t* ctx_lens;
  int64_t max_ctx;               // contexts above this (beyond the block tables) are skipped
  int m, L, page_size;
  int64_t pos0;
  RopeFreqs rf;
  const void* x_new;             // [nseq, C]
  void* ring;                    // [nseq, L, C] (m > 0)
  const void* gate;              // [C]
  const float* bias;             // [L]
  void* kv_pages;                // window cache (rotated rows), nullptr for the indexer part
  const int32_t* kv_bt;
  int kv_max_pages;
  void* pool_pages;              // entries (rotated when rotate != 0)
  const int32_t* pool_bt;
  int pool_max_pages;
  int rotate;
};

// Context length of sequence seq; 0 (the sequence is skipped) when it exceeds max_ctx, a bad
// input the block tables do not cover.
__device__ __forceinline__ int64_t checked_ctx(const AppendPart& a, int seq) {
  const int64_t c = __ldg(a.ctx_lens + seq);
  return c > a.max_ctx ? 0 : c;
}

template <typename T>
__device__ __forceinline__ T* page_row(void* base, const int32_t* bt, int max_pages, int page_size,
                                       int C, int seq, int64_t j) {
  const uint32_t uj = (uint32_t)j, ps = (uint32_t)page_size;  // rows of a sequence fit 32 bits
  const int page = __ldg(bt + (int64_t)seq * max_pages + uj / ps);
  if (page < 0) return nullptr;
  return reinterpret_cast<T*>(base) + ((int64_t)page * ps + uj % ps) * C;
}

// One warp's append of sequence seq when a single warp pools a window (L < 64): the new row to
// the ring and the window pages, and on a closing window the pooled entry.
template <typename T, int V>
__device__ __forceinline__ void append_warp(const AppendPart& a, int seq, int lane,
                                            PoolShared<V, 1>& sh) {
  constexpr int C = 32 * V;
  // the new row does not depend on the context length: its load goes out with ctx's
  const T* x_new = reinterpret_cast<const T*>(a.x_new) + (int64_t)seq * C;
  float v[V];
  load_lane<T, V>(x_new, lane, v);
  const int64_t t = checked_ctx(a, seq) - 1;
  if (t < 0) return;
  T* ring = a.m > 0 ? reinterpret_cast<T*>(a.ring) + (int64_t)seq * a.L * C : nullptr;
  if (ring) store_lane<T, V>(ring + (t % a.L) * C, lane, v);
  if (a.kv_pages) {
    T* dst = page_row<T>(a.kv_pages, a.kv_bt, a.kv_max_pages, a.page_size, C, seq, t);
    if (dst) {
      rotate_lane<V>(v, lane, C, a.rf, a.pos0 + t);
      store_lane<T, V>(dst, lane, v);
    }
  }
  if (a.m == 0 || (t + 1) % a.m != 0) return;
  const int64_t w = (t + 1) / a.m - 1;
  const int64_t hi = (w + 1) * a.m;
  const int64_t lo = hi - a.L < 0 ? 0 : hi - a.L;
  float u[V], acc[V];
  load_lane<T, V>(reinterpret_cast<const T*>(a.gate), lane, u);
  // the entry's page is looked up before the pooling, so its load overlaps the rows'
  T* dst = page_row<T>(a.pool_pages, a.pool_bt, a.pool_max_pages, a.page_size, C, seq, w);
  const int L = a.L;
  pool_window<T, V, 1, rows_in_flight<T, V>(64)>(
      [&](int64_t j) { return j == t ? x_new : ring + (j % L) * C; }, u,
                          a.bias, lo, hi, L, true, 0, lane, sh, acc);
  if (dst == nullptr) return;
  if (a.rotate) rotate_lane<V>(acc, lane, C, a.rf, a.pos0 + w * a.m);
  store_lane<T, V>(dst, lane, acc);
}

// Both parts of a CSA layer's append in one launch: warp 0 the kv row and the main pool, warp 1
// the indexer row and its pool (one launch fewer per decode step).
template <typename T, int V0, int V1>
__global__ void __launch_bounds__(64) append_pair_kernel(AppendPart main_part,
                                                         AppendPart index_part) {
  __shared__ PoolShared<V0, 1> sh0;
  __shared__ PoolShared<V1, 1> sh1;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32)
    append_warp<T, V0>(main_part, blockIdx.x, lane, sh0);
  else
    append_warp<T, V1>(index_part, blockIdx.x, lane, sh1);
}

template <typename T, int V, int WPE>
__global__ void __launch_bounds__(256) append_kernel(AppendPart a) {
  constexpr int C = 32 * V;
  __shared__ PoolShared<V, WPE> sh;
  const int seq = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the new row does not depend on the context length: its load goes out with ctx's
  const T* x_new = reinterpret_cast<const T*>(a.x_new) + (int64_t)seq * C;
  float v[V];
  if (warp == 0) load_lane<T, V>(x_new, lane, v);
  const int64_t t = checked_ctx(a, seq) - 1;
  if (t < 0) return;
  T* ring = a.m > 0 ? reinterpret_cast<T*>(a.ring) + (int64_t)seq * a.L * C : nullptr;
  const bool closing = a.m > 0 && (t + 1) % a.m == 0;
  if (warp == 0) {
    if (ring) store_lane<T, V>(ring + (t % a.L) * C, lane, v);
    if (a.kv_pages) {
      T* dst = page_row<T>(a.kv_pages, a.kv_bt, a.kv_max_pages, a.page_size, C, seq, t);
      if (dst) {
        rotate_lane<V>(v, lane, C, a.rf, a.pos0 + t);
        store_lane<T, V>(dst, lane, v);
      }
    }
  }
  if (!closing) return;

  // The closing window's rows: the new token's row straight from its input, the older ones from
  // the ring (written by earlier calls), so the pooling needs no barrier after the ring write and
  // all of its loads start at once.
  const int64_t w = (t + 1) / a.m - 1;
  const int64_t hi = (w + 1) * a.m;
  const int64_t lo = hi - a.L < 0 ? 0 : hi - a.L;
  float u[V], acc[V];
  load_lane<T, V>(reinterpret_cast<const T*>(a.gate), lane, u);
  // the entry's page is looked up before the pooling, so its load overlaps the rows'
  T* dst = warp == 0 ? page_row<T>(a.pool_pages, a.pool_bt, a.pool_max_pages, a.page_size, C,
                                   seq, w)
                     : nullptr;
  const int L = a.L;
  pool_window<T, V, WPE, rows_in_flight<T, V>(64)>(
      [&](int64_t j) { return j == t ? x_new : ring + (j % L) * C; }, u, a.bias, lo, hi, L,
      WPE > 1 || warp == 0, warp, lane, sh, acc);
  if (warp != 0) return;
  if (dst == nullptr) return;
  if (a.rotate) rotate_lane<V>(acc, lane, C, a.rf, a.pos0 + w * a.m);
  store_lane<T, V>(dst, lane, acc);
}

// ---- prefill chunk: n tokens per sequence, t0 = ctx - n.
// Entries w in [t0 / m, ctx / m) close inside the chunk (their last row (w+1)m - 1 >= t0). Their
// rows j >= t0 come from the chunk's input, rows j < t0 from the ring, which still holds the L rows
// before the chunk (j > t0 - L for every such window), so all entries pool in parallel; the ring
// and page writes of the chunk's rows follow in a second launch.
template <typename T, int V, int WPE>
__global__ void __launch_bounds__(256) chunk_pool_kernel(AppendPart a, int n) {
  constexpr int C = 32 * V;
  constexpr int EPB = 8 / WPE;  // entries per block
  __shared__ PoolShared<V, WPE> sh;
  const int seq = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ctx = checked_ctx(a, seq), t0 = ctx - n;
  if (t0 < 0) return;  // fewer tokens than the chunk: left untouched
  const int64_t w = t0 / a.m + (int64_t)blockIdx.x * EPB + warp / WPE;
  const bool active = w < ctx / a.m;
  if (!__syncthreads_or(active)) return;
  const T* x_new = reinterpret_cast<const T*>(a.x_new) + (int64_t)seq * n * C;
  const T* ring = reinterpret_cast<const T*>(a.ring) + (int64_t)seq * a.L * C;
  const int64_t hi = (w + 1) * a.m;
  const int64_t lo = hi - a.L < 0 ? 0 : hi - a.L;
  float u[V], acc[V];
  load_lane<T, V>(reinterpret_cast<const T*>(a.gate), lane, u);
  const int L = a.L;
  pool_window<T, V, WPE, 4>(
      [&](int64_t j) { return j >= t0 ? x_new + (j - t0) * C : ring + (j % L) * C; }, u, a.bias,
      lo, hi, L, active, warp, lane, sh, acc);
  if (!active || warp % WPE != 0) return;
  T* dst = page_row<T>(a.pool_pages, a.pool_bt, a.pool_max_pages, a.page_size, C, seq, w);
  if (dst == nullptr) return;
  if (a.rotate) rotate_lane<V>(acc, lane, C, a.rf, a.pos0 + w * a.m);
  store_lane<T, V>(dst, lane, acc);
}

// Warp per chunk token: the rotated row into the window pages, the un-rotated row into the ring
// when it is among the sequence's last L rows.
template <typename T, int V>
__global__ void __launch_bounds__(256) chunk_rows_kernel(AppendPart a, int n) {
  constexpr int C = 32 * V;
  const int seq = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t ctx = checked_ctx(a, seq), t0 = ctx - n;
  if (t0 < 0 || i >= n) return;
  const int64_t t = t0 + i;
  float v[V];
  load_lane<T, V>(reinterpret_cast<const T*>(a.x_new) + ((int64_t)seq * n + i) * C, lane, v);
  if (a.m > 0 && t >= ctx - a.L)
    store_lane<T, V>(reinterpret_cast<T*>(a.ring) + ((int64_t)seq * a.L + t % a.L) * C, lane, v);
  if (a.kv_pages) {
    T* dst = page_row<T>(a.kv_pages, a.kv_bt, a.kv_max_pages, a.page_size, C, seq, t);
    if (dst) {
      rotate_lane<V>(v, lane, C, a.rf, a.pos0 + t);
      store_lane<T, V>(dst, lane, v);
    }
  }
}

template <typename T, int V>
cudaError_t chunk_t(const AppendPart& a, int nseq, int n, cudaStream_t st) {
  if (a.m > 0) {
    const int64_t entries = (int64_t)n / a.m + 1;  // closing entries per sequence, at most
    if (a.L >= 64)
      chunk_pool_kernel<T, V, 8><<<dim3((unsigned)entries, nseq), 256, 0, st>>>(a, n);
    else
      chunk_pool_kernel<T, V, 1><<<dim3((unsigned)((entries + 7) / 8), nseq), 256, 0, st>>>(a, n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  chunk_rows_kernel<T, V><<<dim3((unsigned)((n + 7) / 8), nseq), 256, 0, st>>>(a, n);
  return cudaGetLastError();
}

template <typename T>
cudaError_t chunk_dispatch(const AppendPart& a, int C, int nseq, int n, cudaStream_t st) {
  switch (C) {
    case 32: return chunk_t<T, 1>(a, nseq, n, st);
    case 64: return chunk_t<T, 2>(a, nseq, n, st);
    case 128: return chunk_t<T, 4>(a, nseq, n, st);
    case 256: return chunk_t<T, 8>(a, nseq, n, st);
    case 512: return chunk_t<T, 16>(a, nseq, n, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int V>
cudaError_t append_t(const AppendPart& a, int nseq, cudaStream_t st) {
  if (a.m > 0 && a.L >= 64)
    append_kernel<T, V, 8><<<nseq, 256, 0, st>>>(a);
  else
    append_kernel<T, V, 1><<<nseq, 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t append_dispatch(const AppendPart& a, int C, int nseq, cudaStream_t st) {
  switch (C) {
    case 32: return append_t<T, 1>(a, nseq, st);
    case 64: return append_t<T, 2>(a, nseq, st);
    case 128: return append_t<T, 4>(a, nseq, st);
    case 256: return append_t<T, 8>(a, nseq, st);
    case 512: return append_t<T, 16>(a, nseq, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

static AppendPart make_part(const DecodeAppendArgs& a, bool index_part) {
  AppendPart p{};
  p.ctx_lens = a.ctx_lens;
  p.max_ctx = a.max_ctx;
  p.m = a.m;
  p.L = a.L;
  p.page_size = a.page_size;
  p.pos0 = a.pos0;
  p.rf = a.rf;
  p.pool_bt = a.pool_block_table;
  p.pool_max_pages = a.pool_max_pages;
  if (!index_part) {
    p.x_new = a.kv_new;
    p.ring = a.cmp_state;
    p.gate = a.cmp_gate;
    p.bias = a.cmp_bias;
    p.kv_pages = a.kv_pages;
    p.kv_bt = a.kv_block_table;
    p.kv_max_pages = a.kv_max_pages;
    p.pool_pages = a.pool_pages;
    p.rotate = 1;
  } else {
    // the indexer part: its own ring, gate and pool, no window cache, no rotation
    p.x_new = a.k_idx_new;
    p.ring = a.idx_state;
    p.gate = a.idx_gate;
    p.bias = a.idx_bias;
    p.pool_pages = a.idx_pool_pages;
    p.rotate = 0;
  }
  return p;
}

cudaError_t launch_chunk_append(int dtype, const DecodeAppendArgs& a, int n, bool index_part,
                                cudaStream_t st) {
  if (a.nseq == 0 || n == 0) return cudaSuccess;
  const AppendPart p = make_part(a, index_part);
  const int C = index_part ? a.cI : a.D;
  return dtype == 0 ? chunk_dispatch<float>(p, C, a.nseq, n, st)
                    : chunk_dispatch<__nv_bfloat16>(p, C, a.nseq, n, st);
}

bool decode_append_pair_supported(const DecodeAppendArgs& a) {
  return a.D == 512 && a.cI == 128 && a.m > 0 && a.L < 64;
}

cudaError_t launch_decode_append_pair(int dtype, const DecodeAppendArgs& a, cudaStream_t st) {
  if (a.nseq == 0) return cudaSuccess;
  if (!decode_append_pair_supported(a)) return cudaErrorInvalidValue;
  const AppendPart p0 = make_part(a, false), p1 = make_part(a, true);
  if (dtype == 0)
    append_pair_kernel<float, 16, 4><<<a.nseq, 64, 0, st>>>(p0, p1);
  else
    append_pair_kernel<__nv_bfloat16, 16, 4><<<a.nseq, 64, 0, st>>>(p0, p1);
  return cudaGetLastError();
}

cudaError_t launch_decode_append(int dtype, const DecodeAppendArgs& a, bool index_part,
                                 cudaStream_t st) {
  if (a.nseq == 0) return cudaSuccess;
  const AppendPart p = make_part(a, index_part);
  const int C = index_part ? a.cI : a.D;
  return dtype == 0 ? append_dispatch<float>(p, C, a.nseq, st)
                    : append_dispatch<__nv_bfloat16>(p, C, a.nseq, st);
}

}  // namespace sac
