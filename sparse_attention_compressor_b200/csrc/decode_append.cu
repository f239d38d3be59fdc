// Decode-time cache append ("Cache layers": the K=V sliding window plus the compressor's buffer /
// pool / count / overlap state, and the indexer's own copy at index_head_dim; "Hybrid attention":
// entries appear once their source window has closed).
//
// One new token per sequence at t = ctx - 1. Its kv row is rotated at pos0 + t and written to the
// paged window cache. For compressed layers the un-rotated row also goes into a ring of the last
// L rows (slot t mod L): that ring is the compressor buffer, and for CSA (L = 2m) its older half is
// the overlap carried from the previous window. When t + 1 is a multiple of m, entry
// w = (t+1)/m - 1 closes: it pools the ring rows of its window [(w+1)m - L, (w+1)m) (clipped at
// 0) with the same softmax gate as the prefill compressor and is written, rotated at pos0 + w*m,
// to the pool pages. CSA does the same for the indexer key row (no rotation). The token count is
// ctx itself, so the state needs no counter of its own.
//
// One block per sequence; the work is a few kilobytes per token plus one window per m tokens.
#include "sac_kernels.h"

namespace sac {
namespace {

constexpr int kThreads = 256;  // thread i owns channel pair (2i, 2i+1); C <= 512

template <typename T>
__device__ __forceinline__ T* page_row(void* base, const int32_t* bt, int max_pages, int page_size,
                                       int C, int seq, int64_t j) {
  const int page = __ldg(bt + (int64_t)seq * max_pages + j / page_size);
  if (page < 0) return nullptr;
  return reinterpret_cast<T*>(base) + ((int64_t)page * page_size + j % page_size) * C;
}

__device__ __forceinline__ void rotate_pair(float& x, float& y, const RopeFreqs& rf, int C, int c,
                                            int64_t pos) {
  if (c < C - rf.R) return;
  float cs, sn;
  rope_cos_sin(rf, (c - (C - rf.R)) >> 1, pos, cs, sn);
  const float a = x, b = y;
  x = a * cs - b * sn;
  y = a * sn + b * cs;
}

// Pool entry w of one sequence from its ring (slot j mod L holds row j) into out (C channels).
template <typename T>
__device__ void pool_entry(const T* ring, int L, int m, int64_t w, int C, const T* gate,
                           const float* bias, bool rotate, const RopeFreqs& rf, int64_t pos,
                           float* g_s, float* red, T* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t hi = (w + 1) * m;
  const int64_t lo = hi - L < 0 ? 0 : hi - L;
  const int n = (int)(hi - lo);
  // gate logits, a warp per row
  for (int i = warp; i < n; i += kThreads / 32) {
    const int64_t j = lo + i;
    const T* x = ring + (j % L) * C;
    float d = 0.f;
    for (int c = lane; c < C; c += 32) d = fmaf(to_f<T>(x[c]), to_f<T>(gate[c]), d);
    d = warp_sum(d);
    if (lane == 0) g_s[i] = d + __ldg(bias + (j - hi + L));
  }
  __syncthreads();
  // softmax statistics over the window (one warp)
  if (warp == 0) {
    float mx = -INFINITY;
    for (int i = lane; i < n; i += 32) mx = fmaxf(mx, g_s[i]);
    mx = warp_max(mx);
    float z = 0.f;
    for (int i = lane; i < n; i += 32) z += g_s[i] == -INFINITY ? 0.f : __expf(g_s[i] - mx);
    z = warp_sum(z);
    if (lane == 0) {
      red[0] = mx;
      red[1] = z;
    }
  }
  __syncthreads();
  const float mx = red[0], inv_z = 1.f / red[1];
  const int c = 2 * threadIdx.x;
  if (c < C) {
    float a0 = 0.f, a1 = 0.f;
    for (int i = 0; i < n; ++i) {
      const float gi = g_s[i];
      if (gi == -INFINITY) continue;
      const float p = __expf(gi - mx);
      const T* x = ring + ((lo + i) % L) * C;
      a0 = fmaf(p, to_f<T>(x[c]), a0);
      a1 = fmaf(p, to_f<T>(x[c + 1]), a1);
    }
    a0 *= inv_z;
    a1 *= inv_z;
    if (rotate) rotate_pair(a0, a1, rf, C, c, pos);
    out[c] = from_f<T>(a0);
    out[c + 1] = from_f<T>(a1);
  }
  __syncthreads();  // g_s / red are reused by the next call
}

template <typename T>
__global__ void __launch_bounds__(kThreads) decode_append_kernel(DecodeAppendArgs a) {
  extern __shared__ float g_s[];  // [L] gate logits
  __shared__ float red[2];
  const int seq = blockIdx.x;
  const int64_t t = (int64_t)__ldg(a.ctx_lens + seq) - 1;
  if (t < 0) return;
  const int c = 2 * threadIdx.x;
  const int D = a.D, L = a.L;
  const bool compressed = a.m > 0;

  // kv row: rotated into the window cache, un-rotated into the ring
  if (c < D) {
    const T* x = reinterpret_cast<const T*>(a.kv_new) + (int64_t)seq * D;
    float x0 = to_f<T>(x[c]), x1 = to_f<T>(x[c + 1]);
    if (compressed) {
      T* ring = reinterpret_cast<T*>(a.cmp_state) + ((int64_t)seq * L + t % L) * D;
      ring[c] = x[c];
      ring[c + 1] = x[c + 1];
    }
    T* dst = page_row<T>(a.kv_pages, a.kv_block_table, a.kv_max_pages, a.page_size, D, seq, t);
    rotate_pair(x0, x1, a.rf, D, c, a.pos0 + t);
    if (dst) {
      dst[c] = from_f<T>(x0);
      dst[c + 1] = from_f<T>(x1);
    }
  }
  if (a.idx_state != nullptr && c < a.cI) {
    const T* x = reinterpret_cast<const T*>(a.k_idx_new) + (int64_t)seq * a.cI;
    T* ring = reinterpret_cast<T*>(a.idx_state) + ((int64_t)seq * L + t % L) * a.cI;
    ring[c] = x[c];
    ring[c + 1] = x[c + 1];
  }
  if (!compressed || (t + 1) % a.m != 0) return;
  __syncthreads();  // the ring rows written above are read by the whole block below

  const int64_t w = (t + 1) / a.m - 1;
  T* pool = page_row<T>(a.pool_pages, a.pool_block_table, a.pool_max_pages, a.page_size, D, seq, w);
  if (pool)
    pool_entry<T>(reinterpret_cast<const T*>(a.cmp_state) + (int64_t)seq * L * D, L, a.m, w, D,
                  reinterpret_cast<const T*>(a.cmp_gate), a.cmp_bias, true, a.rf,
                  a.pos0 + w * a.m, g_s, red, pool);
  if (a.idx_state != nullptr) {
    T* ipool = page_row<T>(a.idx_pool_pages, a.pool_block_table, a.pool_max_pages, a.page_size,
                           a.cI, seq, w);
    if (ipool)
      pool_entry<T>(reinterpret_cast<const T*>(a.idx_state) + (int64_t)seq * L * a.cI, L, a.m, w,
                    a.cI, reinterpret_cast<const T*>(a.idx_gate), a.idx_bias, false, a.rf, 0, g_s,
                    red, ipool);
  }
}

}  // namespace

cudaError_t launch_decode_append(int dtype, const DecodeAppendArgs& a, cudaStream_t st) {
  if (a.nseq == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * (size_t)(a.L > 0 ? a.L : 1);
  if (dtype == 0) {
    decode_append_kernel<float><<<a.nseq, kThreads, smem, st>>>(a);
  } else {
    decode_append_kernel<__nv_bfloat16><<<a.nseq, kThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sac
