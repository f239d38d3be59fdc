// KV compressor ("Hybrid attention": CSA pool with overlapping windows, HCA pool with
// non-overlapping windows; "Cache layers": compressor buffer / pool / count / overlap) and the
// RoPE rotation of kv rows for the sliding-window branch.
//
// Entry w of a sequence pools the window [(w+1)m - L, (w+1)m) clipped at 0 with softmax weights
// over g_j = <x_j, u> + bias[j - (w+1)m + L]; the result is optionally rotated at pos0 + w*m.
// The pass over the window is a single streaming pass with an online softmax. HBM bound: each
// token row is read once per window that holds it (twice for CSA, from L2 the second time).
#include "pool_window.cuh"
#include "sac_kernels.h"

namespace sac {
namespace {

// WPE warps cooperate on one entry (rows strided by WPE), merging their online-softmax partials.
template <typename T, int V, int WPE>
__global__ void __launch_bounds__(256) compress_kernel(const T* __restrict__ x,
                                                       const T* __restrict__ gate,
                                                       const float* __restrict__ bias, int B,
                                                       int S, int m, int L, int rotate,
                                                       RopeFreqs rf, int64_t pos0,
                                                       T* __restrict__ out) {
  constexpr int C = 32 * V;
  constexpr int EPB = 8 / WPE;  // entries per block
  __shared__ PoolShared<V, WPE> sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t N = S / m;
  const int64_t e = (int64_t)blockIdx.x * EPB + warp / WPE;
  const bool active = e < (int64_t)B * N;
  const int b = active ? (int)(e / N) : 0;
  const int64_t w = active ? e % N : 0;
  const int64_t hi = (w + 1) * m;
  const int64_t lo = hi - L < 0 ? 0 : hi - L;
  float u[V], acc[V];
  load_lane<T, V>(gate, lane, u);
  const T* xb = x + (int64_t)b * S * C;
  pool_window<T, V, WPE>([&](int64_t j) { return xb + j * C; }, u, bias, lo, hi, L, active, warp,
                         lane, sh, acc);
  if (!active || warp % WPE != 0) return;
  if (rotate) rotate_lane<V>(acc, lane, C, rf, pos0 + w * m);
  store_lane<T, V>(out + e * C, lane, acc);
}

template <typename T, int V>
__global__ void __launch_bounds__(256) rotate_rows_kernel(const T* __restrict__ x, int64_t rows,
                                                          int S, RopeFreqs rf, int64_t pos0,
                                                          T* __restrict__ out, int rows_per_pos) {
  constexpr int C = 32 * V;
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  float v[V];
  load_lane<T, V>(x + r * C, lane, v);
  rotate_lane<V>(v, lane, C, rf, pos0 + (r / rows_per_pos) % S);
  store_lane<T, V>(out + r * C, lane, v);
}

template <typename T, int V>
cudaError_t compress_t(const void* x, const void* gate, const float* bias, int B, int S, int m,
                       int L, bool rotate, const RopeFreqs& rf, int64_t pos0, void* out,
                       cudaStream_t st) {
  int64_t entries = (int64_t)B * (S / m);
  if (entries == 0) return cudaSuccess;
  if (L >= 64) {
    int64_t blocks = entries;
    compress_kernel<T, V, 8><<<(unsigned)blocks, 256, 0, st>>>(
        (const T*)x, (const T*)gate, bias, B, S, m, L, rotate, rf, pos0, (T*)out);
  } else {
    int64_t blocks = (entries + 7) / 8;
    compress_kernel<T, V, 1><<<(unsigned)blocks, 256, 0, st>>>(
        (const T*)x, (const T*)gate, bias, B, S, m, L, rotate, rf, pos0, (T*)out);
  }
  return cudaGetLastError();
}

template <typename T, int V>
cudaError_t rotate_t(const void* x, int64_t rows, int S, const RopeFreqs& rf, int64_t pos0,
                     void* out, cudaStream_t st, int rows_per_pos) {
  if (rows == 0) return cudaSuccess;
  rotate_rows_kernel<T, V><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>((const T*)x, rows, S, rf,
                                                                        pos0, (T*)out,
                                                                        rows_per_pos);
  return cudaGetLastError();
}

}  // namespace

#define SAC_DISPATCH_C(C, FN, ...)                                              \
  switch (C) {                                                                  \
    case 32: return FN<T, 1>(__VA_ARGS__);                                      \
    case 64: return FN<T, 2>(__VA_ARGS__);                                      \
    case 128: return FN<T, 4>(__VA_ARGS__);                                     \
    case 256: return FN<T, 8>(__VA_ARGS__);                                     \
    case 512: return FN<T, 16>(__VA_ARGS__);                                    \
    default: return cudaErrorInvalidValue;                                      \
  }

template <typename T>
static cudaError_t compress_dispatch(const void* x, const void* gate, const float* bias, int B,
                                     int S, int C, int m, int L, bool rotate,
                                     const RopeFreqs& rf, int64_t pos0, void* out,
                                     cudaStream_t st) {
  SAC_DISPATCH_C(C, compress_t, x, gate, bias, B, S, m, L, rotate, rf, pos0, out, st)
}

template <typename T>
static cudaError_t rotate_dispatch(const void* x, int64_t rows, int S, int C, const RopeFreqs& rf,
                                   int64_t pos0, void* out, cudaStream_t st, int rows_per_pos) {
  SAC_DISPATCH_C(C, rotate_t, x, rows, S, rf, pos0, out, st, rows_per_pos)
}

cudaError_t launch_compress(int dtype, const void* x, const void* gate, const float* bias, int B,
                            int S, int C, int m, int L, bool rotate, const RopeFreqs& rf,
                            int64_t pos0, void* out, cudaStream_t st) {
  if (dtype == 0)
    return compress_dispatch<float>(x, gate, bias, B, S, C, m, L, rotate, rf, pos0, out, st);
  return compress_dispatch<__nv_bfloat16>(x, gate, bias, B, S, C, m, L, rotate, rf, pos0, out,
                                          st);
}

cudaError_t launch_rotate_rows(int dtype, const void* x, int64_t rows, int S, int C,
                               const RopeFreqs& rf, int64_t pos0, void* out, cudaStream_t st,
                               int rows_per_pos) {
  if (dtype == 0) return rotate_dispatch<float>(x, rows, S, C, rf, pos0, out, st, rows_per_pos);
  return rotate_dispatch<__nv_bfloat16>(x, rows, S, C, rf, pos0, out, st, rows_per_pos);
}

}  // namespace sac
