// KV compressor ("Hybrid attention": CSA pool with overlapping windows, HCA pool with
// non-overlapping windows; "Cache layers": compressor buffer / pool / count / overlap) and the
// RoPE rotation of kv rows for the sliding-window branch.
//
// Entry w of a sequence pools the window [(w+1)m - L, (w+1)m) clipped at 0 with softmax weights
// over g_j = <x_j, u> + bias[j - (w+1)m + L]; the result is optionally rotated at pos0 + w*m.
// The pass over the window is a single streaming pass with an online softmax. HBM bound: each
// token row is read once per window that holds it (twice for CSA, from L2 the second time).
#include "sac_kernels.h"

namespace sac {
namespace {

// Lane owns V contiguous channels [lane*V, lane*V + V) of a C = 32*V row.
template <typename T, int V>
__device__ __forceinline__ void load_lane(const T* row, int lane, float (&v)[V]) {
  const T* p = row + lane * V;
  if constexpr (V * sizeof(T) % 16 == 0) {
#pragma unroll
    for (int i = 0; i < V * (int)sizeof(T) / 16; ++i) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + i);
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int k = 0; k < 16 / (int)sizeof(T); ++k) v[i * (16 / sizeof(T)) + k] = to_f<T>(e[k]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) v[i] = to_f<T>(p[i]);
  }
}

template <typename T, int V>
__device__ __forceinline__ void store_lane(T* row, int lane, const float (&v)[V]) {
  T* p = row + lane * V;
  if constexpr (V * sizeof(T) % 16 == 0) {
#pragma unroll
    for (int i = 0; i < V * (int)sizeof(T) / 16; ++i) {
      uint4 u;
      T* e = reinterpret_cast<T*>(&u);
#pragma unroll
      for (int k = 0; k < 16 / (int)sizeof(T); ++k) e[k] = from_f<T>(v[i * (16 / sizeof(T)) + k]);
      reinterpret_cast<uint4*>(p)[i] = u;
    }
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) p[i] = from_f<T>(v[i]);
  }
}

// Rotate the lane's channels that fall in the trailing R (pairs never straddle lanes: V even).
template <int V>
__device__ __forceinline__ void rotate_lane(float (&v)[V], int lane, int C, const RopeFreqs& rf,
                                            int64_t pos) {
  const int R = rf.R;
#pragma unroll
  for (int i = 0; i + 1 < V; i += 2) {
    int c = lane * V + i;
    if (c >= C - R) {
      float cs, sn;
      rope_cos_sin(rf, (c - (C - R)) >> 1, pos, cs, sn);
      float a = v[i], b = v[i + 1];
      v[i] = a * cs - b * sn;
      v[i + 1] = a * sn + b * cs;
    }
  }
}

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
  __shared__ float s_acc[WPE > 1 ? 8 : 1][WPE > 1 ? C : 1];
  __shared__ float s_mz[8][2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t N = S / m;
  const int64_t e = (int64_t)blockIdx.x * EPB + warp / WPE;
  const int sub = warp % WPE;
  const bool active = e < (int64_t)B * N;
  const int b = active ? (int)(e / N) : 0;
  const int64_t w = active ? e % N : 0;
  const int64_t hi = (w + 1) * m;
  const int64_t lo = hi - L < 0 ? 0 : hi - L;

  float u[V], acc[V];
  load_lane<T, V>(gate, lane, u);
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  float M = -INFINITY, Z = 0.f;
  if (active) {
    for (int64_t j = lo + sub; j < hi; j += WPE) {
      float xv[V];
      load_lane<T, V>(x + ((int64_t)b * S + j) * C, lane, xv);
      float d = 0.f;
#pragma unroll
      for (int i = 0; i < V; ++i) d = fmaf(xv[i], u[i], d);
      float g = warp_sum(d) + __ldg(bias + (j - hi + L));
      if (g == -INFINITY) continue;
      if (g > M) {
        float sc = __expf(M - g);  // 0 when M = -inf
        Z *= sc;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] *= sc;
        M = g;
      }
      float p = __expf(g - M);
      Z += p;
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = fmaf(p, xv[i], acc[i]);
    }
  }
  if constexpr (WPE > 1) {
#pragma unroll
    for (int i = 0; i < V; ++i) s_acc[warp][lane * V + i] = acc[i];
    if (lane == 0) { s_mz[warp][0] = M; s_mz[warp][1] = Z; }
    __syncthreads();
    if (sub != 0) return;
    float Mt = -INFINITY;
    for (int s = 0; s < WPE; ++s) Mt = fmaxf(Mt, s_mz[warp + s][0]);
    float Zt = 0.f;
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    for (int s = 0; s < WPE; ++s) {
      float Ms = s_mz[warp + s][0];
      if (Ms == -INFINITY) continue;
      float sc = __expf(Ms - Mt);
      Zt = fmaf(s_mz[warp + s][1], sc, Zt);
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = fmaf(s_acc[warp + s][lane * V + i], sc, acc[i]);
    }
    Z = Zt;
  }
  if (!active) return;
  float inv = 1.f / Z;
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] *= inv;
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
