// The compressor's pooling of one window ("Hybrid attention": CSA / HCA compressors; "Cache
// layers": compressor buffer), shared by the prefill compressor (compress.cu) and the decode cache
// append (decode_append.cu): entry w pools rows j in [lo, hi) = [(w+1)m - L, (w+1)m) clipped at 0
// with softmax weights over g_j = <x_j, u> + bias[j - hi + L], in one streaming pass with an
// online softmax. Lane l of a warp owns channels [l*V, l*V + V) of a C = 32*V row; WPE warps
// split the rows of one entry and merge their partial (max, sum, accumulator) in shared memory.
#pragma once

#include "sac_common.cuh"

namespace sac {

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

// A lane's V elements of a row kept as loaded (packed), so a batch of rows in flight costs
// V * sizeof(T) / 4 registers a row instead of V.
template <typename T, int V>
struct RawLane {
  static constexpr int kBytes = V * (int)sizeof(T);
  static constexpr int kWords = (kBytes + 3) / 4;
  uint32_t w[kWords];
};
// Rows a lane can keep in flight within about `regs` registers (1 to 16).
template <typename T, int V>
__host__ __device__ constexpr int rows_in_flight(int regs) {
  const int n = regs / RawLane<T, V>::kWords;
  return n < 1 ? 1 : (n > 16 ? 16 : n);
}
template <typename T, int V>
__device__ __forceinline__ void load_lane_raw(const T* row, int lane, RawLane<T, V>& r) {
  constexpr int kBytes = RawLane<T, V>::kBytes;
  const T* src = row + lane * V;
  if constexpr (kBytes % 16 == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < kBytes / 16; ++i) {
      const uint4 u = __ldg(p + i);
      r.w[4 * i] = u.x;
      r.w[4 * i + 1] = u.y;
      r.w[4 * i + 2] = u.z;
      r.w[4 * i + 3] = u.w;
    }
  } else if constexpr (kBytes % 8 == 0) {
    const uint2* p = reinterpret_cast<const uint2*>(src);
#pragma unroll
    for (int i = 0; i < kBytes / 8; ++i) {
      const uint2 u = __ldg(p + i);
      r.w[2 * i] = u.x;
      r.w[2 * i + 1] = u.y;
    }
  } else {
    T* e = reinterpret_cast<T*>(r.w);
#pragma unroll
    for (int i = 0; i < V; ++i) e[i] = src[i];
  }
}
// Elements (2i, 2i+1) of a raw lane (V odd: the last pair's second element is 0).
template <typename T, int V>
__device__ __forceinline__ float2 lane_pair(const RawLane<T, V>& r, int i) {
  if constexpr (sizeof(T) == 4) {
    return make_float2(__uint_as_float(r.w[2 * i]),
                       2 * i + 1 < V ? __uint_as_float(r.w[2 * i + 1]) : 0.f);
  } else {
    const uint32_t w = r.w[i];
    return make_float2(__uint_as_float(w << 16),
                       2 * i + 1 < V ? __uint_as_float(w & 0xFFFF0000u) : 0.f);
  }
}

template <typename T, int V>
__device__ __forceinline__ void unpack_lane(const RawLane<T, V>& r, float (&v)[V]) {
  const T* e = reinterpret_cast<const T*>(r.w);
#pragma unroll
  for (int i = 0; i < V; ++i) v[i] = to_f<T>(e[i]);
}

// Shared memory of pool_window for a block of 8 warps.
template <int V, int WPE>
struct PoolShared {
  float acc[WPE > 1 ? 8 : 1][WPE > 1 ? 32 * V : 1];
  float mz[8][2];
};

// One entry per group of WPE warps (warp = the calling warp's index in the 8-warp block, sub =
// warp % WPE). row(j) gives row j's pointer. On return the group's first warp (sub == 0) holds
// the normalised pooled row in acc; with WPE > 1 every warp of the block must call (it contains
// __syncthreads). Rows whose gate logit is -inf get weight 0.
template <typename T, int V, int WPE, int kBatch = 4, typename RowFn>
__device__ __forceinline__ void pool_window(RowFn row, const float (&u)[V], const float* bias,
                                            int64_t lo, int64_t hi, int L, bool active, int warp,
                                            int lane, PoolShared<V, WPE>& sh, float (&acc)[V]) {
  const int sub = warp % WPE;
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  float M = -INFINITY, Z = 0.f;
  if (active) {
    // rows in batches of kBatch: all loads of a batch are issued before any is used, so a
    // window costs ceil(rows / kBatch) memory latencies instead of one per row; the batch's dot
    // reductions run interleaved and the running max is raised once per batch
    for (int64_t j0 = lo + sub; j0 < hi; j0 += kBatch * WPE) {
      RawLane<T, V> raw[kBatch];
      float bb[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int64_t j = j0 + (int64_t)k * WPE;
        if (j < hi) {
          load_lane_raw<T, V>(row(j), lane, raw[k]);
          bb[k] = __ldg(bias + (j - hi + L));
        } else {
#pragma unroll
          for (int i = 0; i < RawLane<T, V>::kWords; ++i) raw[k].w[i] = 0u;
          bb[k] = 0.f;
        }
      }
      float g[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        float2 d = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < (V + 1) / 2; ++i)
          d = __ffma2_rn(lane_pair<T, V>(raw[k], i),
                         make_float2(u[2 * i], 2 * i + 1 < V ? u[2 * i + 1] : 0.f), d);
        g[k] = d.x + d.y;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < kBatch; ++k) g[k] += __shfl_xor_sync(~0u, g[k], o);
      float bm = -INFINITY;
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        g[k] = j0 + (int64_t)k * WPE < hi ? g[k] + bb[k] : -INFINITY;
        bm = fmaxf(bm, g[k]);
      }
      if (bm > M) {
        const float sc = __expf(M - bm);  // 0 when M = -inf
        Z *= sc;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] *= sc;
        M = bm;
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        if (g[k] == -INFINITY) continue;  // rows past the window, and -inf logits
        const float p = __expf(g[k] - M);
        Z += p;
#pragma unroll
        for (int i = 0; i < (V + 1) / 2; ++i) {
          const float2 x = lane_pair<T, V>(raw[k], i);
          acc[2 * i] = fmaf(p, x.x, acc[2 * i]);
          if (2 * i + 1 < V) acc[2 * i + 1] = fmaf(p, x.y, acc[2 * i + 1]);
        }
      }
    }
  }
  if constexpr (WPE > 1) {
#pragma unroll
    for (int i = 0; i < V; ++i) sh.acc[warp][lane * V + i] = acc[i];
    if (lane == 0) {
      sh.mz[warp][0] = M;
      sh.mz[warp][1] = Z;
    }
    __syncthreads();
    if (sub == 0) {
      float Mt = -INFINITY;
      for (int s = 0; s < WPE; ++s) Mt = fmaxf(Mt, sh.mz[warp + s][0]);
      float Zt = 0.f;
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.f;
      for (int s = 0; s < WPE; ++s) {
        float Ms = sh.mz[warp + s][0];
        if (Ms == -INFINITY) continue;
        float sc = __expf(Ms - Mt);
        Zt = fmaf(sh.mz[warp + s][1], sc, Zt);
#pragma unroll
        for (int i = 0; i < V; ++i) acc[i] = fmaf(sh.acc[warp + s][lane * V + i], sc, acc[i]);
      }
      Z = Zt;
    }
    __syncthreads();  // sh is reused by a following call
  }
  if (sub == 0 && active) {
    const float inv = 1.f / Z;
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] *= inv;
  }
}

}  // namespace sac
