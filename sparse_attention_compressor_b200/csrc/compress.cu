// KV compressor ("Hybrid attention": CSA pool with overlapping windows, HCA pool with
// non-overlapping windows; "Cache layers": compressor buffer / pool / count / overlap) and the
// RoPE rotation of kv rows for the sliding-window branch.
//
// Entry w of a sequence pools the window [(w+1)m - L, (w+1)m) clipped at 0 with softmax weights
// over g_j = <x_j, u> + bias[j - (w+1)m + L]; the result is optionally rotated at pos0 + w*m.
// The pass over the window is a single streaming pass with an online softmax.
//
// HBM bound. Short windows (the CSA main and indexer pools) stream through shared memory: a
// persistent CTA per SM takes chunks of E consecutive entries, whose rows [(w0+1)m - L, w1*m)
// are one contiguous range of the input, and a producer warp brings each chunk in with one bulk
// copy into a 3-stage ring while 16 consumer warps pool the chunks already there. Every input row
// is read from HBM once (plus the L - m overlap rows at each chunk edge) with ~200 KB in flight
// per SM. Long windows (HCA, L = m = 128) keep the direct kernel: 8 warps per entry.
#include "launch_util.h"
#include "pool_window.cuh"
#include "sac_kernels.h"
#include "tc_ptx.cuh"

namespace sac {
namespace {

constexpr int kBulkConsumers = 16;                    // pooling warps
constexpr int kBulkThreads = 32 * (kBulkConsumers + 1);  // + the producer warp
constexpr int kBulkStages = 3;
constexpr int kBulkStageBytes = 68 * 1024;            // 16 CSA entries of 1 KB rows + overlap
constexpr int kBulkPiece = 2048;                       // bytes per bulk copy (multiple of 16)
constexpr int kBulkMaxRows = kBulkStageBytes / 64;     // rows of a stage at the narrowest row

struct BulkArgs {
  const void* x;
  const void* gate;
  const float* bias;
  int B, S, m, L, E;  // E entries per chunk
  int rotate;
  RopeFreqs rf;
  int64_t pos0;
  void* out;
  int* status;
};

// Lane l holds NP pieces of P bytes of a row: piece i at byte (i*32 + l) * P, so a warp reads or
// writes 32*P contiguous bytes per piece (conflict-free in shared memory, coalesced in HBM).
template <typename T, int V>
struct LaneMap {
  static constexpr int kRowBytes = 32 * V * (int)sizeof(T);
  static constexpr int P = V * (int)sizeof(T) < 16 ? V * (int)sizeof(T) : 16;
  static constexpr int NP = V * (int)sizeof(T) / P;
  static constexpr int EPP = P / (int)sizeof(T);  // elements per piece
  static constexpr int NW = (V * (int)sizeof(T) + 3) / 4;
  __device__ static int channel(int lane, int i, int k) { return (i * 32 + lane) * EPP + k; }
};

// The lane's V elements as raw words (NW = 4-byte words; bf16 pairs share a word), converted to
// fp32 only where used, so that a batch of rows costs half the registers in bf16.
template <typename T, int V>
__device__ __forceinline__ void load_row_raw(const uint8_t* row, int lane,
                                             uint32_t (&r)[LaneMap<T, V>::NW]) {
  using M = LaneMap<T, V>;
#pragma unroll
  for (int i = 0; i < M::NP; ++i) {
    const uint8_t* p = row + (i * 32 + lane) * M::P;
    if constexpr (M::P == 16) {
      const uint4 u = *reinterpret_cast<const uint4*>(p);
      r[4 * i] = u.x; r[4 * i + 1] = u.y; r[4 * i + 2] = u.z; r[4 * i + 3] = u.w;
    } else if constexpr (M::P == 8) {
      const uint2 u = *reinterpret_cast<const uint2*>(p);
      r[2 * i] = u.x; r[2 * i + 1] = u.y;
    } else if constexpr (M::P == 4) {
      r[i] = *reinterpret_cast<const uint32_t*>(p);
    } else {
      r[i] = *reinterpret_cast<const uint16_t*>(p);
    }
  }
}

// Element k (0 <= k < V) of a raw row.
template <typename T, int V>
__device__ __forceinline__ float raw_elem(const uint32_t (&r)[LaneMap<T, V>::NW], int k) {
  if constexpr (sizeof(T) == 4) {
    return __uint_as_float(r[k]);
  } else {
    const uint32_t w = r[k >> 1];
    return __uint_as_float((k & 1) ? (w & 0xFFFF0000u) : (w << 16));
  }
}

// Elements (2i, 2i+1) of a raw row (V odd: the last pair's second element is 0).
template <typename T, int V>
__device__ __forceinline__ float2 raw_pair(const uint32_t (&r)[LaneMap<T, V>::NW], int i) {
  if constexpr (sizeof(T) == 4 && V == 1) {
    return make_float2(__uint_as_float(r[0]), 0.f);
  } else if constexpr (sizeof(T) == 4) {
    return make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
  } else {
    const uint32_t w = r[i];
    return make_float2(__uint_as_float(w << 16),
                       2 * i + 1 < V ? __uint_as_float(w & 0xFFFF0000u) : 0.f);
  }
}

// Named barrier 1 over the consumer warps, AND-reducing a per-thread flag.
__device__ __forceinline__ bool consumers_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(kBulkConsumers * 32)
      : "memory");
  return r != 0;
}

template <typename T, int V>
__device__ __forceinline__ void load_row_mapped(const uint8_t* row, int lane, float (&v)[V]) {
  uint32_t r[LaneMap<T, V>::NW];
  load_row_raw<T, V>(row, lane, r);
#pragma unroll
  for (int k = 0; k < V; ++k) v[k] = raw_elem<T, V>(r, k);
}

template <typename T, int V>
__device__ __forceinline__ void store_row_mapped(T* row, int lane, const float (&v)[V]) {
  using M = LaneMap<T, V>;
#pragma unroll
  for (int i = 0; i < M::NP; ++i) {
    uint8_t* p = reinterpret_cast<uint8_t*>(row) + (i * 32 + lane) * M::P;
    if constexpr (M::P == 16) {
      uint4 u;
      T* e = reinterpret_cast<T*>(&u);
#pragma unroll
      for (int k = 0; k < M::EPP; ++k) e[k] = from_f<T>(v[i * M::EPP + k]);
      *reinterpret_cast<uint4*>(p) = u;
    } else if constexpr (M::P == 8) {
      uint2 u;
      T* e = reinterpret_cast<T*>(&u);
#pragma unroll
      for (int k = 0; k < M::EPP; ++k) e[k] = from_f<T>(v[i * M::EPP + k]);
      *reinterpret_cast<uint2*>(p) = u;
    } else {
      T* e = reinterpret_cast<T*>(p);
#pragma unroll
      for (int k = 0; k < M::EPP; ++k) e[k] = from_f<T>(v[i * M::EPP + k]);
    }
  }
}

template <typename T, int V>
__global__ void __launch_bounds__(kBulkThreads, 1) compress_bulk_kernel(BulkArgs a) {
  using M = LaneMap<T, V>;
  constexpr int C = 32 * V;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kBulkStages], empty[kBulkStages];
  __shared__ float g_s[2][kBulkMaxRows];  // gate dots of a chunk's rows, double-buffered
  __shared__ float bias_s[64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t N = a.S / a.m;
  const int64_t cps = (N + a.E - 1) / a.E;  // chunks per sequence
  const int64_t chunks = (int64_t)a.B * cps;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBulkStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kBulkConsumers);
    }
    tc::fence_barrier_init();
  }
  __syncthreads();
  // chunk c: sequence c / cps, entries [w0, w1), input rows [lo, hi)
  auto chunk_rows = [&](int64_t c, int& b, int64_t& w0, int64_t& w1, int64_t& lo, int64_t& hi) {
    b = (int)(c / cps);
    w0 = (c % cps) * a.E;
    w1 = w0 + a.E < N ? w0 + a.E : N;
    lo = (w0 + 1) * a.m - a.L;
    if (lo < 0) lo = 0;
    hi = w1 * a.m;
  };

  if (warp == kBulkConsumers) {
    // ---- producer warp: each chunk goes into the next free stage as pieces of kBulkPiece bytes,
    // issued by all 32 lanes so that many copies are in flight at once
    int64_t issued = 0;
    bool ok = true;
    for (int64_t c = blockIdx.x; c < chunks; c += gridDim.x, ++issued) {
      const int s = (int)(issued % kBulkStages);
      if (issued >= kBulkStages &&
          !__all_sync(~0u, tc::mbar_wait(&empty[s], (uint32_t)((issued / kBulkStages - 1) & 1),
                                         a.status))) {
        ok = false;
        break;
      }
      int b;
      int64_t w0, w1, lo, hi;
      chunk_rows(c, b, w0, w1, lo, hi);
      const uint32_t bytes = (uint32_t)((hi - lo) * M::kRowBytes);
      if (lane == 0) tc::mbar_arrive_expect_tx(&full[s], bytes);
      __syncwarp();
      const uint8_t* src =
          reinterpret_cast<const uint8_t*>(a.x) + ((int64_t)b * a.S + lo) * M::kRowBytes;
      uint8_t* dst = smem + (size_t)s * kBulkStageBytes;
      for (uint32_t off = (uint32_t)lane * kBulkPiece; off < bytes; off += 32u * kBulkPiece) {
        const uint32_t n = bytes - off < (uint32_t)kBulkPiece ? bytes - off : (uint32_t)kBulkPiece;
        tc::bulk_load(dst + off, src + off, n, &full[s]);
      }
    }
    if (!ok && lane == 0) {
      // a consumer gave up: wait (bounded) for the copies still landing in this CTA's stages
      for (int64_t i = issued - kBulkStages < 0 ? 0 : issued - kBulkStages; i < issued; ++i)
        tc::mbar_wait(&full[i % kBulkStages], (uint32_t)((i / kBulkStages) & 1), a.status);
    }
    return;
  }

  // ---- consumers, two passes per chunk. Pass 1: the gate dot <x_j, u> of every row of the chunk,
  // once per row although CSA windows overlap (rows split over the warps, into g_s). Pass 2: warp
  // k pools entries w0 + k, w0 + k + 16, ... with the softmax of (dot + bias) over its window.
  float2 u[(V + 1) / 2];
  {
    float uf[V];
    load_row_mapped<T, V>(reinterpret_cast<const uint8_t*>(a.gate), lane, uf);
#pragma unroll
    for (int i = 0; i < V / 2; ++i) u[i] = make_float2(uf[2 * i], uf[2 * i + 1]);
    if constexpr (V % 2) u[V / 2] = make_float2(uf[V - 1], 0.f);
  }
  for (int i = threadIdx.x; i < a.L; i += kBulkConsumers * 32) bias_s[i] = a.bias[i];
  int64_t it = 0;
  for (int64_t c = blockIdx.x; c < chunks; c += gridDim.x, ++it) {
    const int s = (int)(it % kBulkStages);
    int b;
    int64_t w0, w1, lo, hi;
    chunk_rows(c, b, w0, w1, lo, hi);
    const bool ok =
        __all_sync(~0u, tc::mbar_wait(&full[s], (uint32_t)((it / kBulkStages) & 1), a.status));
    const uint8_t* stage = smem + (size_t)s * kBulkStageBytes;
    float* gs = g_s[it & 1];
    const int nrows = (int)(hi - lo);
    if (ok) {
      for (int r = warp; r < nrows; r += 2 * kBulkConsumers) {
        const int r2 = r + kBulkConsumers < nrows ? r + kBulkConsumers : r;
        uint32_t x0[M::NW], x1[M::NW];
        load_row_raw<T, V>(stage + r * M::kRowBytes, lane, x0);
        load_row_raw<T, V>(stage + r2 * M::kRowBytes, lane, x1);
        float2 d0 = make_float2(0.f, 0.f), d1 = d0;
#pragma unroll
        for (int i = 0; i < (V + 1) / 2; ++i) {
          d0 = __ffma2_rn(raw_pair<T, V>(x0, i), u[i], d0);
          d1 = __ffma2_rn(raw_pair<T, V>(x1, i), u[i], d1);
        }
        float g0 = d0.x + d0.y, g1 = d1.x + d1.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          g0 += __shfl_xor_sync(~0u, g0, o);
          g1 += __shfl_xor_sync(~0u, g1, o);
        }
        if (lane == 0) {
          gs[r] = g0;
          gs[r2] = g1;
        }
      }
    }
    // every consumer has written its dots (and learns whether all of them got the chunk)
    if (!consumers_all(ok)) return;
    for (int64_t w = w0 + warp; w < w1; w += kBulkConsumers) {
      const int64_t whi = (w + 1) * a.m;
      const int64_t wlo = whi - a.L < 0 ? 0 : whi - a.L;
      const int j0 = (int)(wlo - lo), nwin = (int)(whi - wlo), boff = a.L - nwin;
      // softmax weights of the window's rows, lane t holding rows t and t + 32
      const float zA = lane < nwin ? gs[j0 + lane] + bias_s[boff + lane] : -INFINITY;
      const float zB = lane + 32 < nwin ? gs[j0 + lane + 32] + bias_s[boff + lane + 32] : -INFINITY;
      float mx = fmaxf(zA, zB);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(~0u, mx, o));
      const float pA = zA == -INFINITY ? 0.f : __expf(zA - mx);
      const float pB = zB == -INFINITY ? 0.f : __expf(zB - mx);
      float Z = pA + pB;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(~0u, Z, o);
      float2 acc2[(V + 1) / 2];
#pragma unroll
      for (int i = 0; i < (V + 1) / 2; ++i) acc2[i] = make_float2(0.f, 0.f);
      for (int t = 0; t < nwin; t += 2) {
        const int t2 = t + 1 < nwin ? t + 1 : t;
        const float p0 = __shfl_sync(~0u, t < 32 ? pA : pB, t & 31);
        const float p1 = t + 1 < nwin ? __shfl_sync(~0u, t2 < 32 ? pA : pB, t2 & 31) : 0.f;
        uint32_t x0[M::NW], x1[M::NW];
        load_row_raw<T, V>(stage + (j0 + t) * M::kRowBytes, lane, x0);
        load_row_raw<T, V>(stage + (j0 + t2) * M::kRowBytes, lane, x1);
        const float2 q0 = make_float2(p0, p0), q1 = make_float2(p1, p1);
#pragma unroll
        for (int i = 0; i < (V + 1) / 2; ++i) {
          acc2[i] = __ffma2_rn(raw_pair<T, V>(x0, i), q0, acc2[i]);
          acc2[i] = __ffma2_rn(raw_pair<T, V>(x1, i), q1, acc2[i]);
        }
      }
      const float inv = 1.f / Z;
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = ((i & 1) ? acc2[i / 2].y : acc2[i / 2].x) * inv;
      if (a.rotate) {
        const int R = a.rf.R;
        const int64_t pos = a.pos0 + w * a.m;
#pragma unroll
        for (int i = 0; i < M::NP; ++i)
#pragma unroll
          for (int k = 0; k < M::EPP; k += 2) {
            const int ch = M::channel(lane, i, k);
            if (ch >= C - R) {
              float cs, sn;
              rope_cos_sin(a.rf, (ch - (C - R)) >> 1, pos, cs, sn);
              const float x0 = acc[i * M::EPP + k], x1 = acc[i * M::EPP + k + 1];
              acc[i * M::EPP + k] = x0 * cs - x1 * sn;
              acc[i * M::EPP + k + 1] = x0 * sn + x1 * cs;
            }
          }
      }
      store_row_mapped<T, V>(reinterpret_cast<T*>(a.out) + ((int64_t)b * N + w) * C, lane, acc);
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[s]);
  }
}

// WPE warps cooperate on one entry (rows strided by WPE), merging their online-softmax partials.
template <typename T, int V, int WPE, int kRows>
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
  pool_window<T, V, WPE, kRows>([&](int64_t j) { return xb + j * C; }, u, bias, lo, hi, L, active,
                                warp, lane, sh, acc);
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

// Entries per chunk of the streaming kernel (0: the window does not suit it).
template <typename T, int V>
int bulk_entries(int m, int L) {
  constexpr int64_t row_bytes = LaneMap<T, V>::kRowBytes;
  if (L >= 64 || L < m) return 0;
  const int64_t rows = kBulkStageBytes / row_bytes;
  int64_t E = (rows - (L - m)) / m;
  if (E > 64) E = 64;
  return E >= 4 ? (int)E : 0;
}

template <typename T, int V>
cudaError_t compress_t(const void* x, const void* gate, const float* bias, int B, int S, int m,
                       int L, bool rotate, const RopeFreqs& rf, int64_t pos0, void* out,
                       int* status, cudaStream_t st) {
  int64_t entries = (int64_t)B * (S / m);
  if (entries == 0) return cudaSuccess;
  const int E = bulk_entries<T, V>(m, L);
  if (E > 0) {
    BulkArgs a{x, gate, bias, B, S, m, L, E, rotate ? 1 : 0, rf, pos0, out, status};
    const int smem = kBulkStages * kBulkStageBytes;
    cudaError_t e = ensure_smem_limit((const void*)compress_bulk_kernel<T, V>, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t chunks = (int64_t)B * ((S / m + E - 1) / E);
    const int grid = (int)(chunks < sms ? chunks : sms);
    compress_bulk_kernel<T, V><<<grid, kBulkThreads, smem, st>>>(a);
    return cudaGetLastError();
  }
  if (L >= 64) {
    // rows each warp keeps in flight (8 at 16 bf16 channels a lane)
    constexpr int kHcaRows = rows_in_flight<T, V>(64);
    int64_t blocks = entries;
    compress_kernel<T, V, 8, kHcaRows><<<(unsigned)blocks, 256, 0, st>>>(
        (const T*)x, (const T*)gate, bias, B, S, m, L, rotate, rf, pos0, (T*)out);
  } else {
    int64_t blocks = (entries + 7) / 8;
    compress_kernel<T, V, 1, 4><<<(unsigned)blocks, 256, 0, st>>>(
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
                                     const RopeFreqs& rf, int64_t pos0, void* out, int* status,
                                     cudaStream_t st) {
  SAC_DISPATCH_C(C, compress_t, x, gate, bias, B, S, m, L, rotate, rf, pos0, out, status, st)
}

template <typename T>
static cudaError_t rotate_dispatch(const void* x, int64_t rows, int S, int C, const RopeFreqs& rf,
                                   int64_t pos0, void* out, cudaStream_t st, int rows_per_pos) {
  SAC_DISPATCH_C(C, rotate_t, x, rows, S, rf, pos0, out, st, rows_per_pos)
}

cudaError_t launch_compress(int dtype, const void* x, const void* gate, const float* bias, int B,
                            int S, int C, int m, int L, bool rotate, const RopeFreqs& rf,
                            int64_t pos0, void* out, int* status, cudaStream_t st) {
  if (dtype == 0)
    return compress_dispatch<float>(x, gate, bias, B, S, C, m, L, rotate, rf, pos0, out, status,
                                    st);
  return compress_dispatch<__nv_bfloat16>(x, gate, bias, B, S, C, m, L, rotate, rf, pos0, out,
                                          status, st);
}

cudaError_t launch_rotate_rows(int dtype, const void* x, int64_t rows, int S, int C,
                               const RopeFreqs& rf, int64_t pos0, void* out, cudaStream_t st,
                               int rows_per_pos) {
  if (dtype == 0) return rotate_dispatch<float>(x, rows, S, C, rf, pos0, out, st, rows_per_pos);
  return rotate_dispatch<__nv_bfloat16>(x, rows, S, C, rf, pos0, out, st, rows_per_pos);
}

}  // namespace sac
