// Grouped low-rank output projection ("DeepSeek-V4" page, "Grouped Output Projection" bullet; config
// o_groups, o_lora_rank, hidden_size): the attention output o [T, H*D] is cut into G groups of H/G
// heads; group g's (H/G)*D features go through its own o_a_proj matrix to `rank` features, the
// G*rank results are concatenated and o_b_proj maps them to `hidden`.
//
// Both steps are row-major products C[b] = A[b] * W[b]^T (bf16 in, fp32 accumulate, bf16 out) with
// both operands K-major, run by one hand-written tcgen05 GEMM kernel:
//   o_a_proj: batch g, A = o[:, g*Kg : (g+1)*Kg] (read in place, row stride H*D), W = w_a[g],
//             C = mid[:, g*rank : (g+1)*rank];
//   o_b_proj: one batch, A = mid, W = w_b, C = out.
//
// Each persistent CTA computes 256 x 256 output tiles: two M = 128 accumulators (rows 0-127 and
// 128-255 of the tile) share every 256-row W tile, so a K-step of 64 moves 64 KB from L2 for
// 8.4 MFLOP (32 B per cycle per SM at the bf16 rate) instead of the 48 KB per 4.2 MFLOP of a single
// 128 x 256 tile. The two accumulators take all 512 TMEM columns, so the epilogue of a tile drains
// them before the next tile's first MMA; the TMA producer runs ahead meanwhile (3 stages of 64 KB).
// Warps: 0 = TMA producer, 1 and 6 = MMA issuers (warp 1 owns TMEM), 2-5 = epilogue (one TMEM
// lane quarter each: thread = tile row, 256 fp32 columns per accumulator -> bf16 -> global). Each
// issuer feeds one accumulator, so consecutive MMAs of a thread chain on the same accumulator
// (switching accumulators between consecutive MMAs of one thread drains the MMA pipe).
// No cluster multicast: every CTA loads its own tiles.
#include <cuda_bf16.h>

#include "launch_util.h"
#include "sac_kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace sac {
namespace {

constexpr int kBM = 256, kBN = 256, kBK = 64;
constexpr int kStages = 3;
constexpr int kABytes = kBM * kBK * 2;           // 32 KB: 256 rows x 128 B
constexpr int kBBytes = kBN * kBK * 2;           // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;   // 64 KB
constexpr int kOffBar = kStages * kStageBytes;
enum Bar { kFull0, kEmpty0 = kFull0 + kStages, kAccFull = kEmpty0 + kStages, kAccEmpty,
           kNumBars };
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffTmemPtr + 16;
constexpr int kThreads = 224;
constexpr uint32_t kIdesc = tc::idesc_bf16(128, kBN, false, false);

struct GemmArgs {
  int64_t M;          // rows of A and C (tokens)
  int N, K;           // output columns and contraction length per batch
  int batch;
  int a_col_step;     // per batch: column offset of A's block (elements)
  int w_row_step;     // per batch: row offset of W's block
  int c_col_step;     // per batch: column offset of C's block
  int64_t ldc;        // C row stride (elements)
  __nv_bfloat16* c;
  int* status;
};

struct Tile {
  int b, m, n;
};

__device__ __forceinline__ Tile tile_at(const GemmArgs& a, int64_t i, int mt, int nt) {
  Tile t;
  t.n = (int)(i % nt);
  const int64_t r = i / nt;
  t.m = (int)(r % mt);
  t.b = (int)(r / mt);
  return t;
}

__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w,
                   GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = a.status;
  if ((tc::smem_u32(smem) & 1023u) != 0) {  // the 128-byte swizzle needs 1024-byte alignment
    if (threadIdx.x == 0 && status) atomicExch(status, tc::kStatusMisaligned);
    return;
  }
  const int mt = (int)((a.M + kBM - 1) / kBM), nt = (a.N + kBN - 1) / kBN;
  const int kt = (a.K + kBK - 1) / kBK;
  const int64_t tiles = (int64_t)mt * nt * a.batch;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bar[kFull0 + i], 1);
      tc::mbar_init(&bar[kEmpty0 + i], 2);  // both issuers
    }
    tc::mbar_init(&bar[kAccFull], 2);
    tc::mbar_init(&bar[kAccEmpty], 128);
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_ptr, 512);
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_a);
    tc::tma_prefetch_desc(&tm_w);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_ptr;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int64_t i = blockIdx.x; i < tiles && ok; i += gridDim.x) {
        const Tile t = tile_at(a, i, mt, nt);
        const int32_t ay = t.m * kBM, wy = t.b * a.w_row_step + t.n * kBN;
        for (int k = 0; k < kt && ok; ++k, ++g) {
          const uint32_t s = g % kStages;
          if (g >= kStages) ok = tc::mbar_wait(&bar[kEmpty0 + s], ((g - kStages) / kStages) & 1,
                                               status);
          if (!ok) break;
          uint8_t* st = smem + s * kStageBytes;
          tc::mbar_arrive_expect_tx(&bar[kFull0 + s], kStageBytes);
          tc::tma_load_2d(st, &tm_a, &bar[kFull0 + s], t.b * a.a_col_step + k * kBK, ay);
          tc::tma_load_2d(st + kABytes, &tm_w, &bar[kFull0 + s], k * kBK, wy);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 6) {
    // ------------------------------------------------------------------ MMA issuers
    // warp 1: rows 0-127 of the tile (accumulator at column 0); warp 6: rows 128-255 (column 256)
    const uint32_t half = warp == 6 ? 1u : 0u;
    if (lane == 0) {
      uint32_t g = 0, tc_count = 0;
      bool ok = true;
      for (int64_t i = blockIdx.x; i < tiles && ok; i += gridDim.x, ++tc_count) {
        if (tc_count > 0) ok = tc::mbar_wait(&bar[kAccEmpty], (tc_count - 1) & 1, status);
        if (!ok) break;
        tc::tc_fence_after();
        for (int k = 0; k < kt && ok; ++k, ++g) {
          const uint32_t s = g % kStages;
          ok = tc::mbar_wait(&bar[kFull0 + s], (g / kStages) & 1, status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t a_base = tc::smem_u32(smem + s * kStageBytes);
          const uint32_t w_base = a_base + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc::mma_bf16_ss(tmem + half * kBN,
                            tc::desc_sw128(a_base + half * (kABytes / 2) + kk * 32, 0, 1024),
                            tc::desc_sw128(w_base + kk * 32, 0, 1024), kIdesc,
                            (k > 0 || kk > 0) ? 1u : 0u);
          tc::mma_commit(&bar[kEmpty0 + s]);
        }
        tc::mma_commit(&bar[kAccFull]);
      }
    }
    __syncwarp();
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;                   // TMEM lane quarter this warp may read
    const int r = q * 32 + lane;              // row within each accumulator
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    uint32_t tc_count = 0;
    bool ok = true;
    for (int64_t i = blockIdx.x; i < tiles && ok; i += gridDim.x, ++tc_count) {
      const Tile t = tile_at(a, i, mt, nt);
      ok = __all_sync(~0u, tc::mbar_wait(&bar[kAccFull], tc_count & 1, status));
      if (!ok) break;
      tc::tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int64_t row = (int64_t)t.m * kBM + h * 128 + r;
        const int col0 = t.n * kBN;
        __nv_bfloat16* crow = a.c + row * a.ldc + (int64_t)t.b * a.c_col_step + col0;
#pragma unroll 1
        for (int c = 0; c < kBN; c += 32) {
          uint32_t v0[16], v1[16];
          tc::tmem_ld16(t_lane + h * kBN + c, v0);
          tc::tmem_ld16(t_lane + h * kBN + c + 16, v1);
          tc::tmem_wait_ld();
          if (h == 1 && c + 32 == kBN) {  // every column of both accumulators is read
            tc::tc_fence_before();
            tc::mbar_arrive(&bar[kAccEmpty]);
          }
          if (row >= a.M) continue;
          uint32_t p[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = pack_bf16(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1]));
            p[8 + e] = pack_bf16(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1]));
          }
          if (col0 + c + 32 <= a.N) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              reinterpret_cast<uint4*>(crow + c)[e] =
                  make_uint4(p[4 * e], p[4 * e + 1], p[4 * e + 2], p[4 * e + 3]);
          } else {
            for (int e = 0; e < 16; ++e)
              if (col0 + c + 2 * e < a.N)  // N is a multiple of 8: pairs never straddle it
                reinterpret_cast<uint32_t*>(crow + c)[e] = p[e];
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// C[b] = A[b] W[b]^T over `batch` column / row blocks (see GemmArgs), A [M, lda] and W [rows, K]
// row-major bf16 with K contiguous.
cudaError_t gemm(const void* A, int64_t lda, const void* W, int64_t w_rows, GemmArgs g,
                 cudaStream_t st) {
  if (g.M == 0 || g.N == 0 || g.batch == 0) return cudaSuccess;
  CUtensorMap ta, tw;
  const int64_t a_cols = (int64_t)g.a_col_step * (g.batch - 1) + g.K;
  cudaError_t e = make_tmap_bf16_2d(&ta, A, (uint64_t)g.M, (uint64_t)a_cols, (uint64_t)lda * 2,
                                    kBM, kBK);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16_2d(&tw, W, (uint64_t)w_rows, (uint64_t)g.K, (uint64_t)g.K * 2, kBN, kBK);
  if (e != cudaSuccess) return e;
  e = ensure_smem_limit((const void*)gemm_tc_kernel, kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = ((g.M + kBM - 1) / kBM) * ((g.N + kBN - 1) / kBN) * g.batch;
  const int grid = (int)(tiles < sms ? tiles : sms);
  gemm_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(ta, tw, g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_oproj(const OProjArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int kg = a.H / a.groups * a.D;       // features of one group
  const int64_t ld_o = (int64_t)a.H * a.D;   // row stride of o
  const int64_t ld_mid = (int64_t)a.groups * a.rank;
  // o_a_proj: mid[:, g*rank : (g+1)*rank] = o[:, g*kg : (g+1)*kg] * w_a[g]^T, all groups at once
  GemmArgs ga{a.T, a.rank, kg, a.groups, kg, a.rank, a.rank, ld_mid,
              static_cast<__nv_bfloat16*>(a.mid), a.status};
  cudaError_t e = gemm(a.o, ld_o, a.w_a, (int64_t)a.groups * a.rank, ga, st);
  if (e != cudaSuccess) return e;
  // o_b_proj: out = mid * w_b^T
  GemmArgs gb{a.T, a.hidden, a.groups * a.rank, 1, 0, 0, 0, (int64_t)a.hidden,
              static_cast<__nv_bfloat16*>(a.out), a.status};
  return gemm(a.mid, ld_mid, a.w_b, a.hidden, gb, st);
}

}  // namespace sac
