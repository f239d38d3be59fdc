// Tensor-core (tcgen05) Lightning Indexer score for bf16 layers with 64 indexer heads of dim 128
// ("Hybrid attention", CSA bullet, eq. 13-17): I[t,w] = sum_h w_idx[t,h] * max(0, <q_idx[t,h], KI_w>)
// for the visible entries w < (t+1)//m.
//
// One MMA computes, for 128 pool entries and a block of 4 consecutive queries, all 4 x 64
// head dot products at once: D[entry, (query, head)] = KI[128 x 128] * q_idx[256 x 128]^T
// (M = 128, N = 256, K = 128), fp32 in tensor memory. Two accumulators (2 x 256 columns) let one
// math warpgroup drain a block while the tensor core fills the other. In the drain each thread owns
// one entry (one TMEM lane) and reduces its 64 heads per query with packed fp32 FMAs, so the head
// reduction needs no cross-thread traffic and the score stores are coalesced along entries.
//
// Warps: 0 = TMA producer (q_idx block, head weights, KI blocks), 1 = MMA issuer and TMEM owner,
// 4..7 and 8..11 = the two math warpgroups. Query blocks are taken in descending order of work by
// persistent CTAs; only the causal part (entries < (t_last+1)//m) is streamed.
#include <cuda_bf16.h>

#include "launch_util.h"
#include "sac_kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace sac {
namespace {

constexpr int kNI = 64;                    // indexer heads
constexpr int kCI = 128;                   // indexer head dim
constexpr int kBQ = 4;                     // queries per block
constexpr int kBE = 128;                   // pool entries per block (MMA M)
constexpr int kN = kBQ * kNI;              // MMA N = 256
constexpr int kQStages = 2, kKvStages = 3;
constexpr int kQRegion = kN * 128;         // [256 rows x 128 B] = 32 KB
constexpr int kQBytes = 2 * kQRegion;      // 64 KB
constexpr int kKvRegion = kBE * 128;       // 16 KB
constexpr int kKvBytes = 2 * kKvRegion;    // 32 KB
constexpr int kWBytes = kBQ * kNI * 4;     // 1 KB of head weights per query block

constexpr int kOffQ = 0;
constexpr int kOffKv = kOffQ + kQStages * kQBytes;
constexpr int kOffW = kOffKv + kKvStages * kKvBytes;
constexpr int kOffBar = kOffW + kQStages * kWBytes;
enum Bar { kQFull0, kQFull1, kQEmpty0, kQEmpty1, kKvFull0, kKvFull1, kKvFull2, kKvEmpty0,
           kKvEmpty1, kKvEmpty2, kAccFull0, kAccFull1, kAccEmpty0, kAccEmpty1, kNumBars };
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffTmemPtr + 16;
constexpr uint32_t kIdesc = tc::idesc_bf16(kBE, kN, false, false);

struct Block {
  int64_t t0;   // first query position of the block
  int nq;       // queries in the block (<= 4)
  int nkb;      // entry blocks to stream
};

__device__ __forceinline__ Block block_at(const IndexerTcArgs& a, int64_t i) {
  // blocks in descending order of work: block index i counts from the end of the range
  const int64_t nqb = (a.t1 - a.t0 + kBQ - 1) / kBQ;
  const int64_t qb = nqb - 1 - i;
  Block b;
  b.t0 = a.t0 + qb * kBQ;
  const int64_t tl = b.t0 + kBQ < a.t1 ? b.t0 + kBQ - 1 : a.t1 - 1;
  b.nq = (int)(tl - b.t0 + 1);
  const int64_t nvis = (tl + 1) / a.m;
  b.nkb = (int)((nvis + kBE - 1) / kBE);
  return b;
}

__global__ void __launch_bounds__(384, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kv, IndexerTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = a.status;
  // The 128-byte swizzle needs 1024-byte aligned tiles; the dynamic window starts aligned.
  if ((tc::smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0 && status) atomicExch(status, tc::kStatusMisaligned);
    return;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kQStages; ++i) {
      tc::mbar_init(&bar[kQFull0 + i], 1);
      tc::mbar_init(&bar[kQEmpty0 + i], 1 + 256);
    }
    for (int i = 0; i < kKvStages; ++i) {
      tc::mbar_init(&bar[kKvFull0 + i], 1);
      tc::mbar_init(&bar[kKvEmpty0 + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bar[kAccFull0 + i], 1);
      tc::mbar_init(&bar[kAccEmpty0 + i], 128);
    }
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_ptr, 512);
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_q);
    tc::tma_prefetch_desc(&tm_kv);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const int64_t nqb = (a.t1 - a.t0 + kBQ - 1) / kBQ;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      uint32_t qc = 0, kc = 0;
      bool ok = true;
      for (int64_t i = blockIdx.x; i < nqb && ok; i += gridDim.x) {
        const Block blk = block_at(a, i);
        if (blk.nkb == 0) continue;
        const uint32_t qs = qc % kQStages;
        if (qc >= kQStages)
          ok = tc::mbar_wait(&bar[kQEmpty0 + qs], ((qc - kQStages) / kQStages) & 1, status);
        if (!ok) break;
        const int64_t row = (int64_t)a.seq * a.S + blk.t0;  // flat query row
        tc::mbar_arrive_expect_tx(&bar[kQFull0 + qs], kQBytes + blk.nq * kNI * 4);
        for (int c = 0; c < 2; ++c)
          tc::tma_load_2d(smem + kOffQ + qs * kQBytes + c * kQRegion, &tm_q, &bar[kQFull0 + qs],
                          64 * c, (int32_t)(row * kNI));
        tc::bulk_load(smem + kOffW + qs * kWBytes, a.w_idx + row * kNI, blk.nq * kNI * 4,
                      &bar[kQFull0 + qs]);
        ++qc;
        for (int kb = 0; kb < blk.nkb && ok; ++kb, ++kc) {
          const uint32_t ks = kc % kKvStages;
          if (kc >= kKvStages)
            ok = tc::mbar_wait(&bar[kKvEmpty0 + ks], ((kc - kKvStages) / kKvStages) & 1, status);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(&bar[kKvFull0 + ks], kKvBytes);
          for (int c = 0; c < 2; ++c)
            tc::tma_load_2d(smem + kOffKv + ks * kKvBytes + c * kKvRegion, &tm_kv,
                            &bar[kKvFull0 + ks], 64 * c,
                            (int32_t)((int64_t)a.seq * a.N + (int64_t)kb * kBE));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      uint32_t qc = 0, kc = 0, ac = 0;
      bool ok = true;
      for (int64_t i = blockIdx.x; i < nqb && ok; i += gridDim.x) {
        const Block blk = block_at(a, i);
        if (blk.nkb == 0) continue;
        const uint32_t qs = qc % kQStages;
        ok = tc::mbar_wait(&bar[kQFull0 + qs], (qc / kQStages) & 1, status);
        const uint32_t q_base = tc::smem_u32(smem + kOffQ + qs * kQBytes);
        for (int kb = 0; kb < blk.nkb && ok; ++kb, ++kc, ++ac) {
          const uint32_t ks = kc % kKvStages, acc = ac & 1;
          ok = tc::mbar_wait(&bar[kKvFull0 + ks], (kc / kKvStages) & 1, status);
          if (ok && ac >= 2) ok = tc::mbar_wait(&bar[kAccEmpty0 + acc], ((ac - 2) >> 1) & 1, status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t kv_base = tc::smem_u32(smem + kOffKv + ks * kKvBytes);
#pragma unroll
          for (int kk = 0; kk < kCI / 16; ++kk) {
            tc::mma_bf16_ss(tmem + acc * kN,
                            tc::desc_sw128(kv_base + (kk >> 2) * kKvRegion + (kk & 3) * 32, 0, 1024),
                            tc::desc_sw128(q_base + (kk >> 2) * kQRegion + (kk & 3) * 32, 0, 1024),
                            kIdesc, kk > 0);
          }
          tc::mma_commit(&bar[kKvEmpty0 + ks]);
          tc::mma_commit(&bar[kAccFull0 + acc]);
        }
        tc::mma_commit(&bar[kQEmpty0 + qs]);
        ++qc;
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ math warpgroups
    const int wg = (warp - 4) >> 2;          // which accumulator this warpgroup drains
    const int sp = warp & 3;                 // TMEM sub-partition
    const int e_in = sp * 32 + lane;         // entry within the block (TMEM lane)
    const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16) + wg * kN;
    uint32_t qc = 0, ac = 0;
    bool ok = true;
    for (int64_t i = blockIdx.x; i < nqb && ok; i += gridDim.x) {
      const Block blk = block_at(a, i);
      if (blk.nkb == 0) continue;
      const uint32_t qs = qc % kQStages;
      ok = __all_sync(~0u, tc::mbar_wait(&bar[kQFull0 + qs], (qc / kQStages) & 1, status));
      if (!ok) break;
      const float* wsm = reinterpret_cast<const float*>(smem + kOffW + qs * kWBytes);
      for (int kb = 0; kb < blk.nkb && ok; ++kb, ++ac) {
        if ((ac & 1) != (uint32_t)wg) continue;
        ok = __all_sync(~0u, tc::mbar_wait(&bar[kAccFull0 + wg], (ac >> 1) & 1, status));
        if (!ok) break;
        tc::tc_fence_after();
        const int64_t e = (int64_t)kb * kBE + e_in;
        float res[kBQ];
#pragma unroll
        for (int q = 0; q < kBQ; ++q) {
          float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < kNI; c += 16) {
            uint32_t v[16];
            tc::tmem_ld16(t_lane + q * kNI + c, v);
            tc::tmem_wait_ld();
            const float4* w4 = reinterpret_cast<const float4*>(wsm + q * kNI + c);
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
              const float4 wv = w4[u / 4];
              const float2 x0 = make_float2(fmaxf(__uint_as_float(v[u]), 0.f),
                                            fmaxf(__uint_as_float(v[u + 1]), 0.f));
              const float2 x1 = make_float2(fmaxf(__uint_as_float(v[u + 2]), 0.f),
                                            fmaxf(__uint_as_float(v[u + 3]), 0.f));
              s0 = __ffma2_rn(x0, make_float2(wv.x, wv.y), s0);
              s1 = __ffma2_rn(x1, make_float2(wv.z, wv.w), s1);
            }
          }
          res[q] = (s0.x + s0.y) + (s1.x + s1.y);
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[kAccEmpty0 + wg]);
#pragma unroll
        for (int q = 0; q < kBQ; ++q) {
          const int64_t t = blk.t0 + q;
          if (q < blk.nq && e < (t + 1) / a.m)
            a.scores[(t - a.t0) * (int64_t)a.n_stride + e] = res[q];
        }
      }
      tc::mbar_arrive(&bar[kQEmpty0 + qs]);
      ++qc;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool indexer_tc_supported(int dtype, int nI, int cI) {
  return dtype == 1 && nI == kNI && cI == kCI;
}

cudaError_t launch_indexer_tc(const IndexerTcArgs& a, const void* q_idx_seq_base,
                              int64_t q_rows_total, const void* kpool, int64_t kpool_rows,
                              cudaStream_t st) {
  if (a.t1 <= a.t0) return cudaSuccess;
  CUtensorMap tq, tk;
  cudaError_t e = make_tmap_bf16_2d(&tq, q_idx_seq_base, (uint64_t)q_rows_total * kNI, kCI,
                                    kCI * 2, kN, 64);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16_2d(&tk, kpool, (uint64_t)(kpool_rows > 0 ? kpool_rows : 1), kCI, kCI * 2,
                        kBE, 64);
  if (e != cudaSuccess) return e;
  e = ensure_smem_limit((const void*)indexer_tc_kernel, kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nqb = (a.t1 - a.t0 + kBQ - 1) / kBQ;
  const int grid = (int)(nqb < sms ? nqb : sms);
  indexer_tc_kernel<<<grid, 384, kSmemBytes, st>>>(tq, tk, a);
  return cudaGetLastError();
}

}  // namespace sac
