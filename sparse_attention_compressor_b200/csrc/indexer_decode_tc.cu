// Tensor-core (tcgen05) Lightning Indexer score over a paged indexer pool ("Hybrid attention",
// CSA bullet, eq. 13-17; "Cache layers": paged indexer pool): for each query row at position t
// (a decode step's new token t = ctx - 1, or one of a prefill chunk's last positions),
// I[w] = sum_h w_idx[h] * max(0, <q_idx[h], KI_w>) over the visible entries w < (t + 1) // m,
// bf16 layers with 64 indexer heads of dim 128.
//
// The step reads every visible indexer-pool entry once (256 bytes each) and does 64 x 128 MACs per
// entry, so it is bound by HBM. One MMA per 128 entries puts all 64 head dot products of each
// entry into tensor memory: D[entry, head] = KI[128 x 128] * q_idx[64 x 128]^T (M = 128, N = 64,
// K = 128). In the drain each thread owns one entry (one TMEM lane), so the head reduction needs
// no cross-thread traffic and the score stores are coalesced.
//
// Pool pages may have any size, so entries are gathered with 16-byte cp.async copies: sixteen
// threads per 256-byte entry row (one fully used 512-byte span per warp instruction), three
// 32 KB stages in flight per CTA and two CTAs per SM. Each CTA takes one (query row, 1024-entry
// chunk) pair; chunks past the row's visible entries exit at once.
//
// Warps: 0..3 gather (q_idx once, then entry blocks), 4..7 drain, 8 issues the MMAs and owns TMEM.
#include <cuda_bf16.h>

#include "launch_util.h"
#include "sac_kernels.h"
#include "tc_ptx.cuh"

namespace sac {
namespace {

constexpr int kNI = 64;                   // indexer heads (MMA N)
constexpr int kCI = 128;                  // indexer head dim (MMA K)
constexpr int kBE = 128;                  // entries per block (MMA M)
constexpr int kChunkBlocks = 8;           // blocks per CTA (one query row)
constexpr int kChunkBlocksQ4 = 32;        // blocks per CTA (four rows: fewer, longer CTAs)
constexpr int kStages = 3;
constexpr int kGatherThreads = 128;
constexpr int kThreads = 288;
constexpr int kRegion = kBE * 128;        // one 64-dim half of a block: [128 rows x 128 B]
constexpr int kBlockBytes = 2 * kRegion;  // 32 KB
enum Bar { kFull0, kEmpty0 = kFull0 + kStages, kAccFull0 = kEmpty0 + kStages, kAccEmpty0 = kAccFull0 + 2,
           kNumBars = kAccEmpty0 + 2 };

// Layout for Q query rows per CTA (Q = 1: a decode step; Q = 4: four consecutive rows of one
// sequence in a prefill chunk, which then share every gathered entry block). MMA N = 64 Q.
template <int Q>
struct Cfg {
  static constexpr int kN = kNI * Q;
  static constexpr int kQRegion = kN * 128;  // [N rows x 128 B]
  static constexpr int kQBytes = 2 * kQRegion;
  static constexpr int kOffKv = 0;
  static constexpr int kOffQ = kOffKv + kStages * kBlockBytes;
  static constexpr int kOffW = kOffQ + kQBytes;
  static constexpr int kOffBar = kOffW + kN * 4;
  static constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffTmemPtr + 16;  // Q = 1: two CTAs per SM fit
  static constexpr uint32_t kTmemCols = 2 * kN < 32 ? 32 : 2 * kN;  // two accumulators
  static constexpr uint32_t kIdesc = tc::idesc_bf16(kBE, kN, false, false);
  static constexpr int kChunk = (Q == 1 ? kChunkBlocks : kChunkBlocksQ4) * kBE;  // entries per CTA
};

// cp.async.wait_group with the stage depth as its immediate.
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Swizzled shared-memory offset of 16-byte chunk c (0..15) of row r in a two-region K-major tile
// whose regions hold `rows` rows of 128 bytes (the TMA / MMA 128-byte swizzle pattern).
__device__ __forceinline__ uint32_t sw_off(int r, int c, int region_bytes) {
  return (uint32_t)((c >> 3) * region_bytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int Q>
__global__ void __launch_bounds__(kThreads, 2) indexer_decode_tc_kernel(IndexerArgs a, int* status) {
  using K = Cfg<Q>;
  constexpr int kOffQ = K::kOffQ, kOffW = K::kOffW, kOffBar = K::kOffBar;
  constexpr int kOffKv = K::kOffKv, kOffTmemPtr = K::kOffTmemPtr, kQRegion = K::kQRegion;
  extern __shared__ __align__(1024) uint8_t smem[];
  // rows row .. row + Q - 1 of this launch (q_idx, w_idx and scores start at the launch's first
  // row), all of one sequence, whose block-table row the gathers use
  const int row = blockIdx.y * Q;
  int seq;
  int64_t t_first, t;
  a.qr.locate(a.qr.row0 + row, seq, t_first);
  a.qr.locate(a.qr.row0 + row + Q - 1, seq, t);  // the last row sees the most entries
  const int64_t nvis = t < 0 ? 0 : (t + 1) / a.m;
  const int64_t e_begin = (int64_t)blockIdx.x * K::kChunk;
  if (t < 0 || e_begin >= nvis) return;
  const int64_t e_end = nvis < e_begin + K::kChunk ? nvis : e_begin + K::kChunk;
  const int nkb = (int)((e_end - e_begin + kBE - 1) / kBE);

  // The 128-byte swizzle needs 1024-byte aligned tiles; the dynamic window starts aligned.
  if ((tc::smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0 && status) atomicExch(status, tc::kStatusMisaligned);
    return;
  }
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* pool = reinterpret_cast<const __nv_bfloat16*>(a.kpool.base);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bar[kFull0 + i], kGatherThreads);
      tc::mbar_init(&bar[kEmpty0 + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bar[kAccFull0 + i], 1);
      tc::mbar_init(&bar[kAccEmpty0 + i], 128);
    }
    tc::fence_barrier_init();
  }
  if (warp == 8) tc::tmem_alloc(tmem_ptr, K::kTmemCols);
  // head weights: plain loads before the start barrier (the drain reads them from shared memory)
  for (int i = threadIdx.x - 128; i >= 0 && i < K::kN && threadIdx.x < 256; i += 128)
    reinterpret_cast<float*>(smem + kOffW)[i] = __ldg(a.w_idx + (int64_t)row * kNI + i);

  // Gather thread g copies 16-byte chunk (g & 15) of rows (g >> 4) + 8j; its rows share r & 7, so
  // the swizzle term is fixed per thread. Lane l of gather warp w resolves the address of row
  // (2w + (l & 1)) + 8 (l >> 1), and the copies take it by shuffle.
  const int g = threadIdx.x;
  const int gc = g & 15, gr = g >> 4;
  auto row_ptr = [&](int64_t e) -> const __nv_bfloat16* {
    if (e >= e_end) return nullptr;
    // entry numbers fit 32 bits: 32-bit division by the page size
    const uint32_t ue = (uint32_t)e, ps = (uint32_t)a.kpool.page_size;
    const int64_t page = __ldg(a.kpool.block_table + (int64_t)seq * a.kpool.max_pages + ue / ps);
    if (page < 0) return nullptr;
    return pool + (page * ps + ue % ps) * kCI;
  };
  auto issue_block = [&](int kb, const __nv_bfloat16* my_row) {
    uint8_t* dst = smem + kOffKv + (kb % kStages) * kBlockBytes;
    const int src_base = gr & 1;  // lane parity of the resolving lanes of my rows
#pragma unroll
    for (int j = 0; j < kBE / 8; ++j) {
      const __nv_bfloat16* rp = reinterpret_cast<const __nv_bfloat16*>(
          __shfl_sync(~0u, reinterpret_cast<uintptr_t>(my_row), src_base + 2 * j));
      const int r = gr + 8 * j;
      uint8_t* d = dst + sw_off(r, gc, kRegion);
      if (rp != nullptr) {
        tc::cp_async16(d, rp + gc * 8);
      } else if (kb * kBE + r < e_end - e_begin) {
        *reinterpret_cast<uint4*>(d) = make_uint4(0, 0, 0, 0);  // unallocated page: empty key
      }
    }
    cp_async_commit();
  };

  if (warp < 4) {
    // q_idx [Q rows x 64 heads x 128] (consecutive in memory), then the first blocks, before the
    // start barrier
    const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(a.q_idx) + (int64_t)row * kNI * kCI;
#pragma unroll
    for (int j = 0; j < K::kN / 8; ++j) {
      const int r = gr + 8 * j;
      tc::cp_async16(smem + kOffQ + sw_off(r, gc, kQRegion), q + r * kCI + gc * 8);
    }
    const int res_row = 2 * warp + (lane & 1) + 8 * (lane >> 1);
    // the first blocks' block-table loads all go out before any copy is issued
    const __nv_bfloat16* rp0[kStages];
#pragma unroll
    for (int kb = 0; kb < kStages; ++kb)
      rp0[kb] = kb < nkb ? row_ptr(e_begin + (int64_t)kb * kBE + res_row) : nullptr;
#pragma unroll
    for (int kb = 0; kb < kStages; ++kb)
      if (kb < nkb) issue_block(kb, rp0[kb]);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_ptr;

  if (warp < 4) {
    // ------------------------------------------------------------------ gather
    const int res_row = 2 * warp + (lane & 1) + 8 * (lane >> 1);
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      // block kb was issued kStages-1 groups ago at most: wait until it has landed
      const int ahead = (nkb - 1 - kb) < (kStages - 1) ? (nkb - 1 - kb) : (kStages - 1);
      if (ahead >= 2) cp_async_wait_group<2>();
      else if (ahead == 1) cp_async_wait_group<1>();
      else cp_async_wait_group<0>();
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[kFull0 + kb % kStages]);
      const int nb = kb + kStages;
      if (nb < nkb) {
        const __nv_bfloat16* rp = row_ptr(e_begin + (int64_t)nb * kBE + res_row);
        // stage nb % kStages was last used by block nb - kStages
        ok = __all_sync(~0u, tc::mbar_wait(&bar[kEmpty0 + nb % kStages],
                                           ((nb - kStages) / kStages) & 1, status));
        if (!ok) break;
        issue_block(nb, rp);
      }
    }
    tc::cp_async_wait_all();
  } else if (warp == 8) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer
      const uint32_t q_base = tc::smem_u32(smem + kOffQ);
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int s = kb % kStages, acc = kb & 1;
        ok = tc::mbar_wait(&bar[kFull0 + s], (kb / kStages) & 1, status);
        if (ok && kb >= 2) ok = tc::mbar_wait(&bar[kAccEmpty0 + acc], ((kb - 2) >> 1) & 1, status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t kv_base = tc::smem_u32(smem + kOffKv + s * kBlockBytes);
#pragma unroll
        for (int kk = 0; kk < kCI / 16; ++kk)
          tc::mma_bf16_ss(tmem + acc * K::kN,
                          tc::desc_sw128(kv_base + (kk >> 2) * kRegion + (kk & 3) * 32, 0, 1024),
                          tc::desc_sw128(q_base + (kk >> 2) * kQRegion + (kk & 3) * 32, 0, 1024),
                          K::kIdesc, kk > 0);
        tc::mma_commit(&bar[kEmpty0 + s]);
        tc::mma_commit(&bar[kAccFull0 + acc]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ drain
    const int sp = warp & 3;
    const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16);
    const float4* w4 = reinterpret_cast<const float4*>(smem + kOffW);
    bool ok = true;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int acc = kb & 1;
      ok = __all_sync(~0u, tc::mbar_wait(&bar[kAccFull0 + acc], (kb >> 1) & 1, status));
      if (!ok) break;
      tc::tc_fence_after();
      const int64_t e = e_begin + (int64_t)kb * kBE + sp * 32 + lane;
      float score[Q];
#pragma unroll
      for (int qi = 0; qi < Q; ++qi) {
        float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
        // the row's 64 head sums in two loads and one wait (one TMEM round trip)
        uint32_t vv[kNI];
        tc::tmem_ld32(t_lane + acc * K::kN + qi * kNI, *reinterpret_cast<uint32_t(*)[32]>(vv));
        tc::tmem_ld32(t_lane + acc * K::kN + qi * kNI + 32,
                      *reinterpret_cast<uint32_t(*)[32]>(vv + 32));
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kNI; c += 16) {
          const uint32_t* v = vv + c;
#pragma unroll
          for (int u = 0; u < 16; u += 4) {
            const float4 wv = w4[(qi * kNI + c + u) / 4];
            const float2 x0 = make_float2(fmaxf(__uint_as_float(v[u]), 0.f),
                                          fmaxf(__uint_as_float(v[u + 1]), 0.f));
            const float2 x1 = make_float2(fmaxf(__uint_as_float(v[u + 2]), 0.f),
                                          fmaxf(__uint_as_float(v[u + 3]), 0.f));
            s0 = __ffma2_rn(x0, make_float2(wv.x, wv.y), s0);
            s1 = __ffma2_rn(x1, make_float2(wv.z, wv.w), s1);
          }
        }
        score[qi] = (s0.x + s0.y) + (s1.x + s1.y);
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&bar[kAccEmpty0 + acc]);
      // row qi sees the entries w < (t_first + qi + 1) // m (consecutive positions)
#pragma unroll
      for (int qi = 0; qi < Q; ++qi)
        if (e < e_end && e < (t_first + qi + 1) / a.m)
          a.scores[(int64_t)(row + qi) * a.n_stride + e] = score[qi];
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, K::kTmemCols);
  }
}

template <int Q>
cudaError_t launch_q(const IndexerArgs& a, int max_visible, int* status, cudaStream_t st) {
  using K = Cfg<Q>;
  cudaError_t e = ensure_smem_limit((const void*)indexer_decode_tc_kernel<Q>, K::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int chunk = K::kChunk;
  // one launch per 65535 CTA rows (the grid's y limit), each with its rows' pointers
  constexpr int64_t kMaxRowsPerLaunch = 65535 * (int64_t)Q;
  for (int64_t r0 = 0; r0 < a.nrows; r0 += kMaxRowsPerLaunch) {
    IndexerArgs b = a;
    b.nrows = a.nrows - r0 < kMaxRowsPerLaunch ? a.nrows - r0 : kMaxRowsPerLaunch;
    b.qr.row0 = a.qr.row0 + r0;
    b.q_idx = reinterpret_cast<const __nv_bfloat16*>(a.q_idx) + r0 * kNI * kCI;
    b.w_idx = a.w_idx + r0 * kNI;
    b.scores = a.scores + r0 * a.n_stride;
    dim3 grid((unsigned)((max_visible + chunk - 1) / chunk), (unsigned)(b.nrows / Q));
    indexer_decode_tc_kernel<Q><<<grid, kThreads, K::kSmemBytes, st>>>(b, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

bool indexer_decode_tc_supported(int dtype, int nI, int cI) {
  return dtype == 1 && nI == kNI && cI == kCI;
}

cudaError_t launch_indexer_decode_tc(const IndexerArgs& a, int max_visible, int* status,
                                     cudaStream_t st) {
  if (a.nrows == 0 || max_visible == 0) return cudaSuccess;
  // groups of four rows when every group lies in one sequence (rows per sequence a multiple of 4,
  // launches starting on a sequence boundary)
  const int nq = a.qr.nq > 1 ? a.qr.nq : 1;
  if (a.qr.ctx_lens != nullptr && nq % 4 == 0 && a.qr.row0 % nq == 0 && a.nrows % 4 == 0)
    return launch_q<4>(a, max_visible, status, st);
  return launch_q<1>(a, max_visible, status, st);
}

}  // namespace sac
