// Tensor-core (tcgen05) version of the shared K=V multi-query attention for bf16 layers with
// 64 query heads and head_dim 512 ("Hybrid attention": shared K=V MQA; per-head sink, eq. 27;
// partial RoPE with the -i output rotation, eq. 26; sliding-window branch + compressor entries).
//
// One query row at a time per CTA (persistent over rows). Its 64 heads are the M = 64 rows of
// both contractions:  S = Q K^T  (M=64, N=48 keys, K=512)  and  O += P V  (M=64, N=256 x 2, K=48).
// Because K = V, one shared-memory key tile serves as the K-major B operand of QK^T and as the
// MN-major B operand of PV. Tiles of 48 keys keep three tile buffers resident next to the 64 KB
// query tile. Window rows and HCA entries are consecutive rows and load as 8 TMA boxes per tile;
// CSA selections (and paged rows) are gathered with 16-byte cp.async copies by two producer
// groups that take alternate tiles. Tiles never mix window rows and entries.
//
// QK^T of a tile is 32 MMAs of K=16. Accumulating them into one TMEM tile would chain each MMA
// on its predecessor, so they rotate over four partial accumulators (one per issuing thread) and
// the softmax adds the four partials.
//
// The query tile arrives un-rotated; one warp turns its rope slice in shared memory before the
// first QK^T of the row, so no rotated copy of q is written to HBM.
//
// Tensor memory (512 columns, fp32): O[:, 0:256] in lanes 0-15 of each sub-partition and
// O[:, 256:512] in lanes 16-31 (the M = 64 layout leaves half the lanes free); for each of the two
// S buffers, partials 0/2 in lanes 0-15 and partials 1/3 in lanes 16-31 of 96 columns at 256
// (buffer 0) and 352 (buffer 1). A softmax thread of lane i < 16 and its partner i + 16 own the
// same head: they add their partials, exchange halves, and each finishes 24 of the 48 keys.
//
// Warps: 0 = TMA thread, 1-2 = QK^T issuers (warp 1 also owns TMEM), 3 = query rotation, 4-7 and
// 13-16 = two gather groups of 128 threads taking the gathered tiles in turn (idle when every
// tile arrives by TMA), 8-11 = softmax + output, 12 = PV issuer. Each tcgen05.mma costs its issuing thread a fixed time, so two threads
// issue QK^T and a third issues PV the moment P is written, instead of after the next tile's
// QK^T. An M = 64 MMA occupies one 16-lane half of each TMEM sub-partition, and MMAs into
// opposite halves run side by side: the QK^T partials alternate between the lane halves, and the
// two halves of O sit in opposite lane halves. The softmax keeps the running max in log2 units and moves it
// (rescaling O) only when a tile's max exceeds it by more than 8.
#include <cuda_bf16.h>

#include "launch_util.h"
#include "sac_kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace sac {
namespace {

constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kNK = 48;                          // keys per tile
constexpr int kHalfNK = kNK / 2;
constexpr int kStages = 3;                       // key tiles in flight
constexpr int kQRegion = 64 * 128;               // [64 rows x 128 B]: one swizzle column of Q
constexpr int kKRegion = kNK * 128;              // [48 rows x 128 B]
constexpr int kQBytes = 8 * kQRegion;            // 64 KB
constexpr int kTileBytes = 8 * kKRegion;         // 48 KB
constexpr int kPBytes = kHeads * 128;            // 64 rows x 128 B (48 keys used)
constexpr int kGatherGroups = 2;                 // producer groups taking tiles in turn
constexpr int kGroupThreads = 128;               // threads of one gather group (warps 4-7, 13-16)
constexpr int kThreads = 544;                    // with the gather groups
constexpr int kThreadsTma = 416;                 // every tile by TMA: warps 13-16 not launched

constexpr int kOffQ = 0;
constexpr int kOffTile = kOffQ + kQBytes;
constexpr int kOffP = kOffTile + kStages * kTileBytes;
constexpr int kOffCs = kOffP + 2 * kPBytes;      // [32] (cos, sin) of the query's rope pairs
constexpr int kOffBar = kOffCs + 32 * 8;
enum Bar { kQFull, kQReady, kQEmpty, kKvFull0, kKvEmpty0 = kKvFull0 + kStages,
           kSFull0 = kKvEmpty0 + kStages, kPFull0 = kSFull0 + 2, kPvDone0 = kPFull0 + 2,
           kOFull = kPvDone0 + 2, kOEmpty, kNumBars };
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffTmemPtr + 16;

constexpr uint32_t kColS = 256, kSStride = 2 * kNK;  // S buffer s at kColS + s * kSStride
constexpr uint32_t kIdescQK = tc::idesc_bf16(64, kNK, false, false);
constexpr uint32_t kIdescPV = tc::idesc_bf16(64, 256, false, true);
constexpr int kMaxSplits = 8;  // key-tile splits of one row (decode: few rows, many SMs)
constexpr int kQkIssuers = 2;  // threads issuing QK^T (measured faster than 4 and than 1)
constexpr int kRopeStep = 28;  // K-steps 28..31 read the last region of Q (the rope slice)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;  // move the running max only when a tile exceeds it by 2^8

struct Row {
  int seq;
  int64_t t, lo;
  int nwin, npool, twin, tiles;
  int64_t r;   // query row of the work item
  int sp;      // split of the row's key tiles this item covers
  int j0, j1;  // tile range [j0, j1) of the item
  bool bad;    // the row's context lies beyond the block tables (no key is read)
};

__device__ __forceinline__ Row locate_row(const AttnArgs& a, int64_t r) {
  Row w;
  w.bad = !a.qr.locate(a.qr.row0 + r, w.seq, w.t);
  if (w.t < 0) {  // no key: a bad context, or a chunk row before its sequence's start
    w.lo = 0;
    w.nwin = w.npool = w.twin = w.tiles = 0;
    return w;
  }
  w.lo = w.t - a.W + 1 < 0 ? 0 : w.t - a.W + 1;
  w.nwin = (int)(w.t - w.lo + 1);
  const int nvis = a.pool_mode ? (int)((w.t + 1) / a.m) : 0;
  w.npool = a.pool_mode == 2 ? (nvis < a.k ? nvis : a.k) : nvis;
  w.twin = (w.nwin + kNK - 1) / kNK;
  w.tiles = w.twin + (w.npool + kNK - 1) / kNK;
  return w;
}

// Work item it = (row, split): the row's key tiles are divided into a.splits contiguous ranges
// (a.splits = 1: one item per row, all tiles). Items with an empty range are skipped by every role.
template <bool kSplit>
__device__ __forceinline__ Row locate_item(const AttnArgs& a, int64_t it) {
  const int splits = kSplit ? a.splits : 1;
  const int64_t r = kSplit ? it / splits : it;
  const int sp = kSplit ? (int)(it % splits) : 0;
  Row w = locate_row(a, r);
  w.r = r;
  w.sp = sp;
  w.j0 = kSplit ? (int)((int64_t)w.tiles * sp / splits) : 0;
  w.j1 = kSplit ? (int)((int64_t)w.tiles * (sp + 1) / splits) : w.tiles;
  return w;
}

__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

// QK^T K-steps kk = ME (mod NQK) of one tile (fully unrolled, every offset a constant: the issue
// cost per MMA is what bounds this loop). K-step kk accumulates into partial p = kk & 3 at lanes
// 16 (p & 1), columns + 48 (p >> 1) of the S buffer at d0. With qready set (a query's first tile)
// the K-steps of the rope region wait until the query's rope slice has been rotated.
template <int NQK, int ME>
__device__ __forceinline__ bool issue_qk(uint32_t d0, uint64_t qd, uint64_t kd, uint64_t* qready,
                                         uint32_t qparity, int* status) {
#pragma unroll
  for (int i = 0; i < kDim / 16 / NQK; ++i) {
    const int kk = NQK * i + ME;
    if (kk >= kRopeStep && kk - NQK < kRopeStep && qready != nullptr) {
      if (!tc::mbar_wait(qready, qparity, status)) return false;
      tc::tc_fence_after();
    }
    const int p = kk & 3;
    const uint32_t dp = d0 + ((p & 1) ? (16u << 16) : 0u) + ((p & 2) ? (uint32_t)kNK : 0u);
    const uint32_t qo = ((kk >> 2) * kQRegion + (kk & 3) * 32) >> 4;
    const uint32_t ko = ((kk >> 2) * kKRegion + (kk & 3) * 32) >> 4;
    tc::mma_bf16_ss(dp, qd + qo, kd + ko, kIdescQK, kk >= 4 ? 1u : 0u);
  }
  return true;
}

// Global address of key c of tile j (keys past the tile's count reuse a valid row: masked).
__device__ __forceinline__ const __nv_bfloat16* key_ptr(const AttnArgs& a, const Row& w,
                                                        int64_t r, int j, int c) {
  if (j < w.twin) {
    int x = j * kNK + c;
    if (x >= w.nwin) x = 0;
    const __nv_bfloat16* p = a.win.row<__nv_bfloat16>(w.seq, w.lo + x);
    return p ? p : a.win.row<__nv_bfloat16>(w.seq, w.lo);
  }
  int i = (j - w.twin) * kNK + c;
  if (i >= w.npool) i = 0;
  int64_t e = a.pool_mode == 2 ? (int64_t)__ldg(a.sel + r * a.k + i) : i;
  const __nv_bfloat16* p = a.pool.row<__nv_bfloat16>(w.seq, e < 0 ? 0 : e);
  return p ? p : reinterpret_cast<const __nv_bfloat16*>(a.pool.base);
}

// kNThreads: kThreads when some tile is gathered, else kThreadsTma (the smaller block keeps the
// register budget of the TMA-only layers at 152 per thread instead of 120).
template <bool kSplit, int kNThreads>
__global__ void __launch_bounds__(kNThreads, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_win_box,
                        const __grid_constant__ CUtensorMap tm_pool_box, AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = a.status;
  // the 128-byte swizzle needs 1024-byte aligned tiles; the dynamic window starts aligned
  if ((tc::smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0 && status) atomicExch(status, tc::kStatusMisaligned);
    return;
  }

  // window rows of a prefill are consecutive rows of the rotated kv stream, and so are the
  // entries of an HCA prefill: those tiles load as TMA boxes; the rest are gathered
  const bool win_contig = a.win.block_table == nullptr;
  const bool pool_contig = a.pool_mode == 1 && a.pool.block_table == nullptr;
  const bool any_gather = !win_contig || (a.pool_mode != 0 && !pool_contig);
  if (any_gather && kNThreads < kThreads) {  // the launcher sizes the block from the same rule
    if (threadIdx.x == 0 && status) atomicExch(status, tc::kStatusConfig);
    return;
  }
  const int64_t n_items = kSplit ? a.nrows * a.splits : a.nrows;
  // Who issues PV: with gathered tiles the gather latency decides, and a separate thread issues
  // PV the moment P is ready so that tile buffers free early; with TMA-fed tiles QK^T is the
  // critical step, and the QK^T threads issue PV right after the next tile's QK^T (measured: 17%
  // faster at HCA-32k, slower at CSA-8k).
  const bool pv_by_qk = !any_gather;
  const uint32_t pv_commits = pv_by_qk ? kQkIssuers : 1;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bar[kQFull], 1);
    tc::mbar_init(&bar[kQReady], 32);
    tc::mbar_init(&bar[kQEmpty], kQkIssuers);
    for (int i = 0; i < kStages; ++i) {
      // TMA thread (+ one gather group when some tiles are gathered)
      tc::mbar_init(&bar[kKvFull0 + i], any_gather ? 1 + kGroupThreads : 1);
      tc::mbar_init(&bar[kKvEmpty0 + i], pv_commits);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bar[kSFull0 + i], kQkIssuers);
      tc::mbar_init(&bar[kPFull0 + i], 128);
      tc::mbar_init(&bar[kPvDone0 + i], pv_commits);
    }
    tc::mbar_init(&bar[kOFull], pv_commits);
    tc::mbar_init(&bar[kOEmpty], 128);
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_ptr, 512);
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tm_q);
    tc::tma_prefetch_desc(&tm_win_box);
    tc::tma_prefetch_desc(&tm_pool_box);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_ptr;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA thread
    if (lane == 0) {
      uint32_t g = 0, qi = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const Row w = locate_item<kSplit>(a, it);
        if (w.bad && status) atomicExch(status, tc::kStatusBadInput);
        if (w.j0 == w.j1) continue;
        const int64_t r = w.r;
        if (qi > 0) ok = tc::mbar_wait(&bar[kQEmpty], (qi - 1) & 1, status);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(&bar[kQFull], kQBytes);
        for (int c = 0; c < 8; ++c)
          tc::tma_load_2d(smem + kOffQ + c * kQRegion, &tm_q, &bar[kQFull], 64 * c,
                          (int32_t)(r * kHeads));
        for (int j = w.j0; j < w.j1 && ok; ++j, ++g) {
          const uint32_t b = g % kStages;
          if (g >= kStages) ok = tc::mbar_wait(&bar[kKvEmpty0 + b], ((g - kStages) / kStages) & 1,
                                               status);
          if (!ok) break;
          const bool is_win = j < w.twin;
          if (is_win ? win_contig : pool_contig) {
            tc::mbar_arrive_expect_tx(&bar[kKvFull0 + b], kTileBytes);
            const int64_t y0 = is_win ? a.win.row_index(w.seq, w.lo + (int64_t)j * kNK)
                                      : a.pool.row_index(w.seq, (int64_t)(j - w.twin) * kNK);
            const CUtensorMap* map = is_win ? &tm_win_box : &tm_pool_box;
            uint8_t* tile = smem + kOffTile + b * kTileBytes;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              tc::tma_load_2d(tile + c * kKRegion, map, &bar[kKvFull0 + b], 64 * c, (int32_t)y0);
          } else {
            tc::mbar_arrive(&bar[kKvFull0 + b]);
          }
        }
        ++qi;
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------------ QK^T issuers
    // issuer me takes the K-steps kk = me (mod 2); K-step kk accumulates into partial p = kk & 3,
    // which sits in lanes 16 (p & 1), columns + 48 (p >> 1) of the S buffer
    const uint32_t me = warp - 1;
    if (lane == 0) {
      uint32_t g0 = 0, qi = 0;
      bool ok = true;
      const uint64_t qd = tc::desc_sw128(tc::smem_u32(smem + kOffQ), 0, 1024);
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const Row w = locate_item<kSplit>(a, it);
        if (w.j0 == w.j1) continue;
        // the query tile has landed; its rope region (the last 128-byte column, K-steps 28..31)
        // is still being rotated, so the first QK^T waits for kQReady only before those steps
        ok = tc::mbar_wait(&bar[kQFull], qi & 1, status);
        for (int j = w.j0; j < w.j1 + (pv_by_qk ? 1 : 0) && ok; ++j) {
          if (j < w.j1) {  // S(g) = Q K^T over four partial accumulators
            const uint32_t g = g0 + (j - w.j0), b = g % kStages, s = g & 1;
            ok = tc::mbar_wait(&bar[kKvFull0 + b], (g / kStages) & 1, status);
            if (ok && g >= 2) ok = tc::mbar_wait(&bar[kPFull0 + s], ((g - 2) >> 1) & 1, status);
            if (!ok) break;
            tc::tc_fence_after();
            const uint64_t kd =
                tc::desc_sw128(tc::smem_u32(smem + kOffTile + b * kTileBytes), 0, 1024);
            const uint32_t d0 = tmem + kColS + s * kSStride;
            // the descriptor's start-address field counts 16-byte units: advancing along K adds
            // the byte offset >> 4 to the base descriptor
            uint64_t* qready = j == w.j0 ? &bar[kQReady] : nullptr;
            ok = me == 0 ? issue_qk<kQkIssuers, 0>(d0, qd, kd, qready, qi & 1, status)
                         : issue_qk<kQkIssuers, 1>(d0, qd, kd, qready, qi & 1, status);
            if (!ok) break;
            tc::mma_commit(&bar[kSFull0 + s]);
            if (j == w.j1 - 1) tc::mma_commit(&bar[kQEmpty]);
          }
          if (pv_by_qk && j > w.j0) {  // O[:, 256 me : 256 me + 256] += P(g) V(g), after QK^T(g+1)
            const uint32_t g = g0 + (j - 1 - w.j0), b = g % kStages, s = g & 1;
            ok = tc::mbar_wait(&bar[kPFull0 + s], (g >> 1) & 1, status);
            if (ok && j - 1 == w.j0 && qi > 0)
              ok = tc::mbar_wait(&bar[kOEmpty], (qi - 1) & 1, status);
            if (!ok) break;
            tc::tc_fence_after();
            const uint32_t v_base = tc::smem_u32(smem + kOffTile + b * kTileBytes);
            const uint64_t pd = tc::desc_sw128(tc::smem_u32(smem + kOffP + s * kPBytes), 0, 1024);
            const uint64_t vd = tc::desc_sw128(v_base + me * 4 * kKRegion, kKRegion, 1024);
            const uint32_t od = tmem + (me ? (16u << 16) : 0u);
#pragma unroll
            for (int kk = 0; kk < kNK / 16; ++kk)
              tc::mma_bf16_ss(od, pd + kk * 2, vd + kk * 128, kIdescPV,
                              (j - 1 > w.j0 || kk > 0) ? 1u : 0u);
            tc::mma_commit(&bar[kKvEmpty0 + b]);
            tc::mma_commit(&bar[kPvDone0 + s]);
            if (j == w.j1) tc::mma_commit(&bar[kOFull]);
          }
        }
        g0 += w.j1 - w.j0;
        ++qi;
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------------ query rotation
    // Lane p first writes (cos, sin) of rope pair p at the query's position to a shared table.
    // Then thread i turns the rope pairs of head rows i and i+32 of the staged query tile (row h's
    // 16-byte chunk c of a 128-byte region sits at chunk c ^ (h & 7)); when the rope slice starts
    // on a 16-byte boundary (R a multiple of 8) all of a thread's chunks are loaded before any is
    // used, so the rotation costs one shared-memory round trip instead of one per chunk.
    const int R = a.rf.R;
    const int p0 = (kDim - R) >> 1;  // first rotated pair among the 256 channel pairs
    float2* cs_tab = reinterpret_cast<float2*>(smem + kOffCs);
    uint32_t qi = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const Row w = locate_item<kSplit>(a, it);
      if (w.j0 == w.j1) continue;
      const int64_t t = w.t;
      if (lane < R / 2) {
        float c, sn;
        rope_cos_sin(a.rf, lane, a.pos0 + t, c, sn);
        cs_tab[lane] = make_float2(c, sn);
      }
      __syncwarp();
      ok = __all_sync(~0u, tc::mbar_wait(&bar[kQFull], qi & 1, status));
      if (!ok) break;
      if ((R & 7) == 0) {
        constexpr int kMaxChunks = 8;  // R <= 64: at most 8 chunks of 4 pairs
        const int nch = R >> 3;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int h = hh * 32 + lane;
          uint8_t* row = smem + kOffQ + h * 128;
          uint4 v[kMaxChunks];
#pragma unroll
          for (int c = 0; c < kMaxChunks; ++c) {
            const int pp = p0 + 4 * c;
            if (c < nch)
              v[c] = *reinterpret_cast<const uint4*>(row + (pp >> 5) * kQRegion +
                                                     ((((pp & 31) >> 2) ^ (h & 7)) << 4));
          }
#pragma unroll
          for (int c = 0; c < kMaxChunks; ++c) {
            if (c >= nch) break;
            const int pp = p0 + 4 * c;
            const float4 cs01 = *reinterpret_cast<const float4*>(cs_tab + 4 * c);
            const float4 cs23 = *reinterpret_cast<const float4*>(cs_tab + 4 * c + 2);
            const float cc[4] = {cs01.x, cs01.z, cs23.x, cs23.z};
            const float ss[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
            uint32_t* w4 = reinterpret_cast<uint32_t*>(&v[c]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 x = unpack_bf16(w4[u]);
              w4[u] = pack_bf16(x.x * cc[u] - x.y * ss[u], x.x * ss[u] + x.y * cc[u]);
            }
            *reinterpret_cast<uint4*>(row + (pp >> 5) * kQRegion +
                                      ((((pp & 31) >> 2) ^ (h & 7)) << 4)) = v[c];
          }
        }
      } else {
        for (int hh = 0; hh < 2; ++hh) {
          const int h = hh * 32 + lane;
          uint8_t* row = smem + kOffQ + h * 128;
          for (int q = p0; q < kDim / 2; ++q) {
            uint32_t* word = reinterpret_cast<uint32_t*>(
                row + (q >> 5) * kQRegion + ((((q & 31) >> 2) ^ (h & 7)) << 4) + (q & 3) * 4);
            const float2 cs = cs_tab[q - p0];
            const float2 x = unpack_bf16(*word);
            *word = pack_bf16(x.x * cs.x - x.y * cs.y, x.x * cs.y + x.y * cs.x);
          }
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[kQReady]);
      ++qi;
    }
  } else if (warp < 8 || warp >= 13) {
    if (!any_gather) goto done;  // every tile arrives by TMA
    // ------------------------------------------------------------------ gather groups
    // Warps 4-7 and 13-16 form two groups that take the gathered tiles in turn. Thread t of a
    // group of G threads copies rows t/8, t/8 + G/8, ... of the tile; for each it copies 16-byte
    // slot t%8 of all 8 regions, so a warp instruction reads four whole 128-byte row segments and
    // a thread needs only a few row addresses. Once its copies landed it makes them visible to
    // the tensor core and arrives on the tile's barrier.
    const int grp = warp < 8 ? 0 : 1;
    const int gt = (warp < 8 ? warp - 4 : warp - 13) * 32 + lane;  // thread within the group
    const int row0 = gt >> 3, slot = gt & 7;
    constexpr int kRowStride = kGroupThreads / 8;        // rows a group covers per pass
    constexpr int kRowsPer = kNK / kRowStride;
    // Walk this group's tiles in order across the CTA's query rows. The source rows of the next
    // tile are resolved while the current tile's copies are in flight, so the selection-index
    // loads do not add to each tile's latency.
    struct Cursor {
      int64_t r;
      Row w;
      int j;
      uint32_t g;
    };
    auto valid = [&](const Cursor& c) { return c.r < n_items; };  // c.r: the work item
    auto gathered = [&](const Cursor& c) {
      return !(c.j < c.w.twin ? win_contig : pool_contig);
    };
    auto first_tile = [&](Cursor& c) {  // c.r: the first non-empty item from c.r on
      for (; c.r < n_items; c.r += gridDim.x) {
        c.w = locate_item<kSplit>(a, c.r);
        if (c.w.j0 < c.w.j1) break;
      }
      c.j = c.r < n_items ? c.w.j0 : 0;
    };
    auto advance = [&](Cursor c) {  // next tile of this group after c
      do {
        ++c.g;
        if (++c.j >= c.w.j1) {
          c.r += gridDim.x;
          first_tile(c);
          if (c.r >= n_items) return c;
        }
      } while ((int)(c.g % kGatherGroups) != grp);
      return c;
    };
    auto resolve = [&](const Cursor& c, const __nv_bfloat16* (&src)[kRowsPer]) {
#pragma unroll
      for (int i = 0; i < kRowsPer; ++i) src[i] = key_ptr(a, c.w, c.w.r, c.j, row0 + kRowStride * i);
    };
    Cursor c;
    c.r = blockIdx.x;
    c.g = 0;
    first_tile(c);
    if (valid(c))
      for (int i = 0; i < grp; ++i) c = advance(c);
    const __nv_bfloat16* src[kRowsPer];
    if (valid(c) && gathered(c)) resolve(c, src);
    bool ok = true;
    while (valid(c) && ok) {
      const uint32_t b = c.g % kStages;
      if (c.g >= kStages)
        ok = __all_sync(~0u, tc::mbar_wait(&bar[kKvEmpty0 + b], ((c.g - kStages) / kStages) & 1,
                                           status));
      if (!ok) break;
      const bool gath = gathered(c);
      if (gath) {
        uint8_t* tile = smem + kOffTile + b * kTileBytes;
#pragma unroll
        for (int i = 0; i < kRowsPer; ++i) {
          const int row = row0 + kRowStride * i;
          uint8_t* d = tile + row * 128 + ((slot ^ (row & 7)) << 4);
#pragma unroll
          for (int q = 0; q < 8; ++q) tc::cp_async16(d + q * kKRegion, src[i] + q * 64 + slot * 8);
        }
      }
      const Cursor n = advance(c);
      if (valid(n) && gathered(n)) resolve(n, src);  // overlaps the copies in flight
      if (gath) {
        tc::cp_async_wait_all();
        tc::fence_proxy_async_smem();
      }
      tc::mbar_arrive(&bar[kKvFull0 + b]);
      c = n;
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------------ PV issuer
    // O += P(g) V(g) as soon as the softmax has written P(g), independent of how far the QK^T
    // issuers have got: O[:, 0:256] accumulates in lanes 0-15 and O[:, 256:512] in lanes 16-31,
    // and the two halves' MMAs alternate so both lane halves of the tensor core stay busy.
    if (lane == 0 && !pv_by_qk) {
      uint32_t g0 = 0, qi = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const Row w = locate_item<kSplit>(a, it);
        if (w.j0 == w.j1) continue;
        for (int j = w.j0; j < w.j1 && ok; ++j) {
          const uint32_t g = g0 + (j - w.j0), b = g % kStages, s = g & 1;
          ok = tc::mbar_wait(&bar[kPFull0 + s], (g >> 1) & 1, status);
          if (ok && j == w.j0 && qi > 0) ok = tc::mbar_wait(&bar[kOEmpty], (qi - 1) & 1, status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t v_base = tc::smem_u32(smem + kOffTile + b * kTileBytes);
          const uint64_t pd = tc::desc_sw128(tc::smem_u32(smem + kOffP + s * kPBytes), 0, 1024);
          const uint64_t vd0 = tc::desc_sw128(v_base, kKRegion, 1024);
          const uint64_t vd1 = tc::desc_sw128(v_base + 4 * kKRegion, kKRegion, 1024);
#pragma unroll
          for (int kk = 0; kk < kNK / 16; ++kk) {
            const uint32_t acc = (j > w.j0 || kk > 0) ? 1u : 0u;
            tc::mma_bf16_ss(tmem, pd + kk * 2, vd0 + kk * 128, kIdescPV, acc);
            tc::mma_bf16_ss(tmem + (16u << 16), pd + kk * 2, vd1 + kk * 128, kIdescPV, acc);
          }
          tc::mma_commit(&bar[kKvEmpty0 + b]);
          tc::mma_commit(&bar[kPvDone0 + s]);
          if (j == w.j1 - 1) tc::mma_commit(&bar[kOFull]);
        }
        g0 += w.j1 - w.j0;
        ++qi;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + output
    const int sp = warp & 3;                 // TMEM sub-partition of this warp
    const int half = lane >> 4;              // 0: keys 0..23, O[:,0:256]; 1: keys 24..47, O[:,256:]
    const int h = 16 * sp + (lane & 15);     // head of this thread's row
    const uint32_t t_row = tmem + ((uint32_t)(32 * sp) << 16);
    const float scale_log2 = a.scale * kLog2e;
    const float sink_log2 = __ldg(a.sinks + h) * kLog2e;
    uint32_t g0 = 0, qi = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const Row w = locate_item<kSplit>(a, it);
      if (w.j0 == w.j1) continue;
      const int64_t r = w.r;
      // the sink (logit s_h, zero value) is one more term of the normaliser: here, or in the
      // combine kernel when the row's keys are split
      float m_run = kSplit ? -INFINITY : sink_log2, l_run = kSplit ? 0.f : 1.f;
      for (int j = w.j0; j < w.j1 && ok; ++j) {
        const uint32_t g = g0 + (j - w.j0), s = g & 1;
        ok = __all_sync(~0u, tc::mbar_wait(&bar[kSFull0 + s], (g >> 1) & 1, status));
        if (!ok) break;
        tc::tc_fence_after();
        // own partials: columns [0,48) and [48,96) of this S buffer in this thread's lane
        float own[kNK];
        {
          uint32_t v[16];
#pragma unroll
          for (int c = 0; c < kNK; c += 16) {
            uint32_t u[16];
            tc::tmem_ld16(t_row + kColS + s * kSStride + c, v);
            tc::tmem_ld16(t_row + kColS + s * kSStride + kNK + c, u);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) own[c + e] = __uint_as_float(v[e]) + __uint_as_float(u[e]);
          }
        }
        // exchange: this thread finishes keys [half*24, half*24+24) of the row
        float sv[kHalfNK];
#pragma unroll
        for (int k = 0; k < kHalfNK; ++k) {
          const float send = half ? own[k] : own[kHalfNK + k];
          const float recv = __shfl_xor_sync(~0u, send, 16);
          sv[k] = (half ? own[kHalfNK + k] : own[k]) + recv;
        }
        const int nk = j < w.twin ? min(kNK, w.nwin - j * kNK)
                                  : min(kNK, w.npool - (j - w.twin) * kNK);
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < kHalfNK; ++k) {
          sv[k] = half * kHalfNK + k < nk ? sv[k] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, sv[k]);
        }
        mx = fmaxf(mx, __shfl_xor_sync(~0u, mx, 16));
        const bool move = mx > m_run + kLazy;
        const float m_new = move ? mx : m_run;
        const float alpha = exp2f(m_run - m_new);
        // rescale the rows of O this warp owns (rare: only when some row's max moved)
        if (__any_sync(~0u, move) && j > w.j0) {
          const uint32_t gp = g - 1;
          ok = __all_sync(~0u, tc::mbar_wait(&bar[kPvDone0 + (gp & 1)], (gp >> 1) & 1, status));
          if (!ok) break;
          tc::tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256; c += 16) {
            uint32_t v[16];
            tc::tmem_ld16(t_row + c, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tc::tmem_st16(t_row + c, v);
          }
          tc::tmem_wait_st();
        }
        float sum = 0.f;
        uint32_t pk[kHalfNK / 2];
#pragma unroll
        for (int k = 0; k < kHalfNK; k += 2) {
          const float e0 = exp2f(sv[k] - m_new), e1 = exp2f(sv[k + 1] - m_new);
          sum += e0 + e1;
          pk[k / 2] = pack_bf16(e0, e1);
        }
        sum += __shfl_xor_sync(~0u, sum, 16);
        l_run = l_run * alpha + sum;
        m_run = m_new;
        // P buffer s is free once PV(g-2) completed
        if (g >= 2)
          ok = __all_sync(~0u, tc::mbar_wait(&bar[kPvDone0 + s], ((g - 2) >> 1) & 1, status));
        if (!ok) break;
        uint8_t* prow = smem + kOffP + s * kPBytes + h * 128;
#pragma unroll
        for (int ch = 0; ch < kHalfNK / 8; ++ch) {
          const int cg = half * (kHalfNK / 8) + ch;  // 16-byte chunk of keys 8cg..8cg+7
          *reinterpret_cast<uint4*>(prow + ((cg ^ (h & 7)) << 4)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[kPFull0 + s]);
      }
      if (!ok) break;
      if (kSplit) {
        // ---- split output: this item's O (relative to its running max), max and normaliser in
        // fp32 for the combine kernel
        ok = __all_sync(~0u, tc::mbar_wait(&bar[kOFull], qi & 1, status));
        if (!ok) break;
        tc::tc_fence_after();
        float* po = a.part_o + ((int64_t)it * kHeads + h) * kDim + half * 256;
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 64) {
          uint32_t v[4][16];
#pragma unroll
          for (int q = 0; q < 4; ++q) tc::tmem_ld16(t_row + c0 + 16 * q, v[q]);
          tc::tmem_wait_ld();
          if (c0 + 64 == 256) {
            tc::tc_fence_before();
            tc::mbar_arrive(&bar[kOEmpty]);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int e = 0; e < 16; e += 4)
              *reinterpret_cast<float4*>(po + c0 + 16 * q + e) =
                  make_float4(__uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1]),
                              __uint_as_float(v[q][e + 2]), __uint_as_float(v[q][e + 3]));
        }
        if (half == 0)
          *reinterpret_cast<float2*>(a.part_ml + ((int64_t)it * kHeads + h) * 2) =
              make_float2(m_run, l_run);
        g0 += w.j1 - w.j0;
        ++qi;
        continue;
      }
      // ---- output: O / l, the rope slice turned by -P_t, bf16 store. Lane p holds the cos/sin
      // of rope pair p; the rotation reads them with warp shuffles.
      const int64_t P = a.pos0 + w.t;
      float my_c = 1.f, my_s = 0.f;
      if (lane < a.rf.R / 2) rope_cos_sin(a.rf, lane, -P, my_c, my_s);
      ok = __all_sync(~0u, tc::mbar_wait(&bar[kOFull], qi & 1, status));
      if (!ok) break;
      tc::tc_fence_after();
      const float inv_l = 1.f / l_run;
      __nv_bfloat16* orow =
          reinterpret_cast<__nv_bfloat16*>(a.o) + ((int64_t)r * kHeads + h) * kDim + half * 256;
      const int rope_lo = kDim - a.rf.R;  // first rotated channel (always in the upper half)
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 64) {
        uint32_t v[4][16];
#pragma unroll
        for (int q = 0; q < 4; ++q) tc::tmem_ld16(t_row + c0 + 16 * q, v[q]);
        tc::tmem_wait_ld();
        if (c0 + 64 == 256) {  // last chunk: every upper-half lane holds rope channels here
          tc::tc_fence_before();
          tc::mbar_arrive(&bar[kOEmpty]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = c0 + 16 * q;
          float x[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(v[q][e]) * inv_l;
          if (256 + c + 16 > rope_lo) {  // warp-uniform: some upper-half lane rotates here
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const int ch = half * 256 + c + e;
              const int p = ch >= rope_lo ? (ch - rope_lo) >> 1 : 0;
              const float cc = __shfl_sync(~0u, my_c, p);
              const float ss = __shfl_sync(~0u, my_s, p);
              if (ch >= rope_lo) {
                const float x0 = x[e], x1 = x[e + 1];
                x[e] = x0 * cc - x1 * ss;
                x[e + 1] = x0 * ss + x1 * cc;
              }
            }
          }
          uint4 o0 = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]),
                                pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
          uint4 o1 = make_uint4(pack_bf16(x[8], x[9]), pack_bf16(x[10], x[11]),
                                pack_bf16(x[12], x[13]), pack_bf16(x[14], x[15]));
          reinterpret_cast<uint4*>(orow + c)[0] = o0;
          reinterpret_cast<uint4*>(orow + c)[1] = o1;
        }
      }
      g0 += w.j1 - w.j0;
      ++qi;
    }
  }
done:
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Combine the splits of each row: O = sum_s 2^(m_s - M) O_s / (2^(sink - M) + sum_s 2^(m_s - M) l_s)
// with M = max(sink, max_s m_s) over the non-empty splits (all in log2 units), then the rope
// slice turned by -P_t and the bf16 store. Block (row, group of 4 heads); thread (head, chunk)
// owns 8 consecutive channels, so a warp reads 1 KB of one split's partial O contiguously and
// every split's loads are issued before the first is used.
constexpr int kCombineHeads = 4;
__global__ void __launch_bounds__(256) attention_combine_kernel(AttnArgs a) {
  const int64_t r = blockIdx.x;
  const int h = blockIdx.y * kCombineHeads + (threadIdx.x >> 6);
  const int c = (threadIdx.x & 63) * 8;
  const Row w = locate_row(a, r);
  const int splits = a.splits;
  float wgt[kMaxSplits], lsum[kMaxSplits];
  const float sink = __ldg(a.sinks + h) * kLog2e;
  float M = sink;
#pragma unroll
  for (int sp = 0; sp < kMaxSplits; ++sp) {
    wgt[sp] = -INFINITY;
    lsum[sp] = 0.f;
    if (sp < splits &&
        (int64_t)w.tiles * sp / splits < (int64_t)w.tiles * (sp + 1) / splits) {
      const float2 ml =
          __ldcg(reinterpret_cast<const float2*>(a.part_ml) + (r * splits + sp) * kHeads + h);
      wgt[sp] = ml.x;
      lsum[sp] = ml.y;
    }
    M = fmaxf(M, wgt[sp]);
  }
  float L = exp2f(sink - M);
#pragma unroll
  for (int sp = 0; sp < kMaxSplits; ++sp) {
    wgt[sp] = wgt[sp] == -INFINITY ? 0.f : exp2f(wgt[sp] - M);
    L += wgt[sp] * lsum[sp];
  }
  float4 u[kMaxSplits][2];
#pragma unroll
  for (int sp = 0; sp < kMaxSplits; ++sp) {
    if (wgt[sp] > 0.f) {
      const float4* po = reinterpret_cast<const float4*>(
          a.part_o + ((r * splits + sp) * kHeads + h) * kDim + c);
      u[sp][0] = __ldcs(po);
      u[sp][1] = __ldcs(po + 1);
    } else {
      u[sp][0] = u[sp][1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int sp = 0; sp < kMaxSplits; ++sp) {
    const float g = wgt[sp];
    x[0] = fmaf(g, u[sp][0].x, x[0]); x[1] = fmaf(g, u[sp][0].y, x[1]);
    x[2] = fmaf(g, u[sp][0].z, x[2]); x[3] = fmaf(g, u[sp][0].w, x[3]);
    x[4] = fmaf(g, u[sp][1].x, x[4]); x[5] = fmaf(g, u[sp][1].y, x[5]);
    x[6] = fmaf(g, u[sp][1].z, x[6]); x[7] = fmaf(g, u[sp][1].w, x[7]);
  }
  const float inv_l = 1.f / L;
  const int64_t P = a.pos0 + w.t;
  const int rope_lo = kDim - a.rf.R;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float x0 = x[e] * inv_l, x1 = x[e + 1] * inv_l;
    if (c + e >= rope_lo) {
      float cc, ss;
      rope_cos_sin(a.rf, (c + e - rope_lo) >> 1, -P, cc, ss);
      const float y0 = x0 * cc - x1 * ss, y1 = x0 * ss + x1 * cc;
      x0 = y0;
      x1 = y1;
    }
    x[e] = x0;
    x[e + 1] = x1;
  }
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + (r * kHeads + h) * kDim;
  *reinterpret_cast<uint4*>(orow + c) = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]),
                                                   pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}

}  // namespace

int attention_tc_max_splits() { return kMaxSplits; }

bool attention_tc_supported(const AttnArgs& a, int dtype) {
  return dtype == 1 && a.H == kHeads && a.D == kDim && a.rf.R <= 64 && a.rf.R % 2 == 0;
}

cudaError_t launch_attention_tc(const AttnArgs& a, int64_t win_rows, int64_t pool_rows,
                                cudaStream_t st) {
  if (a.nrows == 0) return cudaSuccess;
  CUtensorMap tq, twb, tpb;
  cudaError_t e = make_tmap_bf16_2d(&tq, a.q, (uint64_t)a.nrows * kHeads, kDim, kDim * 2, 64, 64);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16_2d(&twb, a.win.base, (uint64_t)win_rows, kDim, kDim * 2, kNK, 64);
  if (e != cudaSuccess) return e;
  const bool has_pool = a.pool_mode != 0 && pool_rows > 0;
  e = make_tmap_bf16_2d(&tpb, has_pool ? a.pool.base : a.win.base,
                        (uint64_t)(has_pool ? pool_rows : win_rows), kDim, kDim * 2, kNK, 64);
  if (e != cudaSuccess) return e;
  // the same rule as the kernel's any_gather: paged rows or CSA selections are gathered
  const bool win_contig = a.win.block_table == nullptr;
  const bool pool_contig = a.pool_mode == 1 && a.pool.block_table == nullptr;
  const bool any_gather = !win_contig || (a.pool_mode != 0 && !pool_contig);
  const void* kern = a.splits > 1 ? (any_gather ? (const void*)attention_tc_kernel<true, kThreads>
                                                : (const void*)attention_tc_kernel<true, kThreadsTma>)
                                  : (any_gather ? (const void*)attention_tc_kernel<false, kThreads>
                                                : (const void*)attention_tc_kernel<false, kThreadsTma>);
  e = ensure_smem_limit(kern, kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (a.splits < 1 || a.splits > kMaxSplits || (a.splits > 1 && (!a.part_o || !a.part_ml)))
    return cudaErrorInvalidValue;
  const int64_t items = a.nrows * a.splits;
  const int grid = (int)(items < sms ? items : sms);
  if (a.splits > 1) {
    if (any_gather)
      attention_tc_kernel<true, kThreads><<<grid, kThreads, kSmemBytes, st>>>(tq, twb, tpb, a);
    else
      attention_tc_kernel<true, kThreadsTma><<<grid, kThreadsTma, kSmemBytes, st>>>(tq, twb, tpb, a);
  } else {
    if (any_gather)
      attention_tc_kernel<false, kThreads><<<grid, kThreads, kSmemBytes, st>>>(tq, twb, tpb, a);
    else
      attention_tc_kernel<false, kThreadsTma><<<grid, kThreadsTma, kSmemBytes, st>>>(tq, twb, tpb,
                                                                                    a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || a.splits == 1) return e;
  attention_combine_kernel<<<dim3((unsigned)a.nrows, kHeads / kCombineHeads), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sac
