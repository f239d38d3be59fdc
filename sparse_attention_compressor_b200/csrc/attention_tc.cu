// Tensor-core (tcgen05) version of the shared K=V multi-query attention for bf16 layers with
// 64 query heads and head_dim 512 ("Hybrid attention": shared K=V MQA; per-head sink, eq. 27;
// partial RoPE with the -i output rotation, eq. 26; sliding-window branch + compressor entries).
//
// One query row at a time per CTA (persistent over rows). Both contractions put the 128 keys of a
// tile, or the 128 channels of a dimension block, on the MMA's M = 128 side and the 64 heads on
// N = 64, so every MMA runs at the full tcgen05 rate (an M = 64 MMA of the heads would run at
// half of it):
//   S^T[key, head]  = K[128 keys x 512] . Q^T                  (M = 128, N = 64, K = 512)
//   O^T[dim, head] += V^T[128 dims x 128 keys] . P^T[keys, heads]  per block of 128 dims
//                                                              (M = 128, N = 64, K = 128)
// Because K = V, one key tile in shared memory is the K-major A operand of the first product and
// the MN-major A operand of the second. It is held as four 32 KB dimension blocks ("pairs": two
// 128-byte swizzle columns of 64 channels); the next tile refills a pair as soon as the PV MMAs of
// its block have completed, so the loads of tile g+1 overlap the end of tile g.
//
// MMA issue: one thread issuing a chain of MMAs into the same accumulator keeps them pipelined,
// while switching accumulators between consecutive MMAs of one thread drains the pipe (measured:
// ~55 vs ~220 cycles per M = 128, N = 64 MMA), and two chains already reach the shared-memory
// operand rate (~48 cycles per MMA). So issuers 0 and 1 each compute one partial of S^T over two
// dimension blocks (16 K-steps, accumulator S_c), the softmax adds the two, and issuer i adds
// V^T P^T of dimension block i into O^T block i (8 K-steps of 16 keys).
//
// Tensor memory (512 columns, fp32): O^T block i at columns 64i (128 lanes = 128 channels), S_c at
// 256 + 64c.
//
// Softmax: thread = key (TMEM lane) for 32 of the heads, two warps per TMEM sub-partition; per-head
// running max in shared memory, moved only when a tile's logit exceeds it by more than 2^8 (log2
// units), which a vote of the softmax threads detects; then the exact per-head tile max is taken
// with warp shuffles and O^T is rescaled in TMEM. The normaliser's per-head sums over keys are
// reduce-scattered across each warp with shuffles (lane i keeps one head) and summed over the
// four sub-partitions at the end of the row.
//
// Warps: 0 = TMA producer (query, contiguous key tiles), 1-4 = MMA issuers (warp 1 owns TMEM),
// 5 = query rotation, 6-7 and 16-19 = gather group for tiles whose rows are not consecutive (CSA
// selections, paged caches; idle when every tile arrives by TMA), 8-15 = softmax and output. The
// softmax warpgroups take registers from the others (setmaxnreg).
#include <cuda_bf16.h>

#include "launch_util.h"
#include "sac_kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace sac {
namespace {

constexpr int kHeads = 64;
constexpr int kDim = 512;
constexpr int kNK = 128;                         // keys per tile (MMA M of S^T)
constexpr int kPairs = kDim / 128;               // dimension blocks of a key tile
static_assert(kPairs == 4, "the gather hands over four commit groups");
constexpr int kRegion = kNK * 128;               // 16 KB: 128 keys x 64 channels, 128-B rows
constexpr int kPairBytes = 2 * kRegion;          // 32 KB: one dimension block
constexpr int kQRegion = kHeads * 128;           // 8 KB: 64 heads x 64 channels
constexpr int kQBytes = 8 * kQRegion;            // 64 KB
constexpr int kPBytes = kNK * 128;               // 16 KB: P^T, 128 keys x 64 heads
constexpr int kThreads = 640;                    // 20 warps (five warpgroups)
constexpr int kGroupThreads = 192;               // the gather group: warps 6-7 and 16-19
// Registers: the block launches with 96 a thread; the two softmax warpgroups (8-15) raise theirs
// to 128, warpgroups 0-1 (producer, issuers, rotation, two gather warps) lower theirs to 80 and
// warpgroup 4 (gather only) to 64 (setmaxnreg), which the launch's total covers exactly:
// 2 x 128 x 128 + 2 x 128 x 80 + 128 x 64 = 61440 = 640 x 96.
constexpr int kRegsLaunch = 96, kRegsSoftmax = 128, kRegsOther = 80, kRegsGather = 64;
static_assert(2 * 128 * kRegsSoftmax + 2 * 128 * kRegsOther + 128 * kRegsGather <=
                  kThreads * kRegsLaunch,
              "register split above the launch's registers");
constexpr int kIssuers = kPairs;                 // MMA issuer threads, one per dimension block
constexpr int kSoftmaxWarp0 = 8;                 // warps 8-15: softmax and output
constexpr int kSoftmaxThreads = 256;
constexpr int kQkChains = 2;                     // S^T partial accumulators (2 or 4)
static_assert(kQkChains == 2 || kQkChains == 4, "S^T partials: two or four chains");

constexpr int kOffQ = 0;
constexpr int kOffPair = kOffQ + kQBytes;
constexpr int kOffP = kOffPair + kPairs * kPairBytes;
constexpr int kOffM = kOffP + kPBytes;           // [64] running max per head (log2 units)
constexpr int kOffAlpha = kOffM + 256;           // [64] rescale factors of a moved max
constexpr int kOffL = kOffAlpha + 256;           // [64] normaliser of the output
constexpr int kOffWmax = kOffL + 256;            // [4][64] per-sub-partition maxima / normalisers
constexpr int kOffCs = kOffWmax + 1024;          // [32] (cos, sin) of the query's rope pairs
constexpr int kOffBar = kOffCs + 32 * 8;
enum Bar { kQFull, kQReady, kQEmpty, kPairFull0, kPairEmpty0 = kPairFull0 + kPairs,
           kSFull = kPairEmpty0 + kPairs, kSEmpty, kPFull, kOFull, kOEmpty, kNumBars };
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffTmemPtr + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

constexpr uint32_t kColO = 0, kColS = 256;       // O^T block i at 64 i, S^T partial c at 256 + 64 c
constexpr uint32_t kIdescQK = tc::idesc_bf16(128, kHeads, false, false);
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, kHeads, true, true);
constexpr int kMaxSplits = 8;  // key-tile splits of one row (decode: few rows, many SMs)
constexpr int kRopeStep = 28;  // K-steps 28..31 read the last region of Q (the rope slice)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;  // move the running max only when a tile exceeds it by 2^8
constexpr int kSoftmaxBar = 1; // named barrier of the 128 softmax threads

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

// keys of tile j of a row
__device__ __forceinline__ int tile_keys(const Row& w, int j) {
  return j < w.twin ? min(kNK, w.nwin - j * kNK) : min(kNK, w.npool - (j - w.twin) * kNK);
}

__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

__device__ __forceinline__ void bar_sync_softmax() {
  asm volatile("barrier.sync %0, %1;" ::"r"(kSoftmaxBar), "r"(kSoftmaxThreads) : "memory");
}
// true on every softmax thread when v is true on any of them
__device__ __forceinline__ bool bar_any_softmax(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(kSoftmaxBar), "r"(kSoftmaxThreads)
      : "memory");
  return r != 0;
}

// Reduce-scatter of 32 per-head values over the 32 lanes of a warp (sum, or max with kMax):
// each step keeps the half of the heads that one lane bit selects and combines it with the
// partner lane's copy, so after five steps lane l holds head l. v is left unchanged.
template <bool kMax>
__device__ __forceinline__ float reduce_scatter32(const float (&v)[32], int lane) {
  float t[16];
  const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4, u2 = lane & 2, u1 = lane & 1;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float keep = u16 ? v[e + 16] : v[e];
    const float recv = __shfl_xor_sync(~0u, u16 ? v[e] : v[e + 16], 16);
    t[e] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float keep = u8 ? t[e + 8] : t[e];
    const float recv = __shfl_xor_sync(~0u, u8 ? t[e] : t[e + 8], 8);
    t[e] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float keep = u4 ? t[e + 4] : t[e];
    const float recv = __shfl_xor_sync(~0u, u4 ? t[e] : t[e + 4], 4);
    t[e] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float keep = u2 ? t[e + 2] : t[e];
    const float recv = __shfl_xor_sync(~0u, u2 ? t[e] : t[e + 2], 2);
    t[e] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
  const float keep = u1 ? t[1] : t[0];
  const float recv = __shfl_xor_sync(~0u, u1 ? t[0] : t[1], 1);
  return kMax ? fmaxf(keep, recv) : keep + recv;
}

// Wait on an mbarrier phase from the 256 softmax threads. The group meets at named barriers, so
// whether the wait timed out is decided for the whole group: if any thread gave up, all do.
__device__ __forceinline__ bool softmax_wait(uint64_t* bar, uint32_t parity, int* status) {
  return !bar_any_softmax(!tc::mbar_wait(bar, parity, status));
}

// Global addresses of keys c0 + stride * i (i < N) of tile j. Keys past the tile's count reuse a
// valid row (the softmax masks them); an unallocated page reads its buffer's first row. Each level
// of index loads (the CSA selection, then the block table) is issued for all N keys before any is
// used, so a tile's addresses cost two memory latencies at most, not two per key.
template <int N>
__device__ __forceinline__ void key_ptrs(const AttnArgs& a, const Row& w, int j, int c0,
                                         int stride, const __nv_bfloat16* (&src)[N]) {
  const bool is_win = j < w.twin;
  uint32_t lr[N];  // row of the key in its sequence's stream (window row or pool entry)
  if (is_win) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      int x = j * kNK + min(c0 + stride * i, kNK - 1);
      if (x >= w.nwin) x = 0;
      lr[i] = (uint32_t)(w.lo + x);
    }
  } else {
    int e[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
      int x = (j - w.twin) * kNK + min(c0 + stride * i, kNK - 1);
      if (x >= w.npool) x = 0;
      e[i] = a.pool_mode == 2 ? __ldg(a.sel + w.r * a.k + x) : x;
    }
#pragma unroll
    for (int i = 0; i < N; ++i) lr[i] = (uint32_t)(e[i] < 0 ? 0 : e[i]);
  }
  const RowAddr& ra = is_win ? a.win : a.pool;
  const __nv_bfloat16* base = reinterpret_cast<const __nv_bfloat16*>(ra.base);
  if (ra.block_table == nullptr) {
#pragma unroll
    for (int i = 0; i < N; ++i) src[i] = base + ((int64_t)w.seq * ra.seq_stride + lr[i]) * kDim;
    return;
  }
  const uint32_t ps = (uint32_t)ra.page_size;
  const int32_t* bt = ra.block_table + (int64_t)w.seq * ra.max_pages;
  int pg[N];
#pragma unroll
  for (int i = 0; i < N; ++i) pg[i] = __ldg(bt + lr[i] / ps);
#pragma unroll
  for (int i = 0; i < N; ++i)
    src[i] = pg[i] < 0 ? base : base + ((int64_t)pg[i] * ps + lr[i] % ps) * kDim;
}

// The gather group: 192 threads (warps 6-7 and 16-19; gt = the thread's index in the group) fill
// the tiles whose rows are not consecutive. Thread gt copies 16-byte slot gt % 8 of key rows
// gt / 8 + 24 i of both 64-channel regions of a dimension block, so a warp instruction reads four
// whole 128-byte row segments. A tile's row addresses are resolved before the wait for its first
// block (they overlap the previous tile's work); its four blocks are issued in order as soon as
// each is free, all four in flight at once, and handed over in order as their copies land. The
// pair barriers count this group's threads for every tile, so it also arrives for tiles that TMA
// fills (after the same wait for the block to be free): each party waits for every phase, so no
// parity wait can name a phase other than the one it means.
template <bool kSplit>
__device__ __forceinline__ void gather_tiles(const AttnArgs& a, uint8_t* smem, uint64_t* bar,
                                             int64_t n_items, bool win_contig, bool pool_contig,
                                             int gt, int* status) {
  const int row0 = gt >> 3, slot = gt & 7;
  constexpr int kRowStride = kGroupThreads / 8;                     // 24
  constexpr int kRowsPer = (kNK + kRowStride - 1) / kRowStride;     // 6 (the last only row0 < 8)
  uint32_t g = 0;
  bool ok = true;
  for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
    const Row w = locate_item<kSplit>(a, it);
    if (w.j0 == w.j1) continue;
    for (int j = w.j0; j < w.j1 && ok; ++j, ++g) {
      const bool gath = !(j < w.twin ? win_contig : pool_contig);
      const __nv_bfloat16* src[kRowsPer];
      if (gath) key_ptrs<kRowsPer>(a, w, j, row0, kRowStride, src);
#pragma unroll
      for (int b = 0; b < kPairs; ++b) {
        if (g > 0) ok = __all_sync(~0u, tc::mbar_wait(&bar[kPairEmpty0 + b], (g - 1) & 1, status));
        if (!ok) break;
        if (!gath) {
          tc::mbar_arrive(&bar[kPairFull0 + b]);
          continue;
        }
        uint8_t* pr = smem + kOffPair + b * kPairBytes;
#pragma unroll
        for (int i = 0; i < kRowsPer; ++i) {
          const int row = row0 + kRowStride * i;
          if (row < kNK) {
            uint8_t* d = pr + row * 128 + ((slot ^ (row & 7)) << 4);
            tc::cp_async16(d, src[i] + 128 * b + slot * 8);
            tc::cp_async16(d + kRegion, src[i] + 128 * b + 64 + slot * 8);
          }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      if (!ok || !gath) continue;
      // the four blocks' copies are all in flight (one commit group each, so the latency of the
      // loads is paid once per tile): hand each block over as its group lands, in order
      asm volatile("cp.async.wait_group 3;" ::: "memory");
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[kPairFull0 + 0]);
      asm volatile("cp.async.wait_group 2;" ::: "memory");
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[kPairFull0 + 1]);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[kPairFull0 + 2]);
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[kPairFull0 + 3]);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

template <bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
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
  const int64_t n_items = kSplit ? a.nrows * a.splits : a.nrows;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bar[kQFull], 1);
    tc::mbar_init(&bar[kQReady], 32);
    tc::mbar_init(&bar[kQEmpty], kQkChains);
    for (int b = 0; b < kPairs; ++b) {
      // the TMA thread's arrival (with the bytes of a box load), and with gathered tiles also
      // every gather thread's
      tc::mbar_init(&bar[kPairFull0 + b], any_gather ? 1 + kGroupThreads : 1);
      tc::mbar_init(&bar[kPairEmpty0 + b], 1);
    }
    tc::mbar_init(&bar[kSFull], kQkChains);
    tc::mbar_init(&bar[kSEmpty], kSoftmaxThreads);
    tc::mbar_init(&bar[kPFull], kSoftmaxThreads);
    tc::mbar_init(&bar[kOFull], kIssuers);
    tc::mbar_init(&bar[kOEmpty], kSoftmaxThreads);
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

  // Register split by warpgroup: the two softmax warpgroups raise theirs, the other three lower
  // theirs, each warpgroup at one instruction before its warps take their roles.
  if (warp >= kSoftmaxWarp0 && warp < kSoftmaxWarp0 + 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ------------------------------------------------------------------ softmax + output
    // Warp 8 + 4 hh + sp: keys 32 sp .. 32 sp + 31 of the tile (its TMEM lanes) and heads
    // 32 hh .. 32 hh + 31, so each sub-partition has two softmax warps.
    const int sp = warp & 3;                  // TMEM sub-partition of this warp
    const int h0 = 32 * ((warp - kSoftmaxWarp0) >> 2);  // first head of this warp
    const int tid = threadIdx.x - 32 * kSoftmaxWarp0;  // 0..255
    const int key = 32 * sp + lane;           // key of the tile (TMEM lane) / channel in a block
    const uint32_t t_lane = tmem + ((uint32_t)(32 * sp) << 16);
    float* m_sm = reinterpret_cast<float*>(smem + kOffM);
    float* alpha_sm = reinterpret_cast<float*>(smem + kOffAlpha);
    float* l_sm = reinterpret_cast<float*>(smem + kOffL);
    float* wred_sm = reinterpret_cast<float*>(smem + kOffWmax);
    uint8_t* prow = smem + kOffP + key * 128;
    const float scale_log2 = a.scale * kLog2e;
    const int h_mine = h0 + lane;  // the head whose sums this lane keeps after a reduce-scatter
    uint32_t g = 0, qi = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const Row w = locate_item<kSplit>(a, it);
      if (w.j0 == w.j1) continue;
      // running max per head: starts at the sink logit (unsplit rows) or -inf (splits, whose
      // combine adds the sink); O^T starts fresh with the item's first PV
      if (tid < kHeads) m_sm[tid] = kSplit ? -INFINITY : __ldg(a.sinks + tid) * kLog2e;
      float l_acc = 0.f;  // this warp's sum of p for head h_mine
      bar_sync_softmax();
      for (int j = w.j0; j < w.j1 && ok; ++j, ++g) {
        const bool first = j == w.j0;
        ok = softmax_wait(&bar[kSFull], g & 1, status);
        if (!ok) break;
        tc::tc_fence_after();
        const bool valid = key < tile_keys(w, j);
        float x[32];
#pragma unroll
        for (int c = 0; c < kQkChains; c += 2) {  // the partials of S^T, two per TMEM round trip
          uint32_t va[32], vb[32];
          tc::tmem_ld32(t_lane + kColS + 64 * c + h0, va);
          tc::tmem_ld32(t_lane + kColS + 64 * (c + 1) + h0, vb);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float v = __uint_as_float(va[e]) + __uint_as_float(vb[e]);
            x[e] = c == 0 ? v : x[e] + v;
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = valid ? x[e] * scale_log2 : -INFINITY;
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[kSEmpty]);
        // The running max: on a row's first tile it is set from the exact per-head tile max (the
        // sink as the floor); later it moves only for heads whose logits exceed it by the lazy
        // margin, which a vote of the softmax threads detects first.
        bool exceed = first;
        if (!first) {
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(m_sm + h0 + c);
            exceed |= (x[c] > m4.x + kLazy) | (x[c + 1] > m4.y + kLazy) |
                      (x[c + 2] > m4.z + kLazy) | (x[c + 3] > m4.w + kLazy);
          }
        }
        if (first || bar_any_softmax(exceed)) {
          // per-head maximum over this warp's 32 keys by reduce-scatter (lane i keeps head
          // h0 + i), then over the four sub-partitions
          wred_sm[sp * kHeads + h_mine] = reduce_scatter32<true>(x, lane);
          bar_sync_softmax();
          if (tid < kHeads) {
            const float tm = fmaxf(fmaxf(wred_sm[tid], wred_sm[kHeads + tid]),
                                   fmaxf(wred_sm[2 * kHeads + tid], wred_sm[3 * kHeads + tid]));
            const float old = m_sm[tid];
            const float nm = first ? fmaxf(old, tm) : (tm > old + kLazy ? tm : old);
            alpha_sm[tid] = first ? 1.f : tc::exp2_approx(old - nm);
            m_sm[tid] = nm;
          }
          bar_sync_softmax();
          if (!first) {
            l_acc *= alpha_sm[h_mine];
            // rescale this thread's channel row of every O^T block by alpha per head (this
            // warp's 32 heads); PV of the previous tile has completed: its commit preceded this
            // tile's S commits
#pragma unroll 1
            for (int blk = 0; blk < kPairs; ++blk) {
#pragma unroll
              for (int c = 0; c < 32; c += 16) {
                uint32_t v[16];
                tc::tmem_ld16(t_lane + kColO + 64 * blk + h0 + c, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                  v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha_sm[h0 + c + e]);
                tc::tmem_st16(t_lane + kColO + 64 * blk + h0 + c, v);
              }
            }
            tc::tmem_wait_st();
          }
        }
        // P^T row of this key: 64 heads of bf16 in one 128-byte swizzled row, of which this warp
        // writes 16-byte chunks 4 hh .. 4 hh + 3. The buffer is free: this tile's S came from keys
        // that refilled every dimension block after the previous tile's PV of that block had
        // completed (the pair barriers), so every PV MMA that read the previous P has finished;
        // the same ordering covers the rescale of O^T above.
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const float4 ma = *reinterpret_cast<const float4*>(m_sm + h0 + 8 * ch);
          const float4 mb = *reinterpret_cast<const float4*>(m_sm + h0 + 8 * ch + 4);
          float* xs = x + 8 * ch;
          xs[0] = tc::exp2_approx(xs[0] - ma.x); xs[1] = tc::exp2_approx(xs[1] - ma.y);
          xs[2] = tc::exp2_approx(xs[2] - ma.z); xs[3] = tc::exp2_approx(xs[3] - ma.w);
          xs[4] = tc::exp2_approx(xs[4] - mb.x); xs[5] = tc::exp2_approx(xs[5] - mb.y);
          xs[6] = tc::exp2_approx(xs[6] - mb.z); xs[7] = tc::exp2_approx(xs[7] - mb.w);
          const uint4 pk = make_uint4(pack_bf16(xs[0], xs[1]), pack_bf16(xs[2], xs[3]),
                                      pack_bf16(xs[4], xs[5]), pack_bf16(xs[6], xs[7]));
          const int chunk = (h0 >> 3) + ch;
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (key & 7)) << 4)) = pk;
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[kPFull]);
        // per-head sums of p over this warp's 32 keys (reduce-scatter: lane i keeps head h0 + i)
        l_acc += reduce_scatter32<false>(x, lane);
      }
      if (!ok) break;
      // ---- output of the item: the normaliser per head from the four sub-partitions' sums
      wred_sm[sp * kHeads + h_mine] = l_acc;
      bar_sync_softmax();
      if (tid < kHeads)
        l_sm[tid] = (wred_sm[tid] + wred_sm[kHeads + tid]) +
                    (wred_sm[2 * kHeads + tid] + wred_sm[3 * kHeads + tid]);
      ok = softmax_wait(&bar[kOFull], qi & 1, status);
      if (!ok) break;
      tc::tc_fence_after();
      if (kSplit) {
        // this item's O (relative to its running max), max and normaliser in fp32 for the
        // combine kernel: thread = channel of each block, this warp's 32 heads; the four blocks'
        // columns of one group of 16 heads are loaded together (one TMEM round trip per group)
        float* po = a.part_o + (int64_t)it * kHeads * kDim + key;
#pragma unroll 1
        for (int c = h0; c < h0 + 32; c += 16) {
          uint32_t v[kPairs][16];
#pragma unroll
          for (int blk = 0; blk < kPairs; ++blk) tc::tmem_ld16(t_lane + kColO + 64 * blk + c, v[blk]);
          tc::tmem_wait_ld();
          if (c + 16 == h0 + 32) {
            tc::tc_fence_before();
            tc::mbar_arrive(&bar[kOEmpty]);
          }
#pragma unroll
          for (int blk = 0; blk < kPairs; ++blk)
#pragma unroll
            for (int e = 0; e < 16; ++e)
              __stcg(po + (int64_t)(c + e) * kDim + 128 * blk, __uint_as_float(v[blk][e]));
        }
        if (tid < kHeads)
          *reinterpret_cast<float2*>(a.part_ml + ((int64_t)it * kHeads + tid) * 2) =
              make_float2(m_sm[tid], l_sm[tid]);
        bar_sync_softmax();  // m_sm, l_sm and the warp sums are rewritten by the next item
        ++qi;
        continue;
      }
      // O / (l + sink term), the rope slice turned by -P_t, bf16. A lane pair (2i, 2i+1) holds
      // channels d, d+1: after exchanging halves the even lane stores heads c..c+7 and the odd
      // lane heads c+8..c+15 of each group of 16, as bf16 pairs (64 contiguous bytes per warp and
      // head). The four blocks' columns of one group of 16 heads are loaded together.
      if (tid < kHeads)
        l_sm[tid] = 1.f / (l_sm[tid] + tc::exp2_approx(__ldg(a.sinks + tid) * kLog2e - m_sm[tid]));
      bar_sync_softmax();
      const int64_t P = a.pos0 + w.t;
      const int rope_lo = kDim - a.rf.R;  // first rotated channel
      __nv_bfloat16* obase = reinterpret_cast<__nv_bfloat16*>(a.o) + w.r * kHeads * kDim;
      const int odd = lane & 1;
      // only the last block can hold rope channels (R <= 64 < 128)
      const int d3 = 128 * (kPairs - 1) + key - odd;  // even channel of the pair in the last block
      const bool rot = d3 >= rope_lo;                 // the same for both lanes of a pair
      float cc = 1.f, ss = 0.f;
      if (rot) rope_cos_sin(a.rf, (d3 - rope_lo) >> 1, -P, cc, ss);
#pragma unroll 1
      for (int c = h0; c < h0 + 32; c += 16) {
        uint32_t v[kPairs][16];
#pragma unroll
        for (int blk = 0; blk < kPairs; ++blk) tc::tmem_ld16(t_lane + kColO + 64 * blk + c, v[blk]);
        tc::tmem_wait_ld();
        if (c + 16 == h0 + 32) {
          tc::tc_fence_before();
          tc::mbar_arrive(&bar[kOEmpty]);
        }
#pragma unroll
        for (int blk = 0; blk < kPairs; ++blk) {
          float y[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = __uint_as_float(v[blk][e]) * l_sm[c + e];
          if (blk == kPairs - 1) {
            // rope channels: each lane turns its own coordinate of (x0, x1) = (even, odd), with the
            // partner lane's value of the pair (the same decision for both lanes of a pair)
            float z[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) z[e] = __shfl_xor_sync(~0u, y[e], 1);
            if (rot) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float x0 = odd ? z[e] : y[e], x1 = odd ? y[e] : z[e];
                y[e] = odd ? x0 * ss + x1 * cc : x0 * cc - x1 * ss;
              }
            }
          }
          // pack heads (h, h+1) of this channel into one bf16 pair, swap packed words with the
          // partner lane: the even lane then holds head h of channels (d0, d0+1), the odd lane head
          // h+1 of them, each one 4-byte store
          const int d0 = 128 * blk + key - odd;
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const uint32_t mine = pack_bf16(y[e], y[e + 1]);
            const uint32_t theirs = __shfl_xor_sync(~0u, mine, 1);
            const uint32_t word = odd ? __byte_perm(theirs, mine, 0x7632)
                                      : __byte_perm(mine, theirs, 0x5410);
            *reinterpret_cast<uint32_t*>(obase + (int64_t)(c + e + odd) * kDim + d0) = word;
          }
        }
      }
      bar_sync_softmax();  // m_sm, l_sm and the warp sums are rewritten by the next item
      ++qi;
    }
  } else if (warp >= kSoftmaxWarp0 + 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsGather));
    if (any_gather)
      gather_tiles<kSplit>(a, smem, bar, n_items, win_contig, pool_contig,
                           64 + (warp - kSoftmaxWarp0 - 8) * 32 + lane, status);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        uint32_t g = 0, qi = 0;
        bool ok = true;
        for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
          const Row w = locate_item<kSplit>(a, it);
          if (w.bad && status) atomicExch(status, tc::kStatusBadInput);
          if (w.j0 == w.j1) continue;
          if (qi > 0) ok = tc::mbar_wait(&bar[kQEmpty], (qi - 1) & 1, status);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(&bar[kQFull], kQBytes);
          for (int c = 0; c < 8; ++c)
            tc::tma_load_2d(smem + kOffQ + c * kQRegion, &tm_q, &bar[kQFull], 64 * c,
                            (int32_t)(w.r * kHeads));
          for (int j = w.j0; j < w.j1 && ok; ++j, ++g) {
            const bool is_win = j < w.twin;
            const bool contig = is_win ? win_contig : pool_contig;
            const int64_t y0 = contig ? (is_win ? a.win.row_index(w.seq, w.lo + (int64_t)j * kNK)
                                                : a.pool.row_index(w.seq, (int64_t)(j - w.twin) * kNK))
                                      : 0;
            const CUtensorMap* map = is_win ? &tm_win_box : &tm_pool_box;
            for (int b = 0; b < kPairs && ok; ++b) {
              if (g > 0) ok = tc::mbar_wait(&bar[kPairEmpty0 + b], (g - 1) & 1, status);
              if (!ok) break;
              if (!contig) {  // the gather group fills this block
                tc::mbar_arrive(&bar[kPairFull0 + b]);
                continue;
              }
              uint8_t* dst = smem + kOffPair + b * kPairBytes;
              tc::mbar_arrive_expect_tx(&bar[kPairFull0 + b], kPairBytes);
              tc::tma_load_2d(dst, map, &bar[kPairFull0 + b], 128 * b, (int32_t)y0);
              tc::tma_load_2d(dst + kRegion, map, &bar[kPairFull0 + b], 128 * b + 64, (int32_t)y0);
            }
          }
          ++qi;
        }
      }
      __syncwarp();
    } else if (warp >= 1 && warp <= kIssuers) {
      // ------------------------------------------------------------------ MMA issuers
      // Issuers 0 and 1: S^T partial c = K[:, blocks 2c, 2c+1] Q[:, same channels]^T (16 K-steps,
      // each block as soon as it has arrived). Every issuer i then adds V^T P^T of dimension block i
      // to O^T block i (8 steps of 16 keys). Each chain stays on one accumulator.
      const int bi = warp - 1;
      if (lane == 0) {
        uint32_t g = 0, qi = 0;
        bool ok = true;
        const uint32_t q_base = tc::smem_u32(smem + kOffQ);
        const uint32_t pairs = tc::smem_u32(smem + kOffPair);
        const uint64_t p_desc = tc::desc_sw128(tc::smem_u32(smem + kOffP), 0, 1024);
        const uint32_t s_acc = tmem + kColS + 64 * bi, o_acc = tmem + kColO + 64 * bi;
        const bool qk = bi < kQkChains;
        for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
          const Row w = locate_item<kSplit>(a, it);
          if (w.j0 == w.j1) continue;
          if (qk) ok = tc::mbar_wait(&bar[kQFull], qi & 1, status);
          for (int j = w.j0; j < w.j1 && ok; ++j, ++g) {
            const bool first = j == w.j0, last = j == w.j1 - 1;
            if (qk) {
              // ---- S^T partial bi over dimension blocks 2 bi and 2 bi + 1
              if (g > 0) ok = tc::mbar_wait(&bar[kSEmpty], (g - 1) & 1, status);
              for (int h = 0; h < kPairs / kQkChains && ok; ++h) {
                const int pb = (kPairs / kQkChains) * bi + h;
                ok = tc::mbar_wait(&bar[kPairFull0 + pb], g & 1, status);
                if (!ok) break;
                tc::tc_fence_after();
  #pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  // the rope slice of Q (K-steps 28..31, the last block) is rotated in place before
                  // the row's first tile reads it
                  if (first && 8 * pb + kk == kRopeStep) {
                    ok = tc::mbar_wait(&bar[kQReady], qi & 1, status);
                    if (!ok) break;
                    tc::tc_fence_after();
                  }
                  const uint32_t off =
                      (uint32_t)(pb * kPairBytes + (kk >> 2) * kRegion + (kk & 3) * 32);
                  const uint32_t qoff = (uint32_t)((2 * pb + (kk >> 2)) * kQRegion + (kk & 3) * 32);
                  tc::mma_bf16_ss(s_acc, tc::desc_sw128(pairs + off, 0, 1024),
                                  tc::desc_sw128(q_base + qoff, 0, 1024), kIdescQK,
                                  (h > 0 || kk > 0) ? 1u : 0u);
                }
              }
              if (!ok) break;
              tc::mma_commit(&bar[kSFull]);
              if (last) tc::mma_commit(&bar[kQEmpty]);
            }
            // ---- O^T block bi += V^T P^T once the softmax has written P (block bi has arrived:
            // this wait names the phase the S chains already saw complete)
            ok = tc::mbar_wait(&bar[kPFull], g & 1, status);
            if (ok) ok = tc::mbar_wait(&bar[kPairFull0 + bi], g & 1, status);
            if (ok && first && qi > 0) ok = tc::mbar_wait(&bar[kOEmpty], (qi - 1) & 1, status);
            if (!ok) break;
            tc::tc_fence_after();
            const uint32_t pair = pairs + bi * kPairBytes;
  #pragma unroll
            for (int kk = 0; kk < kNK / 16; ++kk)
              tc::mma_bf16_ss(o_acc, tc::desc_sw128(pair + kk * 2048, kRegion, 1024),
                              p_desc + (uint64_t)(kk * 2048 >> 4), kIdescPV,
                              (first && kk == 0) ? 0u : 1u);
            tc::mma_commit(&bar[kPairEmpty0 + bi]);
            if (last) tc::mma_commit(&bar[kOFull]);
          }
          ++qi;
        }
      }
      __syncwarp();
    } else if (warp == kIssuers + 1) {
      // ------------------------------------------------------------------ query rotation
      // Lane p first writes (cos, sin) of rope pair p at the query's position to a shared table.
      // Then thread i turns the rope pairs of head rows i and i+32 of the staged query tile (row h's
      // 16-byte chunk c of a 128-byte region sits at chunk c ^ (h & 7)).
      const int R = a.rf.R;
      const int p0 = (kDim - R) >> 1;  // first rotated pair among the 256 channel pairs
      float2* cs_tab = reinterpret_cast<float2*>(smem + kOffCs);
      uint32_t qi = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const Row w = locate_item<kSplit>(a, it);
        if (w.j0 == w.j1) continue;
        if (lane < R / 2) {
          float c, sn;
          rope_cos_sin(a.rf, lane, a.pos0 + w.t, c, sn);
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
    } else if (warp == 6 || warp == 7) {
      if (any_gather)
        gather_tiles<kSplit>(a, smem, bar, n_items, win_contig, pool_contig, (warp - 6) * 32 + lane,
                             status);
    }
  }
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
  // a paged cache's block table addresses its page buffer, whose extent the call does not carry:
  // its maps span every 32-bit row coordinate (the gathers read only the rows the table names)
  constexpr int64_t kPagedRows = (int64_t(1) << 31) - 1;
  if (a.win.block_table) win_rows = kPagedRows;
  if (a.pool_mode != 0 && a.pool.block_table) pool_rows = kPagedRows;
  CUtensorMap tq, twb, tpb;
  cudaError_t e = make_tmap_bf16_2d(&tq, a.q, (uint64_t)a.nrows * kHeads, kDim, kDim * 2, 64, 64);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16_2d(&twb, a.win.base, (uint64_t)win_rows, kDim, kDim * 2, kNK, 64);
  if (e != cudaSuccess) return e;
  const bool has_pool = a.pool_mode != 0 && pool_rows > 0;
  e = make_tmap_bf16_2d(&tpb, has_pool ? a.pool.base : a.win.base,
                        (uint64_t)(has_pool ? pool_rows : win_rows), kDim, kDim * 2, kNK, 64);
  if (e != cudaSuccess) return e;
  const void* kern = a.splits > 1 ? (const void*)attention_tc_kernel<true>
                                  : (const void*)attention_tc_kernel<false>;
  e = ensure_smem_limit(kern, kSmemBytes);
  if (e != cudaSuccess) return e;
  // the register split needs the block launched with kRegsLaunch registers a thread: with fewer,
  // the softmax warpgroups' raise would wait for registers that never come
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < kRegsLaunch) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (a.splits < 1 || a.splits > kMaxSplits || (a.splits > 1 && (!a.part_o || !a.part_ml)))
    return cudaErrorInvalidValue;
  const int64_t items = a.nrows * a.splits;
  const int grid = (int)(items < sms ? items : sms);
  if (a.splits > 1)
    attention_tc_kernel<true><<<grid, kThreads, kSmemBytes, st>>>(tq, twb, tpb, a);
  else
    attention_tc_kernel<false><<<grid, kThreads, kSmemBytes, st>>>(tq, twb, tpb, a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.splits == 1) return e;
  attention_combine_kernel<<<dim3((unsigned)a.nrows, kHeads / kCombineHeads), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sac
