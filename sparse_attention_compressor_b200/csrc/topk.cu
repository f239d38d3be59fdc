// Indexer top-k ("Hybrid attention", CSA bullet, eq. 17; "Attention mask layout", CSA
// paragraph): per query row, the k largest of the (t+1)//m visible scores, ties going to the
// lower entry index; empty slots (fewer than k visible) hold -1.
//
// One block per row; scores become order-preserving uint32 keys (kept in shared memory for short
// rows, re-read from L2 by every pass for long ones).
// The exact k-th largest key T is found by a radix select on digits of 12, 12 and 8 bits. The
// first digit (sign, exponent and 3 mantissa bits) spreads real score distributions over many
// bins, so the histogram atomics rarely collide; the keys in the bin that holds T (usually a few
// hundred) are compacted and the two finer digits only visit them. Every digit is located with a
// block-wide scan of the histogram rather than a serial walk. Each warp owns a contiguous segment
// of the row; the output keeps every key > T plus the first (k - #{key > T}) keys == T in index
// order. For rows of at most kMapEntries scores the compaction pass also records, one ballot word
// per 32 entries, which keys lie above the threshold bin; the candidates then add theirs (> T, and
// == T in a second map), and the ordered output walks these bit maps (one word per 32 entries)
// instead of the row. Longer rows, and rows whose threshold bin overflows the candidate list, take
// a last pass over the row with ballots for the in-warp order and per-warp counts for the rest.
#include "launch_util.h"
#include "sac_kernels.h"

namespace sac {
namespace {

constexpr int kThreads = 512;       // long rows with keys in shared memory
// rows of at most kSmemKeyRows scores, and rows re-read from L2: more rows side by side per SM
// (measured at CSA-8k: 112 us with 512 threads, 87 us with 256, 108 us with 128; CSA-128k rows
// re-read from L2: 0.56 ms a launch with 512 threads, 0.50 ms with 256)
constexpr int kShortThreads = 256;
constexpr int kWideThreads = 1024;  // rows with keys in shared memory when there are few of them
constexpr int kMaxEntries = 1 << 22;  // longest row (pool entries per sequence) accepted
constexpr int kBins = 4096;          // 12-bit digits
constexpr int kCandCap = 2048;       // compacted keys of the threshold bin
constexpr int kSmemKeyRows = 4096;   // rows up to this length keep their keys in shared memory
constexpr int kSmemKeyLimit = 49152; // longest row whose keys fit in shared memory (192 KB)
constexpr int kBatch = 8;            // loads a thread has in flight in the passes over a row
constexpr int kMapWords = 1024;      // selection bit map: one bit per entry
constexpr int kMapEntries = 32 * kMapWords;  // longest row selected through the bit maps

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s + 0.0f);  // -0 and +0 compare equal
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the lanes of a warp; *total gets the warp's sum.
__device__ __forceinline__ int warp_exclusive_sum(int v, int& total) {
  const int lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(~0u, x, o);
    if (lane >= o) x += y;
  }
  total = __shfl_sync(~0u, x, 31);
  return x - v;
}

struct Shared {
  int hist[kBins];
  uint32_t cand[kCandCap];
  int cand_idx[kCandCap];  // entry index of each compacted key
  int warp_tot[32];  // up to 1024 threads
  int warp_gt[32], warp_eq[32];
  uint32_t gt_map[kMapWords];  // bit i: entry i is selected (key > T)
  int n_cand;
  int digit, rem;
};

// Exclusive prefix sum over the block of NT threads (thread order); also returns the total.
template <int NT>
__device__ __forceinline__ int block_exclusive_sum(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(~0u, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const int t = warp_tot[w];
    before += w < warp ? t : 0;
    total += t;
  }
  __syncthreads();  // warp_tot may be reused right after
  return before + x - v;
}

// Given hist[0..nbins) (nbins = 8 * kThreads or fewer), find the digit d holding the rem-th
// largest counted key: sum(hist[d+1..]) < rem <= sum(hist[d..]). Writes sh.digit and sh.rem (the
// rank of T among the keys of digit d).
template <int NT>
__device__ __forceinline__ void find_digit(Shared& sh, int nbins, int rem) {
  const int per = nbins / NT;  // bins per thread; 0 when there are fewer bins than threads
  const int rt = NT - 1 - threadIdx.x;  // thread blocks of bins counted from the top
  int lo, cnt;
  if (per > 0) {
    lo = rt * per;
    cnt = per;
  } else {
    lo = rt - (NT - nbins);
    cnt = lo >= 0 ? 1 : 0;
  }
  int s = 0;
  for (int i = 0; i < cnt; ++i) s += sh.hist[lo + i];
  int total;
  const int above = block_exclusive_sum<NT>(s, sh.warp_tot, total);
  if (cnt > 0 && above < rem && rem <= above + s) {
    int acc = above;
    for (int d = lo + cnt - 1; d >= lo; --d) {
      const int h = sh.hist[d];
      if (acc + h >= rem) {
        sh.digit = d;
        sh.rem = rem - acc;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
}

// kSmemKeys: the row's keys are kept in shared memory (short rows); otherwise every pass
// re-reads the scores, which the first pass has brought into L2, so that a block needs only
// ~25 KB of shared memory and several rows run side by side on each SM.
template <bool kSmemKeys, int NT>
__global__ void __launch_bounds__(NT) topk_kernel(const float* __restrict__ scores,
                                                        int n_stride, QueryRows qr, int m, int k,
                                                        int32_t* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Shared& sh = *reinterpret_cast<Shared*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(Shared));

  const int64_t r = blockIdx.x;
  int seq;
  int64_t t;
  qr.locate(qr.row0 + r, seq, t);
  const int n = (int)((t + 1) / m);
  int32_t* orow = out + r * k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int i = tid; i < k; i += NT) orow[i] = i < n ? i : -1;
    return;
  }
  const float* srow = scores + r * n_stride;
  auto key_at = [&](int i) -> uint32_t {
    return kSmemKeys ? keys[i] : order_key(__ldcg(srow + i));
  };

  // ---- digit 1: bits 31..20. The passes over the row issue all of a batch's loads before using
  // any, so a thread waits for one memory latency per batch rather than per key.
  for (int i = tid; i < kBins; i += NT) sh.hist[i] = 0;
  if (tid == 0) sh.n_cand = 0;
  __syncthreads();
  auto count_key = [&](int i, float v) {
    const uint32_t key = order_key(v);
    if (kSmemKeys) keys[i] = key;
    atomicAdd(&sh.hist[key >> 20], 1);
  };
  // rows on 16-byte boundaries are read as float4 (kBatch / 2 of them in flight a thread: twice
  // the bytes of kBatch scalars, a quarter of the load instructions), the rest key by key
  int i_scalar = 0;
  if ((reinterpret_cast<uintptr_t>(srow) & 15) == 0) {
    constexpr int kVec = kBatch / 2;
    const float4* s4 = reinterpret_cast<const float4*>(srow);
    const int n4 = n >> 2;
    for (int i0 = tid; i0 < n4; i0 += NT * kVec) {
      float4 v[kVec];
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int i = i0 + u * NT;
        v[u] = i < n4 ? __ldcg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kVec; ++u) {
        const int i = i0 + u * NT;
        if (i < n4) {
          count_key(4 * i, v[u].x);
          count_key(4 * i + 1, v[u].y);
          count_key(4 * i + 2, v[u].z);
          count_key(4 * i + 3, v[u].w);
        }
      }
    }
    i_scalar = 4 * n4;
  }
  for (int i0 = i_scalar + tid; i0 < n; i0 += NT * kBatch) {
    float v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * NT;
      v[u] = i < n ? __ldcg(srow + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * NT;
      if (i < n) count_key(i, v[u]);
    }
  }
  __syncthreads();
  find_digit<NT>(sh, kBins, k);
  const uint32_t d1 = (uint32_t)sh.digit;
  int rem = sh.rem;
  const int c1 = sh.hist[d1];
  __syncthreads();  // everyone has read hist before it is cleared

  // Warp w owns the contiguous segment [w*seg, (w+1)*seg) of the row in the passes below.
  const int seg = ((n + (NT / 32) * 32 - 1) / ((NT / 32) * 32)) * 32;
  const int s0 = warp * seg, s1 = min(n, s0 + seg);

  // ---- one pass when the keys of digit d1 fit the candidate list: keys of a higher digit are
  // all selected (each warp counts its own), those of digit d1 are compacted with their entry
  // index, the rest are dropped. Then the finer digits and the per-segment counts of the output
  // need only the candidates, not the row. Otherwise the finer digits scan the whole row.
  const bool compact = c1 <= kCandCap;
  // (rows whose keys sit in shared memory and are short re-read them faster than the maps cost)
  const bool use_map = compact && n <= kMapEntries && (!kSmemKeys || n > kSmemKeyRows);
  int above_d1 = 0;
  if (compact) {
    for (int b0 = s0; b0 < s1; b0 += 32 * kBatch) {
      uint32_t kb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = b0 + 32 * u + lane;
        kb[u] = i < s1 ? key_at(i) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = b0 + 32 * u + lane;
        const uint32_t dg = kb[u] >> 20;
        const uint32_t gt_mask = __ballot_sync(~0u, i < s1 && dg > d1);
        above_d1 += __popc(gt_mask);
        // the warp's 32 entries of this step are one word of the map (segments start at
        // multiples of 32)
        if (use_map && lane == 0 && b0 + 32 * u < s1) sh.gt_map[(b0 + 32 * u) >> 5] = gt_mask;
        const bool hit = i < s1 && dg == d1;
        const uint32_t mask = __ballot_sync(~0u, hit);
        if (mask) {
          int base = 0;
          if (lane == 0) base = atomicAdd(&sh.n_cand, __popc(mask));
          base = __shfl_sync(~0u, base, 0);
          if (hit) {
            const int slot = base + __popc(mask & ((1u << lane) - 1u));
            sh.cand[slot] = kb[u];
            sh.cand_idx[slot] = i;
          }
        }
      }
    }
  }
  const int nc = compact ? c1 : n;
  auto cand_at = [&](int i) -> uint32_t { return compact ? sh.cand[i] : key_at(i); };

  // ---- digit 2: bits 19..8 among keys with digit 1 == d1
  for (int i = tid; i < kBins; i += NT) sh.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < nc; i += NT) {
    const uint32_t key = cand_at(i);
    if ((key >> 20) == d1) atomicAdd(&sh.hist[(key >> 8) & 0xFFFu], 1);
  }
  __syncthreads();
  find_digit<NT>(sh, kBins, rem);
  const uint32_t d2 = (uint32_t)sh.digit;
  rem = sh.rem;
  __syncthreads();

  // ---- digit 3: bits 7..0 among keys with bits 31..8 == (d1, d2)
  const uint32_t hi24 = (d1 << 12) | d2;
  for (int i = tid; i < 256; i += NT) sh.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < nc; i += NT) {
    const uint32_t key = cand_at(i);
    if ((key >> 8) == hi24) atomicAdd(&sh.hist[key & 0xFFu], 1);
  }
  __syncthreads();
  find_digit<NT>(sh, 256, rem);
  const uint32_t T = (hi24 << 8) | (uint32_t)sh.digit;
  const int take_eq = sh.rem;  // keys equal to T to keep, lowest indices first

  if (use_map) {
    // ---- selection through the bit maps: the candidates above T join the keys above digit d1
    // in gt_map, those equal to T go to eq_map (the histogram's storage, free now)
    uint32_t* eq_map = reinterpret_cast<uint32_t*>(sh.hist);
    const int nwords = (n + 31) >> 5;
    for (int i = tid; i < nwords; i += NT) eq_map[i] = 0u;
    __syncthreads();
    for (int c = tid; c < nc; c += NT) {
      const uint32_t key = sh.cand[c];
      const int e = sh.cand_idx[c];
      if (key > T) atomicOr(&sh.gt_map[e >> 5], 1u << (e & 31));
      else if (key == T) atomicOr(&eq_map[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    // warp w's words cover its segment [s0, s1); an empty segment (s0 >= n) has none
    const int w0 = s0 >> 5, w1 = (s1 + 31) >> 5;
    int gt = 0, eq = 0;
    for (int wd = w0 + lane; wd < w1; wd += 32) {
      gt += __popc(sh.gt_map[wd]);
      eq += __popc(eq_map[wd]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(~0u, gt, o);
      eq += __shfl_xor_sync(~0u, eq, o);
    }
    if (lane == 0) {
      sh.warp_gt[warp] = gt;
      sh.warp_eq[warp] = eq;
    }
    __syncthreads();
    int eq_before = 0, sel_before = 0;
    for (int w = 0; w < warp; ++w) {
      const int e = sh.warp_eq[w];
      sel_before += sh.warp_gt[w] + min(max(take_eq - eq_before, 0), e);
      eq_before += e;
    }
    // 32 words (1024 entries) per step, lane l on word wb + l; the keys == T are taken in entry
    // order while the count taken before them stays below take_eq
    for (int wb = w0; wb < w1; wb += 32) {
      const int wd = wb + lane;
      const uint32_t g = wd < w1 ? sh.gt_map[wd] : 0u;
      const uint32_t e = wd < w1 ? eq_map[wd] : 0u;
      const int ne = __popc(e);
      int ne_tot;
      const int ne_before = warp_exclusive_sum(ne, ne_tot);
      int q = take_eq - (eq_before + ne_before);
      uint32_t taken = 0u;
      if (q >= ne) {
        taken = e;
      } else {
        for (uint32_t rest = e; q > 0; --q) {  // the lowest q bits of e
          taken |= rest & (0u - rest);
          rest &= rest - 1u;
        }
      }
      uint32_t sel = g | taken;
      int ns_tot;
      int pos = sel_before + warp_exclusive_sum(__popc(sel), ns_tot);
      while (sel) {
        orow[pos++] = (wd << 5) + (__ffs(sel) - 1);
        sel &= sel - 1u;
      }
      eq_before += ne_tot;
      sel_before += ns_tot;
    }
    return;
  }

  // ---- selection: per-segment counts of keys > T and == T, then the output in entry order
  if (compact) {
    // keys above digit d1 were counted in the pass; the candidates add theirs
    if (lane == 0) {
      sh.warp_gt[warp] = above_d1;
      sh.warp_eq[warp] = 0;
    }
    __syncthreads();
    for (int c = tid; c < nc; c += NT) {
      const uint32_t key = sh.cand[c];
      const int w = sh.cand_idx[c] / seg;
      if (key > T) atomicAdd(&sh.warp_gt[w], 1);
      else if (key == T) atomicAdd(&sh.warp_eq[w], 1);
    }
  } else {
    int gt = 0, eq = 0;
    for (int b0 = s0; b0 < s1; b0 += 32 * kBatch) {
      uint32_t kb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = b0 + 32 * u + lane;
        kb[u] = i < s1 ? key_at(i) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const bool in = b0 + 32 * u + lane < s1;
        gt += __popc(__ballot_sync(~0u, in && kb[u] > T));
        eq += __popc(__ballot_sync(~0u, in && kb[u] == T));
      }
    }
    if (lane == 0) {
      sh.warp_gt[warp] = gt;
      sh.warp_eq[warp] = eq;
    }
  }
  __syncthreads();
  int eq_before = 0, sel_before = 0;
  for (int w = 0; w < warp; ++w) {
    const int e = sh.warp_eq[w];
    const int take = min(max(take_eq - eq_before, 0), e);
    sel_before += sh.warp_gt[w] + take;
    eq_before += e;
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (int b0 = s0; b0 < s1; b0 += 32 * kBatch) {
    uint32_t kb[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = b0 + 32 * u + lane;
      kb[u] = i < s1 ? key_at(i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = b0 + 32 * u + lane;
      const bool is_gt = i < s1 && kb[u] > T;
      const bool is_eq = i < s1 && kb[u] == T;
      const uint32_t eq_mask = __ballot_sync(~0u, is_eq);
      const bool sel = is_gt || (is_eq && eq_before + __popc(eq_mask & lt) < take_eq);
      const uint32_t sel_mask = __ballot_sync(~0u, sel);
      if (sel) orow[sel_before + __popc(sel_mask & lt)] = i;
      eq_before += __popc(eq_mask);
      sel_before += __popc(sel_mask);
    }
  }
}

}  // namespace

int topk_max_entries() { return kMaxEntries; }

cudaError_t launch_topk(const float* scores, int n_stride, QueryRows qr, int m, int64_t nrows,
                        int k, int32_t* out, cudaStream_t st) {
  if (nrows == 0) return cudaSuccess;
  if (n_stride > kMaxEntries) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // keys in shared memory for short rows, and for launches with too few rows to fill the GPU
  // several times over (there the per-row latency of the L2 re-reads would dominate)
  const bool smem_keys = n_stride <= kSmemKeyRows || (nrows <= 4 * (int64_t)sms &&
                                                       n_stride <= kSmemKeyLimit);
  if (smem_keys) {
    const size_t smem = sizeof(Shared) + sizeof(uint32_t) * (size_t)(n_stride > 0 ? n_stride : 1);
    if (n_stride <= kSmemKeyRows) {
      cudaError_t err = ensure_smem_limit((const void*)topk_kernel<true, kShortThreads>, (int)smem);
      if (err != cudaSuccess) return err;
      topk_kernel<true, kShortThreads><<<(unsigned)nrows, kShortThreads, smem, st>>>(
          scores, n_stride, qr, m, k, out);
      return cudaGetLastError();
    }
    if (nrows <= sms) {
      // fewer rows than SMs (decode): 1024 threads a row halve each pass's per-row time
      cudaError_t err = ensure_smem_limit((const void*)topk_kernel<true, kWideThreads>, (int)smem);
      if (err != cudaSuccess) return err;
      topk_kernel<true, kWideThreads><<<(unsigned)nrows, kWideThreads, smem, st>>>(
          scores, n_stride, qr, m, k, out);
      return cudaGetLastError();
    }
    cudaError_t err = ensure_smem_limit((const void*)topk_kernel<true, kThreads>, (int)smem);
    if (err != cudaSuccess) return err;
    topk_kernel<true, kThreads><<<(unsigned)nrows, kThreads, smem, st>>>(scores, n_stride, qr, m,
                                                                         k, out);
  } else {
    topk_kernel<false, kShortThreads><<<(unsigned)nrows, kShortThreads, sizeof(Shared), st>>>(
        scores, n_stride, qr, m, k, out);
  }
  return cudaGetLastError();
}

}  // namespace sac
