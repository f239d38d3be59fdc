// Indexer top-k ("Hybrid attention", CSA bullet, eq. 17; "Attention mask layout", CSA
// paragraph): per query row, the k largest of the (t+1)//m visible scores, ties going to the
// lower entry index; empty slots (fewer than k visible) hold -1.
//
// One block per row. Scores become order-preserving uint32 keys in shared memory; a 4-pass 8-bit
// radix select finds the exact k-th key T; then a block scan keeps every key > T plus the first
// (k - #{key > T}) keys == T in index order, and writes the chosen entries in ascending order.
#include <cub/block/block_scan.cuh>

#include "sac_kernels.h"

namespace sac {
namespace {

constexpr int kThreads = 512;
constexpr int kMaxEntries = 49152;  // 192 KB of keys in shared memory

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s + 0.0f);  // -0 and +0 compare equal
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kThreads) topk_kernel(const float* __restrict__ scores,
                                                        int n_stride, QueryRows qr, int m, int k,
                                                        int32_t* __restrict__ out) {
  extern __shared__ uint32_t keys[];
  __shared__ int hist[256];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;
  using Scan = cub::BlockScan<int, kThreads>;
  __shared__ typename Scan::TempStorage scan_tmp;

  const int64_t r = blockIdx.x;
  int seq;
  int64_t t;
  qr.locate(qr.row0 + r, seq, t);
  const int n = (int)((t + 1) / m);
  int32_t* orow = out + r * k;
  const int tid = threadIdx.x;
  if (n <= k) {
    for (int i = tid; i < k; i += kThreads) orow[i] = i < n ? i : -1;
    return;
  }
  const float* srow = scores + r * n_stride;
  for (int i = tid; i < n; i += kThreads) keys[i] = order_key(__ldg(srow + i));
  if (tid == 0) { s_prefix = 0; s_mask = 0; s_remaining = k; }
  __syncthreads();

  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int i = tid; i < n; i += kThreads) {
      uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid == 0) {
      int rem = s_remaining, d = 255;
      for (; d > 0; --d) {
        if (hist[d] >= rem) break;
        rem -= hist[d];
      }
      s_prefix = prefix | ((uint32_t)d << shift);
      s_mask = mask | (255u << shift);
      s_remaining = rem;
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int take_eq = s_remaining;  // keys equal to T to keep, lowest indices first

  const int seg = (n + kThreads - 1) / kThreads;
  const int i0 = min(n, tid * seg), i1 = min(n, i0 + seg);
  int eq = 0;
  for (int i = i0; i < i1; ++i) eq += keys[i] == T;
  int eq_before;
  Scan(scan_tmp).ExclusiveSum(eq, eq_before);
  __syncthreads();
  int nsel = 0, e = eq_before;
  for (int i = i0; i < i1; ++i) {
    uint32_t key = keys[i];
    if (key > T) {
      ++nsel;
    } else if (key == T) {
      nsel += e < take_eq;
      ++e;
    }
  }
  int pos;
  Scan(scan_tmp).ExclusiveSum(nsel, pos);
  e = eq_before;
  for (int i = i0; i < i1; ++i) {
    uint32_t key = keys[i];
    bool sel = key > T;
    if (key == T) {
      sel = e < take_eq;
      ++e;
    }
    if (sel) orow[pos++] = i;
  }
}

}  // namespace

int topk_max_entries() { return kMaxEntries; }

cudaError_t launch_topk(const float* scores, int n_stride, QueryRows qr, int m, int64_t nrows,
                        int k, int32_t* out, cudaStream_t st) {
  if (nrows == 0) return cudaSuccess;
  size_t smem = sizeof(uint32_t) * (size_t)(n_stride > 0 ? n_stride : 1);
  cudaError_t err = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  topk_kernel<<<(unsigned)nrows, kThreads, smem, st>>>(scores, n_stride, qr, m, k, out);
  return cudaGetLastError();
}

}  // namespace sac
