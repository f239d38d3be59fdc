// Lightning Indexer score ("Hybrid attention", CSA bullet, eq. 13-17; "DeepseekV4Config":
// index_n_heads, index_head_dim): I[t,w] = sum_h w_idx[t,h] * max(0, <q_idx[t,h], KI_w>) for the
// visible entries w < (t+1)//m. CUDA-core version (fp32 math): one block per (query row, 64
// entries); warps split the heads, lanes the entries, and a shared-memory reduction sums heads.
#include "launch_util.h"
#include "sac_kernels.h"

namespace sac {
namespace {

constexpr int kEntriesPerBlock = 64;

template <typename T>
__global__ void __launch_bounds__(256) indexer_simt_kernel(IndexerArgs a) {
  extern __shared__ float smem[];
  const int nI = a.nI, cI = a.cI;
  float* qs = smem;                        // [nI][cI]
  float* wsm = qs + nI * cI;               // [nI]
  float* ks = wsm + nI;                    // [64][cI+1]
  float* red = ks + kEntriesPerBlock * (cI + 1);  // [8][64]
  const int64_t r = blockIdx.x;
  int seq;
  int64_t t;
  a.qr.locate(a.qr.row0 + r, seq, t);
  const int64_t nvis = (t + 1) / a.m;
  const int64_t e0 = (int64_t)blockIdx.y * kEntriesPerBlock;
  if (e0 >= nvis) return;
  const int ne = nvis - e0 < kEntriesPerBlock ? (int)(nvis - e0) : kEntriesPerBlock;
  const T* qrow = reinterpret_cast<const T*>(a.q_idx) + r * nI * cI;
  for (int i = threadIdx.x; i < nI * cI; i += blockDim.x) qs[i] = to_f<T>(qrow[i]);
  for (int i = threadIdx.x; i < nI; i += blockDim.x) wsm[i] = a.w_idx[r * nI + i];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = warp; e < kEntriesPerBlock; e += 8) {
    const T* kr = e < ne ? a.kpool.row<T>(seq, e0 + e) : nullptr;
    for (int c = lane; c < cI; c += 32) ks[e * (cI + 1) + c] = kr ? to_f<T>(kr[c]) : 0.f;
  }
  __syncthreads();
  float acc0 = 0.f, acc1 = 0.f;
  const float* k0 = ks + lane * (cI + 1);
  const float* k1 = ks + (lane + 32) * (cI + 1);
  for (int h = warp; h < nI; h += 8) {
    const float* qh = qs + h * cI;
    float d0 = 0.f, d1 = 0.f;
    for (int c = 0; c < cI; ++c) {
      float qv = qh[c];
      d0 = fmaf(qv, k0[c], d0);
      d1 = fmaf(qv, k1[c], d1);
    }
    float wh = wsm[h];
    acc0 = fmaf(wh, fmaxf(d0, 0.f), acc0);
    acc1 = fmaf(wh, fmaxf(d1, 0.f), acc1);
  }
  red[warp * 64 + lane] = acc0;
  red[warp * 64 + lane + 32] = acc1;
  __syncthreads();
  if (threadIdx.x < ne) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w * 64 + threadIdx.x];
    a.scores[r * a.n_stride + e0 + threadIdx.x] = s;
  }
}

template <typename T>
cudaError_t indexer_t(const IndexerArgs& a, int max_visible, cudaStream_t st) {
  if (a.nrows == 0 || max_visible == 0) return cudaSuccess;
  size_t smem = sizeof(float) * ((size_t)a.nI * a.cI + a.nI +
                                 (size_t)kEntriesPerBlock * (a.cI + 1) + 8 * 64);
  cudaError_t err = ensure_smem_limit((const void*)indexer_simt_kernel<T>, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)a.nrows, (unsigned)((max_visible + kEntriesPerBlock - 1) / kEntriesPerBlock));
  indexer_simt_kernel<T><<<grid, 256, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer(int dtype, const IndexerArgs& a, int max_visible, cudaStream_t st) {
  if (dtype == 0) return indexer_t<float>(a, max_visible, st);
  return indexer_t<__nv_bfloat16>(a, max_visible, st);
}

}  // namespace sac
