// Shared K=V multi-query attention of one query row over its key set, with the per-head sink
// and the partial-RoPE rotations ("Hybrid attention": shared K=V MQA, partial RoPE with the -i
// output rotation (eq. 26), per-head learnable sink (eq. 27), sliding-window branch concatenated
// with the compressor's entries).
//
// Key set of query t: the window rows (t-W, t] of the rotated kv stream, then either nothing
// (sliding layer), every visible entry w < (t+1)//m (HCA) or the entries of its selection list
// (CSA; -1 slots are skipped). p_x = exp(l_x) / (exp(sink_h) + sum_y exp(l_y)), o = sum p_x v_x,
// then o's rope slice is turned by -P_t.
//
// CUDA-core version: fp32 math for both element types. Block = one query row and HG heads (one
// warp per head); keys stream through shared memory 32 at a time (one per lane for the logits,
// then every lane accumulates its D/32 output channels).
#include "launch_util.h"
#include "sac_kernels.h"

namespace sac {
namespace {

constexpr int kMaxV = 16;  // D <= 512

template <typename T>
__device__ __forceinline__ const T* key_row(const AttnArgs& a, int seq, int64_t lo, int nwin,
                                            int64_t row, int x, bool& valid) {
  valid = true;
  const T* r;
  if (x < nwin) {
    r = a.win.row<T>(seq, lo + x);
  } else {
    int i = x - nwin;
    int64_t w = i;
    if (a.pool_mode == 2) w = __ldg(a.sel + row * a.k + i);
    r = w < 0 ? nullptr : a.pool.row<T>(seq, w);
  }
  valid = r != nullptr;
  return r;
}

template <typename T>
__global__ void attention_simt_kernel(AttnArgs a, int HG) {
  extern __shared__ float smem[];
  const int D = a.D;
  const int nv = D / 32;
  float* qs = smem;                    // [HG][D]
  float* ks = qs + HG * D;             // [32][D+1]
  __shared__ int s_valid[32];
  const int64_t row = blockIdx.x;
  const int h0 = blockIdx.y * HG;
  const int nh = min(HG, a.H - h0);
  int seq;
  int64_t t;
  if (!a.qr.locate(a.qr.row0 + row, seq, t) && threadIdx.x == 0 && blockIdx.y == 0 && a.status)
    atomicExch(a.status, 4);  // a context beyond the block tables: the row sees no key
  const int64_t P = a.pos0 + t;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = a.rf.R;

  const T* qrow = reinterpret_cast<const T*>(a.q) + (row * a.H + h0) * D;
  for (int i = threadIdx.x; i < nh * D; i += blockDim.x) qs[i] = to_f<T>(qrow[i]);
  __syncthreads();
  for (int i = threadIdx.x; i < nh * (R / 2); i += blockDim.x) {
    int h = i / (R / 2), p = i % (R / 2);
    float c, s;
    rope_cos_sin(a.rf, p, P, c, s);
    float* x = qs + h * D + (D - R) + 2 * p;
    float u = x[0], v = x[1];
    x[0] = u * c - v * s;
    x[1] = u * s + v * c;
  }

  const int64_t lo = t - a.W + 1 < 0 ? 0 : t - a.W + 1;
  const int nwin = (int)(t - lo + 1);
  int npool = 0;
  if (a.pool_mode == 1) npool = (int)((t + 1) / a.m);
  if (a.pool_mode == 2) npool = a.k;
  const int total = nwin + npool;

  const bool head_active = warp < nh;
  const float sink = head_active ? a.sinks[h0 + warp] : 0.f;
  float m_run = sink, l_run = 1.f;  // the sink's exp(sink - m_run) term
  float acc[kMaxV];
#pragma unroll
  for (int i = 0; i < kMaxV; ++i) acc[i] = 0.f;
  const float* qh = qs + warp * D;

  for (int c0 = 0; c0 < total; c0 += 32) {
    __syncthreads();
    const int nk = min(32, total - c0);
    // stage the chunk's key rows (fp32) in shared memory
    for (int x = warp; x < nk; x += blockDim.x >> 5) {
      bool valid;
      const T* kr = key_row<T>(a, seq, lo, nwin, row, c0 + x, valid);
      for (int c = lane; c < D; c += 32) ks[x * (D + 1) + c] = valid ? to_f<T>(kr[c]) : 0.f;
      if (lane == 0) s_valid[x] = valid;
    }
    __syncthreads();
    if (!head_active) continue;
    float s = -INFINITY;
    if (lane < nk && s_valid[lane]) {
      const float* kr = ks + lane * (D + 1);
      float d = 0.f;
      for (int c = 0; c < D; ++c) d = fmaf(qh[c], kr[c], d);
      s = d * a.scale;
    }
    const float m_new = fmaxf(m_run, warp_max(s));
    const float p = s == -INFINITY ? 0.f : __expf(s - m_new);
    const float corr = __expf(m_run - m_new);
    l_run = l_run * corr + warp_sum(p);
#pragma unroll
    for (int i = 0; i < kMaxV; ++i) acc[i] *= corr;
    for (int j = 0; j < nk; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
      const float* kr = ks + j * (D + 1) + lane;
#pragma unroll
      for (int i = 0; i < kMaxV; ++i)
        if (i < nv) acc[i] = fmaf(pj, kr[32 * i], acc[i]);
    }
    m_run = m_new;
  }
  __syncthreads();
  // normalise, then turn the rope slice back by -P_t (qs is reused as the output staging row)
  if (head_active) {
    const float inv = 1.f / l_run;
#pragma unroll
    for (int i = 0; i < kMaxV; ++i)
      if (i < nv) qs[warp * D + lane + 32 * i] = acc[i] * inv;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nh * (R / 2); i += blockDim.x) {
    int h = i / (R / 2), p = i % (R / 2);
    float c, s;
    rope_cos_sin(a.rf, p, -P, c, s);
    float* x = qs + h * D + (D - R) + 2 * p;
    float u = x[0], v = x[1];
    x[0] = u * c - v * s;
    x[1] = u * s + v * c;
  }
  __syncthreads();
  T* orow = reinterpret_cast<T*>(a.o) + (row * a.H + h0) * D;
  for (int i = threadIdx.x; i < nh * D; i += blockDim.x) orow[i] = from_f<T>(qs[i]);
}

template <typename T>
cudaError_t attention_t(const AttnArgs& a, cudaStream_t st) {
  if (a.nrows == 0) return cudaSuccess;
  const int HG = a.H < 16 ? a.H : 16;
  size_t smem = sizeof(float) * ((size_t)HG * a.D + 32 * (size_t)(a.D + 1));
  cudaError_t err = ensure_smem_limit((const void*)attention_simt_kernel<T>, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)a.nrows, (unsigned)((a.H + HG - 1) / HG));
  attention_simt_kernel<T><<<grid, 32 * HG, smem, st>>>(a, HG);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_simt(int dtype, const AttnArgs& a, cudaStream_t st) {
  if (dtype == 0) return attention_t<float>(a, st);
  return attention_t<__nv_bfloat16>(a, st);
}

}  // namespace sac
