// Shared device helpers of the sm_100a hybrid-attention library: element conversion, the RoPE
// angle table, key-row addressing for contiguous and paged caches, and warp reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sac {

constexpr int kMaxRopePairs = 64;  // R <= 128

// Per-call RoPE frequencies theta^(-2i/R), computed once on the host in double precision.
struct RopeFreqs {
  double inv_freq[kMaxRopePairs];
  int R;
};

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// cos/sin of pair i at absolute position pos. The angle pos * theta^(-2i/R) is formed in fp64 and
// reduced to [-pi, pi] by subtracting the nearest multiple of 2*pi (one fp64 FMA: for positions
// up to 2^20 the reduction error stays below 1e-9 rad); the fp32 sine/cosine of the reduced angle
// then carry an absolute error of about 1e-6, far below bf16 resolution.
__device__ __forceinline__ void rope_cos_sin(const RopeFreqs& rf, int i, int64_t pos, float& c,
                                             float& s) {
  constexpr double kTwoPi = 6.283185307179586476925;
  const double phi = (double)pos * rf.inv_freq[i];
  const double k = rint(phi * (1.0 / kTwoPi));
  const float r = (float)fma(-k, kTwoPi, phi);
  __sincosf(r, &s, &c);
}

// Rows of a key stream: contiguous [seqs, seq_stride, width], or pages [*, page_size, width]
// reached through a block table [seqs, max_pages].
struct RowAddr {
  const void* base;
  const int32_t* block_table;  // nullptr: contiguous
  int64_t seq_stride;          // rows per sequence (contiguous layout)
  int max_pages;
  int page_size;
  int width;                   // elements per row

  template <typename T>
  __device__ __forceinline__ const T* row(int seq, int64_t j) const {
    const T* b = reinterpret_cast<const T*>(base);
    if (block_table == nullptr) return b + ((int64_t)seq * seq_stride + j) * width;
    int page = __ldg(block_table + (int64_t)seq * max_pages + j / page_size);
    if (page < 0) return nullptr;  // unallocated page: read as an empty key
    return b + ((int64_t)page * page_size + (j % page_size)) * width;
  }

  // Row number of row j of sequence seq in the flat [rows, width] view of the base buffer (TMA
  // coordinates). An unallocated page maps to row 0.
  __device__ __forceinline__ int64_t row_index(int seq, int64_t j) const {
    if (block_table == nullptr) return (int64_t)seq * seq_stride + j;
    int page = __ldg(block_table + (int64_t)seq * max_pages + j / page_size);
    if (page < 0) page = 0;
    return (int64_t)page * page_size + (j % page_size);
  }
};

// Query rows: prefill row r = seq*S + t; decode row r = seq with t = ctx_lens[seq] - 1.
struct QueryRows {
  int S;                     // prefill tokens per sequence (0 for decode)
  const int32_t* ctx_lens;   // decode / chunked prefill only
  int64_t row0;              // first flat row of this launch (prefill chunking)
  int nq;                    // with ctx_lens: query rows per sequence, the last nq positions
                             // (0 or 1: one query per sequence, decode)
  int64_t max_ctx;           // with ctx_lens: the longest context the block tables cover
                             // (0: not checked)

  // Sequence and position of row r. A context above max_ctx is a bad input: the row then gets
  // t = -1, so it sees no key and addresses no cache row, and locate returns false. Rows with
  // t < 0 (also those of a context shorter than nq) see no key; their output rows are undefined.
  __device__ __forceinline__ bool locate(int64_t r, int& seq, int64_t& t) const {
    if (ctx_lens != nullptr) {
      const int q = nq > 1 ? nq : 1;
      seq = (int)(r / q);
      const int64_t ctx = __ldg(ctx_lens + seq);
      if (max_ctx > 0 && ctx > max_ctx) {
        t = -1;
        return false;
      }
      t = ctx - q + r % q;
    } else {
      seq = (int)(r / S);
      t = r % S;
    }
    return true;
  }
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace sac
