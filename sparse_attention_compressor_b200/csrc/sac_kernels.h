// Host-side launch interface of the library's kernels (internal; the public ABI is include/sac.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sac_common.cuh"

namespace sac {

// ---- compressor + rotations (compress.cu) --------------------------------------------------
// Pool of x [B,S,C]: entry w pools the window [(w+1)m - L, (w+1)m) (clipped at 0) with a softmax
// gate; with rotate != 0 the entry is then rotated at pos0 + w*m. out [B,N,C].
cudaError_t launch_compress(int dtype, const void* x, const void* gate, const float* bias, int B,
                            int S, int C, int m, int L, bool rotate, const RopeFreqs& rf,
                            int64_t pos0, void* out, int* status, cudaStream_t st);
// out[r] = x[r] with its trailing R channels rotated at pos0 + (r / rows_per_pos) % S.
// x, out [rows, C] (kv: rows_per_pos = 1; q viewed as [B*S*H, D]: rows_per_pos = H).
cudaError_t launch_rotate_rows(int dtype, const void* x, int64_t rows, int S, int C,
                               const RopeFreqs& rf, int64_t pos0, void* out, cudaStream_t st,
                               int rows_per_pos = 1);

// ---- decode cache append (decode_append.cu) -------------------------------------------------
// One new token per sequence at t = ctx_lens[seq] - 1: kv_new rotated into the window pages; for
// m > 0 the un-rotated row into the ring cmp_state [nseq, L, D] (slot t % L) and, when t + 1 is a
// multiple of m, entry (t+1)/m - 1 pooled from the ring into the pool pages (rotated). The
// indexer part (CSA) takes the indexer key row through the same path at width cI (no rotation).
struct DecodeAppendArgs {
  int nseq;
  const int32_t* ctx_lens;
  int64_t max_ctx;            // the longest context the block tables cover; longer: skipped
  int D, cI, m, L;
  int64_t pos0;
  RopeFreqs rf;
  const void* kv_new;         // [nseq, n, D] un-rotated (n = 1 for a decode step)
  const void* k_idx_new;      // [nseq, n, cI] (CSA)
  const void* cmp_gate;       // [D]
  const float* cmp_bias;      // [L]
  const void* idx_gate;       // [cI] (CSA)
  const float* idx_bias;      // [L] (CSA)
  void* kv_pages;
  const int32_t* kv_block_table;
  int kv_max_pages, page_size;
  void* cmp_state;            // [nseq, L, D] (m > 0)
  void* idx_state;            // [nseq, L, cI] (CSA) or nullptr
  void* pool_pages;
  void* idx_pool_pages;
  const int32_t* pool_block_table;
  int pool_max_pages;
};
// index_part = false: the kv row and the main pool; true: the indexer ring and pool (CSA).
cudaError_t launch_decode_append(int dtype, const DecodeAppendArgs& a, bool index_part,
                                 cudaStream_t st);
// Both parts of a CSA layer in one launch, for the shapes decode_append_pair_supported() accepts
// (D = 512, cI = 128, L < 64); other shapes launch the parts one by one.
bool decode_append_pair_supported(const DecodeAppendArgs& a);
cudaError_t launch_decode_append_pair(int dtype, const DecodeAppendArgs& a, cudaStream_t st);
// The same for a prefill chunk of n tokens per sequence at t = ctx - n .. ctx - 1 (two launches:
// the entries that close inside the chunk, then the rows' page and ring writes).
cudaError_t launch_chunk_append(int dtype, const DecodeAppendArgs& a, int n, bool index_part,
                                cudaStream_t st);

// ---- grouped output projection (oproj.cu, tcgen05 GEMM) ----------------------------------
struct OProjArgs {
  int64_t T;             // tokens
  int H, D, groups, rank, hidden;
  const void* o;         // [T, H*D] bf16
  const void* w_a;       // [groups, rank, H/groups*D] bf16 (o_a_proj, nn.Linear layout per group)
  const void* w_b;       // [hidden, groups*rank] bf16 (o_b_proj)
  void* mid;             // [T, groups*rank] bf16 intermediate
  void* out;             // [T, hidden] bf16
  int* status;           // device status word
};
cudaError_t launch_oproj(const OProjArgs& a, cudaStream_t st);

// ---- indexer (indexer.cu) -----------------------------------------------------------------
struct IndexerArgs {
  const void* q_idx;     // [rows, nI, cI] (flat query rows starting at qr.row0)
  const float* w_idx;    // [rows, nI]
  RowAddr kpool;         // indexer pool rows (width cI)
  QueryRows qr;
  int nI, cI, m;
  int64_t nrows;         // rows in this launch
  int n_stride;          // scores row stride (>= largest visible count)
  float* scores;         // [nrows, n_stride]; entries w < (t+1)//m written
};
cudaError_t launch_indexer(int dtype, const IndexerArgs& a, int max_visible, cudaStream_t st);

// ---- indexer on tcgen05 (indexer_tc.cu): bf16, 64 heads x 128 ---------------------------
struct IndexerTcArgs {
  const float* w_idx;    // [B*S, nI] head weights of all query rows
  float* scores;         // [t1 - t0, n_stride] scores of query positions t0..t1-1
  int* status;           // device status word
  int64_t t0, t1;        // query positions of sequence `seq` handled by this launch
  int seq, S, N, m, n_stride;
};
bool indexer_tc_supported(int dtype, int nI, int cI);
// q_idx: [q_rows_total, 64, 128] (all query rows); kpool: [kpool_rows, 128] (all sequences).
cudaError_t launch_indexer_tc(const IndexerTcArgs& a, const void* q_idx, int64_t q_rows_total,
                              const void* kpool, int64_t kpool_rows, cudaStream_t st);

// ---- decode indexer on tcgen05 (indexer_decode_tc.cu): bf16, 64 heads x 128 -------------
// One query per sequence (a.qr.ctx_lens set, a.nrows sequences), paged or contiguous pool rows of
// width 128; scores [nrows, n_stride]; entries w < ctx // m written. status: nullable.
bool indexer_decode_tc_supported(int dtype, int nI, int cI);
cudaError_t launch_indexer_decode_tc(const IndexerArgs& a, int max_visible, int* status,
                                     cudaStream_t st);

// ---- top-k (topk.cu) ----------------------------------------------------------------------
// Per row: the k largest of the first (t+1)//m scores, ties to the lower index, written in
// ascending entry order followed by -1.
cudaError_t launch_topk(const float* scores, int n_stride, QueryRows qr, int m, int64_t nrows,
                        int k, int32_t* out, cudaStream_t st);
int topk_max_entries();

// ---- attention (attention_simt.cu) --------------------------------------------------------
struct AttnArgs {
  const void* q;         // [rows, H, D] un-rotated
  void* o;               // [rows, H, D]
  const float* sinks;    // [H]
  QueryRows qr;
  int64_t nrows;
  int H, D, W;
  float scale;
  int64_t pos0;
  RowAddr win;           // rotated kv rows
  int pool_mode;         // 0: none, 1: all visible entries (t+1)//m, 2: selection list
  RowAddr pool;          // rotated pool rows
  int m;
  const int32_t* sel;    // [rows, k] for pool_mode 2
  int k;
  RopeFreqs rf;
  int* status;           // device status word (tensor-core kernels record wait timeouts)
  // tensor-core kernel only: each row's key tiles split over `splits` CTAs (1 = no split); with
  // splits > 1 the partial results go to part_o [nrows*splits, H, D] and part_ml
  // [nrows*splits, H, 2] (fp32) and a combine kernel writes o
  int splits;
  float* part_o;
  float* part_ml;
};
cudaError_t launch_attention_simt(int dtype, const AttnArgs& a, cudaStream_t st);

// ---- attention on tcgen05 (attention_tc.cu): bf16, 64 heads, head_dim 512 ------------------
// a.q: [nrows, 64, 512] un-rotated (rotated in the kernel); win/pool bases are [rows, 512]
// buffers whose row counts (win_rows, pool_rows) bound the TMA coordinates; a paged cache's
// count is ignored (its block table names the rows read).
bool attention_tc_supported(const AttnArgs& a, int dtype);
int attention_tc_max_splits();
cudaError_t launch_attention_tc(const AttnArgs& a, int64_t win_rows, int64_t pool_rows,
                                cudaStream_t st);

}  // namespace sac
