/*
 * sac.h -- C ABI of the B200 (sm_100a) hybrid long-range attention forward of DeepSeek-V4:
 * compressor, Lightning Indexer + top-k, shared K=V sparse / sliding-window multi-query attention
 * with a per-head sink, and partial interleaved RoPE with the inverse rotation of the output.
 *
 * Source of the operations: the "DeepSeek-V4" model documentation page (Hugging Face
 * Transformers), sections "Hybrid attention (section 2.3)" (three layer types; shared K=V MQA;
 * partial RoPE and the -i output rotation, eq. 26; per-head sink, eq. 27; sliding-window branch),
 * "Attention mask layout" (sliding mask, CSA slots with the -1 sentinel, HCA visibility
 * w < (t+1)//m), "Cache layers" (compressor / indexer buffer, pool, count, overlap) and
 * "DeepseekV4Config" (head_dim, sliding_window, compress_rates, index_* fields, rope bases,
 * o_groups, o_lora_rank), and the "Grouped Output Projection" bullet of the architecture overview.
 *
 * Entry points: prefill (swa/hca/csa_forward, swa_forward_static), decode over paged caches
 * (swa/hca/csa_decode, decode_append), chunked prefill over the same caches
 * (swa/hca/csa_prefill_chunk, prefill_chunk_append), the grouped output projection
 * (o_proj_forward), workspace sizes, the device status word and per-kernel timing.
 *
 * Conventions shared by every entry point
 *  - Tensors are caller-owned DEVICE pointers, dense row-major, 16-byte aligned. The library
 *    never allocates device memory; scratch space is a caller-provided workspace of at least
 *    sac_workspace_size() / sac_decode_workspace_size() / sac_chunk_workspace_size() /
 *    sac_oproj_workspace_size() bytes (256-byte aligned).
 *  - Element type of q, kv, k_idx, q_idx, gates, pools and o is params.dtype (SAC_F32 or
 *    SAC_BF16). Biases, sinks and indexer head weights are always fp32; indices are int32.
 *  - Every call enqueues kernels on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *    default stream) and returns without synchronising. Host-visible errors come back as a
 *    status code; sac_last_error() gives a message for the calling thread's last failure.
 *  - Prefill inputs are un-rotated; the library applies RoPE itself. The softmax scale is
 *    params.softmax_scale (> 0).
 *  - Thread safety: calls on different streams may run concurrently as long as they do not share
 *    a workspace or an output.
 */
#ifndef SAC_H
#define SAC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAC_API __attribute__((visibility("default")))
#else
#define SAC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* element types */
#define SAC_F32 0
#define SAC_BF16 1

/* status codes */
#define SAC_OK 0
#define SAC_ERR_ARG (-1)          /* null pointer, non-positive or inconsistent size, misalignment */
#define SAC_ERR_UNSUPPORTED (-2)  /* a shape or dtype outside the supported envelope              */
#define SAC_ERR_WORKSPACE (-3)    /* workspace missing or smaller than required                    */
#define SAC_ERR_LAUNCH (-4)       /* a CUDA launch or attribute call failed                        */

/* layer kinds for the workspace queries */
#define SAC_KIND_SWA 0
#define SAC_KIND_HCA 1
#define SAC_KIND_CSA 2

/*
 * Attention hyper-parameters of one layer ("DeepseekV4Config" names in brackets).
 *   B, S            batch and tokens per sequence (prefill). For decode, S is an upper bound on
 *                   every context length and B is ignored.
 *   H, D            query heads [num_attention_heads], head_dim [head_dim]; one shared K=V head
 *                   [num_key_value_heads = 1].
 *   R               rope channels [head_dim * partial_rotary_factor]: the trailing R channels of
 *                   each head rotate in interleaved pairs (D-R+2i, D-R+2i+1) by pos*theta^(-2i/R).
 *   rope_theta      base for q, window keys and pool entries of this layer [rope_theta for
 *                   sliding layers, compress_rope_theta for compressed layers].
 *   m, win_len      compression rate and compressor window [compress_rates]: CSA m=4, win_len=8
 *                   (overlapping); HCA m=128, win_len=128; sliding layers m=0.
 *   sliding_window  W [sliding_window]: query t attends tokens (t-W, t].
 *   n_idx_heads, idx_dim, topk   [index_n_heads, index_head_dim, index_topk], CSA only.
 *   softmax_scale   logit scale (e.g. 1/sqrt(D)).
 *   pos0            absolute position of token 0 (prefill); added to every decode position.
 *   dtype           SAC_F32 or SAC_BF16.
 *   rope_factor, rope_orig_max_pos, yarn_beta_fast, yarn_beta_slow
 *                   YaRN frequency scaling of every rotation of the layer [the rope scaling the
 *                   config pairs with compress_rope_theta; the page gives no values]. With
 *                   rope_factor s > 1, pair i (base frequency f_i) completes
 *                   r_i = rope_orig_max_pos * f_i / (2 pi) turns over the original context and
 *                   turns at (1 - g) f_i / s + g f_i, g = clamp((r_i - yarn_beta_slow) /
 *                   (yarn_beta_fast - yarn_beta_slow), 0, 1) (YaRN, Peng et al. 2023; usual values
 *                   32 and 1). YaRN's attention temperature scales the logits only: fold it into
 *                   softmax_scale. rope_factor <= 1: plain RoPE, the other three are ignored.
 */
typedef struct {
  int B, S, H, D, R;
  double rope_theta;
  int m, win_len;
  int sliding_window;
  int n_idx_heads, idx_dim, topk;
  float softmax_scale;
  int64_t pos0;
  int dtype;
  double rope_factor;
  int rope_orig_max_pos;
  double yarn_beta_fast, yarn_beta_slow;
} sac_params;

/* Message of the calling thread's last failed call ("" if none). Static storage. */
SAC_API const char* sac_last_error(void);

/* ABI version (major*100 + minor): 200 (sac_params carries the YaRN fields). */
SAC_API int sac_version(void);

/*
 * Workspace bytes a prefill call of `kind` (SAC_KIND_*) needs for `p`, assuming every nullable
 * output is NULL (a call that passes those outputs never needs more). 0 on invalid params.
 */
SAC_API size_t sac_workspace_size(const sac_params* p, int kind);

/*
 * Sliding-window layer forward ("Hybrid attention": sliding_attention layers; "Attention mask
 * layout": plain causal sliding-window mask).
 *   q      [B,S,H,D]   un-rotated queries
 *   kv     [B,S,D]     un-rotated shared key/value head
 *   sinks  [H] fp32    per-head sink logits (eq. 27)
 *   o      [B,S,H,D]   output; its rope slice is rotated back by -P_t (eq. 26)
 * o[b,t,h] = sum_x p_x v_x with p over {kv_j rotated at P_j : t-W < j <= t} and the sink:
 * p_x = exp(l_x) / (exp(sink_h) + sum_y exp(l_y)), l_x = scale <q~_t,h, k~_x>, q~ rotated at P_t.
 */
SAC_API int swa_forward(const sac_params* p, const void* q, const void* kv, const float* sinks, void* o,
                void* ws, size_t ws_bytes, void* stream);

/*
 * swa_forward without any device allocation by the caller: the same computation and the same
 * kernels as swa_forward (the tensor-core attention for bf16 layers of 64 heads of 512, the
 * CUDA-core one otherwise), with the one piece of scratch swa_forward takes from `ws` -- the
 * rotated kv stream, B*S*D elements of dtype -- held instead in a fixed 16 MiB array inside this
 * library (a static __device__ array present on every GPU that loads the library, until the
 * process exits). The page has no counterpart of this entry point. It exists for callers that
 * cannot call cudaMalloc: code that runs inside a host framework whose caching allocator owns
 * all device memory and does not lend it to plug-ins, and serving loops that forbid any
 * allocation after start-up so that memory use stays fixed.
 *   - Returns SAC_ERR_UNSUPPORTED when B*S*D*sizeof(dtype) exceeds sac_static_scratch_bytes().
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current); make that first call before any stream capture. Later calls
 *     look the address up again whenever their stream is not capturing, so that a context torn
 *     down and created again (cudaDeviceReset) never leaves a stale address behind.
 *   - All calls share the one array and it keeps the last call's contents; every byte a call
 *     reads is first written by the same call. Calls that overlap on the GPU (concurrent streams
 *     sharing a device) race on it: serialise them.
 *   - There is no status word: a tensor-core kernel that gives up a bounded wait returns silently.
 *   - Allocates nothing: no cudaMalloc / cudaFree and no allocating library routine.
 */
SAC_API size_t sac_static_scratch_bytes(void);
SAC_API int swa_forward_static(const sac_params* p, const void* q, const void* kv,
                               const float* sinks, void* o, void* stream);

/*
 * Heavily compressed attention forward ("Hybrid attention": HCA, m'=128, non-overlapping
 * windows, no indexer; "Attention mask layout": entry w visible to t iff w < (t+1)//m).
 *   cmp_gate [D] (dtype), cmp_bias [win_len] fp32: compressor gate. Entry w pools the window
 *            [(w+1)m - win_len, (w+1)m) clipped at 0 by a softmax over g_j = <kv_j, u> + b[o_j],
 *            o_j = j - (w+1)m + win_len; N = floor(S/m) entries per sequence.
 *   pool_out [B,N,D] nullable: the pool as attended, rotated at p_w = pos0 + w*m.
 * The key set of query t is the sliding window plus every visible entry.
 */
SAC_API int hca_forward(const sac_params* p, const void* q, const void* kv, const void* cmp_gate,
                const float* cmp_bias, const float* sinks, void* o, void* pool_out, void* ws,
                size_t ws_bytes, void* stream);

/*
 * Compressed sparse attention forward ("Hybrid attention": CSA, m=4, overlapping windows, plus
 * the Lightning Indexer, eq. 13-17, keeping index_topk entries per query).
 *   cmp_gate, cmp_bias   main compressor gate (as in hca_forward), over kv
 *   q_idx [B,S,nI,cI]    indexer queries; w_idx [B,S,nI] fp32 indexer head weights
 *   k_idx [B,S,cI]       indexer key stream; idx_gate [cI], idx_bias [win_len] fp32: its gate
 *   topk_out [B,S,k]     nullable int32: the selected entries of each query in ascending entry
 *                        order, then -1 for empty slots (queries with fewer than k visible)
 *   pool_out [B,N,D]     nullable: rotated main pool; idx_pool_out [B,N,cI] nullable: indexer pool
 * Score I[t,w] = sum_h w_idx[t,h] * max(0, <q_idx[t,h], KI_w>) over visible w; the k largest win,
 * ties to the lower w. The key set of query t is the sliding window plus its selected entries.
 */
SAC_API int csa_forward(const sac_params* p, const void* q, const void* kv, const void* cmp_gate,
                const float* cmp_bias, const void* q_idx, const float* w_idx, const void* k_idx,
                const void* idx_gate, const float* idx_bias, const float* sinks, void* o,
                int32_t* topk_out, void* pool_out, void* idx_pool_out, void* ws, size_t ws_bytes,
                void* stream);

/*
 * Decode: nseq sequences, one new token each, over paged caches ("Cache layers").
 * Cache contract:
 *   - kv_pages [num_pages, page_size, D] hold kv already rotated at each token's position
 *     (pos0 + j); row j of sequence s is kv_pages[kv_block_table[s*kv_max_pages + j/page_size]]
 *     [j % page_size]. The new token's row is already written.
 *   - pool_pages [.., page_size, D] hold pool entries already rotated at pos0 + w*m;
 *     idx_pool_pages [.., page_size, cI] hold un-rotated indexer entries; both use
 *     pool_block_table [nseq, pool_max_pages] with entry w at page w/page_size, row w%page_size.
 *   - ctx_lens [nseq] int32 (device) counts the new token: the query is token t = ctx-1 at
 *     position pos0 + t, it sees the last min(ctx, W) tokens and floor(ctx/m) entries.
 *     Every ctx must satisfy 1 <= ctx <= p->S. The kernels check the upper bound (the block
 *     tables cover p->S rows): a sequence with ctx > p->S reads no cache row, its output row is
 *     left undefined and status 4 is recorded in the workspace's status word (sac_device_status).
 *   q [nseq,H,D] un-rotated; o [nseq,H,D]; q_idx [nseq,nI,cI], w_idx [nseq,nI] fp32 (CSA);
 *   topk_out [nseq,k] nullable (ascending entries, -1 fill).
 * Workspace: sac_decode_workspace_size() bytes, 16-byte aligned: a 256-byte status word (see
 * sac_device_status); for CSA the scores [nseq, S/m] fp32 and the selection [nseq, k]; and, for
 * bf16 layers with 64 heads of 512 when nseq is at most a quarter of the device's SM count, fp32
 * partial results that let each sequence's keys be split over several CTAs
 * (nseq * splits * H * (D + 2) floats, splits = min(8, SMs / nseq), used only when >= 4). ws is required by csa_decode; swa_decode / hca_decode accept NULL
 * (no status word, no split) or any size of at least 256 bytes (the split is used only when the
 * workspace holds its buffers). Entries on an unallocated page (block table entry < 0) read as
 * zero keys.
 */
SAC_API size_t sac_decode_workspace_size(const sac_params* p, int kind, int nseq);

SAC_API int swa_decode(const sac_params* p, int nseq, const void* q, const void* kv_pages,
               const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
               int page_size, const float* sinks, void* o, void* ws, size_t ws_bytes,
               void* stream);

SAC_API int hca_decode(const sac_params* p, int nseq, const void* q, const void* kv_pages,
               const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
               int page_size, const void* pool_pages, const int32_t* pool_block_table,
               int pool_max_pages, const float* sinks, void* o, void* ws, size_t ws_bytes,
               void* stream);

SAC_API int csa_decode(const sac_params* p, int nseq, const void* q, const void* kv_pages,
               const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
               int page_size, const void* pool_pages, const void* idx_pool_pages,
               const int32_t* pool_block_table, int pool_max_pages, const void* q_idx,
               const float* w_idx, const float* sinks, void* o, int32_t* topk_out, void* ws,
               size_t ws_bytes, void* stream);

/*
 * Decode cache append ("Cache layers": the sliding K=V window plus the compressor buffer / pool /
 * count / overlap state and the indexer's copy of it at index_head_dim; "Hybrid attention": an
 * entry exists once its source window has closed). Call it once per decode step, before
 * *_decode, for the new token of each of nseq sequences; ctx_lens [nseq] (device, int32) already
 * counts that token, which sits at t = ctx - 1 (position pos0 + t). kind: SAC_KIND_*.
 *   kv_new [nseq, D]          the new token's un-rotated kv row; written rotated at pos0 + t to row
 *                             t of kv_pages (same paging as *_decode)
 *   cmp_state [nseq, win_len, D]   HCA / CSA: compressor buffer, a ring of the last win_len
 *                             un-rotated kv rows (row j in slot j mod win_len; for CSA the older
 *                             half is the overlap with the previous window). Caller-owned; after a
 *                             prefill of P tokens seed it with rows P - win_len .. P - 1.
 *   cmp_gate [D], cmp_bias [win_len] fp32   the compressor gate, as in hca_forward
 *   pool_pages, pool_block_table, pool_max_pages   as in hca_decode / csa_decode
 * When t + 1 is a multiple of m, entry w = (t+1)/m - 1 closes: it is pooled over the ring rows of
 * its window [(w+1)m - win_len, (w+1)m) (clipped at 0) with the compressor's softmax gate, exactly
 * as the prefill compressor does, rotated at pos0 + w*m and written to row w of pool_pages.
 * CSA also takes k_idx_new [nseq, cI], idx_state [nseq, win_len, cI], idx_gate [cI], idx_bias
 * [win_len] fp32 and idx_pool_pages, and closes the indexer entry the same way without rotation.
 * SWA uses only kv_new and the kv pages (the other pointers may be NULL). Rows on unallocated
 * pages (block table entry < 0) are skipped, and so are sequences whose ctx lies outside
 * [1, p->S] (the block tables cover p->S rows): nothing of theirs is read or written. No
 * workspace; returns before the kernel runs.
 */
SAC_API int decode_append(const sac_params* p, int kind, int nseq, const int32_t* ctx_lens,
               const void* kv_new, const void* k_idx_new, const void* cmp_gate,
               const float* cmp_bias, const void* idx_gate, const float* idx_bias,
               void* kv_pages, const int32_t* kv_block_table, int kv_max_pages, int page_size,
               void* cmp_state, void* idx_state, void* pool_pages, void* idx_pool_pages,
               const int32_t* pool_block_table, int pool_max_pages, void* stream);

/*
 * Chunked prefill over the paged caches: n query tokens per sequence, the LAST n tokens of each
 * context (t = ctx - n .. ctx - 1, positions pos0 + t), all of which are already in the caches
 * (prefill_chunk_append below). Each query row sees exactly what a decode step at ctx = t + 1
 * would see: the window rows t - W + 1 .. t and the entries closed by then, (t + 1) // m of them
 * (CSA: the indexer's top-k of those). Later tokens of the chunk already in the caches are masked
 * by position, so the chunk attends to the cached prefix plus itself, causally.
 * Arguments as in *_decode, with n rows per sequence: q, o [nseq, n, H, D]; q_idx [nseq, n, nI,
 * cI]; w_idx [nseq, n, nI]; topk_out [nseq, n, k]; every ctx must satisfy n <= ctx <= p->S
 * (rows of a sequence with ctx < n have t < 0, see no key, and their output rows are left
 * undefined; a sequence with ctx > p->S is handled as in decode, with status 4).
 * Workspace: sac_chunk_workspace_size() bytes (the decode layout for nseq * n query rows; the
 * CSA scores hold at most 1 GiB of rows at once, the indexer and top-k then run in row blocks).
 * Decode is the case n = 1.
 */
SAC_API size_t sac_chunk_workspace_size(const sac_params* p, int kind, int nseq, int n);

SAC_API int swa_prefill_chunk(const sac_params* p, int nseq, int n, const void* q,
               const void* kv_pages, const int32_t* kv_block_table, int kv_max_pages,
               const int32_t* ctx_lens, int page_size, const float* sinks, void* o, void* ws,
               size_t ws_bytes, void* stream);

SAC_API int hca_prefill_chunk(const sac_params* p, int nseq, int n, const void* q,
               const void* kv_pages, const int32_t* kv_block_table, int kv_max_pages,
               const int32_t* ctx_lens, int page_size, const void* pool_pages,
               const int32_t* pool_block_table, int pool_max_pages, const float* sinks, void* o,
               void* ws, size_t ws_bytes, void* stream);

SAC_API int csa_prefill_chunk(const sac_params* p, int nseq, int n, const void* q,
               const void* kv_pages, const int32_t* kv_block_table, int kv_max_pages,
               const int32_t* ctx_lens, int page_size, const void* pool_pages,
               const void* idx_pool_pages, const int32_t* pool_block_table, int pool_max_pages,
               const void* q_idx, const float* w_idx, const float* sinks, void* o,
               int32_t* topk_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Cache append of a prefill chunk: decode_append for n tokens per sequence at once. ctx_lens
 * already counts the chunk, whose tokens are t = ctx - n .. ctx - 1; kv_new [nseq, n, D] and
 * (CSA) k_idx_new [nseq, n, cI] are their un-rotated rows; every other argument as in
 * decode_append. Each entry w that closes inside the chunk ((w+1)m - 1 >= ctx - n) is pooled
 * exactly as the prefill compressor pools it, its rows taken from kv_new where they belong to the
 * chunk and from the ring (which holds the win_len rows before the chunk) otherwise; then every
 * chunk row is written rotated to the window pages and the ring keeps the sequence's last
 * win_len rows. Appending a stream chunk by chunk (any sizes, decode steps mixed
 * in) leaves the same caches as appending it token by token. Sequences with ctx < n are left
 * untouched, and so are sequences with ctx > p->S (as in decode_append). No workspace.
 */
SAC_API int prefill_chunk_append(const sac_params* p, int kind, int nseq, int n,
               const int32_t* ctx_lens, const void* kv_new, const void* k_idx_new,
               const void* cmp_gate, const float* cmp_bias, const void* idx_gate,
               const float* idx_bias, void* kv_pages, const int32_t* kv_block_table,
               int kv_max_pages, int page_size, void* cmp_state, void* idx_state,
               void* pool_pages, void* idx_pool_pages, const int32_t* pool_block_table,
               int pool_max_pages, void* stream);

/*
 * Grouped low-rank output projection ("Grouped Output Projection" bullet of the architecture
 * overview; config o_groups, o_lora_rank, hidden_size). The attention output o [T, H, D] of
 * p->H heads of p->D is cut into `groups` groups of H/groups consecutive heads; group g's
 * (H/groups)*D features are projected to `rank` features by its own matrix w_a[g] (o_a_proj), the
 * groups' results are concatenated and projected to `hidden` by w_b (o_b_proj):
 *   mid[t, g*rank + i] = sum_c o[t, g*(H/groups)*D + c] * w_a[g, i, c]
 *   out[t, j]          = sum_i mid[t, i] * w_b[j, i]
 *   o   [T, H*D], w_a [groups, rank, (H/groups)*D], w_b [hidden, groups*rank], out [T, hidden]:
 *   bf16 (p->dtype must be SAC_BF16), row-major; weights in the nn.Linear [out, in] layout.
 * The intermediate mid is stored in bf16 (the layer's activation precision); both products
 * accumulate in fp32. Both products run on the library's tcgen05 GEMM kernel (256 x 256 output
 * tiles, operands streamed by TMA, fp32 accumulators in tensor memory).
 * ws: sac_oproj_workspace_size() bytes (the 256-byte status word of sac_device_status, then mid),
 * 256-byte aligned.
 * Returns SAC_ERR_UNSUPPORTED for fp32, groups not dividing H, rank / hidden not multiples of 8, or
 * a group width (H/groups)*D that is not a multiple of 64.
 */
SAC_API size_t sac_oproj_workspace_size(const sac_params* p, int64_t T, int groups, int rank);
SAC_API int o_proj_forward(const sac_params* p, int64_t T, int groups, int rank, int hidden,
               const void* o, const void* w_a, const void* w_b, void* out, void* ws,
               size_t ws_bytes, void* stream);

/*
 * Device status of the last call that used workspace `ws` (no counterpart on the page: failure
 * reporting). Every prefill call, and every decode call given a workspace, clears the first word
 * of its workspace; a tensor-core kernel that gives up a bounded wait (2 s) writes a nonzero code
 * there and returns instead of hanging. This call waits for `stream`, copies the word to *status
 * (0 = ok, 1 = a wait timed out, 2 = misaligned shared memory, 3 = a kernel launched with a block
 * size its arguments do not allow: an internal error, 4 = a decode / chunk context length above
 * p->S, whose rows were skipped) and returns SAC_OK, or SAC_ERR_LAUNCH if the copy fails.
 */
SAC_API int sac_device_status(const void* ws, int* status, void* stream);

/*
 * Optional per-kernel timing (no counterpart on the page: a measurement aid). Between
 * sac_timing_begin() and sac_timing_end() every kernel the library launches is bracketed by a
 * pair of CUDA events recorded on the launch's own stream. sac_timing_end() waits for those
 * events, fills up to max_entries records (one per kernel name: launches and summed device time)
 * and returns the number of distinct kernels (which may exceed max_entries), or SAC_ERR_LAUNCH.
 * Calls captured into a CUDA graph while timing is on put their event pairs into the graph; the
 * records then hold the times of the graph's most recent replay.
 *
 * CUDA graphs: after one eager call with the same shapes (which performs the one-time per-device
 * setup), the prefill, decode, chunk, append and projection entry points that take a workspace
 * may be captured into a CUDA graph; nothing they enqueue synchronises or allocates.
 */
typedef struct {
  char name[32];
  int launches;
  double total_ms;
} sac_kernel_time;

SAC_API int sac_timing_begin(void);
SAC_API int sac_timing_end(sac_kernel_time* out, int max_entries);

#ifdef __cplusplus
}
#endif

#endif /* SAC_H */
