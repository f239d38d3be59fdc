// C ABI of the hybrid-attention library (declared in include/sac.h): argument validation,
// workspace carving and the launch sequence of each layer type.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "sac.h"
#include "sac_kernels.h"
#include "sac_timing.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SAC_ERR_LAUNCH, "%s: %s", what, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
constexpr size_t kScoresBudget = size_t(1) << 30;  // bytes of indexer scores per prefill chunk

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
size_t esize(int dtype) { return dtype == SAC_F32 ? 4 : 2; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

#define REQUIRE(cond, code, ...) \
  do {                           \
    if (!(cond)) return fail(code, __VA_ARGS__); \
  } while (0)

#define REQUIRE_PTR(ptr)                                                               \
  do {                                                                                 \
    if ((ptr) == nullptr) return fail(SAC_ERR_ARG, "%s must not be NULL", #ptr);       \
    if (!aligned16(ptr)) return fail(SAC_ERR_ARG, "%s must be 16-byte aligned", #ptr); \
  } while (0)

#define OPTIONAL_PTR(ptr)                                                               \
  do {                                                                                  \
    if ((ptr) != nullptr && !aligned16(ptr))                                            \
      return fail(SAC_ERR_ARG, "%s must be 16-byte aligned", #ptr);                     \
  } while (0)

bool pow2_between(int x, int lo, int hi) {
  return x >= lo && x <= hi && (x & (x - 1)) == 0;
}

// Shape checks shared by every layer kind. kind: SAC_KIND_*; decode: p->S bounds the contexts.
int check_params(const sac_params* p, int kind, bool decode) {
  REQUIRE(p != nullptr, SAC_ERR_ARG, "params must not be NULL");
  REQUIRE(p->dtype == SAC_F32 || p->dtype == SAC_BF16, SAC_ERR_UNSUPPORTED, "dtype %d", p->dtype);
  REQUIRE(decode || p->B >= 1, SAC_ERR_ARG, "B must be >= 1 (got %d)", p->B);
  REQUIRE(p->S >= 1, SAC_ERR_ARG, "S must be >= 1 (got %d)", p->S);
  REQUIRE(p->H >= 1, SAC_ERR_ARG, "H must be >= 1 (got %d)", p->H);
  REQUIRE(pow2_between(p->D, 64, 512), SAC_ERR_UNSUPPORTED,
          "head_dim must be 64, 128, 256 or 512 (got %d)", p->D);
  REQUIRE(p->R >= 0 && p->R <= p->D && p->R % 2 == 0 && p->R / 2 <= sac::kMaxRopePairs,
          SAC_ERR_UNSUPPORTED, "rope dim must be even, <= head_dim and <= 128 (got %d)", p->R);
  REQUIRE(p->rope_theta > 0 && std::isfinite(p->rope_theta), SAC_ERR_ARG, "rope_theta must be > 0");
  if (p->rope_factor > 1.0) {
    REQUIRE(std::isfinite(p->rope_factor) && p->rope_orig_max_pos >= 1, SAC_ERR_ARG,
            "YaRN needs a finite rope_factor and rope_orig_max_pos >= 1");
    REQUIRE(std::isfinite(p->yarn_beta_fast) && p->yarn_beta_slow > 0 &&
                p->yarn_beta_fast > p->yarn_beta_slow,
            SAC_ERR_ARG, "YaRN needs yarn_beta_fast > yarn_beta_slow > 0");
  }
  REQUIRE(p->sliding_window >= 1, SAC_ERR_ARG, "sliding_window must be >= 1");
  REQUIRE(p->softmax_scale > 0 && std::isfinite(p->softmax_scale), SAC_ERR_ARG,
          "softmax_scale must be > 0");
  if (kind == SAC_KIND_HCA || kind == SAC_KIND_CSA) {
    REQUIRE(p->m >= 1, SAC_ERR_ARG, "compression rate m must be >= 1 (got %d)", p->m);
    REQUIRE(p->win_len >= 1 && p->win_len <= 4096, SAC_ERR_UNSUPPORTED,
            "compressor window must be in [1, 4096] (got %d)", p->win_len);
  }
  if (kind == SAC_KIND_CSA) {
    REQUIRE(p->n_idx_heads >= 1 && p->n_idx_heads <= 128, SAC_ERR_UNSUPPORTED,
            "index_n_heads must be in [1, 128] (got %d)", p->n_idx_heads);
    REQUIRE(pow2_between(p->idx_dim, 32, 256), SAC_ERR_UNSUPPORTED,
            "index_head_dim must be 32, 64, 128 or 256 (got %d)", p->idx_dim);
    REQUIRE(p->topk >= 1, SAC_ERR_ARG, "index_topk must be >= 1 (got %d)", p->topk);
    REQUIRE(p->S / p->m <= sac::topk_max_entries(), SAC_ERR_UNSUPPORTED,
            "at most %d pool entries per sequence (S/m = %d)", sac::topk_max_entries(),
            p->S / p->m);
    size_t smem = 4 * ((size_t)p->n_idx_heads * p->idx_dim + p->n_idx_heads +
                       64 * (size_t)(p->idx_dim + 1) + 512);
    REQUIRE(smem <= 200 * 1024, SAC_ERR_UNSUPPORTED, "indexer heads x dim too large");
  }
  return SAC_OK;
}

// Frequencies of the layer's rope pairs, in double precision. With rope_factor s > 1 they follow
// YaRN's "NTK-by-parts" interpolation (Peng et al. 2023): a pair that turns fewer than
// yarn_beta_slow times over the original context is slowed by s (position interpolation), one
// that turns more than yarn_beta_fast times is kept, and the pairs between blend the two linearly
// in their turn count.
sac::RopeFreqs rope_freqs(const sac_params* p) {
  sac::RopeFreqs rf;
  std::memset(&rf, 0, sizeof(rf));
  rf.R = p->R;
  constexpr double kTwoPi = 6.283185307179586476925;
  for (int i = 0; i < p->R / 2; ++i) {
    const double f = std::pow(p->rope_theta, -2.0 * i / p->R);
    if (!(p->rope_factor > 1.0)) {
      rf.inv_freq[i] = f;
      continue;
    }
    const double turns = (double)p->rope_orig_max_pos * f / kTwoPi;
    double keep = (turns - p->yarn_beta_slow) / (p->yarn_beta_fast - p->yarn_beta_slow);
    keep = keep < 0.0 ? 0.0 : keep > 1.0 ? 1.0 : keep;
    rf.inv_freq[i] = keep * f + (1.0 - keep) * (f / p->rope_factor);
  }
  return rf;
}

int64_t csa_chunk_rows(const sac_params* p) {
  int64_t rows = (int64_t)p->B * p->S;
  int64_t n = p->S / p->m;
  if (n == 0) return rows;
  int64_t per = (int64_t)(kScoresBudget / ((size_t)n * 4));
  if (per < 1) per = 1;
  return per < rows ? per : rows;
}

// Bump allocator over the caller's workspace.
struct Carve {
  char* base;
  size_t used = 0;
  explicit Carve(void* ws) : base(static_cast<char*>(ws)) {}
  void* take(size_t bytes) {
    void* ptr = base ? base + used : nullptr;
    used += align_up(bytes);
    return ptr;
  }
};

// bf16 layers with 64 heads of 512 run the attention on tcgen05 (attention_tc.cu).
bool use_tc_attention(const sac_params* p) {
  return p->dtype == SAC_BF16 && p->H == 64 && p->D == 512 && p->R <= 64;
}

constexpr size_t kStatusBytes = 256;  // device status word at the start of every workspace

struct Sizes {
  size_t status = kStatusBytes, kv_rot = 0, pool = 0, idx_pool = 0, scores = 0, topk = 0;
  size_t total() const {
    return align_up(status) + align_up(kv_rot) + align_up(pool) + align_up(idx_pool) +
           align_up(scores) + align_up(topk);
  }
};

Sizes prefill_sizes(const sac_params* p, int kind) {
  Sizes s;
  const size_t rows = (size_t)p->B * p->S;
  s.kv_rot = rows * p->D * esize(p->dtype);
  if (kind == SAC_KIND_HCA || kind == SAC_KIND_CSA)
    s.pool = (size_t)p->B * (p->S / p->m) * p->D * esize(p->dtype);
  if (kind == SAC_KIND_CSA) {
    s.idx_pool = (size_t)p->B * (p->S / p->m) * p->idx_dim * esize(p->dtype);
    s.scores = (size_t)csa_chunk_rows(p) * (p->S / p->m) * 4;
    s.topk = rows * p->topk * 4;
  }
  return s;
}

sac::RowAddr contiguous(const void* base, int64_t seq_stride, int width) {
  return sac::RowAddr{base, nullptr, seq_stride, 0, 1, width};
}

sac::RowAddr paged(const void* base, const int32_t* bt, int max_pages, int page_size, int width) {
  return sac::RowAddr{base, bt, 0, max_pages, page_size, width};
}

// The attention step of a call: the tensor-core kernel for bf16 layers with 64 heads of 512 (it
// rotates q itself), the CUDA-core kernel otherwise.
cudaError_t run_attention(const sac_params* p, const sac::AttnArgs& a, int64_t win_rows,
                          int64_t pool_rows, cudaStream_t st, const char* timer = "attention") {
  if (use_tc_attention(p) && sac::attention_tc_supported(a, p->dtype)) {
    return sac::timed(timer, st, [&] {
      return sac::launch_attention_tc(a, win_rows, pool_rows, st);
    });
  }
  return sac::timed(timer, st, [&] { return sac::launch_attention_simt(p->dtype, a, st); });
}

sac::AttnArgs attn_common(const sac_params* p, const void* q, void* o, const float* sinks) {
  sac::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q;
  a.o = o;
  a.sinks = sinks;
  a.H = p->H;
  a.D = p->D;
  a.W = p->sliding_window;
  a.scale = p->softmax_scale;
  a.pos0 = p->pos0;
  a.m = p->m;
  a.k = p->topk;
  a.rf = rope_freqs(p);
  a.splits = 1;
  return a;
}

}  // namespace

extern "C" {

const char* sac_last_error(void) { return g_err; }

int sac_version(void) { return 200; }

size_t sac_workspace_size(const sac_params* p, int kind) {
  if (kind < SAC_KIND_SWA || kind > SAC_KIND_CSA || check_params(p, kind, false) != SAC_OK)
    return 0;
  return prefill_sizes(p, kind).total();
}

int swa_forward(const sac_params* p, const void* q, const void* kv, const float* sinks, void* o,
                void* ws, size_t ws_bytes, void* stream) {
  int rc = check_params(p, SAC_KIND_SWA, false);
  if (rc) return rc;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kv);
  REQUIRE_PTR(sinks);
  REQUIRE_PTR(o);
  Sizes sz = prefill_sizes(p, SAC_KIND_SWA);
  REQUIRE(ws != nullptr && ws_bytes >= sz.total(), SAC_ERR_WORKSPACE,
          "workspace of %zu bytes needed (got %zu)", sz.total(), ws_bytes);
  REQUIRE(aligned16(ws), SAC_ERR_ARG, "ws must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve cv(ws);
  int* status = static_cast<int*>(cv.take(sz.status));
  void* kv_rot = cv.take(sz.kv_rot);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  sac::RopeFreqs rf = rope_freqs(p);
  const int64_t rows = (int64_t)p->B * p->S;
  e = sac::timed("rotate_kv", st, [&] { return sac::launch_rotate_rows(p->dtype, kv, rows, p->S, p->D, rf, p->pos0, kv_rot, st); });
  if (e != cudaSuccess) return cuda_fail(e, "rotate kv");
  sac::AttnArgs a = attn_common(p, q, o, sinks);
  a.qr = sac::QueryRows{p->S, nullptr, 0};
  a.nrows = rows;
  a.win = contiguous(kv_rot, p->S, p->D);
  a.pool_mode = 0;
  a.status = status;
  e = run_attention(p, a, rows, 0, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention");
  return SAC_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// swa_forward_static: the sliding-window forward with its scratch (the rotated kv stream) in a
// fixed device array owned by this library, for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------------------------
namespace {
constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB on every device that loads us
constexpr int kMaxDevices = 64;
}  // namespace

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (the host symbol is only a stand-in:
// kernels must be given this address). The first call on a device looks it up with that device
// current; later calls look it up again whenever their stream is not capturing, so a context torn
// down and created again (cudaDeviceReset) gets the address of its own copy. A capturing stream
// takes the address found by the device's last look-up (none yet: an error).
int static_scratch_address(cudaStream_t st, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  REQUIRE(dev >= 0 && dev < kMaxDevices, SAC_ERR_UNSUPPORTED, "device ordinal %d", dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
  std::lock_guard<std::mutex> lk(g_static_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_scratch_addr[dev] = ptr;
  }
  REQUIRE(g_static_scratch_addr[dev] != nullptr, SAC_ERR_ARG,
          "swa_forward_static: the first call on a device must come before any stream capture");
  *out = g_static_scratch_addr[dev];
  return SAC_OK;
}
}  // namespace

extern "C" {

size_t sac_static_scratch_bytes(void) { return kStaticScratchBytes; }

int swa_forward_static(const sac_params* p, const void* q, const void* kv, const float* sinks,
                       void* o, void* stream) {
  int rc = check_params(p, SAC_KIND_SWA, false);
  if (rc) return rc;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kv);
  REQUIRE_PTR(sinks);
  REQUIRE_PTR(o);
  // the scratch swa_forward takes from its workspace for the rotated kv stream
  const size_t need = (size_t)p->B * p->S * p->D * esize(p->dtype);
  REQUIRE(need <= kStaticScratchBytes, SAC_ERR_UNSUPPORTED,
          "B*S*head_dim needs %zu bytes of scratch; the static scratch holds %zu", need,
          kStaticScratchBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* kv_rot = nullptr;
  rc = static_scratch_address(st, &kv_rot);
  if (rc) return rc;
  sac::RopeFreqs rf = rope_freqs(p);
  const int64_t rows = (int64_t)p->B * p->S;
  cudaError_t e = sac::timed("rotate_kv", st, [&] {
    return sac::launch_rotate_rows(p->dtype, kv, rows, p->S, p->D, rf, p->pos0, kv_rot, st);
  });
  if (e != cudaSuccess) return cuda_fail(e, "rotate kv");
  sac::AttnArgs a = attn_common(p, q, o, sinks);
  a.qr = sac::QueryRows{p->S, nullptr, 0};
  a.nrows = rows;
  a.win = contiguous(kv_rot, p->S, p->D);
  a.pool_mode = 0;
  // no status word: a kernel giving up a bounded wait returns silently
  e = run_attention(p, a, rows, 0, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention");
  return SAC_OK;
}

int hca_forward(const sac_params* p, const void* q, const void* kv, const void* cmp_gate,
                const float* cmp_bias, const float* sinks, void* o, void* pool_out, void* ws,
                size_t ws_bytes, void* stream) {
  int rc = check_params(p, SAC_KIND_HCA, false);
  if (rc) return rc;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kv);
  REQUIRE_PTR(cmp_gate);
  REQUIRE(cmp_bias != nullptr, SAC_ERR_ARG, "cmp_bias must not be NULL");
  REQUIRE_PTR(sinks);
  REQUIRE_PTR(o);
  OPTIONAL_PTR(pool_out);
  Sizes sz = prefill_sizes(p, SAC_KIND_HCA);
  if (pool_out) sz.pool = 0;
  REQUIRE(ws != nullptr && ws_bytes >= sz.total(), SAC_ERR_WORKSPACE,
          "workspace of %zu bytes needed (got %zu)", sz.total(), ws_bytes);
  REQUIRE(aligned16(ws), SAC_ERR_ARG, "ws must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve cv(ws);
  int* status = static_cast<int*>(cv.take(sz.status));
  void* kv_rot = cv.take(sz.kv_rot);
  void* pool = pool_out ? pool_out : cv.take(sz.pool);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  sac::RopeFreqs rf = rope_freqs(p);
  const int64_t rows = (int64_t)p->B * p->S;
  e = sac::timed("rotate_kv", st, [&] { return sac::launch_rotate_rows(p->dtype, kv, rows, p->S, p->D, rf, p->pos0, kv_rot, st); });
  if (e != cudaSuccess) return cuda_fail(e, "rotate kv");
  e = sac::timed("compress", st, [&] { return sac::launch_compress(p->dtype, kv, cmp_gate, cmp_bias, p->B, p->S, p->D, p->m, p->win_len,
                           true, rf, p->pos0, pool, status, st); });
  if (e != cudaSuccess) return cuda_fail(e, "compress");
  sac::AttnArgs a = attn_common(p, q, o, sinks);
  a.qr = sac::QueryRows{p->S, nullptr, 0};
  a.nrows = rows;
  a.win = contiguous(kv_rot, p->S, p->D);
  a.pool_mode = 1;
  a.pool = contiguous(pool, p->S / p->m, p->D);
  a.status = status;
  e = run_attention(p, a, rows, (int64_t)p->B * (p->S / p->m), st);
  if (e != cudaSuccess) return cuda_fail(e, "attention");
  return SAC_OK;
}

int csa_forward(const sac_params* p, const void* q, const void* kv, const void* cmp_gate,
                const float* cmp_bias, const void* q_idx, const float* w_idx, const void* k_idx,
                const void* idx_gate, const float* idx_bias, const float* sinks, void* o,
                int32_t* topk_out, void* pool_out, void* idx_pool_out, void* ws, size_t ws_bytes,
                void* stream) {
  int rc = check_params(p, SAC_KIND_CSA, false);
  if (rc) return rc;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kv);
  REQUIRE_PTR(cmp_gate);
  REQUIRE(cmp_bias != nullptr, SAC_ERR_ARG, "cmp_bias must not be NULL");
  REQUIRE_PTR(q_idx);
  REQUIRE_PTR(w_idx);
  REQUIRE_PTR(k_idx);
  REQUIRE_PTR(idx_gate);
  REQUIRE(idx_bias != nullptr, SAC_ERR_ARG, "idx_bias must not be NULL");
  REQUIRE_PTR(sinks);
  REQUIRE_PTR(o);
  OPTIONAL_PTR(topk_out);
  OPTIONAL_PTR(pool_out);
  OPTIONAL_PTR(idx_pool_out);
  Sizes sz = prefill_sizes(p, SAC_KIND_CSA);
  if (pool_out) sz.pool = 0;
  if (idx_pool_out) sz.idx_pool = 0;
  if (topk_out) sz.topk = 0;
  REQUIRE(ws != nullptr && ws_bytes >= sz.total(), SAC_ERR_WORKSPACE,
          "workspace of %zu bytes needed (got %zu)", sz.total(), ws_bytes);
  REQUIRE(aligned16(ws), SAC_ERR_ARG, "ws must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve cv(ws);
  int* status = static_cast<int*>(cv.take(sz.status));
  void* kv_rot = cv.take(sz.kv_rot);
  void* pool = pool_out ? pool_out : cv.take(sz.pool);
  void* ipool = idx_pool_out ? idx_pool_out : cv.take(sz.idx_pool);
  float* scores = static_cast<float*>(cv.take(sz.scores));
  int32_t* sel = topk_out ? topk_out : static_cast<int32_t*>(cv.take(sz.topk));

  sac::RopeFreqs rf = rope_freqs(p);
  const int64_t rows = (int64_t)p->B * p->S;
  const int N = p->S / p->m;
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  e = sac::timed("rotate_kv", st, [&] { return sac::launch_rotate_rows(p->dtype, kv, rows, p->S, p->D, rf, p->pos0, kv_rot, st); });
  if (e != cudaSuccess) return cuda_fail(e, "rotate kv");
  e = sac::timed("compress", st, [&] { return sac::launch_compress(p->dtype, kv, cmp_gate, cmp_bias, p->B, p->S, p->D, p->m, p->win_len,
                           true, rf, p->pos0, pool, status, st); });
  if (e != cudaSuccess) return cuda_fail(e, "compress");
  e = sac::timed("compress_index", st, [&] { return sac::launch_compress(p->dtype, k_idx, idx_gate, idx_bias, p->B, p->S, p->idx_dim, p->m,
                           p->win_len, false, rf, p->pos0, ipool, status, st); });
  if (e != cudaSuccess) return cuda_fail(e, "compress indexer stream");

  // indexer + top-k in chunks of query rows of one sequence (bounded scores buffer)
  const int64_t chunk = csa_chunk_rows(p);
  const size_t qi_row = (size_t)p->n_idx_heads * p->idx_dim * esize(p->dtype);
  const bool idx_tc = sac::indexer_tc_supported(p->dtype, p->n_idx_heads, p->idx_dim);
  for (int b = 0; b < p->B; ++b) {
    for (int64_t t0 = 0; t0 < p->S; t0 += chunk) {
      const int64_t t1 = t0 + chunk < p->S ? t0 + chunk : p->S;
      const int64_t r0 = (int64_t)b * p->S + t0, nr = t1 - t0;
      sac::QueryRows qr{p->S, nullptr, r0};
      if (idx_tc) {
        sac::IndexerTcArgs ta;
        ta.w_idx = w_idx;
        ta.scores = scores;
        ta.status = status;
        ta.t0 = t0;
        ta.t1 = t1;
        ta.seq = b;
        ta.S = p->S;
        ta.N = N;
        ta.m = p->m;
        ta.n_stride = N;
        e = sac::timed("indexer_score", st, [&] {
          return sac::launch_indexer_tc(ta, q_idx, rows, ipool, (int64_t)p->B * N, st);
        });
      } else {
        sac::IndexerArgs ia;
        ia.q_idx = static_cast<const char*>(q_idx) + (size_t)r0 * qi_row;
        ia.w_idx = w_idx + (size_t)r0 * p->n_idx_heads;
        ia.kpool = contiguous(ipool, N, p->idx_dim);
        ia.qr = qr;
        ia.nI = p->n_idx_heads;
        ia.cI = p->idx_dim;
        ia.m = p->m;
        ia.nrows = nr;
        ia.n_stride = N;
        ia.scores = scores;
        const int max_vis = (int)(t1 / p->m);
        e = sac::timed("indexer_score", st,
                       [&] { return sac::launch_indexer(p->dtype, ia, max_vis, st); });
      }
      if (e != cudaSuccess) return cuda_fail(e, "indexer");
      e = sac::timed("topk", st, [&] {
        return sac::launch_topk(scores, N, qr, p->m, nr, p->topk, sel + r0 * p->topk, st);
      });
      if (e != cudaSuccess) return cuda_fail(e, "top-k");
    }
  }

  sac::AttnArgs a = attn_common(p, q, o, sinks);
  a.qr = sac::QueryRows{p->S, nullptr, 0};
  a.nrows = rows;
  a.win = contiguous(kv_rot, p->S, p->D);
  a.pool_mode = 2;
  a.pool = contiguous(pool, N, p->D);
  a.sel = sel;
  a.status = status;
  e = run_attention(p, a, rows, (int64_t)p->B * N, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention");
  return SAC_OK;
}

int sac_device_status(const void* ws, int* status, void* stream) {
  REQUIRE(ws != nullptr && status != nullptr, SAC_ERR_ARG, "ws and status must not be NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(status, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  return SAC_OK;
}

// ---------------------------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------------------------
// Decode attention on tensor cores splits each sequence's key tiles over several CTAs when there
// are fewer sequences than SMs; the partial results need nseq * splits * H * (D + 2) floats.
static int decode_splits(const sac_params* p, int64_t rows) {
  if (!use_tc_attention(p)) return 1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Splitting pays only when it multiplies the CTAs several times over: at 2 or 3 splits the
  // fp32 partials and the combine launch cost about what the shorter key walk saves (64
  // sequences on 148 SMs: CSA 3% faster, HCA 10% slower split in two; 16 sequences in 8 splits:
  // 29% and 17% faster).
  int64_t sp = sms / rows;
  if (sp > sac::attention_tc_max_splits()) sp = sac::attention_tc_max_splits();
  return sp < 4 ? 1 : (int)sp;
}

static size_t decode_split_bytes(const sac_params* p, int64_t rows) {
  const int sp = decode_splits(p, rows);
  if (sp == 1) return 0;
  return align_up((size_t)rows * sp * p->H * p->D * 4) + align_up((size_t)rows * sp * p->H * 2 * 4);
}

// Point a paged call's attention at its split buffers (after the first `used` bytes of ws) when
// the workspace holds them; otherwise the attention runs unsplit.
static void decode_attach_splits(const sac_params* p, int64_t rows, void* ws, size_t ws_bytes,
                                 size_t used, sac::AttnArgs& a) {
  const int sp = decode_splits(p, rows);
  const size_t need = decode_split_bytes(p, rows);
  if (sp == 1 || ws == nullptr || ws_bytes < used + need) return;
  char* base = static_cast<char*>(ws) + used;
  a.splits = sp;
  a.part_o = reinterpret_cast<float*>(base);
  a.part_ml = reinterpret_cast<float*>(base + align_up((size_t)rows * sp * p->H * p->D * 4));
}

// CSA query rows whose indexer scores share the workspace at once (the rest run in blocks).
static int64_t paged_score_rows(const sac_params* p, int64_t rows) {
  const int64_t n = p->S / p->m;
  int64_t per = n > 0 ? (int64_t)(kScoresBudget / ((size_t)n * 4)) : rows;
  if (per < 1) per = 1;
  return rows < per ? rows : per;
}

static size_t paged_workspace_size(const sac_params* p, int kind, int64_t rows) {
  size_t bytes = kStatusBytes;
  if (kind == SAC_KIND_CSA) {
    const size_t n = (size_t)(p->S / p->m);
    bytes += align_up((size_t)paged_score_rows(p, rows) * n * 4) +
             align_up((size_t)rows * p->topk * 4);
  }
  return bytes + decode_split_bytes(p, rows);
}

size_t sac_decode_workspace_size(const sac_params* p, int kind, int nseq) {
  if (kind < SAC_KIND_SWA || kind > SAC_KIND_CSA || nseq < 1 ||
      check_params(p, kind, true) != SAC_OK)
    return 0;
  return paged_workspace_size(p, kind, nseq);
}

size_t sac_chunk_workspace_size(const sac_params* p, int kind, int nseq, int n) {
  if (kind < SAC_KIND_SWA || kind > SAC_KIND_CSA || nseq < 1 || n < 1 ||
      check_params(p, kind, true) != SAC_OK)
    return 0;
  return paged_workspace_size(p, kind, (int64_t)nseq * n);
}

// Status word of a decode call: the first word of ws when one is given (cleared here), else none
// (the tensor-core kernels then give up timed-out waits silently).
static int decode_status(void* ws, size_t ws_bytes, cudaStream_t st, int** status) {
  *status = nullptr;
  if (ws == nullptr) return SAC_OK;
  REQUIRE(ws_bytes >= kStatusBytes, SAC_ERR_WORKSPACE,
          "a decode workspace holds at least the %zu-byte status word (got %zu)", kStatusBytes,
          ws_bytes);
  REQUIRE(aligned16(ws), SAC_ERR_ARG, "ws must be 16-byte aligned");
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  *status = static_cast<int*>(ws);
  return SAC_OK;
}

static int check_decode_common(const sac_params* p, int kind, int nseq, const void* q,
                               const void* kv_pages, const int32_t* kv_block_table,
                               int kv_max_pages, const int32_t* ctx_lens, int page_size,
                               const float* sinks, void* o) {
  int rc = check_params(p, kind, true);
  if (rc) return rc;
  REQUIRE(nseq >= 1, SAC_ERR_ARG, "nseq must be >= 1 (got %d)", nseq);
  REQUIRE(page_size >= 1, SAC_ERR_ARG, "page_size must be >= 1 (got %d)", page_size);
  REQUIRE(kv_max_pages >= 1, SAC_ERR_ARG, "kv_max_pages must be >= 1");
  REQUIRE((int64_t)kv_max_pages * page_size >= p->S, SAC_ERR_ARG,
          "kv block table too short for contexts up to S=%d", p->S);
  REQUIRE_PTR(q);
  REQUIRE_PTR(kv_pages);
  REQUIRE(kv_block_table != nullptr, SAC_ERR_ARG, "kv_block_table must not be NULL");
  REQUIRE(ctx_lens != nullptr, SAC_ERR_ARG, "ctx_lens must not be NULL");
  REQUIRE_PTR(sinks);
  REQUIRE_PTR(o);
  return SAC_OK;
}

// Attention of nq query rows per sequence (the last nq positions of each context; nq = 1 for a
// decode step) over the paged caches: window keys from the kv pages, HCA pool entries or the CSA
// indexer's top-k of the pool pages.
struct PagedCall {
  int kind, nseq, nq;
  const void *q, *kv_pages;
  const int32_t *kv_block_table, *ctx_lens;
  int kv_max_pages, page_size;
  const void *pool_pages, *idx_pool_pages;
  const int32_t* pool_block_table;
  int pool_max_pages;
  const void* q_idx;
  const float *w_idx, *sinks;
  void* o;
  int32_t* topk_out;
  void* ws;
  size_t ws_bytes;
  void* stream;
  const char* timer;  // attention timer name
};

static int paged_attention(const sac_params* p, const PagedCall& c) {
  int rc = check_decode_common(p, c.kind, c.nseq, c.q, c.kv_pages, c.kv_block_table,
                               c.kv_max_pages, c.ctx_lens, c.page_size, c.sinks, c.o);
  if (rc) return rc;
  REQUIRE(c.nq >= 1, SAC_ERR_ARG, "query rows per sequence must be >= 1 (got %d)", c.nq);
  const int64_t rows = (int64_t)c.nseq * c.nq;
  if (c.kind != SAC_KIND_SWA) {
    REQUIRE(c.pool_pages != nullptr, SAC_ERR_ARG, "pool_pages must not be NULL");
    REQUIRE(aligned16(c.pool_pages), SAC_ERR_ARG, "pool_pages must be 16-byte aligned");
    REQUIRE(c.pool_block_table != nullptr, SAC_ERR_ARG, "pool_block_table must not be NULL");
    REQUIRE((int64_t)c.pool_max_pages * c.page_size >= p->S / p->m, SAC_ERR_ARG,
            "pool block table too short for S/m entries");
  }
  cudaStream_t st = static_cast<cudaStream_t>(c.stream);
  sac::QueryRows qr{0, c.ctx_lens, 0, c.nq, (int64_t)p->S};
  sac::AttnArgs a = attn_common(p, c.q, c.o, c.sinks);
  a.qr = qr;
  a.nrows = rows;
  a.win = paged(c.kv_pages, c.kv_block_table, c.kv_max_pages, c.page_size, p->D);
  a.pool_mode = c.kind == SAC_KIND_SWA ? 0 : c.kind == SAC_KIND_HCA ? 1 : 2;
  if (c.kind != SAC_KIND_SWA)
    a.pool = paged(c.pool_pages, c.pool_block_table, c.pool_max_pages, c.page_size, p->D);
  size_t used = kStatusBytes;
  int* status = nullptr;
  if (c.kind == SAC_KIND_CSA) {
    REQUIRE(c.idx_pool_pages != nullptr, SAC_ERR_ARG, "idx_pool_pages must not be NULL");
    REQUIRE(aligned16(c.idx_pool_pages), SAC_ERR_ARG, "idx_pool_pages must be 16-byte aligned");
    REQUIRE(c.q_idx != nullptr, SAC_ERR_ARG, "q_idx must not be NULL");
    REQUIRE(aligned16(c.q_idx), SAC_ERR_ARG, "q_idx must be 16-byte aligned");
    REQUIRE(c.w_idx != nullptr, SAC_ERR_ARG, "w_idx must not be NULL");
    REQUIRE(aligned16(c.w_idx), SAC_ERR_ARG, "w_idx must be 16-byte aligned");
    REQUIRE(c.topk_out == nullptr || aligned16(c.topk_out), SAC_ERR_ARG,
            "topk_out must be 16-byte aligned");
    const int N = p->S / p->m;
    const int64_t score_rows = paged_score_rows(p, rows);
    const size_t need = kStatusBytes + align_up((size_t)score_rows * N * 4) +
                        (c.topk_out ? 0 : align_up((size_t)rows * p->topk * 4));
    REQUIRE(c.ws != nullptr && c.ws_bytes >= need, SAC_ERR_WORKSPACE,
            "workspace of %zu bytes needed (got %zu)", need, c.ws_bytes);
    rc = decode_status(c.ws, c.ws_bytes, st, &status);
    if (rc) return rc;
    Carve cv(c.ws);
    cv.take(kStatusBytes);
    float* scores = static_cast<float*>(cv.take((size_t)score_rows * N * 4));
    int32_t* sel =
        c.topk_out ? c.topk_out : static_cast<int32_t*>(cv.take((size_t)rows * p->topk * 4));
    used = cv.used;
    const size_t qi_row = (size_t)p->n_idx_heads * p->idx_dim * esize(p->dtype);
    for (int64_t r0 = 0; r0 < rows; r0 += score_rows) {
      const int64_t nr = rows - r0 < score_rows ? rows - r0 : score_rows;
      sac::QueryRows bq{0, c.ctx_lens, r0, c.nq, (int64_t)p->S};
      sac::IndexerArgs ia;
      ia.q_idx = static_cast<const char*>(c.q_idx) + (size_t)r0 * qi_row;
      ia.w_idx = c.w_idx + (size_t)r0 * p->n_idx_heads;
      ia.kpool = paged(c.idx_pool_pages, c.pool_block_table, c.pool_max_pages, c.page_size,
                       p->idx_dim);
      ia.qr = bq;
      ia.nI = p->n_idx_heads;
      ia.cI = p->idx_dim;
      ia.m = p->m;
      ia.nrows = nr;
      ia.n_stride = N;
      ia.scores = scores;
      cudaError_t e = sac::timed("indexer_score", st, [&] {
        if (sac::indexer_decode_tc_supported(p->dtype, p->n_idx_heads, p->idx_dim))
          return sac::launch_indexer_decode_tc(ia, N, status, st);
        return sac::launch_indexer(p->dtype, ia, N, st);
      });
      if (e != cudaSuccess) return cuda_fail(e, "indexer");
      e = sac::timed("topk", st, [&] {
        return sac::launch_topk(scores, N, bq, p->m, nr, p->topk, sel + r0 * p->topk, st);
      });
      if (e != cudaSuccess) return cuda_fail(e, "top-k");
    }
    a.sel = sel;
  } else {
    rc = decode_status(c.ws, c.ws_bytes, st, &status);
    if (rc) return rc;
  }
  a.status = status;
  decode_attach_splits(p, rows, c.ws, c.ws_bytes, used, a);
  cudaError_t e = run_attention(p, a, 0, 0, st, c.timer);  // paged: extents from the tables
  if (e != cudaSuccess) return cuda_fail(e, "attention");
  return SAC_OK;
}

static PagedCall paged_call(int kind, int nseq, int nq, const void* q, const void* kv_pages,
                            const int32_t* kv_block_table, int kv_max_pages,
                            const int32_t* ctx_lens, int page_size, const float* sinks, void* o,
                            void* ws, size_t ws_bytes, void* stream, const char* timer) {
  PagedCall c;
  std::memset(&c, 0, sizeof(c));
  c.kind = kind;
  c.nseq = nseq;
  c.nq = nq;
  c.q = q;
  c.kv_pages = kv_pages;
  c.kv_block_table = kv_block_table;
  c.kv_max_pages = kv_max_pages;
  c.ctx_lens = ctx_lens;
  c.page_size = page_size;
  c.sinks = sinks;
  c.o = o;
  c.ws = ws;
  c.ws_bytes = ws_bytes;
  c.stream = stream;
  c.timer = timer;
  return c;
}

int swa_decode(const sac_params* p, int nseq, const void* q, const void* kv_pages,
               const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
               int page_size, const float* sinks, void* o, void* ws, size_t ws_bytes,
               void* stream) {
  return paged_attention(p, paged_call(SAC_KIND_SWA, nseq, 1, q, kv_pages, kv_block_table,
                                       kv_max_pages, ctx_lens, page_size, sinks, o, ws, ws_bytes,
                                       stream, "swa_decode_attention"));
}

int hca_decode(const sac_params* p, int nseq, const void* q, const void* kv_pages,
               const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
               int page_size, const void* pool_pages, const int32_t* pool_block_table,
               int pool_max_pages, const float* sinks, void* o, void* ws, size_t ws_bytes,
               void* stream) {
  PagedCall c = paged_call(SAC_KIND_HCA, nseq, 1, q, kv_pages, kv_block_table, kv_max_pages,
                           ctx_lens, page_size, sinks, o, ws, ws_bytes, stream,
                           "hca_decode_attention");
  c.pool_pages = pool_pages;
  c.pool_block_table = pool_block_table;
  c.pool_max_pages = pool_max_pages;
  return paged_attention(p, c);
}

int csa_decode(const sac_params* p, int nseq, const void* q, const void* kv_pages,
               const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
               int page_size, const void* pool_pages, const void* idx_pool_pages,
               const int32_t* pool_block_table, int pool_max_pages, const void* q_idx,
               const float* w_idx, const float* sinks, void* o, int32_t* topk_out, void* ws,
               size_t ws_bytes, void* stream) {
  PagedCall c = paged_call(SAC_KIND_CSA, nseq, 1, q, kv_pages, kv_block_table, kv_max_pages,
                           ctx_lens, page_size, sinks, o, ws, ws_bytes, stream,
                           "csa_decode_attention");
  c.pool_pages = pool_pages;
  c.idx_pool_pages = idx_pool_pages;
  c.pool_block_table = pool_block_table;
  c.pool_max_pages = pool_max_pages;
  c.q_idx = q_idx;
  c.w_idx = w_idx;
  c.topk_out = topk_out;
  return paged_attention(p, c);
}

int swa_prefill_chunk(const sac_params* p, int nseq, int n, const void* q, const void* kv_pages,
                      const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
                      int page_size, const float* sinks, void* o, void* ws, size_t ws_bytes,
                      void* stream) {
  return paged_attention(p, paged_call(SAC_KIND_SWA, nseq, n, q, kv_pages, kv_block_table,
                                       kv_max_pages, ctx_lens, page_size, sinks, o, ws, ws_bytes,
                                       stream, "swa_chunk_attention"));
}

int hca_prefill_chunk(const sac_params* p, int nseq, int n, const void* q, const void* kv_pages,
                      const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
                      int page_size, const void* pool_pages, const int32_t* pool_block_table,
                      int pool_max_pages, const float* sinks, void* o, void* ws, size_t ws_bytes,
                      void* stream) {
  PagedCall c = paged_call(SAC_KIND_HCA, nseq, n, q, kv_pages, kv_block_table, kv_max_pages,
                           ctx_lens, page_size, sinks, o, ws, ws_bytes, stream,
                           "hca_chunk_attention");
  c.pool_pages = pool_pages;
  c.pool_block_table = pool_block_table;
  c.pool_max_pages = pool_max_pages;
  return paged_attention(p, c);
}

int csa_prefill_chunk(const sac_params* p, int nseq, int n, const void* q, const void* kv_pages,
                      const int32_t* kv_block_table, int kv_max_pages, const int32_t* ctx_lens,
                      int page_size, const void* pool_pages, const void* idx_pool_pages,
                      const int32_t* pool_block_table, int pool_max_pages, const void* q_idx,
                      const float* w_idx, const float* sinks, void* o, int32_t* topk_out,
                      void* ws, size_t ws_bytes, void* stream) {
  PagedCall c = paged_call(SAC_KIND_CSA, nseq, n, q, kv_pages, kv_block_table, kv_max_pages,
                           ctx_lens, page_size, sinks, o, ws, ws_bytes, stream,
                           "csa_chunk_attention");
  c.pool_pages = pool_pages;
  c.idx_pool_pages = idx_pool_pages;
  c.pool_block_table = pool_block_table;
  c.pool_max_pages = pool_max_pages;
  c.q_idx = q_idx;
  c.w_idx = w_idx;
  c.topk_out = topk_out;
  return paged_attention(p, c);
}

// Cache append of n tokens per sequence (the last n of each context); n = 0 is a decode step
// (one token, the decode kernel), n >= 1 a prefill chunk (the chunk kernels).
static int append_paged(const sac_params* p, int kind, int nseq, int n, const int32_t* ctx_lens,
                        const void* kv_new, const void* k_idx_new, const void* cmp_gate,
                        const float* cmp_bias, const void* idx_gate, const float* idx_bias,
                        void* kv_pages, const int32_t* kv_block_table, int kv_max_pages,
                        int page_size, void* cmp_state, void* idx_state, void* pool_pages,
                        void* idx_pool_pages, const int32_t* pool_block_table, int pool_max_pages,
                        void* stream) {
  REQUIRE(kind >= SAC_KIND_SWA && kind <= SAC_KIND_CSA, SAC_ERR_ARG, "unknown layer kind %d", kind);
  int rc = check_params(p, kind, true);
  if (rc) return rc;
  REQUIRE(nseq >= 1, SAC_ERR_ARG, "nseq must be >= 1 (got %d)", nseq);
  REQUIRE(n >= 0, SAC_ERR_ARG, "chunk tokens must be >= 1 (got %d)", n);
  REQUIRE(page_size >= 1, SAC_ERR_ARG, "page_size must be >= 1 (got %d)", page_size);
  REQUIRE(ctx_lens != nullptr, SAC_ERR_ARG, "ctx_lens must not be NULL");
  REQUIRE_PTR(kv_new);
  REQUIRE_PTR(kv_pages);
  REQUIRE(kv_block_table != nullptr, SAC_ERR_ARG, "kv_block_table must not be NULL");
  REQUIRE(kv_max_pages >= 1 && (int64_t)kv_max_pages * page_size >= p->S, SAC_ERR_ARG,
          "kv block table too short for contexts up to S=%d", p->S);
  sac::DecodeAppendArgs a;
  std::memset(&a, 0, sizeof(a));
  a.nseq = nseq;
  a.ctx_lens = ctx_lens;
  a.max_ctx = p->S;
  a.D = p->D;
  a.pos0 = p->pos0;
  a.rf = rope_freqs(p);
  a.kv_new = kv_new;
  a.kv_pages = kv_pages;
  a.kv_block_table = kv_block_table;
  a.kv_max_pages = kv_max_pages;
  a.page_size = page_size;
  if (kind != SAC_KIND_SWA) {
    REQUIRE_PTR(cmp_state);
    REQUIRE_PTR(cmp_gate);
    REQUIRE(cmp_bias != nullptr, SAC_ERR_ARG, "cmp_bias must not be NULL");
    REQUIRE_PTR(pool_pages);
    REQUIRE(pool_block_table != nullptr, SAC_ERR_ARG, "pool_block_table must not be NULL");
    REQUIRE((int64_t)pool_max_pages * page_size >= p->S / p->m, SAC_ERR_ARG,
            "pool block table too short for S/m entries");
    a.m = p->m;
    a.L = p->win_len;
    a.cmp_gate = cmp_gate;
    a.cmp_bias = cmp_bias;
    a.cmp_state = cmp_state;
    a.pool_pages = pool_pages;
    a.pool_block_table = pool_block_table;
    a.pool_max_pages = pool_max_pages;
  }
  if (kind == SAC_KIND_CSA) {
    REQUIRE_PTR(k_idx_new);
    REQUIRE_PTR(idx_state);
    REQUIRE_PTR(idx_gate);
    REQUIRE(idx_bias != nullptr, SAC_ERR_ARG, "idx_bias must not be NULL");
    REQUIRE_PTR(idx_pool_pages);
    a.cI = p->idx_dim;
    a.k_idx_new = k_idx_new;
    a.idx_gate = idx_gate;
    a.idx_bias = idx_bias;
    a.idx_state = idx_state;
    a.idx_pool_pages = idx_pool_pages;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (n == 0) {
    if (kind == SAC_KIND_CSA && sac::decode_append_pair_supported(a)) {
      // both parts in one launch
      e = sac::timed("decode_append", st, [&] {
        return sac::launch_decode_append_pair(p->dtype, a, st);
      });
    } else {
      e = sac::timed("decode_append", st, [&] {
        return sac::launch_decode_append(p->dtype, a, false, st);
      });
      if (e == cudaSuccess && kind == SAC_KIND_CSA)
        e = sac::timed("decode_append_index", st, [&] {
          return sac::launch_decode_append(p->dtype, a, true, st);
        });
    }
  } else {
    e = sac::timed("chunk_append", st, [&] {
      return sac::launch_chunk_append(p->dtype, a, n, false, st);
    });
    if (e == cudaSuccess && kind == SAC_KIND_CSA)
      e = sac::timed("chunk_append_index", st, [&] {
        return sac::launch_chunk_append(p->dtype, a, n, true, st);
      });
  }
  if (e != cudaSuccess) return cuda_fail(e, "cache append");
  return SAC_OK;
}

int decode_append(const sac_params* p, int kind, int nseq, const int32_t* ctx_lens,
                  const void* kv_new, const void* k_idx_new, const void* cmp_gate,
                  const float* cmp_bias, const void* idx_gate, const float* idx_bias,
                  void* kv_pages, const int32_t* kv_block_table, int kv_max_pages, int page_size,
                  void* cmp_state, void* idx_state, void* pool_pages, void* idx_pool_pages,
                  const int32_t* pool_block_table, int pool_max_pages, void* stream) {
  return append_paged(p, kind, nseq, 0, ctx_lens, kv_new, k_idx_new, cmp_gate, cmp_bias,
                      idx_gate, idx_bias, kv_pages, kv_block_table, kv_max_pages, page_size,
                      cmp_state, idx_state, pool_pages, idx_pool_pages, pool_block_table,
                      pool_max_pages, stream);
}

int prefill_chunk_append(const sac_params* p, int kind, int nseq, int n, const int32_t* ctx_lens,
                         const void* kv_new, const void* k_idx_new, const void* cmp_gate,
                         const float* cmp_bias, const void* idx_gate, const float* idx_bias,
                         void* kv_pages, const int32_t* kv_block_table, int kv_max_pages,
                         int page_size, void* cmp_state, void* idx_state, void* pool_pages,
                         void* idx_pool_pages, const int32_t* pool_block_table,
                         int pool_max_pages, void* stream) {
  REQUIRE(n >= 1, SAC_ERR_ARG, "chunk tokens must be >= 1 (got %d)", n);
  return append_paged(p, kind, nseq, n, ctx_lens, kv_new, k_idx_new, cmp_gate, cmp_bias,
                      idx_gate, idx_bias, kv_pages, kv_block_table, kv_max_pages, page_size,
                      cmp_state, idx_state, pool_pages, idx_pool_pages, pool_block_table,
                      pool_max_pages, stream);
}

size_t sac_oproj_workspace_size(const sac_params* p, int64_t T, int groups, int rank) {
  if (p == nullptr || T < 0 || groups < 1 || rank < 1) return 0;
  return kStatusBytes + align_up((size_t)T * groups * rank * 2);
}

int o_proj_forward(const sac_params* p, int64_t T, int groups, int rank, int hidden,
                   const void* o, const void* w_a, const void* w_b, void* out, void* ws,
                   size_t ws_bytes, void* stream) {
  REQUIRE(p != nullptr, SAC_ERR_ARG, "params must not be NULL");
  REQUIRE(p->dtype == SAC_BF16, SAC_ERR_UNSUPPORTED, "the output projection takes bf16");
  REQUIRE(T >= 0, SAC_ERR_ARG, "T must be >= 0");
  REQUIRE(p->H >= 1 && p->D >= 8 && p->D % 8 == 0, SAC_ERR_ARG, "bad head shape");
  REQUIRE(groups >= 1 && p->H % groups == 0, SAC_ERR_UNSUPPORTED,
          "o_groups (%d) must divide the head count (%d)", groups, p->H);
  REQUIRE(rank >= 8 && rank % 8 == 0 && hidden >= 8 && hidden % 8 == 0, SAC_ERR_UNSUPPORTED,
          "o_lora_rank and hidden must be positive multiples of 8");
  REQUIRE((p->H / groups) * p->D % 64 == 0, SAC_ERR_UNSUPPORTED,
          "a group's features ((H/o_groups)*head_dim) must be a multiple of 64");
  REQUIRE_PTR(o);
  REQUIRE_PTR(w_a);
  REQUIRE_PTR(w_b);
  REQUIRE_PTR(out);
  const size_t need = sac_oproj_workspace_size(p, T, groups, rank);
  REQUIRE(ws != nullptr && ws_bytes >= need, SAC_ERR_WORKSPACE,
          "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  REQUIRE((reinterpret_cast<uintptr_t>(ws) & 255) == 0, SAC_ERR_ARG,
          "ws must be 256-byte aligned");
  if (T == 0) return SAC_OK;  // nothing to do: no device work
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carve cv(ws);
  int* status = static_cast<int*>(cv.take(kStatusBytes));
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  sac::OProjArgs a;
  a.T = T;
  a.H = p->H;
  a.D = p->D;
  a.groups = groups;
  a.rank = rank;
  a.hidden = hidden;
  a.o = o;
  a.w_a = w_a;
  a.w_b = w_b;
  a.out = out;
  a.mid = cv.take((size_t)T * groups * rank * 2);
  a.status = status;
  e = sac::timed("o_proj", st, [&] { return sac::launch_oproj(a, st); });
  if (e != cudaSuccess) return cuda_fail(e, "output projection");
  return SAC_OK;
}

}  // extern "C"
