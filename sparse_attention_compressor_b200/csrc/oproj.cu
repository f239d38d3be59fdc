// Grouped low-rank output projection ("DeepSeek-V4" page, "Grouped Output Projection" bullet; config
// o_groups, o_lora_rank, hidden_size): the attention output o [T, H*D] is cut into G groups of H/G
// heads; group g's (H/G)*D features go through its own o_a_proj matrix to `rank` features, the
// G*rank results are concatenated and o_b_proj maps them to `hidden`.
//
// Both steps are plain dense GEMMs (bf16 in, fp32 accumulate, bf16 out), so they run on cuBLASLt:
// o_a_proj as one strided-batched GEMM over the groups (the group slices of o are column blocks of
// a row-major matrix, read in place), o_b_proj as one GEMM. Row-major C = A * W^T with W in the
// nn.Linear layout [out, in] is the column-major product C^T = W * A^T, which is how the calls
// below are set up.
#include <cublasLt.h>

#include <map>
#include <mutex>

#include "sac_kernels.h"

namespace sac {
namespace {

cublasLtHandle_t lt_handle(int dev) {
  static std::mutex mu;
  static std::map<int, cublasLtHandle_t> handles;
  std::lock_guard<std::mutex> lk(mu);
  auto it = handles.find(dev);
  if (it != handles.end()) return it->second;
  cublasLtHandle_t h = nullptr;
  if (cublasLtCreate(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
  handles[dev] = h;
  return h;
}

// One (possibly batched) row-major GEMM C[b] = A[b] * W[b]^T:
//   A [rows, k] with leading dimension lda (elements), W [n, k] contiguous, C [rows, n] with ldc;
//   batch b offsets: A by stride_a, W by n*k, C by stride_c (elements).
cudaError_t gemm_rm(cublasLtHandle_t h, int64_t rows, int n, int k, const void* A, int64_t lda,
                    int64_t stride_a, const void* W, void* C, int64_t ldc, int64_t stride_c,
                    int batch, void* ws, size_t ws_bytes, cudaStream_t st) {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t lw = nullptr, la = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  cudaError_t err = cudaErrorUnknown;
  const cublasOperation_t tn = CUBLAS_OP_T, nn = CUBLAS_OP_N;
  const float alpha = 1.f, beta = 0.f;
  const int64_t stride_w = (int64_t)n * k;
  cublasLtMatmulHeuristicResult_t res{};
  int found = 0;
  // column-major view: D[n, rows] = op(Wcm)[n, k] * Acm[k, rows], Wcm = W^T [k, n]
  if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS)
    goto done;
  cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &tn, sizeof(tn));
  cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &nn, sizeof(nn));
  if (cublasLtMatrixLayoutCreate(&lw, CUDA_R_16BF, k, n, k) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, k, rows, lda) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatrixLayoutCreate(&lc, CUDA_R_16BF, n, rows, ldc) != CUBLAS_STATUS_SUCCESS)
    goto done;
  if (batch > 1) {
    for (auto* l : {lw, la, lc})
      cublasLtMatrixLayoutSetAttribute(l, CUBLASLT_MATRIX_LAYOUT_BATCH_COUNT, &batch, sizeof(batch));
    cublasLtMatrixLayoutSetAttribute(lw, CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &stride_w,
                                     sizeof(stride_w));
    cublasLtMatrixLayoutSetAttribute(la, CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &stride_a,
                                     sizeof(stride_a));
    cublasLtMatrixLayoutSetAttribute(lc, CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &stride_c,
                                     sizeof(stride_c));
  }
  if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) goto done;
  cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes,
                                       sizeof(ws_bytes));
  if (cublasLtMatmulAlgoGetHeuristic(h, op, lw, la, lc, lc, pref, 1, &res, &found) !=
          CUBLAS_STATUS_SUCCESS ||
      found == 0)
    goto done;
  if (cublasLtMatmul(h, op, &alpha, W, lw, A, la, &beta, C, lc, C, lc, &res.algo, ws, ws_bytes,
                     st) == CUBLAS_STATUS_SUCCESS)
    err = cudaSuccess;
done:
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (lw) cublasLtMatrixLayoutDestroy(lw);
  if (op) cublasLtMatmulDescDestroy(op);
  return err;
}

}  // namespace

size_t oproj_gemm_scratch_bytes() { return size_t(32) << 20; }

cudaError_t launch_oproj(const OProjArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cublasLtHandle_t h = lt_handle(dev);
  if (h == nullptr) return cudaErrorInitializationError;
  const int kg = a.H / a.groups * a.D;       // features of one group
  const int64_t ld_o = (int64_t)a.H * a.D;   // row stride of o
  const int64_t ld_mid = (int64_t)a.groups * a.rank;
  // o_a_proj: mid[:, g*rank : (g+1)*rank] = o[:, g*kg : (g+1)*kg] * w_a[g]^T, all groups at once
  e = gemm_rm(h, a.T, a.rank, kg, a.o, ld_o, kg, a.w_a, a.mid, ld_mid, a.rank, a.groups,
              a.scratch, a.scratch_bytes, st);
  if (e != cudaSuccess) return e;
  // o_b_proj: out = mid * w_b^T
  return gemm_rm(h, a.T, a.hidden, a.groups * a.rank, a.mid, ld_mid, 0, a.w_b, a.out, a.hidden, 0,
                 1, a.scratch, a.scratch_bytes, st);
}

}  // namespace sac
