// Projection GEMMs of the stacked layer (bf16 in, fp32 accumulate, bf16 out)
// through cuBLASLt: the QKV projection [N, 3D] = x W_qkv^T and the output
// projection with the residual, x_out = x + O W_o^T. Both are plain dense
// GEMMs; the attention itself runs in this library's own kernels.
#include <cublasLt.h>

#include <mutex>

#include "common.cuh"
#include "gemm.cuh"

namespace zebra {

static cublasLtHandle_t lt_handle() {
  static std::once_flag once;
  static cublasLtHandle_t h = nullptr;
  std::call_once(once, [] {
    if (cublasLtCreate(&h) != CUBLAS_STATUS_SUCCESS) h = nullptr;
  });
  return h;
}

// Row-major C[M_rows, N_cols] (+)= A[M_rows, K] * B[N_cols, K]^T, all bf16.
// In cuBLASLt's column-major terms: C^T (N_cols x M_rows) = B (N_cols x K) * A^T.
int gemm_bf16_nt(const void* A, const void* B, const void* Cin, void* Cout, long long M_rows, long long N_cols,
                 long long K, float beta, void* ws, size_t ws_bytes, cudaStream_t st) {
  cublasLtHandle_t h = lt_handle();
  if (!h) {
    set_error("cublasLtCreate failed");
    return ZEBRA_ERR_CUDA;
  }
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  int rc = ZEBRA_OK;
  const cublasOperation_t tA = CUBLAS_OP_T, tB = CUBLAS_OP_N;
  // column-major problem: m = N_cols, n = M_rows, k = K
  //   op(A') = B-matrix rows as columns: stored (K x N_cols) col-major, transposed
  //   op(B') = A^T: stored (K x M_rows) col-major
  cublasStatus_t s = cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &tA, sizeof(tA));
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tB, sizeof(tB));
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, K, N_cols, K);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, K, M_rows, K);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&lc, CUDA_R_16BF, N_cols, M_rows, N_cols);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulPreferenceCreate(&pref);
  if (s == CUBLAS_STATUS_SUCCESS)
    s = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes, sizeof(ws_bytes));
  cublasLtMatmulHeuristicResult_t res;
  int found = 0;
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &res, &found);
  if (s == CUBLAS_STATUS_SUCCESS && found == 0) s = CUBLAS_STATUS_NOT_SUPPORTED;
  if (s == CUBLAS_STATUS_SUCCESS) {
    const float alpha = 1.0f;
    ProfScope prof("cublasLt_gemm", st);
    s = cublasLtMatmul(h, op, &alpha, B, la, A, lb, &beta, beta != 0.f ? Cin : Cout, lc, Cout, lc, &res.algo, ws,
                       ws_bytes, st);
  }
  if (s != CUBLAS_STATUS_SUCCESS) {
    set_error(std::string("cuBLASLt matmul failed, status ") + std::to_string((int)s));
    rc = ZEBRA_ERR_CUDA;
  }
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return rc;
}

int gemm_bf16_nt_f32(const void* A, const void* B, float* C, long long M_rows, long long N_cols, long long K,
                     long long ldc, int batch, long long strideA, long long strideB, long long strideC, void* ws,
                     size_t ws_bytes, cudaStream_t st) {
  cublasLtHandle_t h = lt_handle();
  if (!h) {
    set_error("cublasLtCreate failed");
    return ZEBRA_ERR_CUDA;
  }
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  int rc = ZEBRA_OK;
  const cublasOperation_t tA = CUBLAS_OP_T, tB = CUBLAS_OP_N;
  const int32_t bc = batch;
  // column-major problem as in gemm_bf16_nt: C^T (N_cols x M_rows, ld ldc) = B (N_cols x K) * A^T
  cublasStatus_t s = cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &tA, sizeof(tA));
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tB, sizeof(tB));
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, K, N_cols, K);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, K, M_rows, K);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, N_cols, M_rows, ldc);
  auto batch_attr = [&](cublasLtMatrixLayout_t l, long long stride) {
    cublasStatus_t r = cublasLtMatrixLayoutSetAttribute(l, CUBLASLT_MATRIX_LAYOUT_BATCH_COUNT, &bc, sizeof(bc));
    if (r == CUBLAS_STATUS_SUCCESS)
      r = cublasLtMatrixLayoutSetAttribute(l, CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &stride, sizeof(stride));
    return r;
  };
  if (s == CUBLAS_STATUS_SUCCESS) s = batch_attr(la, strideB);
  if (s == CUBLAS_STATUS_SUCCESS) s = batch_attr(lb, strideA);
  if (s == CUBLAS_STATUS_SUCCESS) s = batch_attr(lc, strideC);
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulPreferenceCreate(&pref);
  if (s == CUBLAS_STATUS_SUCCESS)
    s = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes, sizeof(ws_bytes));
  // first heuristic result that does not split K (split-K or stream-K would sum the K products of
  // different output tiles in different orders)
  cublasLtMatmulHeuristicResult_t res[8];
  int found = 0, pick = -1;
  if (s == CUBLAS_STATUS_SUCCESS) s = cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 8, res, &found);
  for (int i = 0; s == CUBLAS_STATUS_SUCCESS && i < found && pick < 0; ++i) {
    int32_t splitk = 1;
    size_t got = 0;
    if (cublasLtMatmulAlgoConfigGetAttribute(&res[i].algo, CUBLASLT_ALGO_CONFIG_SPLITK_NUM, &splitk, sizeof(splitk),
                                             &got) == CUBLAS_STATUS_SUCCESS &&
        splitk <= 1)
      pick = i;
  }
  if (s == CUBLAS_STATUS_SUCCESS && pick < 0) s = CUBLAS_STATUS_NOT_SUPPORTED;
  if (s == CUBLAS_STATUS_SUCCESS) {
    const float alpha = 1.0f, beta = 0.0f;
    s = cublasLtMatmul(h, op, &alpha, B, la, A, lb, &beta, C, lc, C, lc, &res[pick].algo, ws, ws_bytes, st);
  }
  if (s != CUBLAS_STATUS_SUCCESS) {
    set_error(std::string("cuBLASLt score matmul failed, status ") + std::to_string((int)s));
    rc = ZEBRA_ERR_CUDA;
  }
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return rc;
}

}  // namespace zebra
