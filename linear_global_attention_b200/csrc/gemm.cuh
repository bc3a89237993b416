#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

namespace zebra {

constexpr size_t GEMM_WS_BYTES = 32u << 20;

// Row-major Cout[M_rows, N_cols] = A[M_rows, K] * B[N_cols, K]^T + beta * Cin (bf16, fp32 accumulate).
int gemm_bf16_nt(const void* A, const void* B, const void* Cin, void* Cout, long long M_rows, long long N_cols,
                 long long K, float beta, void* ws, size_t ws_bytes, cudaStream_t st);

// Row-major C[b][M_rows, N_cols] (row stride ldc) = A[b][M_rows, K] * B[b][N_cols, K]^T for b < batch,
// bf16 inputs (rows of K contiguous elements), fp32 accumulate and output. The algorithm is taken
// without split-K, so every output element sums its K products in the same order.
int gemm_bf16_nt_f32(const void* A, const void* B, float* C, long long M_rows, long long N_cols, long long K,
                     long long ldc, int batch, long long strideA, long long strideB, long long strideC, void* ws,
                     size_t ws_bytes, cudaStream_t st);

}  // namespace zebra
